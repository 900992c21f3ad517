// Decode kernel (2 <= M <= 32 per launch): y[m, n] = s_x[m] s_ch[n] sum_g s_rel[n, g] sum_{k in g} cb[idx[n, k]] x_q[m, k].
//
// The layer re-reads every weight for every token, so this kernel is bound
// by HBM ("Qwen3.8-27B-AEON-ULTIMATE-UNCENSORED-BF16 -- W4A8 ConvRot for
// ComfyUI" model card, section "Why this exists").  The weights stream once
// through registers with 128-bit loads; the arithmetic per weight has to fit
// in about two issue slots, so:
//   * a lane's 16 index bytes per (tile, chunk) are its mma.sync A
//     fragments for four k16 steps (the layout in common.cuh);
//   * each index byte becomes the fp16 pair (cb[lo], cb[hi]) through a
//     256-entry table in shared memory, replicated per lane (bank = lane,
//     conflict-free); the table sits at a 64 KiB-aligned shared address so
//     that one byte permute forms the lookup address;
//   * one mma.sync m16n8k16 (fp16 x fp16 -> fp32) reduces 16 k for 16 rows
//     and up to 8 tokens; a k16 step is exactly one 16-wide group, so its
//     fp32 partial is scaled by the group's s_rel in fp32 and accumulated in
//     fp32;
//   * (one token runs gemv1.cuh, whose MMA columns hold 8 groups instead of
//     8 tokens, so each lane scales its group partials once per chunk pair);
//   * 17..32 tokens (four blocks of 8 per fragment): the group scale goes
//     into the fragment instead, fp16(fp16(cb) s_rel) as in the prefill
//     kernel, and the MMAs accumulate in fp32 -- 4 multiplies per k16 step
//     instead of 4 per token block;
//   * s_x and s_ch scale the final sum in fp32, and y is rounded to bf16.
//
// Work split ("stream-K"): a unit is (tile pair p, chunk c), i.e. 32 rows x
// 64 k.  The P * C units, in [p][c] order (the order they lie in memory),
// are cut into W equal ranges, one per warp; a CTA's 12 (8 for 17..32
// tokens) warps hold consecutive ranges.  A warp that covers a whole tile
// pair writes y directly.  A pair split between warps is reduced in two
// levels, both in a fixed order (the result is deterministic): the warps of
// a CTA leave their partials in shared memory and one warp adds them after a
// CTA barrier; a pair that also crosses into other CTAs leaves each CTA's
// partial in the workspace: between two CTAs each lane meets its counterpart
// through an exchange word and the second to arrive adds the two; among
// more, the last CTA to finish (an atomic counter, no waiting) adds them in
// CTA order and writes y.
#pragma once

#include <type_traits>

#include "act.cuh"
#include "common.cuh"

namespace w4a8 {

constexpr int kDecWarps = 16;                      // one token
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecWarpsMulti = 12;                 // 2..16 tokens: fewer warps, more registers each
constexpr int kDecWarpsWide = 8;                   // 17..32 tokens (4 blocks of 8): more registers still
__host__ __device__ constexpr int dec_warps(bool single) { return single ? kDecWarps : kDecWarpsMulti; }
// Warps per CTA of the kernel serving m tokens (one launch).
__host__ __device__ constexpr int dec_warps_m(int m) {
  return m == 1 ? kDecWarps : m <= 16 ? kDecWarpsMulti : kDecWarpsWide;
}
__host__ __device__ constexpr int dec_warps_nb(int nb) { return nb >= 4 ? kDecWarpsWide : kDecWarpsMulti; }
constexpr int kDecTG = 2;                          // tiles (16 rows each) per unit
constexpr int kDecMaxCtas = 148;                   // cap on the grid, fixes the workspace size
// The part of a workspace that must hold zeros when a launch starts (every
// completed launch leaves it so): per CTA boundary, 32 exchange words (a row
// pair split between two CTAs) and one arrival counter (a pair split among
// more).  It sits at the workspace's start and has a fixed size, so calls of
// any shape may share a workspace.
constexpr size_t kWsXchBytes = size_t(kDecMaxCtas) * 32 * 8;
constexpr size_t kWsCntOff = kWsXchBytes;
constexpr size_t kWsZeroBytes = (kWsXchBytes + size_t(kDecMaxCtas) * 4 + 255) / 256 * 256;
constexpr size_t kDecSmemBase = 2 * 65536;         // room for a 64 KiB-aligned 64 KiB table
constexpr int kDecSchRows = 1024;                  // row scales staged in shared memory per CTA
// Units in flight per warp (register ring depth) per variant.
constexpr int kDecDepth1 = 3;                      // 2..8 tokens
constexpr int kDecDepth2 = 2;                      // 9..16 tokens
constexpr int kDecDepth4 = 3;                      // 17..32 tokens

struct DecodeParams {
  const uint16_t* x;     // one token's bf16 activations [K] (the kernel that rotates and quantises them itself)
  const uint8_t* units;  // unit region of the packed layer (contiguous 1152-byte units, [pair][chunk])
  const float* sch;      // [N]
  const float* cb;       // [16]
  const uint4* xfrag;    // activations in B-fragment order, [C][NB][32][2] uint4
  const float* s_x;      // [M]
  uint16_t* y;           // [M, N] bf16
  float* slots;          // [2 * CTAs][kDecTG * 16][M]: per-CTA partials of pairs shared with other CTAs
  unsigned long long* xch;  // [kDecMaxCtas][32]: one token, a pair split between CTAs c and c + 1
  unsigned* counters;    // [kDecMaxCtas]: arrivals at a pair whose first CTA is c
  unsigned* err;
  int M, N, K, C, T, P, W, U;
  int R, Rm;  // U / W and U % W: warp w's first unit is w R + floor(w Rm / W)
  // one token (gemv1.cuh): the P C / 2 duos are split over G CTAs, CTA c
  // holding [c Dq + min(c, Dr), (c + 1) Dq + min(c + 1, Dr))
  int G, Dq, Dr;
  // One token in a decode chain (gemv1.cuh), all optional (null: unused):
  //  * producer: outputs [act_off, act_off + act_len) are the next layer's
  //    input; each 256-block of them, once all its rows are written, is
  //    rotated into act_rot (fp32) and its absmax folded into *act_amax
  //    (float bits, an atomic maximum); act_cnt counts written rows per block;
  //  * consumer: the token's rotated values and absmax come from the
  //    previous producer (in_rot, in_amax) instead of x;
  //  * zero_cnt[0 .. zero_n): cleared after the wait (the counters and absmax
  //    word of the set the next producer writes).
  float* act_rot;
  unsigned* act_cnt;
  unsigned* act_amax;
  int act_off, act_len;
  const float* in_rot;
  const unsigned* in_amax;
  unsigned* zero_cnt;
  int zero_n;
  // One token, input from another engine (w4a8_linear_flagged): every CTA
  // waits until x_ready[0] != 0 before reading x; the last CTA to see it
  // clears x_ready[0] and x_ready[1] (its arrival count).  Null: no wait.
  unsigned* x_ready;
};

// Floats of one partial (a tile pair, the first M tokens).
__host__ __device__ inline int dec_slot_floats(int m) { return kDecTG * 16 * m; }

// Dynamic shared memory of a launch: table (+ alignment room), one token's
// activations, and the CTA's per-warp partials.
__host__ __device__ inline size_t dec_smem_bytes(int m, int k, bool single) {
  return kDecSmemBase + (single ? size_t(k) * 2 : 0) + size_t(single ? kDecWarps : dec_warps_m(m)) * 2 *
         dec_slot_floats(m) * 4 +
         kDecSchRows * 4 + 128 + 128 + 64;
}



// Ranges: warp w holds units [floor(w U / W), floor((w+1) U / W)); in 32-bit
// arithmetic as w R + floor(w Rm / W) (w Rm < W^2 < 2^32).  w may be W.
__device__ __forceinline__ int dec_begin(int w, const DecodeParams& p) {
  return w * p.R + int((unsigned(w) * unsigned(p.Rm)) / unsigned(p.W));
}
// CTA c holds warps [16 c, 16 c + 16) (clipped at W).
template <int WARPS>
__device__ __forceinline__ int dec_cta_begin(int c, const DecodeParams& p) {
  return dec_begin(min(c * WARPS, p.W), p);
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds128_(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// D = A B + 0, with the zero C operand passed in as a register the caller
// keeps for the whole loop.
__device__ __forceinline__ void mma_16816z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1, float z) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
}

// D += A B.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Per-unit registers: index bytes and group scales of the two tiles, and (for
// more than one token) the B fragments of the unit's chunk.
template <int NB>
struct DecStage {
  uint4 w[kDecTG];
  uint2 s[kDecTG];
  uint4 x[NB][2];
};

__device__ __forceinline__ uint4 ld_stream_v4(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const uint8_t* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ld_stream_v2(const uint8_t* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// A lane's index words and scale codes of one unit: wp points at the lane's
// 16 index bytes of tile 0 in the unit, sp at its 8 scale bytes of tile 0.
template <int NB>
__device__ __forceinline__ void dec_load_w(DecStage<NB>& st, const uint8_t* wp, const uint8_t* sp) {
  st.w[0] = ld_stream_v4(wp);
  st.w[1] = ld_stream_v4(wp + kChunkIdxBytes);
  st.s[0] = ld_stream_v2(sp);
  st.s[1] = ld_stream_v2(sp + kChunkSrelBytes);
}

template <int NB>
__device__ __forceinline__ void dec_load_x(DecStage<NB>& st, const DecodeParams& p, int c, int lane) {
#pragma unroll
  for (int j = 0; j < NB; ++j) {
    if ((lane >> 2) + 8 * j < p.M) {
      const uint4* src = p.xfrag + (size_t(c * NB + j) * 32 + lane) * 2;
      st.x[j][0] = __ldg(src);
      st.x[j][1] = __ldg(src + 1);
    } else {
      st.x[j][0] = make_uint4(0, 0, 0, 0);
      st.x[j][1] = make_uint4(0, 0, 0, 0);
    }
  }
}

// One unit: all 32 table lookups are issued first, back to back, so their
// latencies overlap; then the 8 x NB MMAs and the fp32 group-scale
// accumulation.
template <int NB>
__device__ __forceinline__ void dec_compute(const DecStage<NB>& st, float (&acc)[kDecTG][NB][4], uint32_t lut_lane) {
  const float zero = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {  // two halves of two k16 steps each
    uint32_t a[kDecTG][2][4];
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
      const int s = 2 * h + s2;
#pragma unroll
      for (int i = 0; i < kDecTG; ++i) {
        const uint32_t word = s == 0 ? st.w[i].x : s == 1 ? st.w[i].y : s == 2 ? st.w[i].z : st.w[i].w;
        // address = table base + (byte << 8) + 4 lane: the byte replaces bits 8..15
        a[i][s2][0] = lds32(prmt(word, lut_lane, 0x7604u));
        a[i][s2][1] = lds32(prmt(word, lut_lane, 0x7614u));
        a[i][s2][2] = lds32(prmt(word, lut_lane, 0x7624u));
        a[i][s2][3] = lds32(prmt(word, lut_lane, 0x7634u));
      }
    }
    uint32_t b[2][NB][2];
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2)
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        const uint4& xv = st.x[j][h];
        b[s2][j][0] = s2 ? xv.z : xv.x;
        b[s2][j][1] = s2 ? xv.w : xv.y;
      }
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
      const int s = 2 * h + s2;
#pragma unroll
      for (int i = 0; i < kDecTG; ++i) {
        const uint32_t pair_codes = ((s < 2) ? st.s[i].x : st.s[i].y) >> (16 * (s & 1));
        if constexpr (NB >= 4) {
          // Four token blocks share each fragment: scale the fragment once
          // (fp16(fp16(cb) s_rel), the prefill kernel's operand) and let the
          // MMAs accumulate in fp32, instead of rescaling 4 NB partials.
          __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(__nv_fp8x2_storage_t(pair_codes & 0xFFFFu), __NV_E4M3);
          const __half2 hh = *reinterpret_cast<const __half2*>(&hr);  // (row g, row g+8), exact
          const __half2 sg = __low2half2(hh), sg8 = __high2half2(hh);
          uint32_t as[4];
          const __half2 m0 = __hmul2(*reinterpret_cast<const __half2*>(&a[i][s2][0]), sg);
          const __half2 m1 = __hmul2(*reinterpret_cast<const __half2*>(&a[i][s2][1]), sg8);
          const __half2 m2 = __hmul2(*reinterpret_cast<const __half2*>(&a[i][s2][2]), sg);
          const __half2 m3 = __hmul2(*reinterpret_cast<const __half2*>(&a[i][s2][3]), sg8);
          as[0] = *reinterpret_cast<const uint32_t*>(&m0);
          as[1] = *reinterpret_cast<const uint32_t*>(&m1);
          as[2] = *reinterpret_cast<const uint32_t*>(&m2);
          as[3] = *reinterpret_cast<const uint32_t*>(&m3);
#pragma unroll
          for (int j = 0; j < NB; ++j) mma_16816(acc[i][j], as[0], as[1], as[2], as[3], b[s2][j][0], b[s2][j][1]);
        } else {
          const float2 sc = e4m3x2_to_float2(pair_codes);  // (row g, row g+8)
#pragma unroll
          for (int j = 0; j < NB; ++j) {
            float d[4];
            mma_16816z(d, a[i][s2][0], a[i][s2][1], a[i][s2][2], a[i][s2][3], b[s2][j][0], b[s2][j][1], zero);
            acc[i][j][0] = fmaf(d[0], sc.x, acc[i][j][0]);
            acc[i][j][2] = fmaf(d[2], sc.y, acc[i][j][2]);
            acc[i][j][1] = fmaf(d[1], sc.x, acc[i][j][1]);
            acc[i][j][3] = fmaf(d[3], sc.y, acc[i][j][3]);
          }
        }
      }
    }
  }
}

// acc element e of (tile i, block j) is row 16 (2 pair + i) + g + 8 (e >> 1),
// token 8 j + 2 t + (e & 1).
// Row scales of the CTA's first kDecSchRows rows (from row0) and the tokens'
// s_x sit in shared memory; rows past those are read from global memory.
struct DecEpi {
  uint32_t sch;  // shared address of row scales [row0, row0 + kDecSchRows)
  uint32_t sx;   // shared address of s_x[0..M)
  int row0;
};

template <int NB>
__device__ __forceinline__ void dec_epilogue(const float (&acc)[kDecTG][NB][4], const DecodeParams& p, int pair,
                                             int lane, const DecEpi& ep) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int i = 0; i < kDecTG; ++i) {
    const int tile = pair * kDecTG + i;
    if (tile >= p.T) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = tile * 16 + g + 8 * h;
      const int rr = row - ep.row0;
      float sc;
      if (rr < kDecSchRows)
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(sc) : "r"(ep.sch + uint32_t(rr) * 4u));
      else
        sc = __ldg(p.sch + row);
#pragma unroll
      for (int j = 0; j < NB; ++j) {
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
          const int tok = 8 * j + 2 * t + e2;
          if (tok < p.M) {
            float sx;
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(sx) : "r"(ep.sx + uint32_t(tok) * 4u));
            const float v = acc[i][j][2 * h + e2] * sc * sx;
            p.y[size_t(tok) * p.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
          }
        }
      }
    }
  }
}

// A partial lives as [tile i][row 16][token m] floats; each lane owns the
// entries of its fragment positions with token < M.
template <int NB>
__device__ __forceinline__ void dec_partial_store_smem(const float (&acc)[kDecTG][NB][4], uint32_t dst, int M,
                                                       int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int i = 0; i < kDecTG; ++i)
#pragma unroll
    for (int j = 0; j < NB; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = 8 * j + 2 * t + (e & 1);
        if (tok < M) {
          const uint32_t a = dst + uint32_t(((i * 16 + g + 8 * (e >> 1)) * M + tok) * 4);
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(acc[i][j][e]));
        }
      }
}

template <int NB>
__device__ __forceinline__ void dec_partial_add_smem(float (&acc)[kDecTG][NB][4], uint32_t src, int M, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int i = 0; i < kDecTG; ++i)
#pragma unroll
    for (int j = 0; j < NB; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = 8 * j + 2 * t + (e & 1);
        if (tok < M) {
          float v;
          asm volatile("ld.shared.f32 %0, [%1];"
                       : "=f"(v)
                       : "r"(src + uint32_t(((i * 16 + g + 8 * (e >> 1)) * M + tok) * 4)));
          acc[i][j][e] += v;
        }
      }
}

template <int NB>
__device__ __forceinline__ void dec_zero(float (&acc)[kDecTG][NB][4]) {
#pragma unroll
  for (int i = 0; i < kDecTG; ++i)
#pragma unroll
    for (int j = 0; j < NB; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
}

// ---------------------------------------------------------------------------
// Work split ("stream-K"): the P * C units, in the order they lie in memory,
// are cut into W equal ranges, one per warp; a CTA's 16 warps hold 16
// consecutive ranges, so each warp streams one contiguous byte range.  A
// warp keeps D units in flight in registers (a ring refilled right after
// each unit is computed).  A warp that covers a whole tile pair writes y
// directly.  A pair split between warps is reduced in two levels, both in a
// fixed order (the result is deterministic): the warps of a CTA leave their
// partials in shared memory and one warp adds them after a CTA barrier; a
// pair that also crosses into other CTAs is finished by the CTA that comes
// last to it (an arrival counter; the last CTA adds the partials in CTA
// order).  This kernel serves 2..32 tokens per launch; one token runs the
// kernel in gemv1.cuh.
struct DecWaitPdl {
  static constexpr int kLoadsAhead = 4;  // kept blocks whose loads are all issued before the first transform
  __device__ __forceinline__ void operator()() const { pdl_wait(); }
};

template <int NB, int D, class Wait>
__device__ __forceinline__ void decode_body(const DecodeParams& p, const Wait& wait_inputs) {
  constexpr int kW = dec_warps_nb(NB);
  constexpr int kThr = kW * 32;
  extern __shared__ __align__(16) uint8_t dec_smem[];
  const uint32_t base = smem_u32(dec_smem);
  const uint32_t lut = (base + 0xFFFFu) & ~0xFFFFu;  // 64 KiB aligned: bits 8..15 are zero
  const uint32_t parts = lut + 65536u;                // [warp][2] partials
  const uint32_t part_bytes = uint32_t(dec_slot_floats(p.M)) * 4u;
  const uint32_t sch_s = parts + uint32_t(kW * 2) * part_bytes;  // row scales
  const uint32_t sx_s = sch_s + kDecSchRows * 4;                          // s_x[0..32)
  const uint32_t wbeg_s = sx_s + 128;  // warp range starts [kW + 1]; at +96 the CTA pair context [4]
  const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
  const int cta_w0 = blockIdx.x * kW;
  const int w = cta_w0 + wl;
  const int u0 = dec_begin(min(w, p.W), p);
  const int u1 = dec_begin(min(w + 1, p.W), p);
  const int n_units = u1 - u0;
  const int first_pair = u0 / p.C;
  const int first_c = u0 - first_pair * p.C;

  // This lane's index bytes and scale bytes in unit u0; every later unit is
  // kUnitBytes further on.
  const uint8_t* wp = p.units + size_t(u0) * kUnitBytes + lane * 16;
  const uint8_t* sp = p.units + size_t(u0) * kUnitBytes + 2 * kChunkIdxBytes + (lane >> 2) * 8;

  // The codebook level this lane puts in the table: loaded ahead of the
  // weight stream so that it does not queue behind it.
  const float level = p.cb[lane & 15];

  DecStage<NB> st[D];
  // Weights do not depend on the previous kernel: start streaming them now,
  // before the wait.  (x comes from it, so it is loaded after the wait.)
#pragma unroll
  for (int d = 0; d < D; ++d)
    if (d < n_units) dec_load_w<NB>(st[d], wp + d * kUnitBytes, sp + d * kUnitBytes);
  wp += D * kUnitBytes;
  sp += D * kUnitBytes;

  // The CTA's range, its warps' range starts and its rows' scales (all
  // independent of the previous kernel).
  const int v0 = dec_cta_begin<kW>(blockIdx.x, p), v1 = dec_cta_begin<kW>(blockIdx.x + 1, p);
  if (lane == 0) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(wbeg_s + uint32_t(wl) * 4u), "r"(u0));
    if (wl == kW - 1) asm volatile("st.shared.u32 [%0], %1;" ::"r"(wbeg_s + uint32_t(kW) * 4u), "r"(v1));
  }
  // The CTA's first and last pairs and the CTAs where those start and end,
  // for the reduction after the loop (worked out now, while the previous
  // grid runs, so that the tail has no divisions).
  const uint32_t ctx_s = wbeg_s + 96u;
  if (threadIdx.x == kThr - 1 && v1 > v0) {
    const int plo = v0 / p.C, phi = (v1 - 1) / p.C;
    int cf = blockIdx.x, cl = blockIdx.x;
    while (cf > 0 && dec_cta_begin<kW>(cf, p) > plo * p.C) --cf;
    while (dec_cta_begin<kW>(cl + 1, p) < (phi + 1) * p.C) ++cl;
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(ctx_s), "r"(plo), "r"(phi), "r"(cf), "r"(cl));
  }
  DecEpi ep;
  ep.sch = sch_s;
  ep.sx = sx_s;
  ep.row0 = (v0 / p.C) * (kDecTG * 16);
  // The CTA's row scales: loaded now, written to shared memory just before
  // the barrier that ends the activation step (no wait for them here).
  const int sch_rows = min(kDecSchRows, min(p.N, (v1 > v0 ? (v1 - 1) / p.C + 1 : 0) * kDecTG * 16) - ep.row0);
  constexpr int kSchPer = (kDecSchRows + kThr - 1) / kThr;
  float sch_r[kSchPer];
#pragma unroll
  for (int j = 0; j < kSchPer; ++j) {
    const int i = int(threadIdx.x) + j * kThr;
    sch_r[j] = i < sch_rows ? __ldg(p.sch + ep.row0 + i) : 0.f;
  }
  // Table: entry b for lane l at lut + 256 b + 4 l holds fp16 (cb[b & 15], cb[b >> 4]).
  for (int b = wl; b < 256; b += kW) {
    const float lo = __shfl_sync(0xffffffffu, level, b & 15);
    const float hi = __shfl_sync(0xffffffffu, level, b >> 4);
    const __half2 h = __floats2half2_rn(lo, hi);
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(lut + (uint32_t(b) << 8) + uint32_t(lane) * 4u),
                 "r"(*reinterpret_cast<const uint32_t*>(&h)));
  }
  wait_inputs();  // activations, scales and counters come from an earlier step
  int cx = first_c;  // chunk of the next x fragment to load
  if (threadIdx.x < p.M)
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(sx_s + threadIdx.x * 4u), "f"(p.s_x[threadIdx.x]));
#pragma unroll
  for (int d = 0; d < D; ++d) {
    if (d < n_units) {
      dec_load_x<NB>(st[d], p, cx, lane);
      if (++cx == p.C) cx = 0;
    }
  }
#pragma unroll
  for (int j = 0; j < kSchPer; ++j) {
    const int i = int(threadIdx.x) + j * kThr;
    if (i < sch_rows) asm volatile("st.shared.f32 [%0], %1;" ::"r"(sch_s + uint32_t(i) * 4u), "f"(sch_r[j]));
  }
  __syncthreads();

  const uint32_t lut_lane = lut + uint32_t(lane) * 4u;
  float acc[kDecTG][NB][4];
  dec_zero<NB>(acc);
  int cur_pair = first_pair, cur_c = first_c, c_first = first_c;
  auto compute = [&](const DecStage<NB>& s) { dec_compute<NB>(s, acc, lut_lane); };
  // A finished or range-ending pair: write y if this warp covered all of it,
  // else park the partial in shared memory (slot 0: the warp's first pair).
  auto close_pair = [&](int c_last) {
    if (c_first == 0 && c_last == p.C - 1) {
      dec_epilogue<NB>(acc, p, cur_pair, lane, ep);
    } else {
      const uint32_t slot = parts + uint32_t(wl * 2 + (cur_pair == first_pair ? 0 : 1)) * part_bytes;
      dec_partial_store_smem<NB>(acc, slot, p.M, lane);
    }
  };
  auto unit_done = [&]() {
    if (++cur_c == p.C) {
      close_pair(p.C - 1);
      dec_zero<NB>(acc);
      cur_c = 0;
      ++cur_pair;
      c_first = 0;
    }
  };
  auto refill = [&](DecStage<NB>& s, int off_units) {
    dec_load_w<NB>(s, wp + off_units * kUnitBytes, sp + off_units * kUnitBytes);
    dec_load_x<NB>(s, p, cx, lane);
    if (++cx == p.C) cx = 0;
  };
  int ub = 0;
  // Full rounds: every stage computes and refills.
  for (; ub + 2 * D <= n_units; ub += D) {
#pragma unroll
    for (int d = 0; d < D; ++d) {
      compute(st[d]);
      refill(st[d], d);
      unit_done();
    }
    wp += D * kUnitBytes;
    sp += D * kUnitBytes;
  }
  // Tail: fewer than 2 D units left.
#pragma unroll
  for (int d2 = 0; d2 < 2 * D; ++d2) {
    const int d = d2 % D;
    if (ub + d2 < n_units) {
      compute(st[d]);
      if (ub + d2 + D < n_units) refill(st[d], d2);
      unit_done();
    }
  }
  if (n_units > 0 && cur_c != 0) close_pair(cur_c - 1);
  __syncthreads();

  // ---- level 2: pairs split between warps, reduced by one warp of the CTA
  if (v0 >= v1) return;
  int wb[kW + 1];  // the CTA's warp range starts (registers are free after the loop)
#pragma unroll
  for (int i = 0; i <= kW; ++i)
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(wb[i]) : "r"(wbeg_s + uint32_t(i) * 4u));
  int pair_lo, pair_hi, cta_first, cta_last;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(pair_lo), "=r"(pair_hi), "=r"(cta_first), "=r"(cta_last)
               : "r"(ctx_s));
  for (int pr = pair_lo + wl; pr <= pair_hi; pr += kW) {
    const int q0 = pr * p.C, q1 = q0 + p.C;  // the pair's units [q0, q1)
    bool whole = false;                       // one warp held all of it (and wrote y)
#pragma unroll
    for (int ww = 0; ww < kW; ++ww) whole |= (wb[ww] <= q0) & (wb[ww + 1] >= q1);
    if (whole) continue;
    // CTAs cf..cl hold parts of the pair: only the CTA's first pair starts
    // before it and only its last one ends after it
    const int cf = pr == pair_lo ? cta_first : int(blockIdx.x);
    const int cl = pr == pair_hi ? cta_last : int(blockIdx.x);
    // the contributors' partials, added in warp order (all loads independent)
    dec_zero<NB>(acc);
#pragma unroll
    for (int ww = 0; ww < kW; ++ww) {
      const bool holds = (wb[ww] < q1) & (wb[ww + 1] > q0) & (wb[ww] < wb[ww + 1]);
      const uint32_t slot = parts + uint32_t(ww * 2 + (wb[ww] >= q0 ? 0 : 1)) * part_bytes;
      float part[kDecTG][NB][4];
      dec_zero<NB>(part);
      dec_partial_add_smem<NB>(part, slot, p.M, lane);
#pragma unroll
      for (int i = 0; i < kDecTG; ++i)
#pragma unroll
        for (int j = 0; j < NB; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[i][j][e] = holds ? acc[i][j][e] + part[i][j][e] : acc[i][j][e];
    }
    if (q0 >= v0 && q1 <= v1) {  // inside this CTA
      dec_epilogue<NB>(acc, p, pr, lane, ep);
      continue;
    }
    // ---- level 3: the pair spans CTAs cf..cl; park this CTA's partial in the workspace
    const int sf = dec_slot_floats(p.M);
    const int g = lane >> 2, t = lane & 3;
    float* mine = p.slots + size_t(blockIdx.x * 2 + (v0 >= q0 ? 0 : 1)) * sf;
#pragma unroll
    for (int i = 0; i < kDecTG; ++i)
#pragma unroll
      for (int j = 0; j < NB; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tok = 8 * j + 2 * t + (e & 1);
          if (tok < p.M) mine[(i * 16 + g + 8 * (e >> 1)) * p.M + tok] = acc[i][j][e];
        }
    if (cl == cf + 1) {
      // Two CTAs: each lane meets its counterpart through one exchange word
      // (the one-token kernel's words at this boundary).  The release orders
      // the lane's partial before the word; the second lane to arrive adds
      // the other's partial (a + b: the same in either order, and the same
      // as the arrival-count path) and writes the lane's values.
      unsigned long long* word = p.xch + size_t(cf) * 32 + lane;
      unsigned long long other;
      asm volatile("atom.acq_rel.gpu.global.exch.b64 %0, [%1], %2;" : "=l"(other) : "l"(word), "l"(1ull) : "memory");
      if (other == 0ull) continue;  // the other CTA finishes this lane's values
      *word = 0ull;                 // ready for the next launch on this workspace
      const int oc = int(blockIdx.x) == cf ? cl : cf;
      const float* theirs = p.slots + size_t(oc * 2 + (dec_cta_begin<kW>(oc, p) >= q0 ? 0 : 1)) * sf;
      float v[kDecTG][NB][4];
#pragma unroll
      for (int i = 0; i < kDecTG; ++i)
#pragma unroll
        for (int j = 0; j < NB; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tok = 8 * j + 2 * t + (e & 1);
            v[i][j][e] = tok < p.M ? __ldcg(theirs + (i * 16 + g + 8 * (e >> 1)) * p.M + tok) : 0.f;
          }
#pragma unroll
      for (int i = 0; i < kDecTG; ++i)
#pragma unroll
        for (int j = 0; j < NB; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[i][j][e] += v[i][j][e];
      dec_epilogue<NB>(acc, p, pr, lane, ep);
      continue;
    }
    __threadfence();
    __syncwarp();
    unsigned old = 0;
    if (lane == 0) old = atomicAdd(p.counters + cf, 1u);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old != unsigned(cl - cf)) continue;  // another CTA finishes this pair
    __threadfence();
    // Sum the CTAs' partials in CTA order; all loads are independent.
    constexpr int kMaxCtaParts = 4 / NB;
    dec_zero<NB>(acc);
    for (int c0 = cf; c0 <= cl; c0 += kMaxCtaParts) {
      float v[kMaxCtaParts][kDecTG][NB][4];
#pragma unroll
      for (int r = 0; r < kMaxCtaParts; ++r) {
        const int cc = c0 + r;
        const bool have = cc <= cl;
        const float* src = p.slots + size_t(cc * 2 + (have && dec_cta_begin<kW>(cc, p) >= q0 ? 0 : 1)) * sf;
#pragma unroll
        for (int i = 0; i < kDecTG; ++i)
#pragma unroll
          for (int j = 0; j < NB; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int tok = 8 * j + 2 * t + (e & 1);
              v[r][i][j][e] = (have && tok < p.M) ? __ldcg(src + (i * 16 + g + 8 * (e >> 1)) * p.M + tok) : 0.f;
            }
      }
#pragma unroll
      for (int r = 0; r < kMaxCtaParts; ++r)
#pragma unroll
        for (int i = 0; i < kDecTG; ++i)
#pragma unroll
          for (int j = 0; j < NB; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] += v[r][i][j][e];
    }
    if (lane == 0) p.counters[cf] = 0u;  // ready for the next launch on this workspace
    dec_epilogue<NB>(acc, p, pr, lane, ep);
  }
}

template <int NB, int D>
__global__ void __launch_bounds__(dec_warps_nb(NB) * 32, 1) decode_kernel(const DecodeParams p) {
  // The next kernel may launch now: it streams its own weights and waits for
  // this grid's completion before it touches anything this grid writes.
  pdl_launch_dependents();
  decode_body<NB, D>(p, DecWaitPdl{});
}

}  // namespace w4a8
