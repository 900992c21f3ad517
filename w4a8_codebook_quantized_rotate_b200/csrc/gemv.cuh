// Decode kernel (M <= 16): y[m, n] = s_x[m] s_ch[n] sum_g s_rel[n, g] sum_{k in g} cb[idx[n, k]] x_q[m, k].
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
//   * s_x and s_ch scale the final sum in fp32, and y is rounded to bf16.
//
// Work split ("stream-K"): a unit is (tile pair p, chunk c), i.e. 32 rows x
// 64 k.  The P * C units, in [p][c] order (the order they lie in memory),
// are cut into W equal ranges, one per warp.  A warp that covers a whole
// tile pair writes y directly; a pair split across warps leaves one fp32
// partial per warp in the workspace, and the last of its warps to finish
// (found with an atomic counter, no waiting) adds the partials in warp order
// -- the sum is deterministic -- and writes y.
#pragma once

#include "common.cuh"

namespace w4a8 {

constexpr int kDecWarps = 16;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecTG = 2;                    // tiles (16 rows each) per unit
constexpr int kDecMaxWarps = 148 * kDecWarps;  // cap on W, fixes the workspace size
constexpr size_t kDecSmemBytes = 2 * 65536;  // room for a 64 KiB-aligned 64 KiB table

struct DecodeParams {
  const uint8_t* idx;    // index plane
  const uint8_t* srel;   // group-scale plane
  const float* sch;      // [N]
  const float* cb;       // [16]
  const uint4* xfrag;    // activations in B-fragment order, [C][NB][32][2] uint4
  const float* s_x;      // [M]
  uint16_t* y;           // [M, N] bf16
  float* slots;          // [2 W][kDecTG * 16 * 8 * NB]
  unsigned* counters;    // [P]
  unsigned* err;
  int M, N, C, T, P, W, U;
};

__host__ __device__ inline int dec_slot_floats(int nb) { return kDecTG * 16 * 8 * nb; }

// The warp whose range holds unit u (ranges are [floor(w U / W), floor((w+1) U / W))).
__device__ __forceinline__ int dec_warp_of(int u, int U, int W) {
  return int((int64_t(u + 1) * W - 1) / U);
}
__device__ __forceinline__ int dec_range_begin(int w, int U, int W) { return int(int64_t(w) * U / W); }

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

template <int NB>
struct DecStage {
  uint4 w[kDecTG];     // index bytes, one 16-byte fragment set per tile
  uint2 s[kDecTG];     // group-scale bytes (rows g, g+8) x 4 steps
  uint4 x[NB][2];      // B fragments for the chunk's four k16 steps
};

template <int NB>
__device__ __forceinline__ void dec_load_weights(DecStage<NB>& st, const DecodeParams& p, int pair, int c,
                                                 int lane) {
#pragma unroll
  for (int i = 0; i < kDecTG; ++i) {
    const int tile = pair * kDecTG + i;
    if (tile < p.T) {
      const size_t blk = size_t(tile) * p.C + c;
      st.w[i] = ld_stream_v4(p.idx + blk * kChunkIdxBytes + lane * 16);
      st.s[i] = ld_stream_v2(p.srel + blk * kChunkSrelBytes + (lane >> 2) * 8);
    } else {
      st.w[i] = make_uint4(0, 0, 0, 0);
      st.s[i] = make_uint2(0, 0);
    }
  }
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

template <int NB, bool SINGLE>
__device__ __forceinline__ void dec_compute(const DecStage<NB>& st, float (&acc)[kDecTG][NB][4],
                                            uint32_t lut_lane) {
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    uint32_t b[NB][2];
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const uint4& xv = st.x[j][s >> 1];
      b[j][0] = (s & 1) ? xv.z : xv.x;
      b[j][1] = (s & 1) ? xv.w : xv.y;
    }
#pragma unroll
    for (int i = 0; i < kDecTG; ++i) {
      const uint32_t word = s == 0 ? st.w[i].x : s == 1 ? st.w[i].y : s == 2 ? st.w[i].z : st.w[i].w;
      // address = lut base + (byte << 8) + 4 lane: the byte replaces bits 8..15
      const uint32_t a0 = lds32(prmt(word, lut_lane, 0x7604u));
      const uint32_t a1 = lds32(prmt(word, lut_lane, 0x7614u));
      const uint32_t a2 = lds32(prmt(word, lut_lane, 0x7624u));
      const uint32_t a3 = lds32(prmt(word, lut_lane, 0x7634u));
      const uint32_t pair_codes = ((s < 2) ? st.s[i].x : st.s[i].y) >> (16 * (s & 1));
      const float2 sc = e4m3x2_to_float2(pair_codes);  // (row g, row g+8)
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        float d[4];
        mma_16816(d, a0, a1, a2, a3, b[j][0], b[j][1]);
        acc[i][j][0] = fmaf(d[0], sc.x, acc[i][j][0]);
        acc[i][j][2] = fmaf(d[2], sc.y, acc[i][j][2]);
        if (!SINGLE) {
          acc[i][j][1] = fmaf(d[1], sc.x, acc[i][j][1]);
          acc[i][j][3] = fmaf(d[3], sc.y, acc[i][j][3]);
        }
      }
    }
  }
}

// acc element e of (tile i, block j) is row 16 tile + g + 8 (e >> 1), token 8 j + 2 t + (e & 1).
template <int NB>
__device__ __forceinline__ void dec_epilogue(const float (&acc)[kDecTG][NB][4], const DecodeParams& p, int pair,
                                             int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int i = 0; i < kDecTG; ++i) {
    const int tile = pair * kDecTG + i;
    if (tile >= p.T) continue;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = tile * 16 + g + 8 * (e >> 1);
        const int tok = 8 * j + 2 * t + (e & 1);
        if (tok < p.M) {
          const float v = acc[i][j][e] * p.sch[row] * p.s_x[tok];
          p.y[size_t(tok) * p.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        }
      }
    }
  }
}

template <int NB>
__device__ __forceinline__ int dec_slot_index(int w, int pair, const DecodeParams& p) {
  const int first_pair = dec_range_begin(w, p.U, p.W) / p.C;
  return 2 * w + (pair == first_pair ? 0 : 1);
}

// Called when a warp leaves tile pair `pair`, having covered chunks
// [c_first, c_last] of it.
template <int NB>
__device__ __forceinline__ void dec_flush(float (&acc)[kDecTG][NB][4], const DecodeParams& p, int pair,
                                          int c_first, int c_last, int w, int lane) {
  if (c_first == 0 && c_last == p.C - 1) {
    dec_epilogue<NB>(acc, p, pair, lane);
    return;
  }
  const int g = lane >> 2, t = lane & 3;
  const int sf = dec_slot_floats(NB);
  float* mine = p.slots + size_t(dec_slot_index<NB>(w, pair, p)) * sf;
#pragma unroll
  for (int i = 0; i < kDecTG; ++i)
#pragma unroll
    for (int j = 0; j < NB; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = 8 * j + 2 * t + (e & 1);
        if (tok < p.M) mine[(i * 16 + g + 8 * (e >> 1)) * (8 * NB) + tok] = acc[i][j][e];
      }
  __threadfence();
  __syncwarp();
  const int w_first = dec_warp_of(pair * p.C, p.U, p.W);
  const int w_last = dec_warp_of(pair * p.C + p.C - 1, p.U, p.W);
  unsigned old = 0;
  if (lane == 0) old = atomicAdd(p.counters + pair, 1u);
  old = __shfl_sync(0xffffffffu, old, 0);
  if (old != unsigned(w_last - w_first)) return;
  __threadfence();
  float sum[kDecTG][NB][4];
#pragma unroll
  for (int i = 0; i < kDecTG; ++i)
#pragma unroll
    for (int j = 0; j < NB; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) sum[i][j][e] = 0.f;
  for (int ww = w_first; ww <= w_last; ++ww) {
    const float* src = p.slots + size_t(dec_slot_index<NB>(ww, pair, p)) * sf;
#pragma unroll
    for (int i = 0; i < kDecTG; ++i)
#pragma unroll
      for (int j = 0; j < NB; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tok = 8 * j + 2 * t + (e & 1);
          if (tok < p.M) sum[i][j][e] += __ldcg(src + (i * 16 + g + 8 * (e >> 1)) * (8 * NB) + tok);
        }
  }
  if (lane == 0) p.counters[pair] = 0u;  // ready for the next launch on this workspace
  dec_epilogue<NB>(sum, p, pair, lane);
}

template <int NB, int D, bool SINGLE>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(16) uint8_t dec_smem[];
  const uint32_t base = smem_u32(dec_smem);
  const uint32_t lut = (base + 0xFFFFu) & ~0xFFFFu;  // 64 KiB aligned: bits 8..15 are zero
  const int lane = threadIdx.x & 31;
  // Fill the table: entry b, lane l at lut + 256 b + 4 l holds fp16 (cb[b & 15], cb[b >> 4]).
  for (int e = threadIdx.x; e < 256 * 32; e += kDecThreads) {
    const int b = e >> 5;
    const __half2 h = __floats2half2_rn(p.cb[b & 15], p.cb[b >> 4]);
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(lut + (uint32_t(b) << 8) + uint32_t(e & 31) * 4u),
                 "r"(*reinterpret_cast<const uint32_t*>(&h)));
  }
  __syncthreads();
  const uint32_t lut_lane = lut + uint32_t(lane) * 4u;
  const int w = blockIdx.x * kDecWarps + (threadIdx.x >> 5);
  if (w >= p.W) return;
  const int u0 = dec_range_begin(w, p.U, p.W);
  const int u1 = dec_range_begin(w + 1, p.U, p.W);

  DecStage<NB> st[D];
  // Weights do not depend on the previous kernel: start streaming them now.
  {
    int pr = u0 / p.C, c = u0 - pr * p.C;
#pragma unroll
    for (int d = 0; d < D; ++d) {
      if (u0 + d < u1) dec_load_weights<NB>(st[d], p, pr, c, lane);
      if (++c == p.C) { c = 0; ++pr; }
    }
  }
  pdl_wait();  // activations, scales and counters come from the previous kernel
  {
    int c = u0 % p.C;
#pragma unroll
    for (int d = 0; d < D; ++d) {
      if (u0 + d < u1) dec_load_x<NB>(st[d], p, c, lane);
      if (++c == p.C) c = 0;
    }
  }

  float acc[kDecTG][NB][4];
#pragma unroll
  for (int i = 0; i < kDecTG; ++i)
#pragma unroll
    for (int j = 0; j < NB; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

  int cur_pair = u0 / p.C;
  int cur_c = u0 - cur_pair * p.C;  // chunk of the unit being computed
  int c_first = cur_c;
  // position of the unit being prefetched (u + D)
  int pf_pair = (u0 + D) / p.C;
  int pf_c = (u0 + D) - pf_pair * p.C;

  for (int ub = u0; ub < u1; ub += D) {
#pragma unroll
    for (int d = 0; d < D; ++d) {
      const int u = ub + d;
      if (u < u1) {
        if (cur_c == 0 && u != u0) {  // entered a new tile pair
          dec_flush<NB>(acc, p, cur_pair - 1, c_first, p.C - 1, w, lane);
#pragma unroll
          for (int i = 0; i < kDecTG; ++i)
#pragma unroll
            for (int j = 0; j < NB; ++j)
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
          c_first = 0;
        }
        dec_compute<NB, SINGLE>(st[d], acc, lut_lane);
        if (u + D < u1) {
          dec_load_weights<NB>(st[d], p, pf_pair, pf_c, lane);
          dec_load_x<NB>(st[d], p, pf_c, lane);
        }
        if (++pf_c == p.C) { pf_c = 0; ++pf_pair; }
        if (++cur_c == p.C) { cur_c = 0; ++cur_pair; }
      }
    }
  }
  // The last unit computed was u1 - 1; its pair is the one still open.
  const int last_pair = (u1 - 1) / p.C;
  dec_flush<NB>(acc, p, last_pair, c_first, (u1 - 1) - last_pair * p.C, w, lane);
}

}  // namespace w4a8
