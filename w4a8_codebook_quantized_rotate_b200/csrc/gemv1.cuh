// One-token decode kernel: y[n] = s_x s_ch[n] sum_g s_rel[n, g] sum_{k in g} cb[idx[n, k]] x_q[k].
//
// The layer re-reads every weight for every token ("Qwen3.8-27B-AEON-
// ULTIMATE-UNCENSORED-BF16 -- W4A8 ConvRot for ComfyUI" model card, section
// "Why this exists"), so a call should take the time HBM needs to deliver
// 0.5625 bytes per weight.  Two things stand between a call and that:
//   * the instructions per weight: each 2048-weight unit costs 32 table
//     lookups (an address permute and a shared load each) and 8 MMAs at
//     least; the loop here adds about 30 more (B-operand masks, group
//     scales, pointer and pair bookkeeping) and nothing per unit beyond
//     that: a warp's range is a whole number of duos (the two units of an
//     even and the following odd chunk), so no unit needs a range check;
//   * the time before the loop (the lookup table, the wait for the
//     previous kernel, the activation step), during which HBM must keep
//     streaming: each warp fills its register ring and asks L2 to prefetch
//     the duos after it as soon as it starts, and keeps prefetching a fixed
//     distance ahead of the ring in the loop, so the loop (faster than HBM)
//     finds most of its bytes in L2.
//
// Per unit the arithmetic is the one of the multi-token kernel in gemv.cuh:
// index bytes become fp16 pairs through a 256-entry table replicated per
// lane in shared memory; one mma.sync m16n8k16 reduces a 16-k group for 16
// rows, with the 8 groups of a duo in the MMA's 8 columns (in step s of a
// chunk of parity q only the lanes of column 4 q + s hold x; every other B
// register is zero), so a lane scales its 4 group partials by s_rel in fp32
// once per duo; s_x and s_ch scale the row sum, and y is rounded to bf16.
//
// Work split: the duos, in memory order, are cut into one contiguous range
// per CTA (sizes differ by one at most), and a CTA's range into 16 warp
// ranges (sizes differ by one at most), with no division by a runtime
// value.  A pair split between warps or CTAs is reduced as in gemv.cuh: in
// shared memory within the CTA, then through one 64-bit exchange word per
// row (two CTAs) or the per-CTA partial slots and an arrival counter (more).
#pragma once

#include "gemv.cuh"

namespace w4a8 {

constexpr int kOneWarps = kDecWarps;        // 16 warps, one CTA per SM
constexpr int kOneThreads = kOneWarps * 32;
#ifndef W4A8_ONE_RING
#define W4A8_ONE_RING 2
#endif
constexpr int kOneRing = W4A8_ONE_RING;     // duos per warp held in registers
static_assert(kOneRing >= 1 && kOneRing <= 4, "the duo loop is unrolled for up to 4 ring slots");
#ifndef W4A8_ONE_PF
#define W4A8_ONE_PF 4
#endif
constexpr int kOnePf = W4A8_ONE_PF;         // duos prefetched into L2 beyond the ring
#ifndef W4A8_ONE_PF_LOOP
#define W4A8_ONE_PF_LOOP 0
#endif
constexpr bool kOnePfLoop = W4A8_ONE_PF_LOOP;  // keep that distance in the loop (else at the start only)
constexpr int kDuoBytes = 2 * kUnitBytes;   // 2304

// First duo of CTA c (c may be the grid size).
__device__ __forceinline__ int one_cta_duo(int c, const DecodeParams& p) { return c * p.Dq + min(c, p.Dr); }

// First duo of warp wl of a CTA holding duos [a, b) (wl may be 16).
__device__ __forceinline__ int one_warp_duo(int wl, int a, int b) {
  const int n = b - a;
  return a + wl * (n >> 4) + min(wl, n & 15);
}

// A lane's share of one unit: index bytes of the two tiles (its mma.sync A
// fragments for the unit's four k16 steps) and its 4 group-scale bytes of
// each tile.
struct OneUnit {
  uint4 w0, w1;
  uint32_t s0, s1;
};

__device__ __forceinline__ void one_load(OneUnit& u, const uint8_t* wp, const uint8_t* sp) {
  u.w0 = ld_stream_v4(wp);
  u.w1 = ld_stream_v4(wp + kChunkIdxBytes);
  u.s0 = ld_stream_u32(sp);
  u.s1 = ld_stream_u32(sp + kChunkSrelBytes);
}

// One unit into dm (the duo's fragment, columns = its 8 groups): 32 table
// lookups, issued back to back per half so that their latencies overlap,
// then 8 MMAs.  bm[s]: all ones in the lanes whose B fragment is live in
// step s of this unit's chunk.  FIRST: the even unit of the duo, whose
// first step starts dm from zero.
template <bool FIRST>
__device__ __forceinline__ void one_compute(const OneUnit& u, float (&dm)[2][4], uint32_t lut_lane, uint2 xv,
                                            const uint32_t (&bm)[4]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t a[2][2][4];
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
      const int s = 2 * h + s2;
      const uint32_t w0 = s == 0 ? u.w0.x : s == 1 ? u.w0.y : s == 2 ? u.w0.z : u.w0.w;
      const uint32_t w1 = s == 0 ? u.w1.x : s == 1 ? u.w1.y : s == 2 ? u.w1.z : u.w1.w;
      // address = table + (byte << 8) + 4 lane: the byte replaces bits 8..15
      a[0][s2][0] = lds32(prmt(w0, lut_lane, 0x7604u));
      a[0][s2][1] = lds32(prmt(w0, lut_lane, 0x7614u));
      a[0][s2][2] = lds32(prmt(w0, lut_lane, 0x7624u));
      a[0][s2][3] = lds32(prmt(w0, lut_lane, 0x7634u));
      a[1][s2][0] = lds32(prmt(w1, lut_lane, 0x7604u));
      a[1][s2][1] = lds32(prmt(w1, lut_lane, 0x7614u));
      a[1][s2][2] = lds32(prmt(w1, lut_lane, 0x7624u));
      a[1][s2][3] = lds32(prmt(w1, lut_lane, 0x7634u));
    }
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
      const int s = 2 * h + s2;
      const uint32_t b0 = xv.x & bm[s], b1 = xv.y & bm[s];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        if (FIRST && s == 0)
          mma_16816z(dm[i], a[i][s2][0], a[i][s2][1], a[i][s2][2], a[i][s2][3], b0, b1, 0.f);
        else
          mma_16816(dm[i], a[i][s2][0], a[i][s2][1], a[i][s2][2], a[i][s2][3], b0, b1);
      }
    }
  }
}

// ga += dm * s_rel in fp32.  Lane (g, t) holds columns 2 t, 2 t + 1 of dm,
// i.e. groups 2 (t & 1), 2 (t & 1) + 1 of the duo's chunk of parity t >> 1;
// its scale bytes of that chunk are (row g, group), (row g + 8, group),
// (row g, group + 1), (row g + 8, group + 1).
__device__ __forceinline__ void one_scale(float (&ga)[2][4], const float (&dm)[2][4], uint32_t sr0, uint32_t sr1) {
  const uint32_t sr[2] = {sr0, sr1};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float2 s02 = e4m3x2_to_float2(sr[i]);
    const float2 s13 = e4m3x2_to_float2(sr[i] >> 16);
    ga[i][0] = fmaf(dm[i][0], s02.x, ga[i][0]);
    ga[i][2] = fmaf(dm[i][2], s02.y, ga[i][2]);
    ga[i][1] = fmaf(dm[i][1], s13.x, ga[i][1]);
    ga[i][3] = fmaf(dm[i][3], s13.y, ga[i][3]);
  }
}

// Row sums of ga over the lane's two group columns and the 4 lanes of a
// row; every lane of the row ends with them (row g: r[i][0], row g + 8:
// r[i][1]), and ga is cleared.
__device__ __forceinline__ void one_rows(float (&ga)[2][4], float (&r)[2][2]) {
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float r0 = ga[i][0] + ga[i][1], r1 = ga[i][2] + ga[i][3];
    r0 += __shfl_xor_sync(0xffffffffu, r0, 1);
    r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
    r0 += __shfl_xor_sync(0xffffffffu, r0, 2);
    r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
    r[i][0] = r0;
    r[i][1] = r1;
#pragma unroll
    for (int e = 0; e < 4; ++e) ga[i][e] = 0.f;
  }
}

// Codes of 8 consecutive rotated values from k0 (a multiple of 8) into the
// B-fragment order in shared memory: the pair (k, k + 1) of chunk c, k16
// step s4, half w, lane t sits at c 128 + t 32 + (2 s4 + w) 4.  With a
// cluster partner (peer_xs != 0) the codes also go to its shared memory.
template <bool FAST>
__device__ __forceinline__ void one_put_codes(uint32_t xs, uint32_t peer_xs, int k0, const float (&v)[8],
                                              const QuantScale& qs) {
  const uint32_t off = uint32_t(k0 >> 6) * 128u + uint32_t(2 * ((k0 >> 4) & 3) + ((k0 >> 3) & 1)) * 4u;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const __half2 h = __floats2half2_rn(quant_code<FAST>(v[2 * t], qs), quant_code<FAST>(v[2 * t + 1], qs));
    const uint32_t hv = *reinterpret_cast<const uint32_t*>(&h);
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(xs + off + uint32_t(t) * 32u), "r"(hv));
    if (peer_xs) asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(peer_xs + off + uint32_t(t) * 32u), "r"(hv));
  }
}

// Consumer in a decode chain: the token's rotated values (fp32, in block
// order) and their absmax were left by the previous layer, so the codes are
// the activation step's last part alone: s = amax / 127 and the same
// quantisation of the same values, i.e. the same codes and s_x.
__device__ __forceinline__ void one_codes_from_rotated(const DecodeParams& p, uint32_t xs, uint32_t sx_s, int wl,
                                                       int lane) {
  const float amax = __uint_as_float(__ldcg(p.in_amax));
  const float s = quant_scale(amax);
  const QuantScale qs = quant_prepare(s);
  if (threadIdx.x == 0) asm volatile("st.shared.f32 [%0], %1;" ::"r"(sx_s), "f"(s));
  const int nblk = p.K / kRotBlock;
  auto body = [&](auto fast) {
    constexpr bool kFast = decltype(fast)::value;
    for (int b0 = wl; b0 < nblk; b0 += 2 * kOneWarps) {  // two blocks' loads in flight
      float v[2][8];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int b = b0 + r * kOneWarps;
        if (b < nblk) {
          const float4* src = reinterpret_cast<const float4*>(p.in_rot + b * kRotBlock + lane * 8);
          const float4 a = __ldcg(src), c = __ldcg(src + 1);
          v[r][0] = a.x; v[r][1] = a.y; v[r][2] = a.z; v[r][3] = a.w;
          v[r][4] = c.x; v[r][5] = c.y; v[r][6] = c.z; v[r][7] = c.w;
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int b = b0 + r * kOneWarps;
        if (b < nblk) one_put_codes<kFast>(xs, 0u, b * kRotBlock + lane * 8, v[r], qs);
      }
    }
  };
  if (qs.fast)
    body(std::true_type{});
  else
    body(std::false_type{});
}

// Producer in a decode chain: this warp has just written `nrows` rows of y
// in pair `pair` (all 32 lanes call it, converged).  Rows in the next
// layer's input range count towards their 256-block; the warp that
// completes a block rotates it (the activation step's transform, on the
// bf16 values just written) into act_rot and folds its absmax into
// *act_amax.  Ordering: each writer fences its stores before the counting
// atomic (acquire-release), and the completing warp reads after it.
__device__ __forceinline__ void one_emit(const DecodeParams& p, int pair, int nrows, int lane) {
  if (!p.act_cnt || nrows == 0) return;
  const int r0 = pair * (kDecTG * 16) - p.act_off;
  if (r0 < 0 || r0 >= p.act_len) return;
  const int blk = r0 >> 8;
  __threadfence();
  __syncwarp();
  unsigned old = 0;
  if (lane == 0)
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
                 : "=r"(old)
                 : "l"(p.act_cnt + blk), "r"(unsigned(nrows))
                 : "memory");
  old = __shfl_sync(0xffffffffu, old, 0);
  if (old + unsigned(nrows) != unsigned(kRotBlock)) return;  // the block is not complete yet
  __syncwarp();  // the lanes' loads come after lane 0's acquire
  float v[8];
  rotate_block_lane(p.y + p.act_off, blk, lane, v);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  float4* dst = reinterpret_cast<float4*>(p.act_rot + blk * kRotBlock + lane * 8);
  dst[0] = make_float4(v[0], v[1], v[2], v[3]);
  dst[1] = make_float4(v[4], v[5], v[6], v[7]);
  if (lane == 0) atomicMax(p.act_amax, __float_as_uint(amax));  // non-negative: bit order = value order
}

// The activation step of one token (the activation kernel's arithmetic:
// the same codes and s_x): rotate x per 256-block (a warp per block), find
// the absmax, quantise into the B-fragment order in shared memory (fp16
// codes; the pair (k, k + 1) of chunk c, k16 step s4, half w, lane t sits
// at c 128 + t 32 + (2 s4 + w) 4).  Launched as clusters of two CTAs, each
// CTA takes every other block and writes its codes into both CTAs' tables.
// s_x goes to sx_s; red_s holds 16 floats of scratch.
// `after_loads` runs once the warp's token loads are issued (the caller
// starts an L2 prefetch there).
template <class Wait, class AfterLoads>
__device__ __forceinline__ void one_activation(const DecodeParams& p, uint32_t xs, uint32_t sx_s, uint32_t red_s,
                                               int wl, int lane, const AfterLoads& after_loads) {
  const uint32_t crank = cluster_ctarank(), ncta = cluster_nctarank();
  const int nblk = p.K / kRotBlock;
  const int nown = (nblk - int(crank) + int(ncta) - 1) / int(ncta);  // blocks crank + ncta j
  constexpr int kKeep = 4;  // blocks a warp keeps rotated in registers (more are rotated again)
  constexpr int kAhead = Wait::kLoadsAhead < kKeep ? Wait::kLoadsAhead : kKeep;
  float amax = 0.f;
  float vk[kKeep][8];
  uint4 raw[kAhead];
#pragma unroll
  for (int jj = 0; jj < kAhead; ++jj) {
    const int j = wl + kOneWarps * jj;
    if (j < nown) raw[jj] = load_block_lane(p.x, int(crank) + int(ncta) * j, lane);
  }
  after_loads();
#pragma unroll
  for (int jj = 0; jj < kKeep; ++jj) {
    const int j = wl + kOneWarps * jj;
    if (j < nown) {
      rotate_words_lane(jj < kAhead ? raw[jj] : load_block_lane(p.x, int(crank) + int(ncta) * j, lane), lane,
                        vk[jj]);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(vk[jj][i]));
    }
  }
  for (int j = wl + kOneWarps * kKeep; j < nown; j += kOneWarps) {
    float v[8];
    rotate_block_lane(p.x, int(crank) + int(ncta) * j, lane, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (lane == 0) asm volatile("st.shared.f32 [%0], %1;" ::"r"(red_s + uint32_t(wl) * 4u), "f"(amax));
  __syncthreads();
#pragma unroll
  for (int i = 0; i < kOneWarps; ++i) {
    float m;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(m) : "r"(red_s + uint32_t(i) * 4u));
    amax = fmaxf(amax, m);
  }
  uint32_t peer_xs = 0;
  if (ncta > 1) {
    // this CTA's maximum goes to s_x[1]'s slot (one token: unused), read by the partner
    if (threadIdx.x == 0) asm volatile("st.shared.f32 [%0], %1;" ::"r"(sx_s + 4u), "f"(amax));
    cluster_sync_all();
    amax = fmaxf(amax, ld_cluster_f32(sx_s + 4u, crank ^ 1u));
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(peer_xs) : "r"(xs), "r"(crank ^ 1u));
  }
  const float s = quant_scale(amax);
  const QuantScale qs = quant_prepare(s);
  if (threadIdx.x == 0) asm volatile("st.shared.f32 [%0], %1;" ::"r"(sx_s), "f"(s));
  auto put_codes = [&](auto fast, int k0, const float (&v)[8]) {
    one_put_codes<decltype(fast)::value>(xs, ncta > 1 ? peer_xs : 0u, k0, v, qs);
  };
  auto quantise = [&](auto fast) {
#pragma unroll
    for (int jj = 0; jj < kKeep; ++jj) {
      const int j = wl + kOneWarps * jj;
      if (j < nown) put_codes(fast, (int(crank) + int(ncta) * j) * kRotBlock + lane * 8, vk[jj]);
    }
    for (int j = wl + kOneWarps * kKeep; j < nown; j += kOneWarps) {
      float v[8];
      const int b = int(crank) + int(ncta) * j;
      rotate_block_lane(p.x, b, lane, v);
      put_codes(fast, b * kRotBlock + lane * 8, v);
    }
  };
  if (qs.fast)
    quantise(std::true_type{});
  else
    quantise(std::false_type{});
  if (ncta > 1) cluster_sync_all();  // both halves of the codes are in place; no remote access after this
}

// The one-token layer.  FUSED: the kernel rotates and quantises x itself;
// otherwise it reads the B fragments and s_x an activation kernel wrote.
// ready_arrival: thread 0's arrival index on p.x_ready[1] (0 without a ready word).
template <bool FUSED, class Wait>
__device__ __forceinline__ void decode_one_body(const DecodeParams& p, const Wait& wait_inputs,
                                                unsigned& ready_arrival) {
  extern __shared__ __align__(16) uint8_t dec_smem[];
  const uint32_t base = smem_u32(dec_smem);
  const uint32_t lut = (base + 0xFFFFu) & ~0xFFFFu;  // 64 KiB aligned: bits 8..15 are zero
  const uint32_t xs = lut + 65536u;                   // the token's codes, C * 128 bytes
  const uint32_t parts = xs + uint32_t(p.C) * 128u;   // [warp][2] partials of 32 rows
  constexpr uint32_t kPartBytes = kDecTG * 16 * 4;
  const uint32_t sch_s = parts + uint32_t(kOneWarps * 2) * kPartBytes;  // row scales
  const uint32_t sx_s = sch_s + kDecSchRows * 4;                         // s_x (+4: the cluster partner's max)
  const uint32_t wbeg_s = sx_s + 64;   // warp range starts in units [17]; at +96 the CTA's pair context [4]
  const uint32_t red_s = wbeg_s + 128;  // per-warp maxima [16]
  const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;

  // This CTA's duos and this warp's (none for CTAs past the split).
  const int cd0 = one_cta_duo(min(int(blockIdx.x), p.G), p);
  const int cd1 = one_cta_duo(min(int(blockIdx.x) + 1, p.G), p);
  const int d0 = one_warp_duo(wl, cd0, cd1), d1 = one_warp_duo(wl + 1, cd0, cd1);
  const int nd = d1 - d0;
  const int v0 = 2 * cd0, v1 = 2 * cd1;  // the CTA's units
  const int u0 = 2 * d0;
  const int first_pair = u0 / p.C;
  const int first_c = u0 - first_pair * p.C;

  // The lane's index bytes (tile 0) and scale bytes (tile 0) in the warp's first unit.
  const uint8_t* wp = p.units + size_t(u0) * kUnitBytes + lane * 16;
  const uint8_t* sp = p.units + size_t(u0) * kUnitBytes + 2 * kChunkIdxBytes + (lane >> 2) * 8 + 4 * (lane & 1);
  const float level = p.cb[lane & 15];  // ahead of the weight stream in the memory queues

  // Register ring: duo j of the range sits in slot j % kOneRing.
  OneUnit st[kOneRing][2];
#pragma unroll
  for (int r = 0; r < kOneRing; ++r)
    if (r < nd) {
      one_load(st[r][0], wp + r * kDuoBytes, sp + r * kDuoBytes);
      one_load(st[r][1], wp + r * kDuoBytes + kUnitBytes, sp + r * kDuoBytes + kUnitBytes);
    }
  // L2 prefetch of the duos after the ring: one bulk prefetch per warp,
  // issued behind the token's loads (ahead of them it delays the activation
  // step more than it saves), so HBM keeps streaming through that step.
  auto prefetch_l2 = [&]() {
    if (kOnePf > 0 && lane == 0 && nd > kOneRing) {
      const int pf = min(nd, kOneRing + kOnePf) - kOneRing;
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.units + size_t(u0 + 2 * kOneRing) *
                                                                                 kUnitBytes),
                   "r"(uint32_t(pf) * uint32_t(kDuoBytes))
                   : "memory");
    }
  };

  // Warp range starts (in units) for the reduction after the loop.
  if (lane == 0) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(wbeg_s + uint32_t(wl) * 4u), "r"(u0));
    if (wl == kOneWarps - 1) asm volatile("st.shared.u32 [%0], %1;" ::"r"(wbeg_s + uint32_t(kOneWarps) * 4u), "r"(v1));
  }
  // The CTA's first and last pairs and the CTAs where those start and end.
  const uint32_t ctx_s = wbeg_s + 96u;
  if (threadIdx.x == kOneThreads - 1 && v1 > v0) {
    const int plo = v0 / p.C, phi = (v1 - 1) / p.C;
    int cf = blockIdx.x, cl = blockIdx.x;
    while (cf > 0 && 2 * one_cta_duo(cf, p) > plo * p.C) --cf;
    while (cl + 1 < p.G && 2 * one_cta_duo(cl + 1, p) < (phi + 1) * p.C) ++cl;
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(ctx_s), "r"(plo), "r"(phi), "r"(cf), "r"(cl));
  }
  DecEpi ep;
  ep.sch = sch_s;
  ep.sx = sx_s;
  ep.row0 = (v0 / p.C) * (kDecTG * 16);
  const int sch_rows = min(kDecSchRows, min(p.N, (v1 > v0 ? (v1 - 1) / p.C + 1 : 0) * kDecTG * 16) - ep.row0);
  constexpr int kSchPer = (kDecSchRows + kOneThreads - 1) / kOneThreads;
  float sch_r[kSchPer];
#pragma unroll
  for (int j = 0; j < kSchPer; ++j) {
    const int i = int(threadIdx.x) + j * kOneThreads;
    sch_r[j] = i < sch_rows ? __ldg(p.sch + ep.row0 + i) : 0.f;
  }
  // Table: entry b for lane l at lut + 256 b + 4 l holds fp16 (cb[b & 15],
  // cb[b >> 4]).  The codebook is part of the weights, which no earlier
  // kernel writes, so the table is built before the wait for the previous
  // kernel (measured: 0.2 us less per call at K=5120, N=17408 than building
  // it after the activation step).
  for (int b = wl; b < 256; b += kOneWarps) {
    const float lo = __shfl_sync(0xffffffffu, level, b & 15);
    const float hi = __shfl_sync(0xffffffffu, level, b >> 4);
    const __half2 h = __floats2half2_rn(lo, hi);
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(lut + (uint32_t(b) << 8) + uint32_t(lane) * 4u),
                 "r"(*reinterpret_cast<const uint32_t*>(&h)));
  }
  if (p.x_ready) {
    // x comes from another engine: wait (bounded) for its ready word, which
    // no earlier kernel touches, so this overlaps the previous kernel.  The
    // arrival's result only says which CTA clears the word, so thread 0
    // compares it after the layer (the kernel wrapper), not here.
    if (threadIdx.x == 0) {
      poll_at_least_bounded(p.x_ready, 1u, p.err, 1u << 21);  // about a second
      ready_arrival = atomicAdd(p.x_ready + 1, 1u);
    }
    __syncthreads();  // the CTA reads x after thread 0's acquire
  }
  wait_inputs();  // x (or the prepared codes) and the workspace come from an earlier step
  if (p.zero_cnt && blockIdx.x == 0)
    for (int i = threadIdx.x; i < p.zero_n; i += kOneThreads) p.zero_cnt[i] = 0u;
  if (FUSED && p.in_rot) {  // a decode chain's consumer: the previous layer rotated the token
    prefetch_l2();
    one_codes_from_rotated(p, xs, sx_s, wl, lane);
  } else if constexpr (FUSED) {
    one_activation<Wait>(p, xs, sx_s, red_s, wl, lane, prefetch_l2);
  } else {
    prefetch_l2();
    if (threadIdx.x == 0) asm volatile("st.shared.f32 [%0], %1;" ::"r"(sx_s), "f"(p.s_x[0]));
    // the token's B fragments: per chunk, lanes t = 0..3 of the fragment layout (128 bytes)
    const uint8_t* src = reinterpret_cast<const uint8_t*>(p.xfrag);
    for (int e = threadIdx.x; e < p.C * 8; e += kOneThreads) {
      const int c = e >> 3, qq = e & 7;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + size_t(c) * 1024 + qq * 16));
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(xs + uint32_t(c) * 128u + uint32_t(qq) * 16u),
                   "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w));
    }
  }
#pragma unroll
  for (int j = 0; j < kSchPer; ++j) {
    const int i = int(threadIdx.x) + j * kOneThreads;
    if (i < sch_rows) asm volatile("st.shared.f32 [%0], %1;" ::"r"(sch_s + uint32_t(i) * 4u), "f"(sch_r[j]));
  }
  __syncthreads();

  // ---- the loop over the warp's duos
  const int g_lane = lane >> 2, t_lane = lane & 3;
  const uint32_t lut_lane = lut + uint32_t(lane) * 4u;
  uint32_t bm_e[4], bm_o[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    bm_e[q] = (g_lane == q) ? 0xFFFFFFFFu : 0u;      // even chunks: lanes g = 0..3
    bm_o[q] = (g_lane == 4 + q) ? 0xFFFFFFFFu : 0u;  // odd chunks: lanes g = 4..7
  }
  // the lane's x pair in the chunk of its parity, relative to the duo's even chunk
  uint32_t xb = xs + uint32_t(lane & 3) * 32u + uint32_t(g_lane & 3) * 8u + uint32_t(g_lane >> 2) * 128u +
                uint32_t(first_c) * 128u;
  const uint32_t xb_pair0 = xb - uint32_t(first_c) * 128u;  // chunk 0 of a pair
  float dm[2][4], ga[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) ga[i][e] = 0.f;
  int cur_pair = first_pair;
  int c_first = first_c;      // the warp's first chunk of cur_pair
  int left = (p.C - first_c) >> 1;  // duos left in cur_pair
  // A finished or range-ending pair (c_last: its last chunk this warp
  // covered): write y if this warp covered all of it, else park the row sums
  // in shared memory (slot 0: the warp's first pair, slot 1: its last).
  auto close_pair = [&](int c_last) {
    float r[2][2];
    one_rows(ga, r);
    if (c_first == 0 && c_last == p.C - 1) {
      if (t_lane == 0) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int tile = cur_pair * kDecTG + i;
          if (tile < p.T) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int row = tile * 16 + g_lane + 8 * h;
              const int rr = row - ep.row0;
              float sc, sx;
              if (rr < kDecSchRows)
                asm volatile("ld.shared.f32 %0, [%1];" : "=f"(sc) : "r"(ep.sch + uint32_t(rr) * 4u));
              else
                sc = __ldg(p.sch + row);
              asm volatile("ld.shared.f32 %0, [%1];" : "=f"(sx) : "r"(ep.sx));
              p.y[row] = __bfloat16_as_ushort(__float2bfloat16_rn(r[i][h] * sc * sx));
            }
          }
        }
      }
      one_emit(p, cur_pair, (cur_pair * kDecTG + 1 < p.T ? 2 : 1) * 16, lane);
    } else if (t_lane == 0) {
      const uint32_t slot = parts + uint32_t(wl * 2 + (cur_pair == first_pair ? 0 : 1)) * kPartBytes;
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(slot + uint32_t(i * 16 + g_lane + 8 * h) * 4u),
                       "f"(r[i][h]));
    }
  };
  // One duo from ring slot R: both units into dm, each refilled right after
  // its MMAs with the duo kOneRing further on (if the range has it), then
  // the group scales, the L2 prefetch kOnePf duos past the ring, and the
  // pair bookkeeping.
  auto duo = [&](auto R, int j) {
    constexpr int r = decltype(R)::value;
    const uint2 xv = lds64(xb);
    const bool refill = j + kOneRing < nd;
    one_compute<true>(st[r][0], dm, lut_lane, xv, bm_e);
    const uint32_t se0 = st[r][0].s0, se1 = st[r][0].s1;
    if (refill) one_load(st[r][0], wp + kOneRing * kDuoBytes, sp + kOneRing * kDuoBytes);
    one_compute<false>(st[r][1], dm, lut_lane, xv, bm_o);
    const uint32_t so0 = st[r][1].s0, so1 = st[r][1].s1;
    if (refill)
      one_load(st[r][1], wp + kOneRing * kDuoBytes + kUnitBytes, sp + kOneRing * kDuoBytes + kUnitBytes);
    one_scale(ga, dm, t_lane < 2 ? se0 : so0, t_lane < 2 ? se1 : so1);
    if (kOnePfLoop && kOnePf > 0 && lane == 0 && j + kOneRing + kOnePf < nd)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(wp + (kOneRing + kOnePf) * kDuoBytes),
                   "n"(kDuoBytes)
                   : "memory");
    wp += kDuoBytes;
    sp += kDuoBytes;
    xb += 256u;
    if (--left == 0) {  // the pair's last duo
      close_pair(p.C - 1);
      ++cur_pair;
      c_first = 0;
      left = p.C >> 1;
      xb = xb_pair0;
    }
  };
  int j = 0;
  for (; j + kOneRing <= nd; j += kOneRing) {
    duo(std::integral_constant<int, 0>{}, j);
    if constexpr (kOneRing > 1) duo(std::integral_constant<int, 1>{}, j + 1);
    if constexpr (kOneRing > 2) duo(std::integral_constant<int, 2>{}, j + 2);
    if constexpr (kOneRing > 3) duo(std::integral_constant<int, 3>{}, j + 3);
  }
  if (j < nd) duo(std::integral_constant<int, 0>{}, j);
  if constexpr (kOneRing > 1) if (j + 1 < nd) duo(std::integral_constant<int, 1>{}, j + 1);
  if constexpr (kOneRing > 2) if (j + 2 < nd) duo(std::integral_constant<int, 2>{}, j + 2);
  if (nd > 0 && left != (p.C >> 1)) close_pair(p.C - 1 - 2 * left);  // the range ends inside a pair
  __syncthreads();

  // ---- level 2: pairs split between warps, reduced by one warp of the CTA
  if (v0 >= v1) return;
  int wb[kOneWarps + 1];
#pragma unroll
  for (int i = 0; i <= kOneWarps; ++i)
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(wb[i]) : "r"(wbeg_s + uint32_t(i) * 4u));
  int pair_lo, pair_hi, cta_first, cta_last;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(pair_lo), "=r"(pair_hi), "=r"(cta_first), "=r"(cta_last)
               : "r"(ctx_s));
  for (int pr = pair_lo + wl; pr <= pair_hi; pr += kOneWarps) {
    const int q0 = pr * p.C, q1 = q0 + p.C;  // the pair's units [q0, q1)
    bool whole = false;                       // one warp held all of it (and wrote y)
#pragma unroll
    for (int ww = 0; ww < kOneWarps; ++ww) whole |= (wb[ww] <= q0) & (wb[ww + 1] >= q1);
    if (whole) continue;
    const int cf = pr == pair_lo ? cta_first : int(blockIdx.x);
    const int cl = pr == pair_hi ? cta_last : int(blockIdx.x);
    float tot = 0.f;
#pragma unroll
    for (int ww = 0; ww < kOneWarps; ++ww) {
      const bool holds = (wb[ww] < q1) & (wb[ww + 1] > q0) & (wb[ww] < wb[ww + 1]);
      const uint32_t slot = parts + uint32_t(ww * 2 + (wb[ww] >= q0 ? 0 : 1)) * kPartBytes;
      float v;
      asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(slot + uint32_t(lane) * 4u));
      tot = holds ? tot + v : tot;
    }
    const int row = pr * (kDecTG * 16) + lane;
    bool mine = true;  // this lane finishes its row of the pair
    if (!(q0 >= v0 && q1 <= v1)) {
      // level 3: the pair spans CTAs cf..cl
      if (cl == cf + 1) {
        unsigned long long* word = p.xch + size_t(cf) * 32 + lane;
        unsigned long long other;
        asm volatile("atom.relaxed.gpu.global.exch.b64 %0, [%1], %2;"
                     : "=l"(other)
                     : "l"(word), "l"((1ull << 32) | __float_as_uint(tot))
                     : "memory");
        if ((other >> 32) == 0) {
          mine = false;  // the other CTA finishes this row
        } else {
          *word = 0ull;  // ready for the next launch on this workspace
          tot += __uint_as_float(unsigned(other));
        }
      } else {
        const int sf = dec_slot_floats(1);
        p.slots[size_t(blockIdx.x * 2 + (v0 >= q0 ? 0 : 1)) * sf + lane] = tot;
        __syncwarp();
        unsigned old = 0;
        if (lane == 0)
          asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(p.counters + cf) : "memory");
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old != unsigned(cl - cf)) {
          mine = false;  // another CTA finishes this pair
        } else {
          __syncwarp();  // the other lanes' loads come after lane 0's acquire
          tot = 0.f;
          for (int c0 = cf; c0 <= cl; c0 += 4) {
            float v[4];
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
              const int cc = c0 + rr;
              v[rr] = cc <= cl ? __ldcg(p.slots + size_t(cc * 2 + (2 * one_cta_duo(cc, p) >= q0 ? 0 : 1)) * sf + lane)
                               : 0.f;
            }
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) tot += v[rr];
          }
          if (lane == 0) p.counters[cf] = 0u;  // ready for the next launch on this workspace
        }
      }
    }
    mine = mine && row < p.N;
    if (mine) {
      const int rr = row - ep.row0;
      float sc, sx;
      if (rr < kDecSchRows)
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(sc) : "r"(ep.sch + uint32_t(rr) * 4u));
      else
        sc = __ldg(p.sch + row);
      asm volatile("ld.shared.f32 %0, [%1];" : "=f"(sx) : "r"(ep.sx));
      p.y[row] = __bfloat16_as_ushort(__float2bfloat16_rn(tot * sc * sx));
    }
    one_emit(p, pr, __popc(__ballot_sync(0xffffffffu, mine)), lane);
  }
}

template <bool FUSED>
__global__ void __launch_bounds__(kOneThreads, 1) decode_one_kernel(const DecodeParams p) {
  // The next kernel may launch now: it streams its own weights and waits for
  // this grid's completion before it touches anything this grid writes.
  pdl_launch_dependents();
  unsigned ready_arrival = 0u;
  decode_one_body<FUSED>(p, DecWaitPdl{}, ready_arrival);
  if (threadIdx.x == 0 && p.x_ready && ready_arrival == gridDim.x - 1) {  // the last CTA to see it clears it
    p.x_ready[0] = 0u;
    p.x_ready[1] = 0u;
  }
}

// ---------------------------------------------------------------------------
// A chain of one-token layers in one persistent launch (a decode step: each
// layer's input is an earlier layer's output).  Every CTA runs every layer
// with the fused body; between layers a grid barrier (all CTAs co-resident:
// cooperative launch) makes the previous layer's y visible.  A layer's
// weights, table and row scales are fetched before the barrier, since
// nothing in the chain writes them.  The barrier counter is bounded: a
// CTA that waits about a second records a timeout and goes on.
struct DecWaitChain {
  static constexpr int kLoadsAhead = 1;  // (registers: the chain keeps more state live)
  unsigned* ctr;    // arrivals: CTAs add 1 after each layer
  unsigned target;  // arrivals that mean the previous layer is complete (0: the first layer)
  unsigned* err;
  __device__ __forceinline__ void operator()() const {
    if (target == 0) {  // the first layer waits for the previous kernel
      pdl_wait();
      return;
    }
    if (threadIdx.x == 0) poll_at_least_bounded(ctr, target, err, 1u << 26);  // about a second
    __syncthreads();
  }
};

__global__ void __launch_bounds__(kOneThreads, 1)
    decode_chain_kernel(const DecodeParams* __restrict__ layers, int n_layers, unsigned* barrier) {
  pdl_launch_dependents();
#pragma unroll 1
  for (int l = 0; l < n_layers; ++l) {
    const DecodeParams p = layers[l];  // a local copy: the body keeps what it uses in registers
    unsigned ready_arrival = 0u;  // a chain has no ready word
    decode_one_body<true>(p, DecWaitChain{barrier, unsigned(l) * gridDim.x, p.err}, ready_arrival);
    __syncthreads();  // this CTA is done with layer l (its y and workspace writes issued)
    if (threadIdx.x == 0) {
      __threadfence();
      atomicAdd(barrier, 1u);
    }
  }
}

}  // namespace w4a8
