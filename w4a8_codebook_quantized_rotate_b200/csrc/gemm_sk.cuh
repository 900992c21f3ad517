// Small-batch kernel (65..256 tokens on a layer of few 128-row tiles; it
// accepts 2..256): the tensor-core GEMM of
// gemm_tc.cuh with one token tile sized to M and a stream-K split of the
// weight stream over every SM.
//
// y[m, n] = s_x[m] s_ch[n] sum_k fp16(fp16(cb[idx[n, k]]) s_rel[n, k / 16]) x_q[m, k]
//
// Between one token and a full prefill tile the layer is still bound by the
// weight stream ("Qwen3.8-27B-AEON-ULTIMATE-UNCENSORED-BF16 -- W4A8 ConvRot
// for ComfyUI" model card, "Why this exists": every token re-reads the
// weights), so what matters is that all SMs stream and that the work per
// weight does not grow with the token count.  Here:
//   * 8 expansion warps turn 128 rows x 64 k of packed indices into fp16
//     W' = fp16(fp16(cb[idx]) s_rel) and store them straight into tensor
//     memory (the MMA's A operand): the same cost per weight for any M;
//   * one thread issues tcgen05.mma kind::f16, M = 128 rows, N = NT (the
//     token count rounded up to 16), into an fp32 accumulator in TMEM;
//   * a TMA warp loads the x_q tile (NT tokens x 64 k, fp16, 128-byte
//     swizzle; rows past M read as zero) for every 64-k chunk (no
//     multicast);
//   * the work items (128-row tile, 64-k chunk) in row-tile-major order are
//     cut into one contiguous range per CTA (sizes differ by one at most).
//     A range holds one or more tile segments; a segment that covers its
//     whole tile writes y from the accumulator, the others park an fp32
//     partial tile in the workspace, and the last CTA to arrive at a tile
//     (an arrival counter owned by the tile's first CTA) adds the partials
//     in CTA order and writes y: the result does not depend on timing.
// With NT <= 128 the accumulator is double-buffered, so the MMAs of a
// CTA's next segment need not wait for the previous segment's epilogue.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "gemm_tc.cuh"

namespace w4a8 {

constexpr int kSkRows = 128;       // weight rows per tile (TMEM lanes, MMA M)
constexpr int kSkMaxTokens = 256;  // largest token tile (MMA N)
constexpr int kSkMaxStagesB = 16;  // x_q stages in shared memory (as many as fit, up to 16)
constexpr int kSkStagesA = 8;      // expanded-weight stages in TMEM (columns [256, 512))
constexpr int kSkPfItems = 16;     // items whose weights the TMA warp prefetches into L2 ahead
constexpr int kSkThreads = 320;    // warp 0 TMA, warp 1 MMA, warps 2..9 expansion + epilogue
constexpr uint32_t kSkACol = 256;  // A stages: TMEM columns [256, 384)
constexpr int kSkMaxCtas = 148;

// x_q stages of a token tile: a small tile makes each MMA short, so many
// stages are in flight to cover the L2 latency of their loads.
__host__ __device__ constexpr int sk_stages_b(int nt) {
  return (232448 - 1024 - 2 * 65536) / (nt * 128) < kSkMaxStagesB ? (232448 - 1024 - 2 * 65536) / (nt * 128)
                                                                   : kSkMaxStagesB;
}
// Dynamic shared memory: [barriers | pad to 64 KiB] [LUT 64 KiB] [B stages].
__host__ __device__ constexpr size_t sk_smem_bytes(int nt) {
  return size_t(1024) + 65536 + 65536 + size_t(sk_stages_b(nt)) * nt * 128;
}

static_assert(sk_stages_b(kSkMaxTokens) >= 3 && sk_smem_bytes(kSkMaxTokens) <= 232448 &&
                  sk_smem_bytes(16) <= 232448, "fits the 227 KB a CTA may use");

struct SkParams {
  const uint8_t* units;  // unit region of the packed layer
  const float* sch;
  const float* cb;
  const float* s_x;      // [M]
  uint16_t* y;           // [M, N] bf16
  float* part;           // [G][2][NT][128]: partial tiles (a CTA's first and last segment)
  unsigned* counters;    // [kSkMaxCtas][8]: per expansion warp, arrivals at a tile whose first CTA is c
  unsigned* err;
  int M, N, K, C, RT, NT;
  int G, Iq, Ir;         // items RT * C over G CTAs: CTA c holds [c Iq + min(c, Ir), ...)
  uint32_t idesc;
};

// One barrier pair per stage (an x_q tile in shared memory and a weight slot
// in TMEM): `full` counts the TMA thread's transfer and the 128 expansion
// threads of the group that filled the slot, `empty` is the MMA thread's
// commit.  The MMA thread waits once and commits once per item (two waits
// and two commits per item cost the prefill kernel ~10 %).
struct SkShared {
  uint64_t full[kSkStagesA];
  uint64_t empty[kSkStagesA];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort;
};

__device__ __forceinline__ int sk_cta_item(int c, const SkParams& p) { return c * p.Iq + min(c, p.Ir); }
// The CTA whose range holds item i.
__device__ __forceinline__ int sk_item_cta(int i, const SkParams& p) {
  const int big = p.Ir * (p.Iq + 1);
  return i < big ? i / (p.Iq + 1) : p.Ir + (i - big) / p.Iq;
}

// Bounded wait (about a second), giving up once another role has aborted.
__device__ __forceinline__ bool sk_wait(uint64_t* bar, uint32_t parity, SkShared* sh, unsigned* err) {
  for (uint32_t i = 0; i < (1u << 20); ++i) {
#if W4A8_SPIN_WAIT
    if (mbar_test_wait(bar, parity)) return true;
#else
    if (mbar_try_wait(bar, parity)) return true;
#endif
    if ((i & 1023u) == 1023u && sh->abort) return false;
  }
  sh->abort = 1;
  record_error(err, kErrTimeout);
  return false;
}

// 32 lanes x 8 columns of 32-bit cells.
__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}

__device__ __forceinline__ void sk_exp_load(ExpStage& e, const SkParams& p, int tile, int kb, int g, bool valid) {
  if (valid) {
    const uint8_t* src = p.units + tile_idx_offset(tile, kb, p.C) + size_t(4 * g) * 16;
#pragma unroll
    for (int t = 0; t < 4; ++t) e.seg[t] = __ldg(reinterpret_cast<const uint4*>(src) + t);
    e.sr = __ldg(reinterpret_cast<const uint2*>(p.units + tile_srel_offset(tile, kb, p.C) + g * 8));
  } else {
#pragma unroll
    for (int t = 0; t < 4; ++t) e.seg[t] = make_uint4(0, 0, 0, 0);
    e.sr = make_uint2(0, 0);
  }
}

__global__ void __launch_bounds__(kSkThreads, 1)
    gemm_sk_kernel(const __grid_constant__ CUtensorMap tmap_x, const SkParams p) {
  extern __shared__ __align__(1024) uint8_t sk_smem[];
  pdl_launch_dependents();
  SkShared* sh = reinterpret_cast<SkShared*>(sk_smem);
  const uint32_t base = smem_u32(sk_smem);
  const uint32_t lut = (base + uint32_t(sizeof(SkShared)) + 0xFFFFu) & ~0xFFFFu;
  const uint32_t bstage0 = lut + 65536u;  // 1024-byte aligned
  const uint32_t stage_b = uint32_t(p.NT) * 128u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i0 = sk_cta_item(min(int(blockIdx.x), p.G), p);
  const int i1 = sk_cta_item(min(int(blockIdx.x) + 1, p.G), p);
  const int n_items = i1 - i0;
  const bool dbl = p.NT <= 128;  // two accumulators fit beside the A stages
  // stages: as many x_q tiles as fit in shared memory, at most the 8 TMEM weight slots
  const int SB = sk_stages_b(p.NT) < kSkStagesA ? sk_stages_b(p.NT) : kSkStagesA;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SB; ++s) {
      mbar_init(&sh->full[s], 129);  // the TMA thread + 128 expansion threads
      mbar_init(&sh->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->acc_full[b], 1);
      mbar_init(&sh->acc_empty[b], 256);
    }
    mbar_init(&sh->drain, 1);
    sh->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
  }
  {  // Table: entry b for lane l at lut + 256 b + 4 l holds fp16 (cb[b & 15], cb[b >> 4]).
    const float level = p.cb[lane & 15];
    for (int b = warp; b < 256; b += kSkThreads / 32) {
      const float lo = __shfl_sync(0xffffffffu, level, b & 15);
      const float hi = __shfl_sync(0xffffffffu, level, b >> 4);
      const __half2 h = __floats2half2_rn(lo, hi);
      asm volatile("st.shared.b32 [%0], %1;" ::"r"(lut + (uint32_t(b) << 8) + uint32_t(lane) * 4u),
                   "r"(*reinterpret_cast<const uint32_t*>(&h)));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer: x_q tiles, one per item
    if (lane == 0 && n_items > 0) {
      // The weights of an item are 4 units (the row tile's 4 pairs, one
      // chunk), 1152 bytes each: prefetch them into L2 kSkPfItems items
      // ahead of the expansion warps (weights do not depend on the previous
      // kernel, so the first ones go out before the wait).
      auto prefetch_item = [&](int it) {
        const int rt = it / p.C, kb = it - rt * p.C;
        const int npairs = (p.N + 31) / 32;
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2) {
          const int pr = rt * 4 + q2;
          if (pr < npairs)
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.units + unit_offset(pr, kb, p.C)),
                         "n"(kUnitBytes)
                         : "memory");
        }
      };
      for (int it = i0; it < min(i1, i0 + kSkPfItems); ++it) prefetch_item(it);
      tma_prefetch_desc(&tmap_x);
      pdl_wait();  // x_q and s_x are written by the previous kernel
      int kb = i0 % p.C, issued = 0;
      for (int j = 0; j < n_items; ++j) {
        const int s = j % SB;
        if (!sk_wait(&sh->empty[s], ((j / SB) & 1) ^ 1, sh, p.err)) break;
        mbar_arrive_expect_tx(&sh->full[s], stage_b);
        tma_load_2d(bstage0 + uint32_t(s) * stage_b, &tmap_x, &sh->full[s], kb * kTcBK, 0);
        ++issued;
        if (++kb == p.C) kb = 0;
        if (j + kSkPfItems < n_items) prefetch_item(i0 + j + kSkPfItems);
      }
      if (sh->abort && issued > 0) {
        // The stage barriers also count the expansion threads, which may have
        // stopped: let the copies in flight land by waiting a fixed, bounded
        // time (a tile lands in microseconds) before the CTA exits.
        unsigned long long t0, t1;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
        do {
          asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
        } while (t1 - t0 < 50000ull);  // 50 us
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0 && n_items > 0) {
      bool ok = true;
      int kb = i0 % p.C, seg = 0;
      for (int j = 0; j < n_items && ok; ++j) {
        const int sa = j % SB;
        const int buf = dbl ? (seg & 1) : 0;
        const int use = dbl ? (seg >> 1) : seg;  // earlier segments on this buffer
        if (j == 0 || kb == 0) {  // a segment starts: its accumulator must be drained
          ok = use == 0 || sk_wait(&sh->acc_empty[buf], (use - 1) & 1, sh, p.err);
          if (!ok) break;
        }
        ok = sk_wait(&sh->full[sa], (j / SB) & 1, sh, p.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem + uint32_t(buf) * uint32_t(p.NT);
#pragma unroll
        for (int s = 0; s < kTcBK / 16; ++s) {
          const uint32_t a = tmem + kSkACol + uint32_t(sa) * 32u + uint32_t(s) * 8u;
          const uint64_t bd = sw128_desc(bstage0 + uint32_t(sa) * stage_b + uint32_t(s) * 32u);
          tc_mma_ts_f16(acc, a, bd, p.idesc, ((j == 0 || kb == 0) && s == 0) ? 0u : 1u);
        }
        tc_commit(&sh->empty[sa]);
        if (++kb == p.C || j == n_items - 1) {  // the segment ends
          tc_commit(&sh->acc_full[buf]);
          kb = kb == p.C ? 0 : kb;
          ++seg;
        }
      }
      if (!ok) {  // wait for the MMAs already issued before the TMEM is freed
        tc_commit(&sh->drain);
        mbar_wait_bounded(&sh->drain, 0, p.err, 1u << 20);
      }
    }
  } else {
    // ------------------------------------------------ expansion, then each segment's epilogue
    // Group G (4 warps, all 128 rows) expands the items j = G, G + 2, ... of
    // the range; both groups meet at every segment's epilogue, each taking
    // half of the token columns.
    const int grp = (warp - 2) >> 2;
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = 32 * q + lane;
    const uint32_t lut_lane = lut + uint32_t(lane) * 4u;
    const uint32_t trow = uint32_t(32 * q) << 16;
    const int half = p.NT >> 1;
    const int col0 = grp * half;
    bool ok = true;
    int seg = 0;
    // item j of the range: tile jt, chunk jk
    int jt = (i0 + grp) / p.C, jk = (i0 + grp) - ((i0 + grp) / p.C) * p.C;
    int seg_tile = i0 / p.C, seg_k0 = i0 - seg_tile * p.C;  // the segment being accumulated
    auto row_of = [&](int tile) { return tile * kSkRows + r; };
    constexpr int PF = 4;
    ExpStage es[PF];
    {
      int t = jt, k = jk;
#pragma unroll
      for (int i = 0; i < PF; ++i) {
        const int jj = grp + 2 * i;
        const int n = row_of(t);
        sk_exp_load(es[i], p, n >> 4, k, n & 7, jj < n_items && n < p.N);
        k += 2;
        if (k >= p.C) { k -= p.C; ++t; }
      }
    }
    // The epilogue of the segment (tile seg_tile, chunks [seg_k0, last_k]):
    // each warp takes its 32 rows x its group's half of the token columns.
    // A whole tile goes to y; a partial one goes to the CTA's slot (0: its
    // first segment, 1: its last), and the warp counts in at the tile's
    // first CTA; the last of the tile's CTAs to arrive adds the slots in CTA
    // order and writes y.  No cross-warp barrier: a warp that gives up on a
    // wait cannot leave another warp waiting on it.
    const int wid = warp - 2;  // (group, quarter): the counter and the share of the tile
    auto epilogue = [&](int last_k) -> bool {
      const int buf = dbl ? (seg & 1) : 0;
      const int use = dbl ? (seg >> 1) : seg;
      int w_ok = (ok && lane == 0) ? int(sk_wait(&sh->acc_full[buf], use & 1, sh, p.err)) : 0;
      if (__shfl_sync(0xffffffffu, w_ok, 0) == 0) return false;
      tc_fence_after();
      pdl_wait();  // s_x comes from the previous kernel
      const int n = row_of(seg_tile);
      const bool valid = n < p.N;
      const bool whole = seg_k0 == 0 && last_k == p.C - 1;
      const int slot = int(blockIdx.x) * 2 + (i0 >= seg_tile * p.C ? 0 : 1);
      const float sch = valid ? p.sch[n] : 0.f;
      const uint32_t acc = tmem + trow + uint32_t(buf) * uint32_t(p.NT);
      for (int c0 = col0; c0 < col0 + half; c0 += 8) {
        uint32_t v[8];
        tmem_ld_32x32b_x8(acc + uint32_t(c0), v);
        tc_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int m = c0 + jj;
          if (m < p.M) {
            if (whole) {
              if (valid)
                p.y[size_t(m) * p.N + n] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[jj]) * sch * p.s_x[m]));
            } else {
              p.part[(size_t(slot) * p.NT + m) * kSkRows + r] = __uint_as_float(v[jj]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sh->acc_empty[buf]);  // this thread is done with the accumulator
      ++seg;
      if (whole) return true;
      const int first = sk_item_cta(seg_tile * p.C, p);
      const int last = sk_item_cta(seg_tile * p.C + p.C - 1, p);
      unsigned* cnt = p.counters + first * 8 + wid;
      __threadfence();
      __syncwarp();
      unsigned old = 0;
      if (lane == 0) old = atomicAdd(cnt, 1u);
      old = __shfl_sync(0xffffffffu, old, 0);
      if (old != unsigned(last - first)) return true;  // another CTA finishes this share
      __threadfence();
      // Sum the CTAs' partials in CTA order.  Loads go out 8 tokens x 4 CTAs
      // at a time (a token-by-token loop waits one L2 round trip per token:
      // measured 28-50 us of a 105-129 us call).
      const int m_end = min(col0 + half, p.M);
      for (int mc = col0; mc < m_end; mc += 8) {
        float tot[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) tot[jj] = 0.f;
        for (int c0 = first; c0 <= last; c0 += 4) {
          float v[4][8];
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int cc = c0 + qq;
            const bool have = cc <= last;
            const int sl = have ? cc * 2 + (sk_cta_item(cc, p) >= seg_tile * p.C ? 0 : 1) : 0;
            const float* src = p.part + (size_t(sl) * p.NT + mc) * kSkRows + r;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) v[qq][jj] = (have && mc + jj < m_end) ? __ldcg(src + jj * kSkRows) : 0.f;
          }
#pragma unroll
          for (int qq = 0; qq < 4; ++qq)
            if (c0 + qq <= last) {  // only the CTAs that exist: the same additions as one at a time
#pragma unroll
              for (int jj = 0; jj < 8; ++jj) tot[jj] += v[qq][jj];
            }
        }
        if (valid) {
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int m = mc + jj;
            if (m < m_end)
              p.y[size_t(m) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(tot[jj] * sch * p.s_x[m]));
          }
        }
      }
      __syncwarp();
      if (lane == 0) *cnt = 0u;  // ready for the next launch on this workspace
      return true;
    };
    // One item of this group (stage I of the load ring); false once the
    // range (and its last epilogue) is done or a wait gave up.
    auto step = [&](auto I, int jj) -> bool {
      constexpr int i = decltype(I)::value;
      // segments that end before this item (or at the range's end) get their epilogue first
      const int item = i0 + min(jj, n_items);
      while (ok && seg_tile * p.C + p.C <= item && seg_tile * p.C + seg_k0 < i1) {
        ok = epilogue(p.C - 1);
        ++seg_tile;
        seg_k0 = 0;
      }
      if (jj >= n_items) {
        if (ok && seg_tile * p.C + seg_k0 < i1) ok = epilogue((i1 - 1) - seg_tile * p.C);
        return false;
      }
      if (!ok) return false;
      const int sa = jj % SB;
      uint32_t v[32];
      const int n = row_of(jt);
      exp_compute(es[i], lut_lane, (n >> 3) & 1, v);
      if (n >= p.N) {
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = 0u;
      }
      {  // refill this stage with the group's item jj + 2 PF
        int t = jt, k = jk + 2 * PF;
        while (k >= p.C) { k -= p.C; ++t; }
        const int nn = row_of(t);
        sk_exp_load(es[i], p, nn >> 4, k, nn & 7, jj + 2 * PF < n_items && nn < p.N);
      }
      int w_ok = lane == 0 ? int(sk_wait(&sh->empty[sa], ((jj / SB) & 1) ^ 1, sh, p.err)) : 0;
      ok = __shfl_sync(0xffffffffu, w_ok, 0) != 0;
      if (!ok) return false;
      tc_fence_after();
      tmem_st_32x32b_x32(tmem + trow + kSkACol + uint32_t(sa) * 32u, v);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&sh->full[sa]);
      jk += 2;
      if (jk >= p.C) { jk -= p.C; ++jt; }
      return true;
    };
    static_assert(PF == 4, "the item loop is unrolled for 4 load stages");
    for (int jb = grp;; jb += 2 * PF) {
      if (!step(std::integral_constant<int, 0>{}, jb)) break;
      if (!step(std::integral_constant<int, 1>{}, jb + 2)) break;
      if (!step(std::integral_constant<int, 2>{}, jb + 4)) break;
      if (!step(std::integral_constant<int, 3>{}, jb + 6)) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace w4a8
