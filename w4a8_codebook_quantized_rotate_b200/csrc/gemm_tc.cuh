// Prefill kernel (M > 64; on a layer of few 128-row tiles, M > 256):
// tensor-core GEMM on tcgen05 with the codebook
// expansion fused into the operand path.
//
// The product is computed transposed, D^T[n, m] = sum_k W'[n, k] x_q[m, k],
// so that the expanded weight is the MMA's A operand, which tcgen05 can read
// from tensor memory:
//   * 4 expansion warps turn a 128-row x 64-k block of packed indices into
//     fp16 W' = fp16(fp16(cb[idx]) * s_rel) and store it straight into TMEM
//     with tcgen05.st -- the expansion never touches shared-memory
//     bandwidth, which the B operand and the TMA engine need;
//   * a TMA warp loads x_q (fp16, integer-valued, exact) tiles of 256 tokens
//     x 64 k into 128-byte-swizzled shared memory (no multicast);
//   * one thread issues tcgen05.mma kind::f16 (M = 128 weight rows, N = 256
//     tokens, K = 16) into an fp32 accumulator in TMEM;
//   * the expansion warps then read the accumulator back (tcgen05.ld), scale
//     by s_ch[n] s_x[m] in fp32 and store y in bf16.
// "Qwen3.8-27B-AEON-ULTIMATE-UNCENSORED-BF16 -- W4A8 ConvRot for ComfyUI"
// model card, "Why this exists" and "Format": the layer runs a tensor-core
// GEMM with a codebook dequantisation step on top.  The pages' int8 operand
// cannot hold the three-tier weight within the output tolerance, so the
// operand here is fp16 (the accumulation is fp32 either way).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace w4a8 {

constexpr int kTcRows = 128;      // weight rows per tile (TMEM lanes, MMA M)
constexpr int kTcTokens = 256;    // tokens per tile (MMA N)
constexpr int kTcBK = 64;         // k per pipeline stage
// Pipeline stages: an x_q tile in shared memory + an expanded-weight tile in
// TMEM.  Three lie above the table; a fourth goes in the table's alignment
// room when that room holds it (it does for a kernel without static shared
// memory; the kernel checks), so 128 KB of activation tiles are in flight.
constexpr int kTcStages = 4;
constexpr int kTcStagesHigh = 3;
constexpr int kTcThreads = 320;   // warp 0 TMA, warp 1 MMA, warps 2..9 expansion + epilogue (2 groups)
constexpr uint32_t kTcStageBBytes = kTcTokens * kTcBK * 2;  // 32 KiB
constexpr uint32_t kTcTmemCols = 512;
constexpr uint32_t kTcAccCol = 0;     // accumulator: columns [0, 256)
constexpr uint32_t kTcACol = 256;     // A stages: columns [256, 384)
// dynamic shared memory: [barriers | pad to the next 64 KiB boundary] [LUT 64 KiB] [B stages]
constexpr size_t kTcSmemBytes = 1024 + 65536 + 65536 + size_t(kTcStagesHigh) * kTcStageBBytes;

struct TcParams {
  const uint8_t* units;   // unit region of the packed layer
  const float* sch;
  const float* cb;
  const float* s_x;
  uint16_t* y;
  unsigned* err;
  int M, N, K, C, T;
};

// One barrier pair per stage: `full` completes when the stage's x_q tile has
// landed (the TMA thread's arrive with the transfer bytes) and its weight
// tile is in TMEM (128 expansion threads' arrivals); `empty` when the MMAs
// that read both have completed.  The MMA thread then waits once and
// commits once per 64-k block: its per-block work is what bounds the
// pipeline (measured: two waits and two commits per block held the tensor
// pipe at 45 %).
struct TcShared {
  uint64_t full[kTcStages];
  uint64_t empty[kTcStages];
  uint64_t acc_full;
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort;
};

// Instruction descriptor, kind::f16: fp16 A and B, fp32 D, both K-major,
// M = 128 (bits 24..28 hold M >> 4), N = 256 (bits 17..22 hold N >> 3).
constexpr uint32_t kTcIdesc = (1u << 4) | (uint32_t(kTcTokens >> 3) << 17) | (uint32_t(kTcRows >> 4) << 24);

// Shared-memory descriptor of a K-major tile with 128-byte swizzling: rows
// of 128 bytes, 8-row groups 1024 bytes apart (SBO), LBO unused (1), format
// version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  return uint64_t((smem_addr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Bounded wait that also gives up once another role has aborted.  About a
// million polls, each of which may suspend the thread briefly: on the order
// of a second before the kernel records a timeout and unwinds.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, TcShared* sh, unsigned* err) {
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

struct ExpStage {
  uint4 seg[4];  // the four 16-byte lane segments holding this row's index bytes
  uint2 sr;      // group-scale bytes of rows (g, g+8) for the chunk's 4 groups
};

__device__ __forceinline__ void exp_load(ExpStage& e, const TcParams& p, int tile, int kb, int g, bool valid) {
  if (valid && kb < p.C) {
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

// Expand one row's 64 k of one chunk into 32 fp16 pairs (TMEM column
// 8 s + b holds k = 16 s + 2 b, 2 b + 1 of the chunk).
__device__ __forceinline__ void exp_compute(const ExpStage& e, uint32_t lut_lane, int h, uint32_t (&out)[32]) {
  const uint32_t sel_lo = 0x7604u | (uint32_t(h) << 4);        // byte h of a word: (row, b = t)
  const uint32_t sel_hi = 0x7604u | (uint32_t(h + 2) << 4);    // byte h+2: (row, b = t + 4)
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const uint32_t codes = (s < 2 ? e.sr.x : e.sr.y) >> (16 * (s & 1) + 8 * h);
    __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)(codes & 0xFFu), __NV_E4M3);
    const __half sh = *reinterpret_cast<__half*>(&hr);
    const __half2 sc = __halves2half2(sh, sh);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t word = s == 0 ? e.seg[t].x : s == 1 ? e.seg[t].y : s == 2 ? e.seg[t].z : e.seg[t].w;
      uint32_t lo = lds_u32(prmt(word, lut_lane, sel_lo));
      uint32_t hi = lds_u32(prmt(word, lut_lane, sel_hi));
      __half2 vlo = __hmul2(*reinterpret_cast<__half2*>(&lo), sc);
      __half2 vhi = __hmul2(*reinterpret_cast<__half2*>(&hi), sc);
      out[8 * s + t] = *reinterpret_cast<uint32_t*>(&vlo);
      out[8 * s + t + 4] = *reinterpret_cast<uint32_t*>(&vhi);
    }
  }
}

__global__ void __launch_bounds__(kTcThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const TcParams p) {
  extern __shared__ __align__(1024) uint8_t tc_smem[];
  pdl_launch_dependents();
  TcShared* sh = reinterpret_cast<TcShared*>(tc_smem);
  const uint32_t base = smem_u32(tc_smem);
  // 64 KiB aligned (bits 8..15 zero), past the barrier block
  const uint32_t lut = (base + uint32_t(sizeof(TcShared)) + 0xFFFFu) & ~0xFFFFu;
  const uint32_t bstage0 = lut + 65536u;  // 1024-byte aligned
  // stage 3 in the room below the table, if it fits there
  const uint32_t low_stage = (base + uint32_t(sizeof(TcShared)) + 1023u) & ~1023u;
  const int S = low_stage + kTcStageBBytes <= lut ? kTcStages : kTcStagesHigh;
  auto bstage = [&](int st) { return st < kTcStagesHigh ? bstage0 + uint32_t(st) * kTcStageBBytes : low_stage; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kTcRows;
  const int m0 = blockIdx.y * kTcTokens;
  const int KB = p.C;  // k blocks of 64

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&sh->full[s], 129);  // 128 expansion threads + the TMA thread
      mbar_init(&sh->empty[s], 1);
    }
    mbar_init(&sh->acc_full, 1);
    mbar_init(&sh->drain, 1);
    sh->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, kTcTmemCols);
    tmem_relinquish();
  }
  // Table: entry b for lane l at lut + 256 b + 4 l holds fp16 (cb[b & 15], cb[b >> 4]).
  // Each lane reads one level once; the pairs come from shuffles.
  {
    const float level = p.cb[lane & 15];
    for (int b = warp; b < 256; b += kTcThreads / 32) {
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
    // ------------------------------------------------ TMA producer: x_q tiles
    if (lane == 0) {
      tma_prefetch_desc(&tmap_x);
      pdl_wait();  // x_q and s_x are written by the previous kernel
      int issued = 0, s = 0;
      uint32_t phase = 0;
      for (int kb = 0; kb < KB; ++kb) {
        if (!tc_wait(&sh->empty[s], phase ^ 1u, sh, p.err)) break;
        mbar_arrive_expect_tx(&sh->full[s], kTcStageBBytes);
        tma_load_2d(bstage(s), &tmap_x, &sh->full[s], kb * kTcBK, m0);
        ++issued;
        if (++s == S) {
          s = 0;
          phase ^= 1u;
        }
      }
      if (sh->abort && issued > 0) {
        // The stage barriers also count the expansion threads, which may have
        // stopped: let the copies in flight land by waiting a fixed, bounded
        // time (a 32 KB tile lands in microseconds) before the CTA exits.
        unsigned long long t0, t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
        do {
          asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        } while (t - t0 < 50000ull);  // 50 us
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      // descriptor of stage 0's first k16 step; a stage adds kTcStageBBytes and a
      // k16 step 32 bytes to the address field (in 16-byte units; no carry:
      // the stages lie below 256 KiB)
      const uint64_t bd_first = sw128_desc(bstage0), bd_low = sw128_desc(low_stage);
      int s = 0;
      uint32_t phase = 0;
      for (int kb = 0; kb < KB && ok; ++kb) {
        ok = tc_wait(&sh->full[s], phase, sh, p.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a0 = tmem + kTcACol + uint32_t(s) * 32u;
#pragma unroll
        for (int j = 0; j < kTcBK / 16; ++j)
          tc_mma_ts_f16(tmem + kTcAccCol, a0 + uint32_t(j) * 8u,
                        (s < kTcStagesHigh ? bd_first + uint64_t(s) * (kTcStageBBytes >> 4) : bd_low) + uint64_t(2 * j),
                        kTcIdesc,
                        (kb | j) != 0 ? 1u : 0u);
        tc_commit(&sh->empty[s]);
        if (++s == S) {
          s = 0;
          phase ^= 1u;
        }
      }
      if (ok) {
        tc_commit(&sh->acc_full);
      } else {  // wait for the MMAs already issued before the TMEM is freed
        tc_commit(&sh->drain);
        mbar_wait_bounded(&sh->drain, 0, p.err, 1u << 20);
      }
    }
  } else {
    // ------------------------------------------------ expansion, then epilogue
    // Two groups of 4 warps: group G expands the k blocks kb = G, G+2, ...
    // (each group covers all 128 rows), which doubles the time each warp has
    // per block; the epilogue splits the 256 accumulator columns between them.
    const int grp = (warp - 2) >> 2;
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = 32 * q + lane;
    const int n = n0 + r;
    const bool valid = n < p.N;
    const int tile = n >> 4, g = n & 7, h = (n >> 3) & 1;
    const uint32_t lut_lane = lut + uint32_t(lane) * 4u;
    const uint32_t trow = uint32_t(32 * q) << 16;
    constexpr int PF = 4;
    ExpStage es[PF];
#pragma unroll
    for (int i = 0; i < PF; ++i) exp_load(es[i], p, tile, grp + 2 * i, g, valid);
    bool ok = true;
    for (int kb0 = grp; kb0 < KB && ok; kb0 += 2 * PF) {
#pragma unroll
      for (int i = 0; i < PF; ++i) {
        const int kb = kb0 + 2 * i;
        if (kb < KB && ok) {
          const int sa = kb % S;
          uint32_t v[32];
          exp_compute(es[i], lut_lane, h, v);
          if (!valid) {
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c] = 0u;
          }
          exp_load(es[i], p, tile, kb + 2 * PF, g, valid);
          // lane 0 polls; the outcome is made warp-uniform before the
          // .sync.aligned TMEM store
          int w_ok = lane == 0 ? int(tc_wait(&sh->empty[sa], ((kb / S) & 1) ^ 1, sh, p.err)) : 0;
          ok = __shfl_sync(0xffffffffu, w_ok, 0) != 0;
          if (ok) {
            tc_fence_after();
            tmem_st_32x32b_x32(tmem + trow + kTcACol + uint32_t(sa) * 32u, v);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&sh->full[sa]);
          }
        }
      }
    }
    int acc_ok = (ok && lane == 0) ? int(tc_wait(&sh->acc_full, 0, sh, p.err)) : 0;
    if (__shfl_sync(0xffffffffu, acc_ok, 0) != 0) {
      tc_fence_after();
      pdl_wait();  // s_x comes from the previous kernel
      const float sch = valid ? p.sch[n] : 0.f;
      // every stage is free once the accumulator is complete: stage 0 holds each warp's 32 x 32 bf16 block
      const uint32_t tbuf = bstage0 + uint32_t(warp - 2) * 2048u;
#pragma unroll 1
      for (int ci = grp * (kTcTokens / 64); ci < (grp + 1) * (kTcTokens / 64) && m0 + 32 * ci < p.M; ++ci) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + trow + kTcAccCol + uint32_t(ci) * 32u, v);
        tc_wait_ld();
        const int mc = m0 + 32 * ci;
        store_block_transposed(p.y, p.M, p.N, mc, n0 + 32 * q, tbuf, lane, [&](int j) {
          const float sx = mc + j < p.M ? p.s_x[mc + j] : 0.f;
          return __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j]) * sch * sx));
        });
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTcTmemCols);
}

}  // namespace w4a8
