// NVFP4 comparison layer: 4-bit weights AND 4-bit activations on the
// block-scaled FP4 tensor cores (tcgen05.mma kind::mxf4nvf4), as the speed
// and accuracy foil of the codebook layer.
//
// Format ("Qwen3.8-27B-Uncensored-NVFP4: En runbook för servering på
// Blackwell-GPU:er", section "Vad NVFP4 är, och hur det skiljer sig från FP8
// och från INT8/AWQ"): E2M1 values (1 sign, 2 exponent, 1 mantissa bit),
// one e4m3 scale per 16 values, one fp32 scalar per tensor.  Readings where
// the page is silent: bias-1 E2M1 (0, 0.5, 1, 1.5, 2, 3, 4, 6), round to
// nearest even with saturation, g = amax / (6 * 448), weights one g per
// tensor and activations one g per token, both operands in the codebook
// layer's rotated basis (256-blocks times H_256 / 16).  Decisions in fp32:
//   d = g * 6,  s = e4m3(bmax / d),  S = e4m3val(s) * g,  code = e2m1(x / S).
//
// Layouts:
//   codes   [R][K/2] bytes, two codes per byte, even k in the low nibble
//           (the tensor core's packed FP4 order).
//   scales  the tensor core's order, rows padded to 128: chunks of 128 rows x
//           64 k (512 bytes) in [row block][k64 step] order; inside a chunk
//           the scale of (row r, 16-block c) is byte 16 (r % 32) +
//           4 ((r % 128) / 32) + c % 4.  A chunk's 16-byte row i is the
//           content of TMEM lane i (of every lane quarter) over four columns
//           (row r -> lane r % 32, column (r % 128) / 32, byte c % 4), the
//           layout the block-scaled MMA reads for M = 128 and scale_vec::4X.
//   g       [R] fp32.
//
// GEMM: D^T[n, m] = sum_k W[n, k] x[m, k] with the weights as the MMA's A
// operand (M = 128 rows, the TMEM lanes) and NT tokens as B; a stage is
// 256 k: 128 bytes of codes per row by TMA (128-byte swizzle, no multicast),
// the scale chunks by plain bulk copies, moved into per-stage TMEM columns by
// the four epilogue warps (tcgen05.st, each warp its lane quarter; with
// tcgen05.cp issued by the MMA thread, 8 copies per stage held the tensor pipe
// near a third busy), so the MMA thread waits once and issues its four
// K = 64 MMAs per stage.  The epilogue scales by g_w[n] g_x[m] and stores
// bf16.
#pragma once

#include <cuda.h>
#include <cuda_fp4.h>

#include "act.cuh"
#include "common.cuh"

namespace w4a8 {

constexpr int kNvBlock = 16;          // values per e4m3 scale
constexpr int kNvSfChunk = 512;       // scale bytes of 128 rows x 64 k
constexpr int kNvRows = 128;          // weight rows per tile (MMA M)
constexpr int kNvBK = 256;            // k per pipeline stage
constexpr int kNvThreads = 192;       // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kNvQuantThreads = 256;  // quantiser: 8 warps per row
constexpr float kNvGDiv = 2688.0f;    // 6 * 448
constexpr uint32_t kNvTmemCols = 512;
constexpr size_t kNvMaxSmem = 232448;

__host__ __device__ inline size_t nv_sf_offset(int64_t r, int64_t c, int64_t K) {
  const int64_t steps = K / 64;
  return size_t((r >> 7) * steps + (c >> 2)) * kNvSfChunk + size_t((r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3));
}
__host__ __device__ inline size_t nv_sf_bytes(int64_t R, int64_t K) {
  return size_t((R + 127) / 128) * 128 * size_t(K / kNvBlock);
}

// ------------------------------------------------------------------ quantiser

struct NvQuantParams {
  const void* x;               // [R][K] bf16 or fp32
  const unsigned* amax_word;   // the tensor's |max| as float bits (one g per tensor), or null (one g per row)
  uint8_t* codes;              // [R][K/2]
  uint8_t* sf;                 // tensor-core order, nv_sf_bytes(R, K)
  float* g;                    // [R]
  int R, K, in_f32, rotate;
};

// Lane's 8 consecutive values (positions 256 b + 8 lane ..) of row r, rotated if asked.
__device__ __forceinline__ void nv_load_lane(const NvQuantParams& p, int64_t r, int b, int lane, float (&v)[8]) {
  const int64_t off = r * p.K + int64_t(b) * kRotBlock + lane * 8;
  if (p.in_f32) {
    const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(p.x) + off);
    const float4 a = __ldg(src), c = __ldg(src + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
  } else {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) + off));
    const uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(wds[i] << 16);
      v[2 * i + 1] = __uint_as_float(wds[i] & 0xFFFF0000u);
    }
  }
  if (p.rotate) rotate_vals_lane(v, lane);
}

__device__ __forceinline__ float nv_warp_max(float m) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

// The tensor's |max| over all rows (rotated if asked), for one g per tensor.
// A grid-stride loop over rows; one atomic per CTA (atomics on one word
// serialise: one per warp and row took 130 us for 17408 rows).  *amax_out
// must start at 0.
__global__ void __launch_bounds__(kNvQuantThreads) nvfp4_amax_kernel(const NvQuantParams p, unsigned* amax_out) {
  __shared__ float red[kNvQuantThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float m = 0.f;
  for (int64_t r = blockIdx.x; r < p.R; r += gridDim.x) {
    for (int b = warp; b < p.K / kRotBlock; b += kNvQuantThreads / 32) {
      float v[8];
      nv_load_lane(p, r, b, lane, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
    }
  }
  m = nv_warp_max(m);
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 1; w < kNvQuantThreads / 32; ++w) m = fmaxf(m, red[w]);
    atomicMax(amax_out, __float_as_uint(m));  // non-negative floats order as their bits
  }
}

// One CTA per row of the padded row count (rows >= R write zero scales).
// The rotated row is staged in shared memory until its maximum is known.
__global__ void __launch_bounds__(kNvQuantThreads) nvfp4_quant_kernel(const NvQuantParams p) {
  extern __shared__ float nv_row[];
  __shared__ float red[kNvQuantThreads / 32];
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r = blockIdx.x;
  pdl_wait();  // x may come from the previous kernel; the scale buffers may still be read by it
  if (r >= p.R) {
    for (int c = threadIdx.x; c < p.K / kNvBlock; c += kNvQuantThreads) p.sf[nv_sf_offset(r, c, p.K)] = 0;
    return;
  }
  float m = 0.f;
  for (int b = warp; b < p.K / kRotBlock; b += kNvQuantThreads / 32) {
    float v[8];
    nv_load_lane(p, r, b, lane, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
    float4* dst = reinterpret_cast<float4*>(nv_row + b * kRotBlock + lane * 8);
    dst[0] = make_float4(v[0], v[1], v[2], v[3]);
    dst[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
  m = nv_warp_max(m);
  if (lane == 0) red[warp] = m;
  __syncthreads();
  float amax;
  if (p.amax_word) {
    amax = __uint_as_float(*p.amax_word);
  } else {
    amax = red[0];
#pragma unroll
    for (int w = 1; w < kNvQuantThreads / 32; ++w) amax = fmaxf(amax, red[w]);
  }
  const float g = __fdiv_rn(amax, kNvGDiv);
  const float d = __fmul_rn(g, 6.0f);
  if (threadIdx.x == 0) p.g[r] = g;
  uint32_t* codes = reinterpret_cast<uint32_t*>(p.codes + r * (p.K / 2));
  // a thread takes 8 consecutive values, half a 16-block; lanes 2i and 2i+1
  // share a block (K / 8 is a multiple of 32, so whole warps iterate)
  for (int j = threadIdx.x; j < p.K / 8; j += kNvQuantThreads) {
    const float4 a = reinterpret_cast<const float4*>(nv_row)[2 * j];
    const float4 c = reinterpret_cast<const float4*>(nv_row)[2 * j + 1];
    const float v[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
    float bm = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) bm = fmaxf(bm, fabsf(v[i]));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
    uint32_t s = 0;
    float S = 0.f;
    if (d > 0.f) {
      s = __nv_cvt_float_to_fp8(__fdiv_rn(bm, d), __NV_SATFINITE, __NV_E4M3);
      S = __fmul_rn(e4m3_to_float(s), g);
    }
    uint32_t word = 0;
    if (S > 0.f) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 q = make_float2(__fdiv_rn(v[2 * i], S), __fdiv_rn(v[2 * i + 1], S));
        word |= uint32_t(__nv_cvt_float2_to_fp4x2(q, __NV_E2M1, cudaRoundNearest)) << (8 * i);
      }
    }
    codes[j] = word;
    if ((lane & 1) == 0) p.sf[nv_sf_offset(r, j >> 1, p.K)] = uint8_t(s);
  }
}

// Row-major scales [R][K/16] -> the tensor-core order (rows padded to 128
// with zero scales).  One thread per output byte.
__global__ void nvfp4_pack_scales_kernel(const uint8_t* __restrict__ rows, int R, int K, uint8_t* __restrict__ out) {
  const int64_t cols = K / kNvBlock;
  const int64_t total = int64_t((R + 127) / 128) * 128 * cols;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / cols, c = i % cols;
    out[nv_sf_offset(r, c, K)] = r < R ? rows[r * cols + c] : uint8_t(0);
  }
}

// ------------------------------------------------------------------ GEMM

template <int NT, int CPS = 1>  // CPS: CTAs resident per SM (each takes its share of shared memory and TMEM)
struct NvCfg {
  static constexpr uint32_t kA = kNvRows * 128;                 // weight codes: 128 rows x 128 bytes
  static constexpr uint32_t kB = NT * 128;                      // token codes
  static constexpr uint32_t kSfa = 4 * kNvSfChunk;              // 4 k64 steps of 128 rows
  static constexpr int kSfbBlocks = (NT + 127) / 128;           // 128-row scale blocks of the token tile
  static constexpr uint32_t kSfb = kSfbBlocks * 4 * kNvSfChunk;
  static constexpr uint32_t kStage = kA + kB + kSfa + kSfb;     // a multiple of 1024
  // a CTA's share of the SM's 228 KiB (1 KiB of each CTA's share is reserved)
  static constexpr size_t kBudget = CPS == 1 ? kNvMaxSmem : size_t(233472 / CPS) - 1024;
  static constexpr int kStages = int((kBudget - 2048) / kStage) > 8 ? 8 : int((kBudget - 2048) / kStage);
  static constexpr size_t kSmem = 2048 + size_t(kStages) * kStage;
  static constexpr uint32_t kSfaCols = 16;                      // 4 steps x 4 columns
  static constexpr uint32_t kSfbStepCols = 4 * kSfbBlocks;      // columns of one k64 step's token scales
  static constexpr uint32_t kSfCols = kSfaCols + 4 * kSfbStepCols;
  // kind::mxf4nvf4: E2M1 A and B (format 1), ue4m3 scales (bit 23 = 0),
  // K-major both, N >> 3 at bit 17, M >> 4 at bit 24, dense K = 64.
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (uint32_t(NT >> 3) << 17) | (uint32_t(kNvRows >> 4) << 24);
  static_assert(kStage % 1024 == 0, "stages stay 1024-byte aligned");
  // TMEM columns: the accumulator, then each stage's scale columns; a power of two of at least 32
  static constexpr uint32_t kCols = NT + kStages * kSfCols;
  static constexpr uint32_t kTmemCols = kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128 : kCols <= 256 ? 256 : 512;
  static_assert(kCols <= kNvTmemCols / CPS, "accumulator and scale columns fit the SM's share");
  static_assert(kStages >= 2, "a pipeline");
  static_assert(NT % 32 == 0 && NT >= 32 && NT <= 256, "token tile");
};

struct NvGemmParams {
  const uint8_t* sfa;   // weight scales, tensor-core order
  const uint8_t* sfb;   // activation scales, tensor-core order
  const float* gw;      // [N]
  const float* gx;      // [M]
  uint16_t* y;          // bf16 [M][N]
  unsigned* err;
  int M, N, K;
};

// Per stage: `loaded` completes when the stage's code tiles and scale chunks
// have landed (the TMA thread's transfer); `full` when the four epilogue
// warps have moved the scale chunks into the stage's TMEM columns; `empty`
// when the MMAs that read the stage have completed.
struct NvShared {
  uint64_t loaded[8];
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full;
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort;
};

// Bounded wait that also gives up once another role has aborted (about a
// second of polls before it records a timeout).
__device__ __forceinline__ bool nv_wait(uint64_t* bar, uint32_t parity, NvShared* sh, unsigned* err) {
  for (uint32_t i = 0; i < (1u << 20); ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 1023u && sh->abort) return false;
  }
  sh->abort = 1;
  record_error(err, kErrTimeout);
  return false;
}

// Shared-memory descriptor of a K-major 128-byte-swizzled operand tile
// (8-row groups 1024 bytes apart; the k64 step adds 32 bytes).
__device__ __forceinline__ uint64_t nv_sw128_desc(uint32_t smem_addr) {
  return uint64_t((smem_addr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// 32 lanes x 4 columns of 32-bit cells (thread i: lane quarter base + i).
__device__ __forceinline__ void tmem_st_32x32b_x4(uint32_t taddr, const uint4& v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// D[tmem] (+)= (A * SFA) (B * SFB)^T, E2M1 operands from shared memory,
// ue4m3 scales per 16 k from TMEM.
__device__ __forceinline__ void tc_mma_fp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Epilogue of one warp: its 32 accumulator lanes (rows nb .. nb + 31) x NT
// columns (tokens m0 ..), 32 columns at a time, stored through shared memory
// (store_block_transposed).
template <int NT>
__device__ __forceinline__ void nv_epilogue(const NvGemmParams& p, uint32_t tmem_rows, uint32_t tbuf, int nb, int m0,
                                            int lane) {
  const int n = nb + lane;
  const float gw = n < p.N ? p.gw[n] : 0.f;
#pragma unroll 1
  for (int c = 0; c < NT / 32 && m0 + 32 * c < p.M; ++c) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(tmem_rows + uint32_t(32 * c), v);
    tc_wait_ld();
    const int mc = m0 + 32 * c;
    store_block_transposed(p.y, p.M, p.N, mc, nb, tbuf, lane, [&](int j) {
      const float gx = mc + j < p.M ? p.gx[mc + j] : 0.f;
      return __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j]) * gw * gx));
    });
  }
}

template <int NT, int CPS = 1>
__global__ void __launch_bounds__(kNvThreads, CPS)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                      const NvGemmParams p) {
  using C = NvCfg<NT, CPS>;
  extern __shared__ __align__(1024) uint8_t nv_smem[];
  pdl_launch_dependents();
  NvShared* sh = reinterpret_cast<NvShared*>(nv_smem);
  const uint32_t stage0 = (smem_u32(nv_smem) + uint32_t(sizeof(NvShared)) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kNvRows;
  const int m0 = blockIdx.y * NT;
  const int KT = p.K / kNvBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&sh->loaded[s], 1);
      mbar_init(&sh->full[s], 4);  // one arrival per epilogue warp
      mbar_init(&sh->empty[s], 1);
    }
    mbar_init(&sh->acc_full, 1);
    mbar_init(&sh->drain, 1);
    sh->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------ producer: codes by TMA, scales by bulk copy
    if (lane == 0) {
      tma_prefetch_desc(&tmap_w);
      tma_prefetch_desc(&tmap_x);
      pdl_wait();  // the activation codes and scales come from the previous kernel
      const int steps = p.K / 64;
      const int xblocks = (p.M + 127) / 128;
      int nb = 0;  // token scale blocks that exist (the tile's last one may lie past M)
      for (int i = 0; i < C::kSfbBlocks; ++i) nb += (m0 / 128 + i < xblocks) ? 1 : 0;
      const uint32_t bytes = C::kA + C::kB + C::kSfa + uint32_t(nb) * 4u * kNvSfChunk;
      const uint8_t* sfa = p.sfa + size_t(n0 / 128) * steps * kNvSfChunk;
      const uint8_t* sfb = p.sfb + size_t(m0 / 128) * steps * kNvSfChunk;
      int s = 0, issued = 0;
      uint32_t phase = 0;
      for (int kt = 0; kt < KT; ++kt) {
        if (!nv_wait(&sh->empty[s], phase ^ 1u, sh, p.err)) break;
        const uint32_t a = stage0 + uint32_t(s) * C::kStage;
        mbar_arrive_expect_tx(&sh->loaded[s], bytes);
        tma_load_2d(a, &tmap_w, &sh->loaded[s], kt * 128, n0);
        tma_load_2d(a + C::kA, &tmap_x, &sh->loaded[s], kt * 128, m0);
        bulk_load(a + C::kA + C::kB, sfa + size_t(kt) * 4 * kNvSfChunk, C::kSfa, &sh->loaded[s]);
        for (int i = 0; i < nb; ++i)
          bulk_load(a + C::kA + C::kB + C::kSfa + uint32_t(i) * 4u * kNvSfChunk,
                    sfb + (size_t(i) * steps + size_t(kt) * 4) * kNvSfChunk, 4u * kNvSfChunk, &sh->loaded[s]);
        ++issued;
        if (++s == C::kStages) {
          s = 0;
          phase ^= 1u;
        }
      }
      if (sh->abort && issued > 0) {
        // let the copies in flight land before the CTA exits (bounded: 50 us)
        unsigned long long t0, t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
        do {
          asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        } while (t - t0 < 50000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      int s = 0;
      uint32_t phase = 0;
      for (int kt = 0; kt < KT; ++kt) {
        ok = nv_wait(&sh->full[s], phase, sh, p.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a = stage0 + uint32_t(s) * C::kStage;
        const uint32_t sfa_t = tmem + uint32_t(NT) + uint32_t(s) * C::kSfCols;
        const uint32_t sfb_t = sfa_t + C::kSfaCols;
        const uint64_t ad = nv_sw128_desc(a), bd = nv_sw128_desc(a + C::kA);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tc_mma_fp4(tmem, ad + uint64_t(2 * j), bd + uint64_t(2 * j), C::kIdesc, sfa_t + 4u * j,
                     sfb_t + C::kSfbStepCols * j, (kt | j) != 0 ? 1u : 0u);
        tc_commit(&sh->empty[s]);
        if (++s == C::kStages) {
          s = 0;
          phase ^= 1u;
        }
      }
      if (ok) {
        tc_commit(&sh->acc_full);
      } else {  // wait for the tensor-core work already issued before the TMEM is freed
        tc_commit(&sh->drain);
        mbar_wait_bounded(&sh->drain, 0, p.err, 1u << 20);
      }
    }
  } else {
    // ------------------------------------------------ scale chunks into TMEM, then the epilogue
    const int q = warp & 3;  // the TMEM lane quarter this warp may access
    // Per stage: every chunk (32 rows of 16 bytes: 128 rows x 4 scales of a k64 step) goes to 4 TMEM
    // columns of this warp's 32 lanes; the four warps write the same data, which is the layout the
    // block-scaled MMA reads (row r at lane r % 32 of every quarter, column (r % 128) / 32).  Moving
    // them here keeps the MMA thread to one wait, four MMAs and one commit per stage.
    bool ok = true;
    {
      int s = 0;
      uint32_t phase = 0;
      const uint32_t lanebase = uint32_t(32 * q) << 16;
      for (int kt = 0; kt < KT && ok; ++kt) {
        const int w_ok = lane == 0 ? int(nv_wait(&sh->loaded[s], phase, sh, p.err)) : 0;
        ok = __shfl_sync(0xffffffffu, w_ok, 0) != 0;
        if (!ok) break;
        const uint32_t sfa_s = stage0 + uint32_t(s) * C::kStage + C::kA + C::kB, sfb_s = sfa_s + C::kSfa;
        const uint32_t sfa_t = tmem + lanebase + uint32_t(NT) + uint32_t(s) * C::kSfCols;
        const uint32_t sfb_t = sfa_t + C::kSfaCols;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 v;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(sfa_s + uint32_t(j) * kNvSfChunk + uint32_t(lane) * 16u));
          tmem_st_32x32b_x4(sfa_t + 4u * j, v);
#pragma unroll
          for (int i = 0; i < C::kSfbBlocks; ++i) {
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(sfb_s + uint32_t(i) * 4u * kNvSfChunk + uint32_t(j) * kNvSfChunk +
                               uint32_t(lane) * 16u));
            tmem_st_32x32b_x4(sfb_t + C::kSfbStepCols * j + 4u * i, v);
          }
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->full[s]);
        if (++s == C::kStages) {
          s = 0;
          phase ^= 1u;
        }
      }
    }
    // ---- epilogue: y[m, n] = D[n, m] g_w[n] g_x[m]
    const int acc_ok = (ok && lane == 0) ? int(nv_wait(&sh->acc_full, 0, sh, p.err)) : 0;
    if (__shfl_sync(0xffffffffu, acc_ok, 0) != 0) {
      tc_fence_after();
      pdl_wait();  // g_x comes from the previous kernel
      // every stage is free once the accumulator is complete: stage 0 holds each warp's 32 x 32 bf16 block
      const uint32_t tbuf = stage0 + uint32_t(q) * 2048u;
      nv_epilogue<NT>(p, tmem + (uint32_t(32 * q) << 16), tbuf, n0 + 32 * q, m0, lane);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

}  // namespace w4a8
