// Activation rotation and per-token int8 quantisation.
//
// x_rot[m, 256 b + j] = (1/16) sum_i x[m, 256 b + i] H_256[i, j]  (Sylvester H)
// s_x[m] = max_k |x_rot[m, k]| / 127,  q = clamp(rint(x_rot / s_x), -127, 127)
//
// "Qwen3.8-27B-AEON-ULTIMATE-UNCENSORED-BF16 -- W4A8 ConvRot for ComfyUI"
// model card, section "Format" (group-wise Hadamard rotation, group 256);
// "Qwen3.8-27B-W4A8" model card, section "Model Overview" (int8
// activations).  The weights were rotated by the same orthonormal H_256/16,
// so x_rot . W_rot = x . W.
//
// One CTA per token.  Each warp transforms whole 256-blocks: a lane holds 8
// consecutive values, the three butterfly stages inside a lane run in
// registers and the five across lanes use shuffles.  The rotated row is
// staged in shared memory until the row maximum is known.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace w4a8 {

enum ActOut : int {
  kActI8Row = 0,    // int8 [M, K] row-major (the C ABI's rotate-quant call)
  kActF16Row = 1,   // fp16 [M, K] row-major, the tensor-core GEMM's operand
};

constexpr int kActMaxThreads = 1024;

// Threads per token: 8 warps (a warp takes every 8th 256-block).  Fewer
// threads than blocks lets more tokens share an SM (measured: 29 vs 38 us
// for 4096 tokens at K = 5120 against one warp per block).
__host__ __device__ inline int act_threads(int64_t) { return 256; }

// Index (in half2 units) of element (m, k) in the decode B-fragment layout:
// [chunk][n8 block j][lane 32][8 half2], lane = 4 (m % 8) + t, half2
// register 2 s + w holds k = 64 chunk + 16 s + 2 t + 8 w and k + 1.
__host__ __device__ inline int64_t frag_half2_index(int64_t m, int64_t k, int nb) {
  const int64_t c = k >> 6;
  const int s = int(k >> 4) & 3, w = int(k >> 3) & 1, t = int(k >> 1) & 3;
  const int64_t j = m >> 3;
  const int g = int(m & 7);
  return (((c * nb + j) * 32 + 4 * g + t) * 8) + 2 * s + w;
}

__device__ __forceinline__ void fwht8_in_lane(float (&v)[8]) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
}

// The lane's 16 bytes of 256-block b of a bf16 row (positions 256 b + 8 lane
// .. + 7), from L2 only: a chain of layers rewrites its activation buffers
// within one launch.
__device__ __forceinline__ uint4 load_block_lane(const uint16_t* __restrict__ row, int b, int lane) {
  return __ldcg(reinterpret_cast<const uint4*>(row + b * kRotBlock + lane * 8));
}

// Rotate a 256-block held 8 consecutive values per lane (lane l holds
// positions 8 l .. 8 l + 7), in place: three butterfly stages inside the
// lane, five across lanes (shuffles), then the exact 1/16.
__device__ __forceinline__ void rotate_vals_lane(float (&v)[8], int lane) {
  fwht8_in_lane(v);
#pragma unroll
  for (int bit = 1; bit < 32; bit <<= 1) {
    const bool upper = (lane & bit) != 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float p = __shfl_xor_sync(0xffffffffu, v[i], bit);
      v[i] = upper ? (p - v[i]) : (v[i] + p);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] *= 0.0625f;  // 1/16, exact
}

// Lane's 8 values of a rotated 256-block, from the lane's 16 bytes of it (bf16).
__device__ __forceinline__ void rotate_words_lane(const uint4 raw, int lane, float (&v)[8]) {
  const uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(wds[i] << 16);
    v[2 * i + 1] = __uint_as_float(wds[i] & 0xFFFF0000u);
  }
  rotate_vals_lane(v, lane);
}

// Lane's 8 values of the rotated 256-block b of a bf16 row.
__device__ __forceinline__ void rotate_block_lane(const uint16_t* __restrict__ row, int b, int lane, float (&v)[8]) {
  rotate_words_lane(load_block_lane(row, b, lane), lane, v);
}

// Per-token scale and code: s = amax / 127 (IEEE division), q = clamp(rint(v / s), -127, 127)
// with v / s the correctly rounded fp32 quotient.
//
// A token's codes take one division each, in every CTA that needs them, so
// the quotient is formed from the correctly rounded reciprocal r = 1/s and
// one correction step, q0 = v r, q = q0 + (v - q0 s) r (two fused
// multiply-adds): P. Markstein, "Computation of elementary functions on the
// IBM RISC System/6000 processor", IBM J. Res. Develop. 34 (1990), which
// gives the correctly rounded quotient when r is the correctly rounded
// reciprocal and nothing overflows or underflows.  The sign of a zero
// quotient is taken from v.  Scales outside [2^-100, 2^100] use the
// division itself.
struct QuantScale {
  float s;     // amax / 127
  float r;     // 1 / s, correctly rounded (when fast)
  bool fast;
};
__device__ __forceinline__ float quant_scale(float amax) { return __fdiv_rn(amax, 127.0f); }
__device__ __forceinline__ QuantScale quant_prepare(float s) {
  QuantScale q;
  q.s = s;
  q.fast = s >= 0x1p-100f && s <= 0x1p100f;
  q.r = q.fast ? __frcp_rn(s) : 0.f;
  return q;
}
// FAST: the scale is in the reciprocal's range (QuantScale::fast); callers
// branch on it once per token, so each loop carries one form only.
template <bool FAST>
__device__ __forceinline__ float quant_code(float v, const QuantScale& q) {
  if constexpr (FAST) {
    const float q0 = v * q.r;
    return fminf(fmaxf(rintf(copysignf(fmaf(fmaf(-q0, q.s, v), q.r, q0), v)), -127.f), 127.f);
  } else {
    return q.s > 0.f ? fminf(fmaxf(rintf(__fdiv_rn(v, q.s)), -127.f), 127.f) : 0.f;
  }
}

template <int OUT>
__global__ void __launch_bounds__(kActMaxThreads) rotate_quant_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                                  void* __restrict__ out, float* __restrict__ s_x) {
  extern __shared__ float xr[];  // [K] rotated row
  __shared__ float warp_max[kActMaxThreads / 32];
  const int nwarps = blockDim.x >> 5;
  // The previous kernel may still read this workspace: wait for it before
  // writing.  Then the next kernel may launch (it streams its weights, and
  // waits for this grid before reading what it writes).
  pdl_wait();
  pdl_launch_dependents();
  const int m = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nblocks = K / kRotBlock;
  float amax = 0.f;
  for (int b = warp; b < nblocks; b += nwarps) {
    float v[8];
    rotate_block_lane(x + int64_t(m) * K, b, lane, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    float4* dst = reinterpret_cast<float4*>(xr + b * kRotBlock + lane * 8);
    dst[0] = make_float4(v[0], v[1], v[2], v[3]);
    dst[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (lane == 0) warp_max[warp] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int i = 1; i < nwarps; ++i) amax = fmaxf(amax, warp_max[i]);
  const float s = quant_scale(amax);
  const QuantScale qs = quant_prepare(s);
  if (threadIdx.x == 0) s_x[m] = s;
  // Quantise 8 consecutive values per thread per step.
  auto quantise = [&](auto fast) {
    for (int k0 = threadIdx.x * 8; k0 < K; k0 += blockDim.x * 8) {
      const float4 a = *reinterpret_cast<const float4*>(xr + k0);
      const float4 c = *reinterpret_cast<const float4*>(xr + k0 + 4);
      const float v[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
      float q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        q[i] = quant_code<decltype(fast)::value>(v[i], qs);
      }
      if constexpr (OUT == kActI8Row) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          lo |= (uint32_t(int(q[i])) & 0xFFu) << (8 * i);
          hi |= (uint32_t(int(q[i + 4])) & 0xFFu) << (8 * i);
        }
        *reinterpret_cast<uint2*>(static_cast<int8_t*>(out) + int64_t(m) * K + k0) = make_uint2(lo, hi);
      } else {
        __half2 h[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(q[2 * i], q[2 * i + 1]);
        *reinterpret_cast<uint4*>(static_cast<__half*>(out) + int64_t(m) * K + k0) =
            *reinterpret_cast<uint4*>(h);
      }
    }
  };
  if (qs.fast)
    quantise(std::true_type{});
  else
    quantise(std::false_type{});
}

// The decode operand for a few tokens, one token per thread-block cluster:
// CTA c of the cluster rotates 256-blocks [16 c, 16 c + 16) (a warp each,
// the values stay in registers), the CTAs exchange their absmax through
// distributed shared memory, and each quantises its own blocks.  Same
// arithmetic as rotate_quant_kernel (rotate_block_lane, quant_scale,
// quant_code): the same codes and s_x.  Splitting the token over up to 8
// SMs cuts the latency of the step before a decode GEMV.
constexpr int kActClusterBlocks = 16;  // 256-blocks per CTA (one per warp)

// Blocks of 8 tokens of a decode launch of m tokens: 1 (up to 8), 2 (up to
// 16) or 4 (up to 32) -- the decode kernel's variants.
__host__ __device__ constexpr int dec_blocks(int m) { return m <= 8 ? 1 : m <= 16 ? 2 : 4; }
constexpr int kActClusterThreads = kActClusterBlocks * 32;

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Reads a float at a shared address of CTA `rank` of this cluster.
__device__ __forceinline__ float ld_cluster_f32(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// Tokens are laid out in slices of `slice_m` (16 or 32; the decode kernel
// runs one launch per slice): token m goes to slice m / slice_m,
// `slice_half2` half2 units apart, as token m % slice_m of a slice with
// dec_blocks(tokens in the slice) blocks of 8 (1, 2 or 4: the decode
// kernel's variants).
// The first CTA also clears `zero_count` 16-byte words at `zero_vec` (the
// decode workspace's split-K counters).
__global__ void __launch_bounds__(kActClusterThreads) rotate_quant_frag_cluster_kernel(
    const uint16_t* __restrict__ x, int M, int K, __half2* __restrict__ out, float* __restrict__ s_x,
    int slice_half2, uint4* __restrict__ zero_vec, int zero_count, int slice_m) {
  __shared__ float warp_max[kActClusterBlocks];
  __shared__ float cta_max;
  // The previous kernel may still read the workspace: wait before writing.
  pdl_wait();
  pdl_launch_dependents();
  const int m = blockIdx.y;
  const uint32_t rank = cluster_ctarank(), ncta = cluster_nctarank();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (zero_vec && m == 0 && rank == 0) {
    for (int i = threadIdx.x; i < zero_count; i += blockDim.x) zero_vec[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  const int b = int(rank) * kActClusterBlocks + warp;
  const bool mine = b < K / kRotBlock;
  float v[8];
  float amax = 0.f;
  if (mine) {
    rotate_block_lane(x + int64_t(m) * K, b, lane, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (lane == 0) warp_max[warp] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = warp_max[0];
    for (int i = 1; i < kActClusterBlocks; ++i) a = fmaxf(a, warp_max[i]);
    cta_max = a;
  }
  cluster_sync_all();  // every CTA's maximum is written and visible cluster-wide
  float tmax = 0.f;
  for (uint32_t r = 0; r < ncta; ++r) tmax = fmaxf(tmax, ld_cluster_f32(smem_u32(&cta_max), r));
  const float s = quant_scale(tmax);
  const QuantScale qs = quant_prepare(s);
  if (rank == 0 && threadIdx.x == 0) s_x[m] = s;
  if (mine) {
    const int sl = m / slice_m, ml = m - sl * slice_m;
    const int nb = dec_blocks(min(slice_m, M - slice_m * sl));
    __half2* o = out + int64_t(sl) * slice_half2;
    const int k0 = b * kRotBlock + lane * 8;
    auto put = [&](auto fast) {
      constexpr bool kFast = decltype(fast)::value;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o[frag_half2_index(ml, k0 + 2 * i, nb)] =
            __floats2half2_rn(quant_code<kFast>(v[2 * i], qs), quant_code<kFast>(v[2 * i + 1], qs));
    };
    if (qs.fast)
      put(std::true_type{});
    else
      put(std::false_type{});
  }
  cluster_sync_all();  // no CTA leaves while another may still read its cta_max
}

}  // namespace w4a8
