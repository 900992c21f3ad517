// Fidelity checks of a stored layer ("Qwen3.8-27B-AEON-ULTIMATE-UNCENSORED-BF16
// -- W4A8 ConvRot for ComfyUI" model card, sections "Verification": the
// stored layer's dequantised weights against a fresh quantisation of the
// same source tensor, expected ~0; and "Accuracy": the quantised layer's
// output against the full-precision one, ~1 %).
//
// Two building blocks:
//   * compare: sum (a - ref)^2, sum ref^2 and max |a - ref| over n values, in
//     fp64, with a fixed grid and a fixed reduction order (deterministic);
//   * dense reference: y[m, n] = sum_k x[m, k] W[n, k] in fp64 from bf16 x and
//     fp32 W (the unquantised layer in the original basis).
#pragma once

#include "common.cuh"

namespace w4a8 {

constexpr int kCmpBlocks = 1024;  // fixed grid: the reduction order does not depend on the device
constexpr int kCmpThreads = 256;

template <bool A_BF16>
__global__ void __launch_bounds__(kCmpThreads) compare_kernel(const void* __restrict__ a, const float* __restrict__ ref,
                                                              int64_t n, double* __restrict__ part) {
  __shared__ double s_d2[kCmpThreads], s_r2[kCmpThreads], s_mx[kCmpThreads];
  double d2 = 0.0, r2 = 0.0, mx = 0.0;
  for (int64_t i = int64_t(blockIdx.x) * kCmpThreads + threadIdx.x; i < n; i += int64_t(kCmpBlocks) * kCmpThreads) {
    double av;
    if constexpr (A_BF16) av = double(__uint_as_float(uint32_t(static_cast<const uint16_t*>(a)[i]) << 16));
    else av = double(static_cast<const float*>(a)[i]);
    const double r = double(ref[i]);
    const double d = av - r;
    d2 += d * d;
    r2 += r * r;
    mx = fmax(mx, fabs(d));
  }
  s_d2[threadIdx.x] = d2;
  s_r2[threadIdx.x] = r2;
  s_mx[threadIdx.x] = mx;
  __syncthreads();
  for (int h = kCmpThreads / 2; h > 0; h >>= 1) {
    if (threadIdx.x < h) {
      s_d2[threadIdx.x] += s_d2[threadIdx.x + h];
      s_r2[threadIdx.x] += s_r2[threadIdx.x + h];
      s_mx[threadIdx.x] = fmax(s_mx[threadIdx.x], s_mx[threadIdx.x + h]);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    part[3 * blockIdx.x + 0] = s_d2[0];
    part[3 * blockIdx.x + 1] = s_r2[0];
    part[3 * blockIdx.x + 2] = s_mx[0];
  }
}

// out = {sum (a - ref)^2, sum ref^2, max |a - ref|}: the blocks' partials in block order.
__global__ void compare_final_kernel(const double* __restrict__ part, double* __restrict__ out) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  double d2 = 0.0, r2 = 0.0, mx = 0.0;
  for (int b = 0; b < kCmpBlocks; ++b) {
    d2 += part[3 * b + 0];
    r2 += part[3 * b + 1];
    mx = fmax(mx, part[3 * b + 2]);
  }
  out[0] = d2;
  out[1] = r2;
  out[2] = mx;
}

// One warp per weight row n: lanes take k = lane, lane + 32, ...; a fixed
// butterfly adds the lanes' sums.
constexpr int kRefWarps = 8;
__global__ void __launch_bounds__(kRefWarps * 32) dense_reference_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                                         int64_t K, const float* __restrict__ w,
                                                                         int64_t N, float* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int64_t n = int64_t(blockIdx.x) * kRefWarps + (threadIdx.x >> 5);
  if (n >= N) return;
  const float* wr = w + n * K;
  for (int64_t m = 0; m < M; ++m) {
    const uint16_t* xr = x + m * K;
    double acc = 0.0;
    for (int64_t k = lane; k < K; k += 32)
      acc = fma(double(__uint_as_float(uint32_t(xr[k]) << 16)), double(wr[k]), acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) y[m * N + n] = float(acc);
  }
}

}  // namespace w4a8
