// Weight converter on the GPU: fp32 W[N, K] -> the four stored tensors
// (packed 4-bit indices, e4m3 group scales, fp32 row scales, 16-level
// codebook).  "Qwen3.8-27B-AEON-ULTIMATE-UNCENSORED-BF16 -- W4A8 ConvRot for
// ComfyUI" model card, sections "Format" (rotate by the group-256 Hadamard,
// three scaling tiers, Lloyd-Max codebook, two indices per byte) and
// "Reproducing" (the fit samples the values with a fixed seed).
//
// Per row (one CTA), in fp64 so that every decision is the one an fp64
// evaluation of the formulas takes:
//   R[k]      = (1/16) sum_i W[256 b + i] H_256[i, k - 256 b]      (fast WHT)
//   s_ch      = fp32(max_k |R[k]|)
//   s_rel[g]  = e4m3_rne(max_{k in g} |R[k]| / s_ch)                (0 if s_ch = 0)
//   v[k]      = R[k] / (s_rel[g] s_ch)                             (0 where that is 0)
//   idx[k]    = number of level midpoints strictly below v[k]      (ties go low)
// The sums of the transform are exact in fp64 for any realistic weight (a
// block's 256 fp32 values span far less than the 2^29 of headroom), so the
// order of the butterflies does not matter.
//
// Codebook fit (Lloyd-Max): the normalised values v at the sample positions
// are gathered, sorted (bitonic network), prefix-summed exactly in 128-bit
// fixed point, and one CTA iterates: boundaries = level midpoints (a value
// on a midpoint belongs to the lower cell), level = mean of its cell (an
// empty cell keeps its level), until no level moves by tol or max_iter
// rounds.  It starts at the sample's (i + 1/2)/16 quantiles (linear
// interpolation between order statistics).
#pragma once

#include "common.cuh"

namespace w4a8 {

constexpr int kCvtThreads = 256;  // 8 warps per row
constexpr int kFixShift = 80;     // fixed point of the exact sums: v * 2^80

// ---------------------------------------------------------------- fp64 helpers

// e4m3fn code of x, round half to even, saturating at 448; NaN -> 0x7F; the
// sign bit is kept (so -0 -> 0x80).
__device__ __forceinline__ uint32_t e4m3_rne_f64(double x) {
  const uint32_t sign = signbit(x) ? 0x80u : 0u;
  double a = fabs(x);
  if (isnan(a)) return 0x7Fu;
  if (a > 896.0) a = 896.0;  // past the saturation point; keeps the exponent small
  uint32_t code;
  if (a < 0.015625) {  // below 2^-6: subnormal multiples of 2^-9
    code = uint32_t(rint(ldexp(a, 9)));
  } else {
    const int e = ilogb(a);                         // a in [2^e, 2^(e+1))
    const uint32_t t = uint32_t(rint(ldexp(a, 3 - e)));  // 8..16
    code = uint32_t((e + 7) * 8) + t - 8u;          // t = 16 rolls into the next binade
  }
  if (code > 0x7Eu) code = 0x7Eu;
  return code | sign;
}

__device__ __forceinline__ double e4m3_to_f64(uint32_t c) {
  const int e = int(c >> 3) & 15, m = int(c & 7u);
  double mag;
  if (e == 15 && m == 7) mag = __longlong_as_double(0x7FF8000000000000ll);
  else if (e == 0) mag = ldexp(double(m), -9);
  else mag = ldexp(double(8 + m), e - 10);
  return (c & 0x80u) ? -mag : mag;
}

// 8 values held by a lane of a warp that transforms one 256-block: positions
// 8 lane .. 8 lane + 7.  Three stages in the lane, five across lanes.
__device__ __forceinline__ void fwht256_f64(double (&v)[8], int lane) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((i & h) == 0) {
        const double a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
#pragma unroll
  for (int bit = 1; bit < 32; bit <<= 1) {
    const bool upper = (lane & bit) != 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const double p = __shfl_xor_sync(0xffffffffu, v[i], bit);
      v[i] = upper ? (p - v[i]) : (v[i] + p);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] *= 0.0625;
}

__device__ __forceinline__ void load_block_f64(const float* __restrict__ row, int b, int lane, double (&v)[8]) {
  const float4* src = reinterpret_cast<const float4*>(row + b * kRotBlock + lane * 8);
  const float4 a = src[0], c = src[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
}

// ---------------------------------------------------------------- per-row conversion

struct CvtParams {
  const float* w;             // [N, K]
  const float* cb;            // [16] ascending (ASSIGN)
  uint8_t* idx;               // [N, K/2] (ASSIGN)
  uint8_t* s_rel;             // [N, K/16]
  float* s_ch;                // [N]
  const uint64_t* sample_bits;  // GATHER: bit n K + k set = sample that value; null = every live value
  double* samples;            // GATHER: out, appended in any order
  unsigned long long* n_samples;  // GATHER: counter
  int64_t N, K;
};

// MODE 0: scales + indices (ASSIGN).  MODE 1: scales + gather the sample (GATHER).
template <int MODE>
__global__ void __launch_bounds__(kCvtThreads) convert_row_kernel(const CvtParams p) {
  extern __shared__ double gmax_s[];  // [K/16] group absmax
  __shared__ double red_s[kCvtThreads / 32];
  __shared__ double mids_s[15];
  const int64_t n = blockIdx.x;
  const int K = int(p.K), nblk = K / kRotBlock;
  const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
  const float* row = p.w + n * p.K;
  if (MODE == 0 && threadIdx.x < 15)
    mids_s[threadIdx.x] = 0.5 * (double(p.cb[threadIdx.x]) + double(p.cb[threadIdx.x + 1]));

  // pass 1: rotated row -> group and row absmax
  double rmax = 0.0;
  for (int b = wl; b < nblk; b += kCvtThreads / 32) {
    double v[8];
    load_block_f64(row, b, lane, v);
    fwht256_f64(v, lane);
    double g = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) g = fmax(g, fabs(v[i]));
    g = fmax(g, __shfl_xor_sync(0xffffffffu, g, 1));  // a group is two lanes
    if ((lane & 1) == 0) gmax_s[b * 16 + (lane >> 1)] = g;
    rmax = fmax(rmax, g);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) rmax = fmax(rmax, __shfl_xor_sync(0xffffffffu, rmax, off));
  if (lane == 0) red_s[wl] = rmax;
  __syncthreads();
  rmax = red_s[0];
#pragma unroll
  for (int i = 1; i < kCvtThreads / 32; ++i) rmax = fmax(rmax, red_s[i]);
  const float sch32 = __double2float_rn(rmax);
  const double sch = double(sch32);
  if (threadIdx.x == 0) p.s_ch[n] = sch32;
  // group scales: the ratio to the stored row scale, rounded to e4m3
  for (int g = threadIdx.x; g < K / kGroup; g += kCvtThreads) {
    const uint32_t code = sch > 0.0 ? e4m3_rne_f64(gmax_s[g] / sch) : 0u;
    p.s_rel[n * (p.K / kGroup) + g] = uint8_t(code);
    gmax_s[g] = e4m3_to_f64(code) * sch;  // the divisor of the group (exact product)
  }
  __syncthreads();

  // pass 2: normalised values -> indices, or the sample
  for (int b = wl; b < nblk; b += kCvtThreads / 32) {
    double v[8];
    load_block_f64(row, b, lane, v);
    fwht256_f64(v, lane);
    const double den = gmax_s[b * 16 + (lane >> 1)];
    const bool live = den > 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = live ? v[i] / den : 0.0;
    if constexpr (MODE == 0) {
      uint32_t packed = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint32_t c = 0;
#pragma unroll
        for (int j = 0; j < 15; ++j) c += mids_s[j] < v[i] ? 1u : 0u;
        packed |= c << (4 * i);
      }
      *reinterpret_cast<uint32_t*>(p.idx + n * (p.K / 2) + b * 128 + lane * 4) = packed;
    } else {
      if (live) {
        const int64_t pos0 = n * p.K + int64_t(b) * kRotBlock + lane * 8;
        uint32_t take = 0xFFu;
        if (p.sample_bits) take = uint32_t(p.sample_bits[pos0 >> 6] >> (pos0 & 63)) & 0xFFu;
        const int cnt = __popc(take);
        if (cnt) {
          const unsigned long long at = atomicAdd(p.n_samples, (unsigned long long)cnt);
          int j = 0;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if ((take >> i) & 1u) p.samples[at + j++] = v[i];
        }
      }
    }
  }
}

// ---------------------------------------------------------------- sample handling

// Marks the sample positions in a bit set of N K bits (cleared beforehand).
__global__ void sample_bits_kernel(const int64_t* __restrict__ pos, int64_t n, uint64_t* bits, int64_t total,
                                   unsigned* err) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int64_t q = pos[i];
  if (q < 0 || q >= total) {
    record_error(err, kErrInput);
    return;
  }
  atomicOr(reinterpret_cast<unsigned long long*>(bits) + (q >> 6), 1ull << (q & 63));
}

__global__ void fill_u64_kernel(uint64_t* a, int64_t n, uint64_t v) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
    a[i] = v;
}

// One compare-exchange step of a bitonic sorting network over n (a power of
// two) doubles, ascending; +inf pads sort to the end.
__global__ void bitonic_step_kernel(double* a, int64_t n, int64_t j, int64_t k) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int64_t l = i ^ j;
  if (l <= i) return;
  const double x = a[i], y = a[l];
  const bool up = (i & k) == 0;
  if ((x > y) == up) {
    a[i] = y;
    a[l] = x;
  }
}

// The same network for all strides j < 2 * kBitonicTile inside one block's
// tile of shared memory (k, the run length, is the outer loop).
constexpr int kBitonicTile = 2048;
__global__ void __launch_bounds__(kBitonicTile / 2) bitonic_local_kernel(double* a, int64_t k, int64_t j_first) {
  __shared__ double t[kBitonicTile];
  const int64_t base = int64_t(blockIdx.x) * kBitonicTile;
  for (int i = threadIdx.x; i < kBitonicTile; i += blockDim.x) t[i] = a[base + i];
  __syncthreads();
  for (int64_t j = j_first; j > 0; j >>= 1) {
    for (int i = threadIdx.x; i < kBitonicTile; i += blockDim.x) {
      const int l = i ^ int(j);
      if (l > i) {
        const double x = t[i], y = t[l];
        const bool up = ((base + i) & k) == 0;
        if ((x > y) == up) {
          t[i] = y;
          t[l] = x;
        }
      }
    }
    __syncthreads();
  }
  for (int i = threadIdx.x; i < kBitonicTile; i += blockDim.x) a[base + i] = t[i];
}

// v * 2^kFixShift as a 128-bit integer, truncated toward zero (exact for
// |v| >= 2^-27; smaller values lose bits below 2^-80).
__device__ __forceinline__ __int128 to_fixed(double v) {
  if (v == 0.0 || !isfinite(v)) return 0;
  int e;
  const double m = frexp(fabs(v), &e);                  // |v| = m 2^e, m in [0.5, 1)
  const long long mi = (long long)ldexp(m, 53);          // 53-bit integer mantissa
  const int sh = e - 53 + kFixShift;                     // |v| 2^80 = mi 2^sh
  __int128 r;
  if (sh >= 0) r = __int128(mi) << sh;
  else if (sh > -64) r = __int128(mi >> (-sh));
  else r = 0;
  return v < 0 ? -r : r;
}

// Round-to-nearest-even conversion of a 128-bit integer to fp64.
__device__ __forceinline__ double fixed_to_f64(__int128 x) {
  if (x == 0) return 0.0;
  const bool neg = x < 0;
  unsigned __int128 u = neg ? (unsigned __int128)(-x) : (unsigned __int128)x;
  const uint64_t hi = uint64_t(u >> 64), lo = uint64_t(u);
  const int top = hi ? 127 - __clzll((long long)hi) : 63 - __clzll((long long)lo);  // highest set bit
  double r;
  if (top < 53) {
    r = double(lo);  // exact
  } else {
    const int drop = top - 52;
    const unsigned __int128 keep = u >> drop;
    const unsigned __int128 rem = u - (keep << drop);
    const unsigned __int128 half = (unsigned __int128)1 << (drop - 1);
    unsigned __int128 q = keep;
    if (rem > half || (rem == half && (keep & 1))) q += 1;
    r = ldexp(double(uint64_t(q)), drop);  // q < 2^54: exact in fp64 after the shift
  }
  return neg ? -r : r;
}

// Per-block sums of the fixed-point values (the first step of an exact scan).
constexpr int kScanThreads = 256;
constexpr int kScanItems = 8;  // values per thread
__global__ void __launch_bounds__(kScanThreads) scan_blocks_kernel(const double* __restrict__ s, int64_t n,
                                                                   __int128* __restrict__ block_sum) {
  __shared__ __int128 part[kScanThreads];
  const int64_t base = int64_t(blockIdx.x) * kScanThreads * kScanItems;
  __int128 acc = 0;
  for (int i = 0; i < kScanItems; ++i) {
    const int64_t q = base + int64_t(threadIdx.x) * kScanItems + i;
    if (q < n) acc += to_fixed(s[q]);
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    __int128 t = 0;
    for (int i = 0; i < kScanThreads; ++i) t += part[i];
    block_sum[blockIdx.x] = t;
  }
}

// Exclusive prefix of the block sums, in place (one thread; a few thousand blocks).
__global__ void scan_offsets_kernel(__int128* block_sum, int64_t nblocks) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  __int128 run = 0;
  for (int64_t b = 0; b < nblocks; ++b) {
    const __int128 t = block_sum[b];
    block_sum[b] = run;
    run += t;
  }
  block_sum[nblocks] = run;
}

// prefix[q] = sum of the fixed-point values s[0 .. q), q = 0 .. n (exact).
__global__ void __launch_bounds__(kScanThreads) scan_final_kernel(const double* __restrict__ s, int64_t n,
                                                                  const __int128* __restrict__ block_off,
                                                                  __int128* __restrict__ prefix) {
  __shared__ __int128 part[kScanThreads];
  const int64_t base = int64_t(blockIdx.x) * kScanThreads * kScanItems;
  __int128 mine[kScanItems];
  __int128 acc = 0;
  for (int i = 0; i < kScanItems; ++i) {
    const int64_t q = base + int64_t(threadIdx.x) * kScanItems + i;
    mine[i] = q < n ? to_fixed(s[q]) : 0;
    acc += mine[i];
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {  // exclusive scan of the thread sums (serial: exact and deterministic)
    __int128 run = block_off[blockIdx.x];
    for (int i = 0; i < kScanThreads; ++i) {
      const __int128 t = part[i];
      part[i] = run;
      run += t;
    }
  }
  __syncthreads();
  __int128 run = part[threadIdx.x];
  for (int i = 0; i < kScanItems; ++i) {
    const int64_t q = base + int64_t(threadIdx.x) * kScanItems + i;
    if (q < n) prefix[q] = run;
    run += mine[i];
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) prefix[n] = block_off[gridDim.x];
}

// Number of sorted values <= x (searchsorted, side "right").
__device__ __forceinline__ int64_t count_le(const double* s, int64_t n, double x) {
  int64_t lo = 0, hi = n;
  while (lo < hi) {
    const int64_t mid = (lo + hi) >> 1;
    if (s[mid] <= x) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// Lloyd-Max iterations on the sorted sample (one warp; lane i < 16 owns level i).
__global__ void lloyd_kernel(const double* __restrict__ s, const unsigned long long* __restrict__ n_samples,
                             const __int128* __restrict__ prefix, int max_iter, double tol, float* cb_out,
                             int* rounds_out, unsigned* err) {
  const int lane = threadIdx.x;
  const int64_t n = int64_t(*n_samples);
  if (n == 0) {
    if (lane < 16) cb_out[lane] = 0.f;
    if (lane == 0 && rounds_out) *rounds_out = 0;
    if (lane == 0) record_error(err, kErrInput);
    return;
  }
  double c = 0.0;
  if (lane < 16) {  // start: the (lane + 1/2)/16 quantile, linear between order statistics
    const double h = double(n - 1) * ((lane + 0.5) / 16.0);
    const int64_t lo = int64_t(floor(h));
    const int64_t hi = lo + 1 < n ? lo + 1 : n - 1;
    const double t = h - double(lo), a = s[lo], b = s[hi];
    const double d = b - a;
    c = t < 0.5 ? a + d * t : b - d * (1.0 - t);
  }
  int it = 0;
  for (it = 1; it <= max_iter; ++it) {
    // cell i = sorted positions [end(i - 1), end(i)), end(i) = count of values <= midpoint i
    const double up = __shfl_down_sync(0xffffffffu, c, 1);
    int64_t end = n;
    if (lane < 15) end = count_le(s, n, 0.5 * (c + up));
    const int64_t start_raw = __shfl_up_sync(0xffffffffu, end, 1);
    const int64_t start = lane == 0 ? 0 : start_raw;
    double nc = c;
    if (lane < 16 && end > start) {
      const __int128 sum = prefix[end] - prefix[start];
      nc = ldexp(fixed_to_f64(sum), -kFixShift) / double(end - start);
    }
    double moved = lane < 16 ? fabs(nc - c) : 0.0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) moved = fmax(moved, __shfl_xor_sync(0xffffffffu, moved, off));
    c = nc;
    if (moved < tol) break;
  }
  if (it > max_iter) it = max_iter;
  if (lane < 16) cb_out[lane] = __double2float_rn(c);
  if (lane == 0 && rounds_out) *rounds_out = it;
}

}  // namespace w4a8
