// Layout packing and standalone dequantisation.
//
// pack: canonical stored tensors -> device layout (see common.cuh).
// dequant: device layout -> W_hat[n, k] = fp32(fp32(cb[idx] * s_rel) * s_ch),
// "Qwen3.8-27B-AEON-ULTIMATE-UNCENSORED-BF16 -- W4A8 ConvRot for ComfyUI"
// model card, section "Format" (three tiers of scaling).
#pragma once

#include "common.cuh"

namespace w4a8 {

// One thread per (tile, chunk, lane) over 2 * pairs tiles: gathers the
// lane's 16 index bytes from the canonical [N, K/2] plane; lanes 0..15 also
// move 4 group-scale bytes.  The missing last tile of an odd tile count is
// written as zeros.
__global__ void __launch_bounds__(256) pack_kernel(const uint8_t* __restrict__ idx,
                                                   const uint8_t* __restrict__ s_rel, int64_t N, int64_t K,
                                                   uint8_t* __restrict__ units) {
  const int64_t chunks = K / kChunkK;
  const int64_t tiles = N / kTileRows;
  const int64_t tiles_padded = 2 * ((tiles + 1) / 2);
  const int64_t gtid = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t block = gtid >> 5;  // (tile, chunk) block
  const int lane = int(gtid & 31);
  if (block >= tiles_padded * chunks) return;
  const int64_t tile = block / chunks;
  const int64_t chunk = block - tile * chunks;
  const bool real = tile < tiles;
  const int g = lane >> 2, t = lane & 3;
  const int64_t row_bytes = K / 2;
  uint32_t w[4] = {0, 0, 0, 0};
  if (real) {
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      uint32_t v = 0;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int64_t row = tile * kTileRows + g + 8 * (r & 1);
        const int64_t col = chunk * 32 + 8 * s + t + 4 * (r >> 1);
        v |= uint32_t(idx[row * row_bytes + col]) << (8 * r);
      }
      w[s] = v;
    }
  }
  *reinterpret_cast<uint4*>(units + tile_idx_offset(tile, chunk, chunks) + lane * 16) =
      make_uint4(w[0], w[1], w[2], w[3]);
  if (lane < 16) {
    const int64_t row_groups = K / kGroup;
    uint32_t v = 0;
    if (real) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int q = lane * 4 + e;  // byte 8 g + 2 s + h of the tile's 64
        const int gg = q >> 3, s = (q >> 1) & 3, h = q & 1;
        const int64_t row = tile * kTileRows + gg + 8 * h;
        v |= uint32_t(s_rel[row * row_groups + chunk * 4 + s]) << (8 * e);
      }
    }
    *reinterpret_cast<uint32_t*>(units + tile_srel_offset(tile, chunk, chunks) + lane * 4) = v;
  }
}

__global__ void copy_scales_kernel(const float* __restrict__ s_channel, const float* __restrict__ codebook,
                                   int64_t N, float* __restrict__ sch_out, float* __restrict__ cb_out) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < N) sch_out[i] = s_channel[i];
  if (i < 16) cb_out[i] = codebook[i];
}

// One warp per (tile, chunk) block.  Each lane rebuilds its 32 weights and
// writes them as float2 pairs; across the warp every 32-byte sector of the
// output rows is written whole.
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ units,
                                                      const float* __restrict__ sch, const float* __restrict__ cb,
                                                      int64_t N, int64_t K, float* __restrict__ w_hat) {
  __shared__ float cb_s[16];
  if (threadIdx.x < 16) cb_s[threadIdx.x] = cb[threadIdx.x];
  __syncthreads();
  const int64_t chunks = K / kChunkK;
  const int64_t tiles = N / kTileRows;
  const int64_t block = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (block >= tiles * chunks) return;
  const int64_t tile = block / chunks;
  const int64_t chunk = block - tile * chunks;
  const int g = lane >> 2, t = lane & 3;
  const uint4 wv = *reinterpret_cast<const uint4*>(units + tile_idx_offset(tile, chunk, chunks) + lane * 16);
  const uint2 sv = *reinterpret_cast<const uint2*>(units + tile_srel_offset(tile, chunk, chunks) + g * 8);
  const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
  const float s_row[2] = {sch[tile * kTileRows + g], sch[tile * kTileRows + g + 8]};
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const uint32_t pair = (s < 2 ? sv.x : sv.y) >> (16 * (s & 1));  // (row g, row g+8) codes
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int h = r & 1;
      const float sr = e4m3_to_float(pair >> (8 * h));
      const uint32_t byte = (words[s] >> (8 * r)) & 0xFFu;
      const int64_t row = tile * kTileRows + g + 8 * h;
      const int64_t k = chunk * kChunkK + 16 * s + 2 * (t + 4 * (r >> 1));
      float2 out;
      out.x = __fmul_rn(__fmul_rn(cb_s[byte & 15u], sr), s_row[h]);
      out.y = __fmul_rn(__fmul_rn(cb_s[byte >> 4], sr), s_row[h]);
      *reinterpret_cast<float2*>(w_hat + row * K + k) = out;
    }
  }
}

}  // namespace w4a8
