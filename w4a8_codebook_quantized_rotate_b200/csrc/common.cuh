// Shared definitions for the W4A8 ConvRot kernels (sm_100a).
//
// Device layout of one packed layer (written by the pack kernel, read by the
// dequant, decode and prefill kernels).  All region offsets are multiples of
// 256 bytes.
//
//   [cb]     16 fp32 codebook levels
//   [sch]    N fp32 row scales
//   [units]  [pair = ceil(N/32)][chunk = K/64][1152 bytes]
//
// A unit covers the 32 rows of a tile pair (tiles 2p and 2p+1, 16 rows
// each) and 64 k.  Its 1152 bytes are
//   [0, 512)      index bytes of tile 2p
//   [512, 1024)   index bytes of tile 2p+1
//   [1024, 1088)  group-scale bytes of tile 2p
//   [1088, 1152)  group-scale bytes of tile 2p+1
// (a missing last tile, when N/16 is odd, is zero).  A unit is contiguous,
// and units lie in [pair][chunk] order, so any range of units is one
// contiguous run of memory that a single bulk copy can move.
//
// A tile's 512 index bytes are laid out in the register order of the
// mma.sync m16n8k16 A operand, so that a lane's 16 bytes are exactly its A
// fragments for the chunk's four k16 steps: lane = 4 g + t (g = lane / 4,
// t = lane % 4), byte j = 4 s + r (s = k16 step, r = fragment register)
// holds the canonical byte (two 4-bit indices, even k in the low nibble) of
//     row  16 tile + g + 8 (r & 1)
//     k    64 chunk + 16 s + 2 (t + 4 (r >> 1)), and k + 1.
// A tile's 64 group-scale bytes are [g 8][s 4][h 2]:
//     byte 8 g + 2 s + h = s_rel[16 tile + g + 8 h][4 chunk + s].
// One 16-bit half word then holds the pair (row g, row g + 8) of a k16 step,
// which is the pair a lane needs to scale its accumulator fragment.
#pragma once

#include <cstdint>
#include <cstddef>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace w4a8 {

#ifndef W4A8_SPIN_WAIT
#define W4A8_SPIN_WAIT 0
#endif

constexpr int kRotBlock = 256;
constexpr int kGroup = 16;
constexpr int kTileRows = 16;     // rows per (tile, chunk) block
constexpr int kChunkK = 64;       // k per (tile, chunk) block
constexpr int kChunkIdxBytes = 512;     // one tile's index bytes per chunk
constexpr int kChunkSrelBytes = 64;     // one tile's group-scale bytes per chunk
constexpr int kUnitBytes = 2 * kChunkIdxBytes + 2 * kChunkSrelBytes;  // 1152
constexpr int kMaxK = 32768;

// Device-side error word values (bit flags).
constexpr unsigned kErrTimeout = 1u;
constexpr unsigned kErrInput = 2u;  // a device-side input check failed

struct PackedLayout {
  int64_t N, K, tiles, pairs, chunks;
  size_t off_cb, off_sch, off_units, total;
};

__host__ __device__ inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline PackedLayout packed_layout(int64_t N, int64_t K) {
  PackedLayout L;
  L.N = N;
  L.K = K;
  L.tiles = N / kTileRows;
  L.pairs = (L.tiles + 1) / 2;
  L.chunks = K / kChunkK;
  L.off_cb = 0;
  L.off_sch = 256;
  L.off_units = L.off_sch + round_up(size_t(N) * 4, 256);
  L.total = round_up(L.off_units + size_t(L.pairs) * L.chunks * kUnitBytes, 256);
  return L;
}

// Byte offsets, within the units region, of tile `tile`'s index bytes and
// group-scale bytes for chunk `chunk`.
__host__ __device__ inline size_t unit_offset(int64_t pair, int64_t chunk, int64_t chunks) {
  return size_t(pair * chunks + chunk) * kUnitBytes;
}
__host__ __device__ inline size_t tile_idx_offset(int64_t tile, int64_t chunk, int64_t chunks) {
  return unit_offset(tile >> 1, chunk, chunks) + size_t(tile & 1) * kChunkIdxBytes;
}
__host__ __device__ inline size_t tile_srel_offset(int64_t tile, int64_t chunk, int64_t chunks) {
  return unit_offset(tile >> 1, chunk, chunks) + 2 * kChunkIdxBytes + size_t(tile & 1) * kChunkSrelBytes;
}

// ---------------------------------------------------------------- small device helpers

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Two e4m3 codes (low byte first) -> fp32 pair, exact.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two_codes) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two_codes & 0xFFFFu), __NV_E4M3);
  __half2 hh = *reinterpret_cast<__half2*>(&h);
  return __half22float2(hh);
}

__device__ __forceinline__ float e4m3_to_float(uint32_t code) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)(code & 0xFFu), __NV_E4M3);
  return __half2float(*reinterpret_cast<__half*>(&h));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void record_error(unsigned* err, unsigned code) {
  if (err) atomicOr(err, code);
}

// ---------------------------------------------------------------- programmatic dependent launch

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking probe of a barrier phase (returns at once).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on a barrier phase.  Returns false (and records a timeout in
// the error word) if the phase did not complete within `max_tries` polls;
// each poll itself suspends for a hardware-chosen time, so the bound is on
// the order of seconds.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, unsigned* err,
                                                  uint32_t max_tries = (1u << 24)) {
  for (uint32_t i = 0; i < max_tries; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
  }
  record_error(err, kErrTimeout);
  return false;
}

// Bounded poll of a global word until it reaches `target` (acquire loads,
// one L2 round trip each).  Returns false (and records a timeout in the
// error word) if it did not within `max_tries` polls.
__device__ __forceinline__ bool poll_at_least_bounded(const unsigned* word, unsigned target, unsigned* err,
                                                      uint32_t max_tries) {
  for (uint32_t i = 0; i < max_tries; ++i) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(word) : "memory");
    if (v >= target) return true;
  }
  record_error(err, kErrTimeout);
  return false;
}

// ---------------------------------------------------------------- TMA (no multicast)

__device__ __forceinline__ void tma_prefetch_desc(const void* desc) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(desc) : "memory");
}

// 2-D tiled load into shared memory (shared-window address `smem_dst`),
// completing `bytes` on the mbarrier.  x is the innermost coordinate.
__device__ __forceinline__ void tma_load_2d(uint32_t smem_dst, const void* desc, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_dst),
      "l"(desc), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned addresses, size a multiple
// of 16), completing `bytes` on the mbarrier.  No multicast.
__device__ __forceinline__ void bulk_load(uint32_t smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_dst),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------- tcgen05 (cta_group::1)

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Arrive on `bar` once every tcgen05 operation this thread issued so far has
// completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16 (fp16 x fp16 -> fp32).
__device__ __forceinline__ void tc_mma_ts_f16(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 columns of 32-bit cells; thread i of the warp owns lane
// (32 * (warp % 4) + i), register j is column (base + j).
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// ---------------------------------------------------------------- transposed bf16 epilogue

// One warp stores a 32 x 32 block of a row-major bf16 matrix y [M, N]: rows
// (tokens) mc .. mc + 31, columns (outputs) nb .. nb + 31, where thread i
// holds column nb + i for the 32 rows (value(j) is row mc + j, as bf16
// bits).  The block goes through 2 KiB of shared memory [row][column], so
// the global stores are 16 bytes of 8 consecutive columns (4 threads cover
// the block's 64-byte run of a row) rather than one 2-byte store per value.
// Rows >= M and columns >= N are not written.
template <typename Value>
__device__ __forceinline__ void store_block_transposed(uint16_t* __restrict__ y, int M, int N, int mc, int nb,
                                                       uint32_t tbuf, int lane, Value value) {
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint16_t b = value(j);
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(tbuf + uint32_t(j) * 64u + uint32_t(lane) * 2u), "h"(b));
  }
  __syncwarp();
  const bool vec = (N & 7) == 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = lane + 32 * i, row = idx >> 2, part = idx & 3;
    const int m = mc + row, n = nb + 8 * part;
    if (m < M && n < N) {
      uint32_t w[4];
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                   : "r"(tbuf + uint32_t(row) * 64u + uint32_t(part) * 16u));
      uint16_t* dst = y + size_t(m) * N + n;
      if (vec) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (n + e < N) dst[e] = uint16_t(w[e >> 1] >> (16 * (e & 1)));
      }
    }
  }
  __syncwarp();
}

}  // namespace w4a8
