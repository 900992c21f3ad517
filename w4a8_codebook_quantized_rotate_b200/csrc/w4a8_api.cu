// C ABI of the W4A8 ConvRot linear layer: argument checks, per-device set-up
// and kernel launches.  The declarations, with argument meaning, layout,
// ownership and error behaviour, are in include/w4a8.h.
#include <algorithm>
#include <mutex>
#include <new>
#include <vector>

#include <cuda.h>  // driver types for the stream write below (resolved at run time, not linked)

#include "w4a8.h"

#include "act.cuh"
#include "common.cuh"
#include "convert.cuh"
#include "gemm_sk.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "gemv1.cuh"
#include "nvfp4.cuh"
#include "pack.cuh"
#include "verify.cuh"

namespace w4a8 {

// Device-side error word (bit flags, kErrTimeout); read and cleared by
// w4a8_get_device_error.
__device__ unsigned g_error_word;

// Built-in scratch for w4a8_linear_decode_static (callers that cannot
// allocate device memory).  Every GPU that loads the library holds this
// array until the process exits.  In host code the name is only a stand-in
// for the array: its device address comes from cudaGetSymbolAddress.
constexpr size_t kStaticScratchBytes = size_t(W4A8_STATIC_SCRATCH_BYTES);
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  bool arch_ok = false;
  int sms = 0;
  unsigned* err = nullptr;
};

DeviceState g_devices[kMaxDevices];
std::mutex g_mutex;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool weight_shape_ok(int64_t N, int64_t K) {
  return N > 0 && N % kTileRows == 0 && N <= (int64_t(1) << 24) && K > 0 && K % kRotBlock == 0 && K <= kMaxK;
}

// Token counts up to 65535 tiles of 256 (the GEMM's grid has one y index per token tile).
constexpr int64_t kMaxTokens = int64_t(65535) * 256;

bool act_shape_ok(int64_t M, int64_t K) {
  return M > 0 && M <= kMaxTokens && K > 0 && K % kRotBlock == 0 && K <= kMaxK;
}

template <typename Kern>
cudaError_t allow_smem(Kern k, size_t bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
}

// Per-device state: architecture check, SM count, error-word address and
// the shared-memory opt-ins of the large kernels.  Done once per device.
w4a8_status device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return W4A8_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& d = g_devices[dev];
  if (!d.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return W4A8_ERR_CUDA;
    d.arch_ok = (major == 10 && minor == 0);
    d.sms = sms;
    if (d.arch_ok) {
      void* sym = nullptr;
      if (cudaGetSymbolAddress(&sym, g_error_word) != cudaSuccess) return W4A8_ERR_CUDA;
      d.err = static_cast<unsigned*>(sym);
      if (allow_smem(rotate_quant_kernel<kActI8Row>, size_t(kMaxK) * 4) != cudaSuccess ||
          allow_smem(rotate_quant_kernel<kActF16Row>, size_t(kMaxK) * 4) != cudaSuccess ||
          allow_smem(decode_one_kernel<false>, dec_smem_bytes(1, kMaxK, true)) != cudaSuccess ||
          allow_smem(decode_one_kernel<true>, dec_smem_bytes(1, kMaxK, true)) != cudaSuccess ||
          allow_smem(decode_chain_kernel, dec_smem_bytes(1, kMaxK, true)) != cudaSuccess ||
          allow_smem(decode_kernel<1, kDecDepth1>, dec_smem_bytes(8, kMaxK, false)) != cudaSuccess ||
          allow_smem(decode_kernel<2, kDecDepth2>, dec_smem_bytes(16, kMaxK, false)) != cudaSuccess ||
          allow_smem(decode_kernel<4, kDecDepth4>, dec_smem_bytes(32, kMaxK, false)) != cudaSuccess ||
          allow_smem(gemm_tc_kernel, kTcSmemBytes) != cudaSuccess ||
          allow_smem(gemm_sk_kernel, 232448) != cudaSuccess ||  // the largest sk_smem_bytes over token tiles
          allow_smem(nvfp4_quant_kernel, size_t(kMaxK) * 4) != cudaSuccess ||
          allow_smem(nvfp4_gemm_kernel<256>, NvCfg<256>::kSmem) != cudaSuccess ||
          allow_smem(nvfp4_gemm_kernel<128>, NvCfg<128>::kSmem) != cudaSuccess ||
          allow_smem(nvfp4_gemm_kernel<128, 2>, NvCfg<128, 2>::kSmem) != cudaSuccess ||
          allow_smem(nvfp4_gemm_kernel<64>, NvCfg<64>::kSmem) != cudaSuccess)
        return W4A8_ERR_CUDA;
    }
    d.ready = true;
  }
  if (!d.arch_ok) return W4A8_ERR_ARCH;
  *out = &d;
  return W4A8_OK;
}

w4a8_status launch_status() { return cudaGetLastError() == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA; }

// ------------------------------------------------------------------ linear workspace

// One token runs the one-token decode kernel, 2..16 tokens the mma.sync
// decode kernel in one launch, 17..64 in launches of up to 32 tokens, more
// the prefill GEMM -- except that 65..256 tokens on a layer with few 128-row
// tiles (the GEMM would leave most SMs idle: 40 CTAs at N = 5120) run the
// small-batch tensor-core kernel, which splits the weight stream over every
// SM.  (Measured at K = 17408, N = 5120: 32 tokens 42 us in one launch
// against 52 us in two of 16; 64 tokens 76 us in two launches of 32 against
// 99 us on the small-batch kernel; 256 tokens 108 us on the small-batch kernel
// against 128 us on the GEMM.)
constexpr int kDecodeSliceM = 16;      // the slice of up to 16 tokens (also the static-scratch limit)
constexpr int kDecodeWideSliceM = 32;  // the slice when M > 16
constexpr int kDecodeMaxM = 64;
#ifndef W4A8_SK_MIN_M
#define W4A8_SK_MIN_M 65
#endif
constexpr int64_t kSkMinM = W4A8_SK_MIN_M;
constexpr int64_t kSkMaxRowTiles = 100;  // more 128-row tiles than this keep the GEMM busy enough
constexpr int64_t kSkMaxM = 256;         // its largest token tile (measured ahead of the GEMM up to there)

static_assert(size_t(kSkMaxCtas) * 8 * 4 <= kWsXchBytes, "the small-batch counters fit in the zero region");

struct LinearPlan {
  bool decode;
  bool sk;         // the small-batch tensor-core kernel
  int nt;          // sk: token tile (M rounded up to 16)
  size_t off_part; // sk: partial tiles
  int nb;          // decode: token blocks of 8 of a full slice
  int slice_m;     // decode: tokens per launch (16 up to 16 tokens, else 32)
  int slices;      // decode: launches of up to slice_m tokens
  size_t slice_bytes;  // decode: B-fragment bytes of one slice
  size_t off_sx, off_xq, off_slots, total;  // [0, kWsZeroBytes): exchange words and counters
  int T, P, C;
};

LinearPlan linear_plan(int64_t M, int64_t K, int64_t N, bool allow_sk = true) {
  LinearPlan L{};
  L.sk = allow_sk && M >= kSkMinM && M <= kSkMaxM && (N + kSkRows - 1) / kSkRows < kSkMaxRowTiles;
  L.decode = !L.sk && M <= kDecodeMaxM;
  L.T = int(N / kTileRows);
  L.C = int(K / kChunkK);
  L.P = (L.T + kDecTG - 1) / kDecTG;
  if (L.decode) {
    L.slice_m = M <= kDecodeSliceM ? kDecodeSliceM : kDecodeWideSliceM;
    const int64_t mslice = M < L.slice_m ? M : L.slice_m;
    L.nb = dec_blocks(int(mslice));
    L.slices = int((M + L.slice_m - 1) / L.slice_m);
    L.slice_bytes = size_t(K) * L.nb * 16;
    L.off_sx = kWsZeroBytes;
    L.off_xq = L.off_sx + 256;  // s_x: at most 64 floats
    L.off_slots = round_up(L.off_xq + L.slice_bytes * L.slices, 256);
    L.total = round_up(L.off_slots + size_t(2) * kDecMaxCtas * dec_slot_floats(int(mslice)) * 4, 256);
  } else {
    L.nb = 0;
    L.slices = 0;
    L.slice_bytes = 0;
    L.off_sx = kWsZeroBytes;  // the zero region is left as it is
    L.off_xq = round_up(L.off_sx + size_t(M) * 4, 256);
    L.off_slots = 0;
    L.total = round_up(L.off_xq + size_t(M) * K * 2, 256);
    if (L.sk) {
      L.nt = int((M + 15) / 16 * 16);
      L.off_part = L.total;  // [CTAs][2][nt][128] fp32
      L.total = round_up(L.off_part + size_t(kSkMaxCtas) * 2 * L.nt * kSkRows * 4, 256);
    }
  }
  return L;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// launch_pdl with a 1-D thread-block cluster of `cluster_x` CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, unsigned cluster_x, size_t smem,
                               cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace

// Waits (bounded) until ready[0] != 0, clears ready[0] and ready[1], then
// waits for the previous kernel (so that the next kernel's wait covers it
// too).  One thread.
__global__ void flag_wait_kernel(unsigned* ready, unsigned* err) {
  pdl_launch_dependents();
  poll_at_least_bounded(ready, 1u, err, 1u << 21);  // about a second
  ready[0] = 0u;
  ready[1] = 0u;
  pdl_wait();
}

// A word nothing ever writes: the self-test's flag.
__device__ unsigned g_never_set;

// The library's two kinds of bounded device wait, each on something that
// never completes: an mbarrier phase nobody arrives at (the GEMM's role
// handshakes) and a global word nobody sets (the chain's grid barrier).
// Each gives up after `tries` polls and records a timeout.
__global__ void wait_timeout_selftest_kernel(unsigned* err, uint32_t tries) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_wait_bounded(&bar, 0, err, tries);
    poll_at_least_bounded(&g_never_set, 1u, err, tries);
  }
}
}  // namespace w4a8

using namespace w4a8;

extern "C" {

size_t w4a8_packed_bytes(int64_t N, int64_t K) {
  if (!weight_shape_ok(N, K)) return 0;
  return packed_layout(N, K).total;
}

w4a8_status w4a8_pack_layout(const uint8_t* idx, const uint8_t* s_rel, const float* s_channel,
                             const float* codebook, int64_t N, int64_t K, void* packed, size_t packed_bytes,
                             void* stream) {
  if (!idx || !s_rel || !s_channel || !codebook || !packed) return W4A8_ERR_NULL;
  if (!weight_shape_ok(N, K)) return W4A8_ERR_SHAPE;
  if (!aligned16(idx) || !aligned16(s_rel) || !aligned16(s_channel) || !aligned16(codebook) || !aligned16(packed))
    return W4A8_ERR_ALIGN;
  const PackedLayout L = packed_layout(N, K);
  if (packed_bytes < L.total) return W4A8_ERR_WORKSPACE;
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(packed);
  const int64_t threads = 2 * L.pairs * L.chunks * 32;
  pack_kernel<<<unsigned((threads + 255) / 256), 256, 0, s>>>(idx, s_rel, N, K, base + L.off_units);
  copy_scales_kernel<<<unsigned((N + 255) / 256), 256, 0, s>>>(s_channel, codebook, N,
                                                                reinterpret_cast<float*>(base + L.off_sch),
                                                                reinterpret_cast<float*>(base + L.off_cb));
  return launch_status();
}

w4a8_status w4a8_unpack_dequant(const void* packed, int64_t N, int64_t K, float* w_hat, void* stream) {
  if (!packed || !w_hat) return W4A8_ERR_NULL;
  if (!weight_shape_ok(N, K)) return W4A8_ERR_SHAPE;
  if (!aligned16(packed) || !aligned16(w_hat)) return W4A8_ERR_ALIGN;
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  const PackedLayout L = packed_layout(N, K);
  const uint8_t* base = static_cast<const uint8_t*>(packed);
  const int64_t threads = L.tiles * L.chunks * 32;
  dequant_kernel<<<unsigned((threads + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      base + L.off_units, reinterpret_cast<const float*>(base + L.off_sch),
      reinterpret_cast<const float*>(base + L.off_cb), N, K, w_hat);
  return launch_status();
}

w4a8_status w4a8_rotate_quant_act(const uint16_t* x, int64_t M, int64_t K, int8_t* x_q, float* s_x,
                                  void* stream) {
  if (!x || !x_q || !s_x) return W4A8_ERR_NULL;
  if (!act_shape_ok(M, K)) return W4A8_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(x_q) || !aligned16(s_x)) return W4A8_ERR_ALIGN;
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  rotate_quant_kernel<kActI8Row><<<unsigned(M), act_threads(K), size_t(K) * 4, static_cast<cudaStream_t>(stream)>>>(
      x, int(M), int(K), x_q, s_x);
  return launch_status();
}

size_t w4a8_linear_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  if (!act_shape_ok(M, K) || !weight_shape_ok(N, K)) return 0;
  return linear_plan(M, K, N).total;
}

static w4a8_status linear_checks(int64_t M, int64_t K, int64_t N, const void* workspace, size_t workspace_bytes,
                                 LinearPlan* plan, DeviceState** d) {
  if (!workspace) return W4A8_ERR_NULL;
  if (!act_shape_ok(M, K) || !weight_shape_ok(N, K)) return W4A8_ERR_SHAPE;
  if (!aligned16(workspace)) return W4A8_ERR_ALIGN;
  *plan = linear_plan(M, K, N);
  if (workspace_bytes < plan->total) return W4A8_ERR_WORKSPACE;
  return device_state(d);
}

// One token with K above this: the fused kernel runs as pairs of CTAs that
// split the activation step (below it the pair's two cluster barriers cost
// more than the halved rotation saves).
#ifndef W4A8_DEC_PAIR_K
#define W4A8_DEC_PAIR_K 8192
#endif
constexpr int64_t kDecPairK = W4A8_DEC_PAIR_K;

// One-token work split (gemv1.cuh): the P C / 2 duos over G CTAs.
static void one_token_split(DecodeParams& p, int ctas_avail) {
  const int duos = p.P * p.C / 2;
  p.G = duos < ctas_avail ? duos : ctas_avail;
  p.Dq = duos / p.G;
  p.Dr = duos % p.G;
}

// Decode launches (M <= 64, one per slice of plan.slice_m tokens).  With x
// given (one token) the kernel also rotates
// and quantises the token; otherwise it reads what w4a8_linear_prepare left
// in the workspace.
static w4a8_status launch_decode(const LinearPlan& plan, const DeviceState* d, int64_t M, int64_t K, int64_t N,
                                 const uint8_t* pk, uint16_t* y, uint8_t* ws, cudaStream_t s, const uint16_t* x,
                                 unsigned* x_ready = nullptr) {
  const PackedLayout L = packed_layout(N, K);
  for (int sl = 0; sl < plan.slices; ++sl) {
    const int64_t m0 = int64_t(sl) * plan.slice_m;
    const int64_t ms = M - m0 < plan.slice_m ? M - m0 : plan.slice_m;
    DecodeParams p{};  // the decode-chain fields stay null
    p.x = x;
    p.units = pk + L.off_units;
    p.sch = reinterpret_cast<const float*>(pk + L.off_sch);
    p.cb = reinterpret_cast<const float*>(pk + L.off_cb);
    p.xfrag = reinterpret_cast<const uint4*>(ws + plan.off_xq + plan.slice_bytes * sl);
    p.s_x = reinterpret_cast<const float*>(ws + plan.off_sx) + m0;
    p.y = y + m0 * N;
    p.slots = reinterpret_cast<float*>(ws + plan.off_slots);
    p.xch = reinterpret_cast<unsigned long long*>(ws);
    p.counters = reinterpret_cast<unsigned*>(ws + kWsCntOff);
    p.err = d->err;
    p.x_ready = x_ready;
    p.M = int(ms);
    p.N = int(N);
    p.K = int(K);
    p.C = plan.C;
    p.T = plan.T;
    p.P = plan.P;
    p.U = plan.P * plan.C;
    const int wpc = dec_warps_m(int(ms));  // warps per CTA of this variant
    const int ctas_avail = d->sms < kDecMaxCtas ? d->sms : kDecMaxCtas;
    const int warps_avail = ctas_avail * wpc;
    p.W = p.U < warps_avail ? p.U : warps_avail;
    p.R = p.U / p.W;
    p.Rm = p.U % p.W;
    one_token_split(p, ctas_avail);
    const dim3 grid(ms == 1 ? unsigned(p.G) : unsigned((p.W + wpc - 1) / wpc));
    const size_t smem = dec_smem_bytes(int(ms), int(K), ms == 1);
    const int nb = dec_blocks(int(ms));
    cudaError_t e;
    if (x && K > kDecPairK)  // pairs of CTAs share the activation step (an even grid; extra CTAs hold no units)
      e = launch_pdl_cluster(decode_one_kernel<true>, dim3((grid.x + 1) & ~1u), dim3(kOneThreads), 2, smem, s, p);
    else if (x)
      e = launch_pdl(decode_one_kernel<true>, grid, dim3(kOneThreads), smem, s, p);
    else if (ms == 1)
      e = launch_pdl(decode_one_kernel<false>, grid, dim3(kOneThreads), smem, s, p);
    else if (nb == 1)
      e = launch_pdl(decode_kernel<1, kDecDepth1>, grid, dim3(wpc * 32), smem, s, p);
    else if (nb == 2)
      e = launch_pdl(decode_kernel<2, kDecDepth2>, grid, dim3(wpc * 32), smem, s, p);
    else
      e = launch_pdl(decode_kernel<4, kDecDepth4>, grid, dim3(wpc * 32), smem, s, p);
    if (e != cudaSuccess) return W4A8_ERR_CUDA;
  }
  return W4A8_OK;
}

// The activation step before w4a8_linear_run.  `zero_from` is where the
// activation kernel starts clearing the workspace's zero region (the split-K
// counters by default; the static-scratch call clears it whole).
static w4a8_status prepare_impl(const uint16_t* x, int64_t M, int64_t K, int64_t N, void* workspace,
                                size_t workspace_bytes, void* stream, size_t zero_from) {
  if (!x) return W4A8_ERR_NULL;
  if (!aligned16(x)) return W4A8_ERR_ALIGN;
  LinearPlan plan;
  DeviceState* d = nullptr;
  if (w4a8_status st = linear_checks(M, K, N, workspace, workspace_bytes, &plan, &d); st != W4A8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* s_x = reinterpret_cast<float*>(ws + plan.off_sx);
  if (plan.decode) {
    // one cluster of up to 8 CTAs per token (16 blocks of 256 per CTA)
    const unsigned cl = unsigned((K / kRotBlock + kActClusterBlocks - 1) / kActClusterBlocks);
    if (launch_pdl_cluster(rotate_quant_frag_cluster_kernel, dim3(cl, unsigned(M)), dim3(kActClusterThreads), cl, 0,
                           s, x, int(M), int(K), reinterpret_cast<__half2*>(ws + plan.off_xq), s_x,
                           int(plan.slice_bytes / 4), reinterpret_cast<uint4*>(ws + zero_from),
                           int((kWsZeroBytes - zero_from) / 16), plan.slice_m) != cudaSuccess)
      return W4A8_ERR_CUDA;
  } else {
    if (launch_pdl(rotate_quant_kernel<kActF16Row>, dim3(unsigned(M)), dim3(act_threads(K)), size_t(K) * 4, s, x,
                   int(M), int(K), (void*)(ws + plan.off_xq), s_x) != cudaSuccess)
      return W4A8_ERR_CUDA;
  }
  return launch_status();
}

w4a8_status w4a8_linear_prepare(const uint16_t* x, int64_t M, int64_t K, int64_t N, void* workspace,
                                size_t workspace_bytes, void* stream) {
  return prepare_impl(x, M, K, N, workspace, workspace_bytes, stream, kWsCntOff);
}

w4a8_status w4a8_linear_run(int64_t M, int64_t K, const void* packed, int64_t N, uint16_t* y, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (!packed || !y) return W4A8_ERR_NULL;
  if (!aligned16(packed) || !aligned16(y)) return W4A8_ERR_ALIGN;
  LinearPlan plan;
  DeviceState* d = nullptr;
  if (w4a8_status st = linear_checks(M, K, N, workspace, workspace_bytes, &plan, &d); st != W4A8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const PackedLayout L = packed_layout(N, K);
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* s_x = reinterpret_cast<float*>(ws + plan.off_sx);

  if (plan.decode) return launch_decode(plan, d, M, K, N, pk, y, ws, s, nullptr);

  __half* xq = reinterpret_cast<__half*>(ws + plan.off_xq);
  EncodeTiledFn enc = encode_fn();
  if (!enc) return W4A8_ERR_CUDA;
  CUtensorMap tmap;
  const cuuint64_t gdim[2] = {cuuint64_t(K), cuuint64_t(M)};
  const cuuint64_t gstride[1] = {cuuint64_t(K) * 2};
  const cuuint32_t box[2] = {uint32_t(kTcBK), uint32_t(plan.sk ? plan.nt : kTcTokens)};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, xq, gdim, gstride, box, estride,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return W4A8_ERR_CUDA;
  if (plan.sk) {
    SkParams q;
    q.units = pk + L.off_units;
    q.sch = reinterpret_cast<const float*>(pk + L.off_sch);
    q.cb = reinterpret_cast<const float*>(pk + L.off_cb);
    q.s_x = s_x;
    q.y = y;
    q.part = reinterpret_cast<float*>(ws + plan.off_part);
    q.counters = reinterpret_cast<unsigned*>(ws);  // inside the zero region (the exchange words' place)
    q.err = d->err;
    q.M = int(M);
    q.N = int(N);
    q.K = int(K);
    q.C = plan.C;
    q.RT = int((N + kSkRows - 1) / kSkRows);
    q.NT = plan.nt;
    const int items = q.RT * q.C;
    const int ctas = d->sms < kSkMaxCtas ? d->sms : kSkMaxCtas;
    q.G = items < ctas ? items : ctas;
    q.Iq = items / q.G;
    q.Ir = items % q.G;
    q.idesc = (1u << 4) | (uint32_t(q.NT >> 3) << 17) | (uint32_t(kSkRows >> 4) << 24);
    const cudaError_t e =
        launch_pdl(gemm_sk_kernel, dim3(unsigned(q.G)), dim3(kSkThreads), sk_smem_bytes(q.NT), s, tmap, q);
    return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
  }
  TcParams p;
  p.units = pk + L.off_units;
  p.sch = reinterpret_cast<const float*>(pk + L.off_sch);
  p.cb = reinterpret_cast<const float*>(pk + L.off_cb);
  p.s_x = s_x;
  p.y = y;
  p.err = d->err;
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  p.C = plan.C;
  p.T = plan.T;
  const dim3 grid(unsigned((N + kTcRows - 1) / kTcRows), unsigned((M + kTcTokens - 1) / kTcTokens));
  const cudaError_t e = launch_pdl(gemm_tc_kernel, grid, dim3(kTcThreads), kTcSmemBytes, s, tmap, p);
  return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

w4a8_status w4a8_linear(const uint16_t* x, int64_t M, int64_t K, const void* packed, int64_t N, uint16_t* y,
                        void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !packed || !y || !workspace) return W4A8_ERR_NULL;
  if (!aligned16(packed) || !aligned16(y)) return W4A8_ERR_ALIGN;
  if (M == 1) {  // one token: a single kernel makes the layer
    if (!aligned16(x)) return W4A8_ERR_ALIGN;
    LinearPlan plan;
    DeviceState* d = nullptr;
    if (w4a8_status st = linear_checks(M, K, N, workspace, workspace_bytes, &plan, &d); st != W4A8_OK) return st;
    return launch_decode(plan, d, M, K, N, static_cast<const uint8_t*>(packed), y, static_cast<uint8_t*>(workspace),
                         static_cast<cudaStream_t>(stream), x);
  }
  w4a8_status st = w4a8_linear_prepare(x, M, K, N, workspace, workspace_bytes, stream);
  if (st != W4A8_OK) return st;
  return w4a8_linear_run(M, K, packed, N, y, workspace, workspace_bytes, stream);
}

w4a8_status w4a8_linear_flagged(const uint16_t* x, int64_t M, int64_t K, const void* packed, int64_t N, uint16_t* y,
                                unsigned* x_ready, void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !packed || !y || !workspace || !x_ready) return W4A8_ERR_NULL;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(y) || (reinterpret_cast<uintptr_t>(x_ready) & 7u))
    return W4A8_ERR_ALIGN;
  LinearPlan plan;
  DeviceState* d = nullptr;
  if (w4a8_status st = linear_checks(M, K, N, workspace, workspace_bytes, &plan, &d); st != W4A8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 1)  // the layer's single kernel waits for the flag itself
    return launch_decode(plan, d, M, K, N, static_cast<const uint8_t*>(packed), y, static_cast<uint8_t*>(workspace), s,
                         x, x_ready);
  if (launch_pdl(flag_wait_kernel, dim3(1), dim3(1), 0, s, x_ready, d->err) != cudaSuccess) return W4A8_ERR_CUDA;
  w4a8_status st = w4a8_linear_prepare(x, M, K, N, workspace, workspace_bytes, stream);
  if (st != W4A8_OK) return st;
  return w4a8_linear_run(M, K, packed, N, y, workspace, workspace_bytes, stream);
}

// cuStreamWriteValue32 of the driver, looked up once through the runtime
// (the library links no driver library).  Null if the driver lacks it.
using WriteValue32Fn = CUresult (*)(CUstream, CUdeviceptr, cuuint32_t, unsigned int);
static WriteValue32Fn stream_write_value32() {
  static const WriteValue32Fn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuStreamWriteValue32", &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return WriteValue32Fn(nullptr);
    return reinterpret_cast<WriteValue32Fn>(f);
  }();
  return fn;
}

w4a8_status w4a8_signal_ready(unsigned* x_ready, void* stream) {
  if (!x_ready) return W4A8_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(x_ready) & 7u) return W4A8_ERR_ALIGN;
  const WriteValue32Fn fn = stream_write_value32();
  if (!fn) return W4A8_ERR_CUDA;
  // default flags: the write is ordered after every earlier write of the stream
  if (fn(static_cast<CUstream>(stream), reinterpret_cast<CUdeviceptr>(x_ready), 1u, 0u) != CUDA_SUCCESS)
    return W4A8_ERR_CUDA;
  return W4A8_OK;
}

// Device address of g_static_scratch, looked up once per device with that
// device current (the first w4a8_linear_decode_static call on the device).
static void* g_static_scratch_ptr[kMaxDevices];
static std::mutex g_static_scratch_mutex;

// The largest scratch a call may need: M = 16 at the largest K (the plan
// does not depend on N).  The array's size is checked against it once, and
// a CPU test checks the header's constant against w4a8_linear_workspace_bytes.
static_assert(kStaticScratchBytes % 256 == 0, "the scratch size is a whole number of 256-byte blocks");

w4a8_status w4a8_linear_decode_static(const uint16_t* x, int64_t M, int64_t K, const void* packed, int64_t N,
                                      uint16_t* y, void* stream) {
  if (!x || !packed || !y) return W4A8_ERR_NULL;
  if (M > kDecodeSliceM || !act_shape_ok(M, K) || !weight_shape_ok(N, K)) return W4A8_ERR_SHAPE;
  if (linear_plan(M, K, N).total > kStaticScratchBytes) return W4A8_ERR_WORKSPACE;
  // architecture first: on another GPU the array's lookup would fail with no kernel image
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return W4A8_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
    if (!g_static_scratch_ptr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
        cudaGetLastError();  // leave no error behind for a later launch check
        return W4A8_ERR_CUDA;
      }
      g_static_scratch_ptr[dev] = p;
    }
    scratch = g_static_scratch_ptr[dev];
  }
  // Every call clears the whole zero region (exchange words and arrival
  // counters, at the start of the scratch) before the layer's kernel runs --
  // in the decode path's activation kernel, else with a memset -- so a call
  // cut short (a timeout) leaves nothing that a later call could trip on.
  // Nothing else in the scratch has to start at a known value.
  if (linear_plan(M, K, N).sk &&
      cudaMemsetAsync(scratch, 0, kWsZeroBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return W4A8_ERR_CUDA;
  w4a8_status st = prepare_impl(x, M, K, N, scratch, kStaticScratchBytes, stream, 0);
  if (st != W4A8_OK) return st;
  return w4a8_linear_run(M, K, packed, N, y, scratch, kStaticScratchBytes, stream);
}

// ------------------------------------------------------------------ weight converter

struct ConvertPlan {
  int64_t n_cap, n_pad, scan_blocks;
  size_t off_bits, off_samples, off_bsum, off_prefix, total;
};

static ConvertPlan convert_plan(int64_t N, int64_t K, int64_t n_sample) {
  ConvertPlan c{};
  c.n_cap = n_sample > 0 ? n_sample : N * K;
  c.n_pad = int64_t(kBitonicTile);
  while (c.n_pad < c.n_cap) c.n_pad <<= 1;
  c.scan_blocks = (c.n_pad + kScanThreads * kScanItems - 1) / (kScanThreads * kScanItems);
  c.off_bits = 256;  // [0, 8): sample counter
  c.off_samples = round_up(c.off_bits + size_t((N * K + 63) / 64) * 8, 256);
  c.off_bsum = round_up(c.off_samples + size_t(c.n_pad) * 8, 256);
  c.off_prefix = round_up(c.off_bsum + size_t(c.scan_blocks + 1) * 16, 256);
  c.total = round_up(c.off_prefix + size_t(c.n_pad + 1) * 16, 256);
  return c;
}

size_t w4a8_convert_workspace_bytes(int64_t N, int64_t K, int64_t n_sample) {
  if (!weight_shape_ok(N, K) || n_sample > N * K) return 0;
  return convert_plan(N, K, n_sample).total;
}

w4a8_status w4a8_convert_weight(const float* w, int64_t N, int64_t K, const float* codebook_in,
                                const int64_t* sample_pos, int64_t n_sample, int32_t max_iter, double tol,
                                uint8_t* idx_packed, uint8_t* s_rel, float* s_channel, float* codebook_out,
                                int32_t* fit_rounds, void* workspace, size_t workspace_bytes, void* stream) {
  if (!w || !idx_packed || !s_rel || !s_channel || !codebook_out) return W4A8_ERR_NULL;
  if (!weight_shape_ok(N, K) || max_iter < 1 || !(tol >= 0.0)) return W4A8_ERR_SHAPE;
  if (sample_pos && (n_sample < 1 || n_sample > N * K)) return W4A8_ERR_SHAPE;
  if (!aligned16(w) || !aligned16(idx_packed)) return W4A8_ERR_ALIGN;
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CvtParams p{};
  p.w = w;
  p.idx = idx_packed;
  p.s_rel = s_rel;
  p.s_ch = s_channel;
  p.N = N;
  p.K = K;
  const size_t smem = size_t(K / kGroup) * 8;
  if (codebook_in) {
    p.cb = codebook_in;
    convert_row_kernel<0><<<unsigned(N), kCvtThreads, smem, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return W4A8_ERR_CUDA;
    if (codebook_out != codebook_in &&
        cudaMemcpyAsync(codebook_out, codebook_in, 16 * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return W4A8_ERR_CUDA;
    if (fit_rounds && cudaMemsetAsync(fit_rounds, 0, sizeof(int32_t), s) != cudaSuccess) return W4A8_ERR_CUDA;
    return W4A8_OK;
  }
  // fit the codebook first
  if (!workspace) return W4A8_ERR_NULL;
  if (!aligned16(workspace)) return W4A8_ERR_ALIGN;
  const ConvertPlan c = convert_plan(N, K, sample_pos ? n_sample : 0);
  if (workspace_bytes < c.total) return W4A8_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto* counter = reinterpret_cast<unsigned long long*>(ws);
  auto* bits = reinterpret_cast<uint64_t*>(ws + c.off_bits);
  auto* samples = reinterpret_cast<double*>(ws + c.off_samples);
  auto* bsum = reinterpret_cast<__int128*>(ws + c.off_bsum);
  auto* prefix = reinterpret_cast<__int128*>(ws + c.off_prefix);
  const int fill_grid = int(d->sms) * 8;
  if (cudaMemsetAsync(counter, 0, 8, s) != cudaSuccess) return W4A8_ERR_CUDA;
  fill_u64_kernel<<<fill_grid, 256, 0, s>>>(reinterpret_cast<uint64_t*>(samples), c.n_pad,
                                             0x7FF0000000000000ull);  // +inf: sorts past the sample
  if (sample_pos) {
    fill_u64_kernel<<<fill_grid, 256, 0, s>>>(bits, (N * K + 63) / 64, 0ull);
    sample_bits_kernel<<<unsigned((n_sample + 255) / 256), 256, 0, s>>>(sample_pos, n_sample, bits, N * K, d->err);
  }
  p.sample_bits = sample_pos ? bits : nullptr;
  p.samples = samples;
  p.n_samples = counter;
  convert_row_kernel<1><<<unsigned(N), kCvtThreads, smem, s>>>(p);
  // sort (bitonic network; strides below the tile size run in shared memory)
  const unsigned sort_grid = unsigned(c.n_pad / 256);
  for (int64_t k = 2; k <= c.n_pad; k <<= 1) {
    int64_t j = k >> 1;
    for (; j >= kBitonicTile; j >>= 1) bitonic_step_kernel<<<sort_grid, 256, 0, s>>>(samples, c.n_pad, j, k);
    bitonic_local_kernel<<<unsigned(c.n_pad / kBitonicTile), kBitonicTile / 2, 0, s>>>(samples, k, j);
  }
  scan_blocks_kernel<<<unsigned(c.scan_blocks), kScanThreads, 0, s>>>(samples, c.n_pad, bsum);
  scan_offsets_kernel<<<1, 1, 0, s>>>(bsum, c.scan_blocks);
  scan_final_kernel<<<unsigned(c.scan_blocks), kScanThreads, 0, s>>>(samples, c.n_pad, bsum, prefix);
  lloyd_kernel<<<1, 32, 0, s>>>(samples, counter, prefix, max_iter, tol, codebook_out, fit_rounds, d->err);
  p.cb = codebook_out;
  convert_row_kernel<0><<<unsigned(N), kCvtThreads, smem, s>>>(p);
  return launch_status();
}

// ------------------------------------------------------------------ chains of one-token layers

// [0, 256): grid-barrier counter; then the decode zero region (exchange words
// and split-K counters, shared by the layers); then the per-CTA partials.
constexpr size_t kChainZeroOff = 256;
constexpr size_t kChainSlotsOff = kChainZeroOff + kWsZeroBytes;

size_t w4a8_chain_plan_bytes(int64_t n_layers) {
  return n_layers < 1 ? 0 : round_up(size_t(n_layers) * sizeof(DecodeParams), 256);
}

size_t w4a8_chain_workspace_bytes(const w4a8_chain_layer* layers, int64_t n_layers) {
  if (!layers || n_layers < 1) return 0;
  for (int64_t i = 0; i < n_layers; ++i)
    if (!weight_shape_ok(layers[i].N, layers[i].K)) return 0;
  return kChainSlotsOff +
         round_up(size_t(2) * kDecMaxCtas * dec_slot_floats(1) * 4, 256);
}

w4a8_status w4a8_chain_plan(const w4a8_chain_layer* layers, int64_t n_layers, void* plan, size_t plan_bytes,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (!layers || !plan || !workspace) return W4A8_ERR_NULL;
  if (n_layers < 1 || n_layers > (int64_t(1) << 20)) return W4A8_ERR_SHAPE;
  for (int64_t i = 0; i < n_layers; ++i) {
    const w4a8_chain_layer& L = layers[i];
    if (!L.packed || !L.x || !L.y) return W4A8_ERR_NULL;
    if (!weight_shape_ok(L.N, L.K)) return W4A8_ERR_SHAPE;
    if (!aligned16(L.packed) || !aligned16(L.x) || !aligned16(L.y)) return W4A8_ERR_ALIGN;
  }
  if (plan_bytes < w4a8_chain_plan_bytes(n_layers) ||
      workspace_bytes < w4a8_chain_workspace_bytes(layers, n_layers))
    return W4A8_ERR_WORKSPACE;
  if (!aligned16(plan) || !aligned16(workspace)) return W4A8_ERR_ALIGN;
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  unsigned long long* xch = reinterpret_cast<unsigned long long*>(ws + kChainZeroOff);
  unsigned* counters = reinterpret_cast<unsigned*>(ws + kChainZeroOff + kWsCntOff);
  float* slots = reinterpret_cast<float*>(ws + kChainSlotsOff);
  const int ctas = d->sms < kDecMaxCtas ? d->sms : kDecMaxCtas;  // the cooperative grid
  const int warps_avail = ctas * kDecWarps;
  DecodeParams* host = new (std::nothrow) DecodeParams[size_t(n_layers)];
  if (!host) return W4A8_ERR_SHAPE;
  for (int64_t i = 0; i < n_layers; ++i) {
    const w4a8_chain_layer& L = layers[i];
    const PackedLayout PL = packed_layout(L.N, L.K);
    const uint8_t* pk = static_cast<const uint8_t*>(L.packed);
    DecodeParams p{};
    p.x = L.x;
    p.units = pk + PL.off_units;
    p.sch = reinterpret_cast<const float*>(pk + PL.off_sch);
    p.cb = reinterpret_cast<const float*>(pk + PL.off_cb);
    p.xfrag = nullptr;
    p.s_x = nullptr;
    p.y = L.y;
    p.slots = slots;
    p.xch = xch;
    p.counters = counters;
    p.err = d->err;
    p.M = 1;
    p.N = int(L.N);
    p.K = int(L.K);
    p.C = int(L.K / kChunkK);
    p.T = int(L.N / kTileRows);
    p.P = (p.T + kDecTG - 1) / kDecTG;
    p.U = p.P * p.C;
    p.W = p.U < warps_avail ? p.U : warps_avail;
    p.R = p.U / p.W;
    p.Rm = p.U % p.W;
    one_token_split(p, ctas);
    host[i] = p;
  }
  // From pageable memory: the call returns once the table has been staged.
  const cudaError_t e = cudaMemcpyAsync(plan, host, size_t(n_layers) * sizeof(DecodeParams),
                                        cudaMemcpyHostToDevice, static_cast<cudaStream_t>(stream));
  delete[] host;
  return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

w4a8_status w4a8_chain_run(const void* plan, int64_t n_layers, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (!plan || !workspace) return W4A8_ERR_NULL;
  if (n_layers < 1 || n_layers > (int64_t(1) << 20)) return W4A8_ERR_SHAPE;
  if (workspace_bytes < kChainSlotsOff) return W4A8_ERR_WORKSPACE;
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the barrier and the split-K counters start at zero
  const size_t zero = kChainSlotsOff;
  if (cudaMemsetAsync(workspace, 0, zero, s) != cudaSuccess) return W4A8_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(d->sms < kDecMaxCtas ? d->sms : kDecMaxCtas));
  cfg.blockDim = dim3(kOneThreads);
  cfg.dynamicSmemBytes = dec_smem_bytes(1, kMaxK, true);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the grid barrier can complete
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_chain_kernel, static_cast<const DecodeParams*>(plan),
                                           int(n_layers), static_cast<unsigned*>(workspace));
  return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

// ------------------------------------------------------------------ decode chains with fused activations

namespace {

constexpr int kActSets = 3;  // activation sets in rotation among producers

struct ActSetLayout {
  size_t rot_off, cnt_off, set_bytes, total;  // one set: [rot K_max fp32][cnt K_max/256 + amax]
  int cnt_words;
};

ActSetLayout act_sets(int64_t kmax) {
  ActSetLayout a{};
  a.cnt_words = int(kmax / kRotBlock) + 1;  // block counters, then the absmax word
  a.rot_off = 0;
  a.cnt_off = round_up(size_t(kmax) * 4, 256);
  a.set_bytes = round_up(a.cnt_off + size_t(a.cnt_words) * 4, 256);
  a.total = a.set_bytes * kActSets;
  return a;
}

// [0, kWsZeroBytes): exchange words and split-K counters (left at zero by
// every layer); then the per-CTA partial slots; then the activation sets.
constexpr size_t kDecChainSlotsOff = kWsZeroBytes;
constexpr size_t kDecChainSetsOff = kDecChainSlotsOff + (size_t(2) * kDecMaxCtas * kDecTG * 16 * 4 + 255) / 256 * 256;

struct ChainLink {
  int producer = -1;   // the layer whose output this layer reads (fused), or -1
  int64_t off = 0;     // producer: the outputs the consumers read start here
  int64_t len = 0;     // and are this many (0: not a producer)
  int set = -1;        // producer: its activation set
  int zero_set = -1;   // this layer clears that set (the next layer produces into it)
};

// Which layers read which earlier layer's output, and the sets.
void link_chain(const w4a8_chain_layer* L, int64_t n, ChainLink* link) {
  for (int64_t i = 0; i < n; ++i) {
    const uint16_t* x = L[i].x;
    // the latest earlier layer whose output range overlaps this input
    for (int64_t j = i - 1; j >= 0; --j) {
      const uint16_t* y = L[j].y;
      const bool overlaps = x < y + L[j].N && y < x + L[i].K;
      if (!overlaps) continue;
      const int64_t off = x - y;
      const bool inside = off >= 0 && off % kRotBlock == 0 && off + L[i].K <= L[j].N;
      if (inside && (link[j].len == 0 || (link[j].off == off && link[j].len == L[i].K))) {
        link[j].off = off;
        link[j].len = L[i].K;
        link[i].producer = int(j);
      }
      break;
    }
  }
  // sets in rotation; a set is cleared by the layer before its next producer,
  // so every reader of the set's previous contents must come before that
  std::vector<int64_t> producers;
  for (int64_t i = 0; i < n; ++i)
    if (link[i].len > 0) producers.push_back(i);
  for (size_t a = 0; a < producers.size(); ++a) link[producers[a]].set = int(a % kActSets);
  for (size_t a = 0; a + kActSets < producers.size(); ++a) {
    const int64_t next = producers[a + kActSets];  // the next producer into this set
    for (int64_t c = next - 1; c < n; ++c)
      if (link[c].producer == producers[a]) link[c].producer = -1;  // would read a cleared set: use x
  }
  for (size_t a = kActSets; a < producers.size(); ++a) link[producers[a] - 1].zero_set = link[producers[a]].set;
}

}  // namespace

size_t w4a8_decode_chain_workspace_bytes(const w4a8_chain_layer* layers, int64_t n_layers) {
  if (!layers || n_layers < 1) return 0;
  int64_t kmax = 0;
  for (int64_t i = 0; i < n_layers; ++i) {
    if (!weight_shape_ok(layers[i].N, layers[i].K)) return 0;
    kmax = layers[i].K > kmax ? layers[i].K : kmax;
  }
  return kDecChainSetsOff + act_sets(kmax).total;
}

w4a8_status w4a8_decode_chain(const w4a8_chain_layer* layers, int64_t n_layers, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!layers || !workspace) return W4A8_ERR_NULL;
  if (n_layers < 1 || n_layers > (int64_t(1) << 20)) return W4A8_ERR_SHAPE;
  int64_t kmax = 0;
  for (int64_t i = 0; i < n_layers; ++i) {
    const w4a8_chain_layer& L = layers[i];
    if (!L.packed || !L.x || !L.y) return W4A8_ERR_NULL;
    if (!weight_shape_ok(L.N, L.K)) return W4A8_ERR_SHAPE;
    if (!aligned16(L.packed) || !aligned16(L.x) || !aligned16(L.y)) return W4A8_ERR_ALIGN;
    kmax = L.K > kmax ? L.K : kmax;
  }
  if (!aligned16(workspace)) return W4A8_ERR_ALIGN;
  if (workspace_bytes < w4a8_decode_chain_workspace_bytes(layers, n_layers)) return W4A8_ERR_WORKSPACE;
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::vector<ChainLink> link(static_cast<size_t>(n_layers));
  link_chain(layers, n_layers, link.data());
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const ActSetLayout A = act_sets(kmax);
  uint8_t* sets = ws + kDecChainSetsOff;
  auto set_rot = [&](int k) { return reinterpret_cast<float*>(sets + k * A.set_bytes + A.rot_off); };
  auto set_cnt = [&](int k) { return reinterpret_cast<unsigned*>(sets + k * A.set_bytes + A.cnt_off); };
  // every set's counters and absmax start at zero
  for (int k = 0; k < kActSets; ++k)
    if (cudaMemsetAsync(set_cnt(k), 0, size_t(A.cnt_words) * 4, s) != cudaSuccess) return W4A8_ERR_CUDA;
  const int ctas = d->sms < kDecMaxCtas ? d->sms : kDecMaxCtas;
  for (int64_t i = 0; i < n_layers; ++i) {
    const w4a8_chain_layer& L = layers[i];
    const PackedLayout PL = packed_layout(L.N, L.K);
    const uint8_t* pk = static_cast<const uint8_t*>(L.packed);
    DecodeParams p{};
    p.x = L.x;
    p.units = pk + PL.off_units;
    p.sch = reinterpret_cast<const float*>(pk + PL.off_sch);
    p.cb = reinterpret_cast<const float*>(pk + PL.off_cb);
    p.y = L.y;
    p.slots = reinterpret_cast<float*>(ws + kDecChainSlotsOff);
    p.xch = reinterpret_cast<unsigned long long*>(ws);
    p.counters = reinterpret_cast<unsigned*>(ws + kWsCntOff);
    p.err = d->err;
    p.M = 1;
    p.N = int(L.N);
    p.K = int(L.K);
    p.C = int(L.K / kChunkK);
    p.T = int(L.N / kTileRows);
    p.P = (p.T + kDecTG - 1) / kDecTG;
    p.U = p.P * p.C;
    p.W = p.U < ctas * kDecWarps ? p.U : ctas * kDecWarps;
    p.R = p.U / p.W;
    p.Rm = p.U % p.W;
    one_token_split(p, ctas);
    const ChainLink& k = link[size_t(i)];
    if (k.len > 0) {
      p.act_rot = set_rot(k.set);
      p.act_cnt = set_cnt(k.set);
      p.act_amax = set_cnt(k.set) + (A.cnt_words - 1);
      p.act_off = int(k.off);
      p.act_len = int(k.len);
    }
    if (k.producer >= 0) {
      const int ps = link[size_t(k.producer)].set;
      p.in_rot = set_rot(ps);
      p.in_amax = set_cnt(ps) + (A.cnt_words - 1);
    }
    if (k.zero_set >= 0) {
      p.zero_cnt = set_cnt(k.zero_set);
      p.zero_n = A.cnt_words;
    }
    const size_t smem = dec_smem_bytes(1, p.K, true);
    cudaError_t e;
    if (!p.in_rot && p.K > kDecPairK)
      e = launch_pdl_cluster(decode_one_kernel<true>, dim3((unsigned(p.G) + 1) & ~1u), dim3(kOneThreads), 2, smem, s,
                             p);
    else
      e = launch_pdl(decode_one_kernel<true>, dim3(unsigned(p.G)), dim3(kOneThreads), smem, s, p);
    if (e != cudaSuccess) return W4A8_ERR_CUDA;
  }
  return W4A8_OK;
}

// ------------------------------------------------------------------ fidelity checks

// ------------------------------------------------------------------ NVFP4 comparison layer

#ifndef W4A8_NV_PREFILL_NT
#define W4A8_NV_PREFILL_NT 128
#endif
#ifndef W4A8_NV_PREFILL_CPS
#define W4A8_NV_PREFILL_CPS 2
#endif
constexpr int kNvPrefillNT = W4A8_NV_PREFILL_NT;    // token tile beyond 128 tokens
constexpr int kNvPrefillCPS = W4A8_NV_PREFILL_CPS;  // its CTAs per SM
static_assert((kNvPrefillNT == 256 && kNvPrefillCPS == 1) || (kNvPrefillNT == 128 && kNvPrefillCPS <= 2),
              "a compiled prefill configuration");

static bool nv_shape_ok(int64_t R, int64_t K) {
  return R > 0 && R <= (int64_t(1) << 24) && K > 0 && K % kNvBK == 0 && K <= kMaxK;
}

size_t w4a8_nvfp4_scale_bytes(int64_t R, int64_t K) { return nv_shape_ok(R, K) ? nv_sf_bytes(R, K) : 0; }

static w4a8_status nv_quantize(const void* x, int32_t x_is_f32, int64_t R, int64_t K, int32_t rotate,
                               unsigned* amax_word, uint8_t* codes, uint8_t* scales, float* g, cudaStream_t s) {
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  NvQuantParams p;
  p.x = x;
  p.amax_word = amax_word;
  p.codes = codes;
  p.sf = scales;
  p.g = g;
  p.R = int(R);
  p.K = int(K);
  p.in_f32 = x_is_f32 ? 1 : 0;
  p.rotate = rotate ? 1 : 0;
  if (amax_word) {
    if (cudaMemsetAsync(amax_word, 0, sizeof(unsigned), s) != cudaSuccess) return W4A8_ERR_CUDA;
    const unsigned grid = unsigned(std::min<int64_t>(R, int64_t(d->sms) * 8));
    nvfp4_amax_kernel<<<grid, kNvQuantThreads, 0, s>>>(p, amax_word);
    if (launch_status() != W4A8_OK) return W4A8_ERR_CUDA;
  }
  const unsigned rows = unsigned((R + 127) / 128 * 128);
  const cudaError_t e = launch_pdl(nvfp4_quant_kernel, dim3(rows), dim3(kNvQuantThreads), size_t(K) * 4, s, p);
  return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

w4a8_status w4a8_nvfp4_quantize(const void* x, int32_t x_is_f32, int64_t R, int64_t K, int32_t rotate,
                                int32_t per_tensor, uint8_t* codes, uint8_t* scales, float* g,
                                unsigned* amax_scratch, void* stream) {
  if (!x || !codes || !scales || !g || (per_tensor && !amax_scratch)) return W4A8_ERR_NULL;
  if (!nv_shape_ok(R, K)) return W4A8_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(g) ||
      (per_tensor && !aligned16(amax_scratch)))
    return W4A8_ERR_ALIGN;
  return nv_quantize(x, x_is_f32, R, K, rotate, per_tensor ? amax_scratch : nullptr, codes, scales, g,
                     static_cast<cudaStream_t>(stream));
}

w4a8_status w4a8_nvfp4_pack_scales(const uint8_t* scales_rows, int64_t R, int64_t K, uint8_t* scales,
                                   void* stream) {
  if (!scales_rows || !scales) return W4A8_ERR_NULL;
  if (!nv_shape_ok(R, K)) return W4A8_ERR_SHAPE;
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  const int64_t total = int64_t(nv_sf_bytes(R, K));
  const unsigned blocks = unsigned(std::min<int64_t>((total + 255) / 256, int64_t(d->sms) * 8));
  nvfp4_pack_scales_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(scales_rows, int(R), int(K),
                                                                                  scales);
  return launch_status();
}

static w4a8_status nv_gemm(const uint8_t* x_codes, const uint8_t* x_scales, const float* g_x, int64_t M,
                           const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w, int64_t N, int64_t K,
                           uint16_t* y, const DeviceState* d, cudaStream_t s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return W4A8_ERR_CUDA;
  // token tile: 64 / 128 for few tokens (one CTA per SM); beyond, the prefill tile
  const int nt = M > 128 ? kNvPrefillNT : M > 64 ? 128 : 64;
  const int cps = M > 128 ? kNvPrefillCPS : 1;
  CUtensorMap tw, tx;
  const cuuint64_t gw_dim[2] = {cuuint64_t(K / 2), cuuint64_t(N)};
  const cuuint64_t gx_dim[2] = {cuuint64_t(K / 2), cuuint64_t(M)};
  const cuuint64_t gstride[1] = {cuuint64_t(K / 2)};
  const cuuint32_t box_w[2] = {128u, uint32_t(kNvRows)};
  const cuuint32_t box_x[2] = {128u, uint32_t(nt)};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(w_codes), gw_dim, gstride, box_w, estride,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
      enc(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(x_codes), gx_dim, gstride, box_x, estride,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return W4A8_ERR_CUDA;
  NvGemmParams p;
  p.sfa = w_scales;
  p.sfb = x_scales;
  p.gw = g_w;
  p.gx = g_x;
  p.y = y;
  p.err = d->err;
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  const dim3 grid(unsigned((N + kNvRows - 1) / kNvRows), unsigned((M + nt - 1) / nt));
  cudaError_t e;
  if (nt == 256)
    e = launch_pdl(nvfp4_gemm_kernel<256>, grid, dim3(kNvThreads), NvCfg<256>::kSmem, s, tw, tx, p);
  else if (nt == 128 && cps == 2)
    e = launch_pdl(nvfp4_gemm_kernel<128, 2>, grid, dim3(kNvThreads), NvCfg<128, 2>::kSmem, s, tw, tx, p);
  else if (nt == 128)
    e = launch_pdl(nvfp4_gemm_kernel<128>, grid, dim3(kNvThreads), NvCfg<128>::kSmem, s, tw, tx, p);
  else
    e = launch_pdl(nvfp4_gemm_kernel<64>, grid, dim3(kNvThreads), NvCfg<64>::kSmem, s, tw, tx, p);
  return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

// The GEMM's grid has one y index per token tile (up to 128 tokens each): at most 65535.
constexpr int64_t kNvMaxTokens = int64_t(65535) * 128;

w4a8_status w4a8_nvfp4_gemm(const uint8_t* x_codes, const uint8_t* x_scales, const float* g_x, int64_t M,
                            const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w, int64_t N, int64_t K,
                            uint16_t* y, void* stream) {
  if (!x_codes || !x_scales || !g_x || !w_codes || !w_scales || !g_w || !y) return W4A8_ERR_NULL;
  if (!nv_shape_ok(M, K) || !nv_shape_ok(N, K) || M > kNvMaxTokens) return W4A8_ERR_SHAPE;
  if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(y))
    return W4A8_ERR_ALIGN;
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  return nv_gemm(x_codes, x_scales, g_x, M, w_codes, w_scales, g_w, N, K, y, d, static_cast<cudaStream_t>(stream));
}

struct NvLinearWs {
  size_t off_codes, off_sf, off_g, total;
};
static NvLinearWs nv_linear_ws(int64_t M, int64_t K) {
  NvLinearWs w;
  w.off_codes = 0;
  w.off_sf = round_up(size_t(M) * size_t(K / 2), 256);
  w.off_g = w.off_sf + round_up(nv_sf_bytes(M, K), 256);
  w.total = w.off_g + round_up(size_t(M) * 4, 256);
  return w;
}

size_t w4a8_nvfp4_linear_workspace_bytes(int64_t M, int64_t K) {
  return nv_shape_ok(M, K) ? nv_linear_ws(M, K).total : 0;
}

w4a8_status w4a8_nvfp4_linear(const uint16_t* x, int64_t M, int64_t K, const uint8_t* w_codes,
                              const uint8_t* w_scales, const float* g_w, int64_t N, uint16_t* y, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!x || !w_codes || !w_scales || !g_w || !y || !workspace) return W4A8_ERR_NULL;
  if (!nv_shape_ok(M, K) || !nv_shape_ok(N, K) || M > kNvMaxTokens) return W4A8_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(y) || !aligned16(workspace))
    return W4A8_ERR_ALIGN;
  const NvLinearWs w = nv_linear_ws(M, K);
  if (workspace_bytes < w.total) return W4A8_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  float* gx = reinterpret_cast<float*>(ws + w.off_g);
  if (w4a8_status st = nv_quantize(x, 0, M, K, 1, nullptr, ws + w.off_codes, ws + w.off_sf, gx, s); st != W4A8_OK)
    return st;
  return nv_gemm(ws + w.off_codes, ws + w.off_sf, gx, M, w_codes, w_scales, g_w, N, K, y, d, s);
}

size_t w4a8_compare_workspace_bytes(void) { return size_t(kCmpBlocks) * 3 * sizeof(double); }

w4a8_status w4a8_compare(const void* a, int32_t a_is_bf16, const float* ref, int64_t n, double* out,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (!a || !ref || !out || !workspace) return W4A8_ERR_NULL;
  if (n < 1) return W4A8_ERR_SHAPE;
  if (workspace_bytes < w4a8_compare_workspace_bytes()) return W4A8_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(out) & 7u) || (reinterpret_cast<uintptr_t>(workspace) & 7u)) return W4A8_ERR_ALIGN;
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double* part = static_cast<double*>(workspace);
  if (a_is_bf16) compare_kernel<true><<<kCmpBlocks, kCmpThreads, 0, s>>>(a, ref, n, part);
  else compare_kernel<false><<<kCmpBlocks, kCmpThreads, 0, s>>>(a, ref, n, part);
  compare_final_kernel<<<1, 32, 0, s>>>(part, out);
  return launch_status();
}

w4a8_status w4a8_dense_reference(const uint16_t* x, int64_t M, int64_t K, const float* w, int64_t N, float* y,
                                 void* stream) {
  if (!x || !w || !y) return W4A8_ERR_NULL;
  if (M < 1 || M > (int64_t(1) << 24) || K < 1 || N < 1 || N > (int64_t(1) << 30)) return W4A8_ERR_SHAPE;
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  dense_reference_kernel<<<unsigned((N + kRefWarps - 1) / kRefWarps), kRefWarps * 32, 0,
                           static_cast<cudaStream_t>(stream)>>>(x, M, K, w, N, y);
  return launch_status();
}

w4a8_status w4a8_selftest_timeout(void* stream) {
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(d->err, 1024u);
  return launch_status();
}

w4a8_status w4a8_get_device_error(void* stream) {
  DeviceState* d = nullptr;
  if (w4a8_status st = device_state(&d); st != W4A8_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return W4A8_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(v)) != cudaSuccess) return W4A8_ERR_CUDA;
  if (v) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return W4A8_ERR_CUDA;
  }
  if (v & kErrTimeout) return W4A8_ERR_TIMEOUT;
  return (v & kErrInput) ? W4A8_ERR_INPUT : W4A8_OK;
}

const char* w4a8_status_string(w4a8_status status) {
  switch (status) {
    case W4A8_OK: return "ok";
    case W4A8_ERR_NULL: return "a required pointer is NULL";
    case W4A8_ERR_SHAPE: return "shape outside the supported rules (K % 256, N % 16, K <= 32768, M, N > 0)";
    case W4A8_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case W4A8_ERR_WORKSPACE: return "buffer smaller than the size function requires";
    case W4A8_ERR_CUDA: return "a CUDA call failed";
    case W4A8_ERR_TIMEOUT: return "a bounded device wait gave up";
    case W4A8_ERR_ARCH: return "the current device is not sm_100";
    case W4A8_ERR_INPUT: return "a device-side input check failed";
  }
  return "unknown status";
}

}  // extern "C"
