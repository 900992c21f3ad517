/*
 * w4a8.h -- C ABI of the asym_w4a8_int8 ConvRot linear layer on NVIDIA B200
 * (sm_100a).
 *
 * The layer computes y = x * W_hat^T where
 *   - x[M, K] are bf16 activations, rotated per 256-block of K by the
 *     normalised Sylvester Hadamard matrix H_256 / 16 and quantised to int8
 *     per token (symmetric absmax / 127, round half to even);
 *   - W_hat[n, k] = codebook[idx[n, k]] * s_rel[n, k / 16] * s_channel[n] is
 *     the weight in the same rotated basis, rebuilt from four stored tensors:
 *     packed 4-bit indices, fp8 e4m3 group scales (one per 16 values), fp32
 *     row scales and a 16-entry fp32 codebook.
 * Sources: "Qwen3.8-27B-AEON-ULTIMATE-UNCENSORED-BF16 -- W4A8 ConvRot for
 * ComfyUI" model card, sections "Why this exists" and "Format" (the four
 * tensors, three tiers of scaling, rotation group 256, codebook group 16);
 * "Qwen3.8-27B-W4A8" model card, section "Model Overview" (group sizes,
 * int8 activations, per-group fp8 scales, fp32 channel scales).
 *
 * Conventions for every call below:
 *   - All buffer pointers are DEVICE pointers owned by the caller.  The
 *     library allocates no device memory and keeps no reference to any
 *     buffer after the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Work is enqueued on it asynchronously; no call synchronises
 *     except w4a8_get_device_error.
 *   - Arguments are checked on the host before anything is launched.  On a
 *     failed check nothing is launched and the status says why.
 *   - Shapes: K must be a multiple of 256 (the rotation block; a layer whose
 *     input width is not, such as 4304 = 16 x 269, stays unquantised on the
 *     pages) and at most W4A8_MAX_K; N must be a positive multiple of 16,
 *     at most 2^24; M must be positive and at most 16 776 960 (65535 tiles of
 *     256 tokens).
 *   - Every pointer must be 16-byte aligned.
 *   - The calls run on the current CUDA device, which must be sm_100.
 */
#ifndef W4A8_H_
#define W4A8_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define W4A8_ROT_BLOCK 256   /* rotation block along K */
#define W4A8_GROUP 16        /* values per fp8 group scale */
#define W4A8_LEVELS 16       /* codebook entries */
#define W4A8_MAX_K 32768     /* largest supported K */

typedef enum w4a8_status {
  W4A8_OK = 0,
  W4A8_ERR_NULL = 1,       /* a required pointer is NULL */
  W4A8_ERR_SHAPE = 2,      /* M, N or K outside the rules above */
  W4A8_ERR_ALIGN = 3,      /* a pointer is not 16-byte aligned */
  W4A8_ERR_WORKSPACE = 4,  /* a buffer is smaller than the size function says */
  W4A8_ERR_CUDA = 5,       /* a CUDA call failed (launch or device query) */
  W4A8_ERR_TIMEOUT = 6,    /* a bounded device wait gave up (see get_device_error) */
  W4A8_ERR_ARCH = 7,       /* the current device is not sm_100 */
  W4A8_ERR_INPUT = 8       /* a device-side input check failed (see get_device_error) */
} w4a8_status;

/*
 * Size in bytes of the device layout produced by w4a8_pack_layout for an
 * [N, K] weight, or 0 if (N, K) break the shape rules.  About 0.5625 bytes
 * per weight (0.5 for the indices, 1/16 for the group scales) plus 4 bytes
 * per row and 64 bytes for the codebook, each region padded to 256 bytes;
 * rows are stored in blocks of 32, so an N that is an odd multiple of 16
 * carries 16 rows of zero padding.
 */
size_t w4a8_packed_bytes(int64_t N, int64_t K);

/*
 * Re-lay the four stored tensors of one layer into the library's device
 * layout (ConvRot card, "Format": the four tensors of a quantised layer).
 *   idx        [N, K/2] uint8, row-major.  Byte c of row n holds the index
 *              of k = 2c in its low nibble and of k = 2c + 1 in its high
 *              nibble ("packed int4 indices, two per byte").
 *   s_rel      [N, K/16] uint8, row-major: e4m3fn bit patterns, one per
 *              group of 16 consecutive k.
 *   s_channel  [N] fp32: one scale per output row.
 *   codebook   [16] fp32: the levels the indices point into.
 *   packed     output, `packed_bytes` >= w4a8_packed_bytes(N, K).  Its
 *              content is opaque; it is read by w4a8_unpack_dequant and
 *              w4a8_linear.
 * Errors: NULL, SHAPE, ALIGN, WORKSPACE (packed_bytes too small), CUDA.
 */
w4a8_status w4a8_pack_layout(const uint8_t* idx, const uint8_t* s_rel,
                             const float* s_channel, const float* codebook,
                             int64_t N, int64_t K, void* packed,
                             size_t packed_bytes, void* stream);

/*
 * Rebuild the weight in the rotated basis (ConvRot card, "Format": "three
 * tiers of scaling -- codebook shape, group magnitude, row magnitude"):
 *   w_hat[n, k] = fp32(fp32(codebook[idx[n,k]] * s_rel[n, k/16]) * s_channel[n])
 * with both products rounded to nearest even (bit-exact).
 *   packed  a buffer filled by w4a8_pack_layout for the same (N, K).
 *   w_hat   output [N, K] fp32, row-major.
 * Errors: NULL, SHAPE, ALIGN, CUDA.
 */
w4a8_status w4a8_unpack_dequant(const void* packed, int64_t N, int64_t K,
                                float* w_hat, void* stream);

/*
 * Rotate and quantise activations (ConvRot card, "Format": group-wise
 * Hadamard rotation, group 256; "Qwen3.8-27B-W4A8" card, "Model Overview":
 * int8 activations):
 *   x_rot[m, 256b + j] = (1/16) * sum_i x[m, 256b + i] * H_256[i, j]
 *   s_x[m]             = max_k |x_rot[m, k]| / 127           (fp32)
 *   x_q[m, k]          = clamp(round_half_even(x_rot / s_x), -127, 127)
 * The rotation runs in fp32; an all-zero token gives s_x = 0 and x_q = 0.
 *   x    [M, K] bf16 bit patterns (uint16), row-major.
 *   x_q  output [M, K] int8, row-major.
 *   s_x  output [M] fp32.
 * Errors: NULL, SHAPE, ALIGN, CUDA.
 */
w4a8_status w4a8_rotate_quant_act(const uint16_t* x, int64_t M, int64_t K,
                                  int8_t* x_q, float* s_x, void* stream);

/*
 * Bytes of device workspace w4a8_linear needs for (M, K, N), or 0 if the
 * shape breaks the rules.  The workspace holds the quantised activations,
 * their scales, the split-K partial sums and, at its start, the words that
 * join partial sums across CTAs (arrival counters, exchange words).  Fill a
 * new workspace with zeros before its first use (for example
 * cudaMemsetAsync): the decode kernel needs those words at zero when it
 * starts, and every completed call leaves them at zero again.  They sit at
 * the same offsets, with the same size, for every shape and nothing else
 * writes there, so one workspace may serve calls of different shapes.
 * After a call that reported W4A8_ERR_TIMEOUT, zero the workspace again.
 * Everything else in it is scratch between calls.
 */
size_t w4a8_linear_workspace_bytes(int64_t M, int64_t K, int64_t N);

/*
 * The layer: y[m, n] = bf16( s_x[m] * sum_k x_q[m,k] * W_hat[n,k] ), the
 * sum accumulated in fp32 (ConvRot card, "Why this exists": the 4-bit
 * weights are re-read on every token; "Format": the three scaling tiers).
 *   x          [M, K] bf16 bit patterns (uint16), row-major.
 *   packed     a buffer filled by w4a8_pack_layout for the same (N, K).
 *   y          output [M, N] bf16 bit patterns (uint16), row-major.
 *   workspace  scratch of at least w4a8_linear_workspace_bytes(M, K, N).
 * M <= 64 runs the decode kernel (a weight-streaming GEMV: one launch for
 * up to 16 tokens, else one per slice of up to 32); larger M runs the
 * tensor-core GEMM, except that
 * 65 <= M <= 256 on a layer of fewer than 100 row tiles of 128 (where the
 * GEMM would leave most SMs idle) runs a small-batch tensor-core kernel
 * that splits the weight stream over every SM.  For one token a single
 * kernel rotates, quantises and applies the layer (every CTA quantises the
 * token itself, with the activation kernel's arithmetic); otherwise the call
 * is w4a8_linear_prepare followed by w4a8_linear_run.  Two calls sharing one
 * workspace must be ordered on the GPU (same stream, or synchronised).
 * Errors: NULL, SHAPE, ALIGN, WORKSPACE, ARCH, CUDA.
 */
w4a8_status w4a8_linear(const uint16_t* x, int64_t M, int64_t K,
                        const void* packed, int64_t N, uint16_t* y,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * w4a8_linear for an input that another engine delivers (ConvRot card, "Why
 * this exists": a decode step is bound by streaming memory, so its host
 * transfers should overlap the previous layer).  Instead of a stream
 * dependency on the copy that brings x, the call's first kernel waits on the
 * GPU until x_ready[0] != 0, and once every CTA of that kernel has seen it,
 * clears x_ready[0] and x_ready[1] (an arrival count).  The caller copies x
 * and then writes a non-zero word to x_ready[0] (for example a second
 * cudaMemcpyAsync on the copy stream, which orders it after the data), and
 * orders its next write of the same x, x_ready and y after this call
 * (events on the compute stream).  A compute stream holding only kernels
 * keeps the overlap of consecutive layers (programmatic dependent launch);
 * a kernel that also waits on a copy event loses it (measured: 18.5 vs
 * 14.2 us per one-token step).
 *   x_ready  device, 2 words, 8-byte aligned, [1] zero before the first call;
 *            a buffer set per call in flight.  The wait is bounded (about a
 *            second); if it runs out, w4a8_get_device_error reports
 *            W4A8_ERR_TIMEOUT and the output is undefined.
 * For one token the layer's single kernel waits (before its wait for the
 * previous kernel, so the two overlap); otherwise a one-thread kernel waits
 * and then w4a8_linear_prepare and w4a8_linear_run follow.
 * Other arguments and errors as w4a8_linear.
 */
w4a8_status w4a8_linear_flagged(const uint16_t* x, int64_t M, int64_t K,
                                const void* packed, int64_t N, uint16_t* y,
                                unsigned* x_ready, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * Writes 1 to x_ready[0] in stream order: after everything issued earlier on
 * `stream` (in particular the copy that brings x), with the ordering of a
 * stream write of the driver (cuStreamWriteValue32, default flags: earlier
 * writes of the stream are visible first).  The companion of
 * w4a8_linear_flagged for a caller whose copy stream should carry x alone:
 * the word is written by the stream itself, not copied from host memory.
 * Can be captured into a CUDA graph.
 *   x_ready  device, 2 words, 8-byte aligned (as for w4a8_linear_flagged);
 *            only word 0 is written.
 * Errors: W4A8_ERR_NULL, W4A8_ERR_ALIGN before anything is issued;
 * W4A8_ERR_CUDA if the driver lacks the call or refuses it.
 */
w4a8_status w4a8_signal_ready(unsigned* x_ready, void* stream);

/*
 * The two halves of w4a8_linear, for callers that apply several layers of
 * the same shape to one activation or that time the GEMM on its own.
 *
 * w4a8_linear_prepare: rotate and quantise x [M, K] (bf16 bits) into
 *   `workspace`, laid out for a layer of N output rows (ConvRot card,
 *   "Format": group-256 Hadamard rotation; W4A8 card, "Model Overview": int8
 *   activations).
 * w4a8_linear_run: y [M, N] = the layer applied to the activations the last
 *   prepare on this workspace wrote.  It must be called with the same (M, K,
 *   N) as that prepare, may be called any number of times after it (each run
 *   leaves the workspace ready for another), and must be ordered after it on
 *   the GPU.
 * Errors: as w4a8_linear.
 */
w4a8_status w4a8_linear_prepare(const uint16_t* x, int64_t M, int64_t K, int64_t N,
                                void* workspace, size_t workspace_bytes, void* stream);
w4a8_status w4a8_linear_run(int64_t M, int64_t K, const void* packed, int64_t N,
                            uint16_t* y, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * w4a8_linear for decode sizes (M <= 16) without any caller-provided
 * workspace.  The pages have no counterpart to this call; it exists for
 * callers that cannot allocate device memory where they run the layer: a
 * plugin whose host application owns the device heap and hands it no
 * scratch, code on a latency-critical path that must not allocate
 * (cudaMalloc can synchronise the whole device), or a host program that
 * drives the library through a foreign-function interface with no device
 * allocator of its own.
 *
 * Instead of a workspace it uses a scratch array built into the library: a
 * file-scope __device__ array of W4A8_STATIC_SCRATCH_BYTES (2 MiB; the
 * largest plan, M = 16 at K = W4A8_MAX_K, needs about 1.62 MiB), which every
 * GPU that loads the library holds until the process exits.  The call
 * allocates nothing and calls no allocating routine.  Its first call on a
 * device looks up the array's device address once (cudaGetSymbolAddress,
 * with that device current, after the architecture check); make that first
 * call before any stream capture.  All calls on a device share the one
 * array and leave their scratch in it: calls whose work overlaps on the GPU
 * (different streams without ordering, or other host threads) race and give
 * wrong results, so order them.  Each call runs the activation kernel, which
 * clears the words the decode kernel needs at zero (exchange words and
 * arrival counters), and then the decode kernel (one token too); so a call
 * that reported W4A8_ERR_TIMEOUT needs no reset before the next one.
 *   x, packed, y  as for w4a8_linear (device pointers owned by the caller).
 * Limits: M <= 16 (larger M returns W4A8_ERR_SHAPE); a shape needing more
 * scratch than the array holds would return W4A8_ERR_WORKSPACE (no accepted
 * (N, K) does at M <= 16).
 * Errors: NULL, SHAPE, WORKSPACE, ALIGN, ARCH, CUDA.
 */
#define W4A8_STATIC_SCRATCH_BYTES (2u << 20)
w4a8_status w4a8_linear_decode_static(const uint16_t* x, int64_t M, int64_t K,
                                      const void* packed, int64_t N, uint16_t* y,
                                      void* stream);

/*
 * A chain of one-token layers in one persistent launch: a decode step, where
 * each layer's input is an earlier layer's output (ConvRot card, "Why this
 * exists": a decode step re-reads every layer's weights for one token).
 * Layer i computes y_i = w4a8_linear(x_i) for M = 1, with every CTA
 * rotating and quantising x_i itself; between layers a grid barrier makes
 * the previous layer's y visible, and each layer's weights are fetched
 * before that barrier.  Results equal the layer-by-layer w4a8_linear calls
 * bit for bit.
 *   layers     host array of n_layers descriptors: packed (w4a8_pack_layout
 *              buffer for (N, K)), x (device, K bf16), y (device, N bf16).
 *              An x may be an earlier layer's y (or part of it).  Layers run
 *              strictly in order (a grid barrier separates them), so a later
 *              layer may also overwrite a buffer that an earlier one read.
 * w4a8_chain_plan: check the layers and write their launch table into
 *   `plan` (device, w4a8_chain_plan_bytes(n) bytes; the call returns once
 *   the table has been staged) for the given `workspace` (device,
 *   w4a8_chain_workspace_bytes(layers, n) bytes, owned by the caller).
 * w4a8_chain_run: run the planned chain on `stream` (capturable in a CUDA
 *   graph; zeroes the workspace's barrier and counters first).  The launch
 *   is cooperative (one CTA per SM, all resident); W4A8_ERR_CUDA if the
 *   device cannot host it.  Two runs sharing a workspace must be ordered.
 * Errors: NULL, SHAPE, ALIGN, WORKSPACE, ARCH, CUDA; a grid-barrier wait
 * that gives up is reported by w4a8_get_device_error as W4A8_ERR_TIMEOUT.
 */
typedef struct {
  const void* packed;
  int64_t N, K;
  const uint16_t* x;
  uint16_t* y;
} w4a8_chain_layer;

size_t w4a8_chain_plan_bytes(int64_t n_layers);
size_t w4a8_chain_workspace_bytes(const w4a8_chain_layer* layers, int64_t n_layers);
w4a8_status w4a8_chain_plan(const w4a8_chain_layer* layers, int64_t n_layers, void* plan,
                            size_t plan_bytes, void* workspace, size_t workspace_bytes,
                            void* stream);
w4a8_status w4a8_chain_run(const void* plan, int64_t n_layers, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * A decode step as one launch per one-token layer, each layer quantising the
 * next layer's activation in its own epilogue (ConvRot card, "Why this
 * exists": a decode step re-reads every layer's weights for one token, so
 * the per-layer work besides that stream must shrink).  The layers are the
 * chain descriptors above.  A layer whose input x lies inside an earlier
 * layer's output y (at a multiple of 256 elements, wholly inside, and
 * written by no layer in between) reads that output already rotated: the
 * producing layer rotates each 256-block of the consumer's input as soon as
 * all its rows are written (the last writer of the block does it) and keeps
 * the running absmax, so the consumer only quantises (same arithmetic, so
 * the same codes and s_x as w4a8_linear on the same bf16 x).  Other layers
 * rotate their x themselves.  Results equal the layer-by-layer w4a8_linear
 * calls bit for bit; y buffers are written as those calls would.
 *   layers     host array of n_layers descriptors (as for w4a8_chain_plan),
 *              run strictly in order.
 *   workspace  device, w4a8_decode_chain_workspace_bytes(layers, n) bytes,
 *              zero-filled before its first use (like a w4a8_linear
 *              workspace: its first 38,656 bytes must be zero when a call
 *              starts, and every completed call leaves them so).
 * The call issues one small memset and one kernel launch per layer on
 * `stream` (capturable in a CUDA graph).  Two calls sharing a workspace must
 * be ordered.  Errors: NULL, SHAPE, ALIGN, WORKSPACE, ARCH, CUDA.
 */
size_t w4a8_decode_chain_workspace_bytes(const w4a8_chain_layer* layers, int64_t n_layers);
w4a8_status w4a8_decode_chain(const w4a8_chain_layer* layers, int64_t n_layers, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * Weight converter on the GPU: fp32 W [N, K] -> the four stored tensors
 * (ConvRot card, "Format": rotate by the group-256 Hadamard, a per-row scale
 * and a per-16 e4m3 scale, 16-level Lloyd-Max codebook, two indices per
 * byte; "Reproducing": the codebook fit samples the values with a fixed
 * seed).  Per row, in fp64:
 *   R = W rotated (each 256-block times H_256 / 16)
 *   s_channel[n]  = fp32(max_k |R[n,k]|)
 *   s_rel[n, g]   = e4m3 (round half to even, saturating) of
 *                   max_{k in g} |R[n,k]| / s_channel[n]   (0 if s_channel is 0)
 *   v[n, k]       = R[n,k] / (s_rel[n, g] * s_channel[n])  (0 where that is 0)
 *   idx[n, k]     = the number of midpoints between consecutive codebook
 *                   levels that are strictly below v (a value on a midpoint
 *                   takes the lower level)
 * With `codebook_in` given (16 fp32 levels, strictly ascending) those levels
 * are used.  With `codebook_in` NULL the levels are fitted first (Lloyd-Max):
 * the fit uses v at `sample_pos` (n_sample flat positions n*K + k, each a
 * position whose group scale and row scale are non-zero; the caller draws
 * them), or every such value when `sample_pos` is NULL; it starts at the
 * sample's (i + 1/2)/16 quantiles (linear interpolation between order
 * statistics) and alternates boundaries = level midpoints (a value on a
 * midpoint belongs to the lower cell) and level = mean of its cell (an empty
 * cell keeps its level) until no level moves by `tol` or after `max_iter`
 * rounds.  Cell sums are exact (128-bit fixed point).
 *   w            [N, K] fp32, row-major, 16-byte aligned.
 *   idx_packed   out [N, K/2] uint8 (low nibble = even k).
 *   s_rel        out [N, K/16] uint8 e4m3fn codes.
 *   s_channel    out [N] fp32.
 *   codebook_out out [16] fp32 (the fitted levels, or a copy of codebook_in).
 *   fit_rounds   out, device int32 (rounds the fit took; 0 when given), or NULL.
 *   workspace    w4a8_convert_workspace_bytes(N, K, n_sample) bytes (only
 *                the fit uses it; n_sample <= 0 sizes it for every value).
 * Errors: NULL, SHAPE, ALIGN, WORKSPACE, ARCH, CUDA; an out-of-range sample
 * position or an empty sample is reported by w4a8_get_device_error as
 * W4A8_ERR_INPUT.
 */
size_t w4a8_convert_workspace_bytes(int64_t N, int64_t K, int64_t n_sample);
w4a8_status w4a8_convert_weight(const float* w, int64_t N, int64_t K, const float* codebook_in,
                                const int64_t* sample_pos, int64_t n_sample, int32_t max_iter,
                                double tol, uint8_t* idx_packed, uint8_t* s_rel,
                                float* s_channel, float* codebook_out, int32_t* fit_rounds,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * Fidelity checks of a stored layer (ConvRot card, "Verification": a stored
 * layer's dequantised weights compared with a fresh quantisation of the same
 * source tensor, expected ~0; "Accuracy": the quantised layer's output
 * against the full-precision one, ~1 %).  The binding's verify_layer
 * composes them with w4a8_convert_weight, w4a8_unpack_dequant and
 * w4a8_linear.
 *
 * w4a8_compare: out[0] = sum_i (a[i] - ref[i])^2, out[1] = sum_i ref[i]^2,
 *   out[2] = max_i |a[i] - ref[i]|, all in fp64 (device memory, 8-byte
 *   aligned).  a is fp32 (a_is_bf16 = 0) or bf16 bit patterns (1); ref is
 *   fp32; n values each.  The reduction order is fixed (same result on every
 *   call and device).  workspace: w4a8_compare_workspace_bytes() bytes.
 *   Errors: NULL, SHAPE, WORKSPACE, ALIGN, ARCH, CUDA.
 * w4a8_dense_reference: y [M, N] fp32 = x [M, K] (bf16 bits) times W^T
 *   (W [N, K] fp32, unquantised, original basis), each sum in fp64 then
 *   rounded once.  Errors: NULL, SHAPE, ARCH, CUDA.
 */
size_t w4a8_compare_workspace_bytes(void);
w4a8_status w4a8_compare(const void* a, int32_t a_is_bf16, const float* ref, int64_t n,
                         double* out, void* workspace, size_t workspace_bytes, void* stream);
w4a8_status w4a8_dense_reference(const uint16_t* x, int64_t M, int64_t K, const float* w,
                                 int64_t N, float* y, void* stream);

/* ------------------------------------------------------------------------
 * NVFP4 comparison layer (the speed and accuracy foil of the codebook layer)
 *
 * Format: "Qwen3.8-27B-Uncensored-NVFP4: En runbook för servering på
 * Blackwell-GPU:er", section "Vad NVFP4 är, och hur det skiljer sig från FP8
 * och från INT8/AWQ": E2M1 values (1 sign, 2 exponent, 1 mantissa bit), one
 * e4m3 scale per 16 values, one fp32 scalar per tensor; Blackwell runs the
 * FP4 matmul natively.  Both operands are 4-bit here (the native block-scaled
 * FP4 tensor-core instruction takes FP4 on both sides).  Readings taken where
 * the page is silent: E2M1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; round to
 * nearest even, saturating; g = amax / (6 * 448); weights one g per tensor,
 * activations one g per token; both operands rotated like the codebook layer
 * (each 256-block of K times H_256 / 16).  In fp32: d = g * 6, block scale
 * s = e4m3(bmax / d), S = value(s) * g, code = e2m1(x / S) (0 where S = 0).
 *
 * Layouts (all device memory, caller-owned):
 *   codes   uint8 [R, K/2]: two codes per byte, even k in the low nibble.
 *   scales  uint8 e4m3 codes in the tensor cores' order, rows padded to a
 *           multiple of 128 (w4a8_nvfp4_scale_bytes): 512-byte chunks of 128
 *           rows x 64 k in [row block][k/64] order; inside a chunk the scale
 *           of (row r, 16-block c) is byte 16 (r % 32) + 4 ((r % 128) / 32)
 *           + c % 4.  Pad rows hold 0.
 *   g       fp32 [R].
 * Shapes: R, N in [1, 2^24]; M in [1, 8 388 480] (65535 tiles of 128
 * tokens); K a multiple of 256, at most W4A8_MAX_K.
 * Pointers 16-byte aligned.  Calls are asynchronous on `stream`.
 * ------------------------------------------------------------------------ */

/* Bytes of a scale buffer for R rows of K values (0 for a bad shape). */
size_t w4a8_nvfp4_scale_bytes(int64_t R, int64_t K);

/*
 * Quantise R rows of x [R, K] (bf16 bits when x_is_f32 == 0, else fp32) to
 * NVFP4: codes, scales (tensor-core order) and g.  rotate != 0 rotates each
 * row first.  per_tensor != 0 takes one g for the whole tensor (weights; it
 * then needs `amax_scratch`, one device word the call overwrites); else one g
 * per row (activations; `amax_scratch` may be NULL).
 * Errors: NULL, SHAPE, ALIGN, ARCH, CUDA.
 */
w4a8_status w4a8_nvfp4_quantize(const void* x, int32_t x_is_f32, int64_t R, int64_t K,
                                int32_t rotate, int32_t per_tensor, uint8_t* codes,
                                uint8_t* scales, float* g, unsigned* amax_scratch,
                                void* stream);

/*
 * Row-major e4m3 scale codes [R, K/16] -> the tensor-core order
 * (w4a8_nvfp4_scale_bytes(R, K) bytes; pad rows 0).  For scales made
 * elsewhere.  Errors: NULL, SHAPE, ARCH, CUDA.
 */
w4a8_status w4a8_nvfp4_pack_scales(const uint8_t* scales_rows, int64_t R, int64_t K,
                                   uint8_t* scales, void* stream);

/*
 * y [M, N] (bf16 bits) = g_x[m] g_w[n] sum_k (e2m1 x e4m3)(x)[m, k]
 * (e2m1 x e4m3)(w)[n, k], on the block-scaled FP4 tensor cores
 * (tcgen05.mma kind::mxf4nvf4, fp32 accumulation).  x_codes [M, K/2],
 * x_scales, g_x [M]; w_codes [N, K/2], w_scales, g_w [N].  A bounded wait
 * that gives up leaves y undefined and is reported by w4a8_get_device_error.
 * Errors: NULL, SHAPE, ALIGN, ARCH, CUDA.
 */
w4a8_status w4a8_nvfp4_gemm(const uint8_t* x_codes, const uint8_t* x_scales, const float* g_x,
                            int64_t M, const uint8_t* w_codes, const uint8_t* w_scales,
                            const float* g_w, int64_t N, int64_t K, uint16_t* y, void* stream);

/* Workspace bytes of w4a8_nvfp4_linear for M tokens of K values. */
size_t w4a8_nvfp4_linear_workspace_bytes(int64_t M, int64_t K);

/*
 * The NVFP4 layer: rotate and quantise x [M, K] (bf16 bits, one g per token)
 * into `workspace`, then w4a8_nvfp4_gemm against weights quantised with
 * rotate != 0.  Errors: as the two calls, WORKSPACE if the workspace is
 * smaller than w4a8_nvfp4_linear_workspace_bytes.
 */
w4a8_status w4a8_nvfp4_linear(const uint16_t* x, int64_t M, int64_t K, const uint8_t* w_codes,
                              const uint8_t* w_scales, const float* g_w, int64_t N, uint16_t* y,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronise `stream`, then report and clear the device-side error word of
 * the current device: W4A8_ERR_TIMEOUT if a bounded wait inside a kernel
 * gave up since the last call (the affected outputs are then undefined),
 * W4A8_ERR_INPUT if a kernel found an input it cannot use (a converter
 * sample position out of range, or an empty sample), W4A8_ERR_CUDA if the
 * synchronisation itself failed, else W4A8_OK.
 */
w4a8_status w4a8_get_device_error(void* stream);

/*
 * Self-test of the device error path (the pages have no counterpart): one
 * small kernel runs the library's two kinds of bounded wait, an mbarrier
 * phase and a global word, on things that never complete, so both give up
 * after a short bound (about a millisecond at most) and record a timeout.
 * The next w4a8_get_device_error on the stream then returns
 * W4A8_ERR_TIMEOUT and clears the word; the context stays usable.  Nothing
 * traps or hangs.  Errors: ARCH, CUDA.
 */
w4a8_status w4a8_selftest_timeout(void* stream);

/* Static English description of a status code. */
const char* w4a8_status_string(w4a8_status status);

#ifdef __cplusplus
}
#endif

#endif /* W4A8_H_ */
