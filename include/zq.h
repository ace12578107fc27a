/*
 * zq.h — C ABI of the weight-only quantized linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer computes y = x · dequant(W)^T, the projection that dominates every
 * decode and prefill step of a pre-quantized LLM inference engine.
 *
 * Sources (cited by page title and section):
 *   [wiki]  "ZSE - open-source движок для запуска LLM локально на GPU - 2026"
 *           (wiki.iphoster.net). Section "Формат модели .zse": asymmetric
 *           group-wise quantization with groups of 128, scale = (max-min)/15,
 *           zero = min, q = clamp(round((w-zero)/scale), 0, 15), two INT4 codes
 *           per byte with the low nibble first, fp16 scales and zeros, and
 *           quantization done once at conversion time. Section "Оркестратор и
 *           GPU-ядра": INT4 GEMV with 128-bit weight loads, batched launches and
 *           graph capture to cut launch latency.
 *   [lavx]  "ZSE: A Memory-Efficient LLM Inference Engine with Smart Resource
 *           Orchestration", section "Technical Architecture": per-tensor INT2-8
 *           mixed precision (zQuantize).
 *
 * Tensor format (all buffers row-major and contiguous):
 *   W       N x K weights (output features x input features; y = x W^T).
 *   bits    b in {2, 3, 4, 8}, chosen per tensor.  L = 2^b - 1.  (bits = 16:
 *           fp16 weights kept unquantized, see zq_linear.)
 *   group   g consecutive weights along K share one fp16 scale and one fp16
 *           zero: g = 128 (the pages' figure), or 64 or 32 (the encoding
 *           variants).  K must be a multiple of 128.  G = K / g.
 *   packed  uint32 N x (K*b/32).  The codes of one row form a little-endian
 *           bitstream: code k occupies stream bits [k*b, k*b+b), and stream bit
 *           t is bit (t % 32) of word t / 32.  At b = 4 this is the pages'
 *           "two codes per byte, low nibble first".  At b = 3 codes straddle
 *           word boundaries; a group is always exactly 4*b words.
 *   scales  fp16 (as uint16 bit patterns) N x G.
 *   zeros   fp16 (as uint16 bit patterns) N x G.  The zero is the group's
 *           float minimum, not an integer zero point:
 *           dequant(W)[n][k] = q[n][k] * scale[n][k/128] + zero[n][k/128].
 *   x       fp16 M x K activations;  out  fp16 M x N.
 *   Arithmetic: fp16 in, fp32 accumulation, fp16 out (round to nearest even).
 *
 * Conventions for every entry point:
 *   - Pointers are device pointers unless stated otherwise, and must be
 *     16-byte aligned.  The caller owns every buffer.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued on it; zq_linear and zq_linear_stack return without waiting.
 *   - Errors: a non-OK status is returned and nothing is enqueued when the
 *     arguments are rejected.  zq_last_error() gives a message for the most
 *     recent failure on the calling thread.  ZQ_ERR_CUDA means a CUDA call
 *     failed (launch error, out of memory); the CUDA error is in the message.
 *   - Stream order: a call's kernels read their inputs only after all work
 *     enqueued earlier on `stream` has completed (programmatic dependent
 *     launch is used only to overlap launch latency, never to read early).
 *   - Workspace: zq_linear and zq_linear_stack use one device buffer per
 *     (device, stream) for activation staging, split-K partial sums and work
 *     counters.  The calls themselves never allocate, free or synchronise: the
 *     buffer is reserved beforehand with zq_reserve_workspace (the library
 *     allocates it) or attached with zq_attach_workspace (the caller owns it),
 *     sized by zq_linear_workspace_bytes / zq_linear_stack_workspace_bytes.  A
 *     call that needs more than its stream holds returns ZQ_ERR_INVALID_ARG
 *     and enqueues nothing.  Streams are told apart by their unique id
 *     (cudaStreamGetId), so a handle reused by CUDA after cudaStreamDestroy
 *     starts without a workspace; release a stream's workspace
 *     (zq_release_workspace) before destroying the stream.  Calls on the same
 *     stream are ordered; calls on different streams use different buffers.
 */
#ifndef ZQ_H
#define ZQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ZQ_API __attribute__((visibility("default")))
#else
#define ZQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *zq_stream_t; /* identical to cudaStream_t */

typedef enum {
    ZQ_OK = 0,
    ZQ_ERR_INVALID_ARG = 1, /* bad size, null or misaligned pointer          */
    ZQ_ERR_UNSUPPORTED = 2, /* bits not in {2,3,4,8} or group not in {32,64,128} */
    ZQ_ERR_NONFINITE = 3,   /* a weight is NaN/Inf or |w| > 65504 (fp16 max)  */
    ZQ_ERR_CUDA = 4,        /* a CUDA runtime call failed                     */
    ZQ_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up             */
} zq_status;

/* Number of uint32 words of a packed N x K tensor: N * K * bits / 32
 * ([wiki] "Формат модели .zse": b-bit codes packed densely, two INT4 codes per
 * byte; [lavx] "Technical Architecture": b from 2 to 8 per tensor).
 * Returns 0 for unsupported bits or sizes (K % 128 != 0, N <= 0, K <= 0). */
ZQ_API size_t zq_packed_words(int N, int K, int bits);

/* Quantize and pack a weight tensor on the GPU, [wiki] "Формат модели .zse",
 * generalised to L = 2^bits - 1 ([lavx] "Technical Architecture").
 *   w       device, fp32 N x K row-major.
 *   packed  device, uint32 N x (K*bits/32), written.
 *   scales  device, fp16 bits N x (K/128), written.
 *   zeros   device, fp16 bits N x (K/128), written.
 * Per group: zero = fp16(min), scale = fp16((max - min) / L) computed in fp64
 * and rounded once; q = clamp(round_half_even((w - zero) / scale), 0, L) with
 * the stored fp16 scale and zero, in fp64; a group whose fp16 scale is 0 gets
 * all q = 0.  Bit-exact with the reference quantizer.
 * SYNCHRONOUS: the call waits for `stream` so it can report ZQ_ERR_NONFINITE
 * (any NaN, Inf or |w| > 65504); then the outputs are unspecified.  Not
 * capturable into a CUDA graph. */
ZQ_API zq_status zq_quantize_pack(const float *w, int N, int K, int bits, int group,
                           uint32_t *packed, uint16_t *scales, uint16_t *zeros,
                           zq_stream_t stream);

/* Symmetric variant of zq_quantize_pack ([wiki] "Формат модели .zse" lists
 * symmetric INT8 quantization, reserved, without a formula; the same step is
 * offered for every supported width).  Arguments, layout, synchronisation and
 * errors as zq_quantize_pack.  Per group of 128, with Q = 2^(bits-1) - 1:
 * scale = fp16(max|w| / Q) computed in fp64 and rounded once;
 * q = clamp(round_half_even(w / scale), -Q, Q) with the stored fp16 scale
 * (q = 0 when the scale is 0).  The result is stored in the ordinary format:
 * code = q + 2^(bits-1) and zero = -2^(bits-1) * scale (exact), so zq_linear
 * and every other consumer compute code*scale + zero = q*scale unchanged.
 * Bit-exact with the reference quantizer.  ZQ_ERR_NONFINITE also when a
 * group's zero would fall below -65504 (max|w| above about 65000 at 8 bits,
 * 32752 at 2 bits). */
ZQ_API zq_status zq_quantize_pack_symmetric(const float *w, int N, int K, int bits, int group,
                                            uint32_t *packed, uint16_t *scales, uint16_t *zeros,
                                            zq_stream_t stream);

/* y = x · dequant(W)^T, the quantized projection of [wiki] "Оркестратор и
 * GPU-ядра" (INT4 GEMV for decode, tiled matmul for prefill) over the format
 * of [wiki] "Формат модели .zse" (dequant(W) = q * scale + zero per group).
 *   x       device, fp16 M x K.      out  device, fp16 M x N (written).
 *   packed/scales/zeros as produced by zq_quantize_pack.
 * M <= 32 runs the decode kernel (mma.sync skinny GEMM streaming the packed
 * weights once through a shared-memory ring); larger M, and groups of 32 or
 * 64 at any M, run the tcgen05 tile kernel (256-token x 256-row output tiles,
 * so at M <= 256 the weights are again streamed once; with b-bit codes and
 * some M >= 512 in the call, 512 x 256 tiles computed by pairs of CTAs on two
 * SMs with tcgen05.mma.cta_group::2).
 * bits = 16 is the fp16 passthrough of the .zse format ([wiki] "Формат
 * модели .zse": tensors kept unquantized): `packed` then holds the weights as
 * fp16 N x K, `scales`, `zeros` and `group` are not read (may be NULL / any).
 * Needs a workspace of zq_linear_workspace_bytes(bits, M, N, K) on `stream`
 * (see Conventions; the size for group 128 covers every group size).
 * Asynchronous; fp32 accumulation, fp16 output rounded to nearest even. */
ZQ_API zq_status zq_linear(const uint16_t *x, const uint32_t *packed,
                    const uint16_t *scales, const uint16_t *zeros,
                    int bits, int group, int M, int N, int K,
                    uint16_t *out, zq_stream_t stream);

/* zq_linear with bfloat16 activations and output (the encoding variants next
 * to [wiki] "Формат модели .zse"; the pages fix no activation type).
 *   x    device, bfloat16 bit patterns M x K.   out  device, bfloat16 M x N.
 * Weights, formats, kernels and errors as zq_linear.  The products still run
 * in fp16 on the tensor cores: each activation group (decode kernel) or token
 * row (tile kernel) is scaled by a power of two into fp16's range, exactly
 * for every value within 2^24 of the largest, and the factor is divided out
 * in fp32; activations of magnitude 2^55 or more are out of range.  The tile
 * kernel keeps that fp16 copy in the workspace: size it with
 * zq_linear_bf16_workspace_bytes.  Output rounded once to bfloat16 (nearest
 * even).  Asynchronous. */
ZQ_API zq_status zq_linear_bf16(const uint16_t *x, const uint32_t *packed, const uint16_t *scales,
                                const uint16_t *zeros, int bits, int group, int M, int N, int K,
                                uint16_t *out, zq_stream_t stream);

/* Workspace bytes of zq_linear_bf16 with these sizes (0 for invalid sizes). */
ZQ_API size_t zq_linear_bf16_workspace_bytes(int bits, int M, int N, int K);

/* Allocation-free zq_linear, for callers that cannot allocate device memory:
 * code running inside a CUDA stream capture (where cudaMalloc is not
 * allowed), code under a fixed device-memory budget, or latency-critical
 * paths that must not risk the device-wide synchronisation cudaMalloc and
 * cudaFree can cause.  zq_linear keeps a workspace per (device, stream) that
 * it allocates on first use; this entry point instead uses one fixed 4 MiB
 * device array compiled into the library, which every GPU that loads the
 * library holds until the process exits.  (The pages describe no
 * counterpart: this is a service of the library, not part of the method.)
 *   Arguments and result: as zq_linear, with 1 <= M <= 8.
 *   Limits: M > 8, or a call whose scratch (staged activations and split-K
 *   partial sums) would exceed 4 MiB, returns ZQ_ERR_UNSUPPORTED.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 *   Every call shares the one array and clears its counters with an
 *   asynchronous memset on `stream`: calls that overlap on the GPU (other
 *   streams, other host threads) race and must be serialised by the caller.
 *   Calls no cudaMalloc, cudaFree or allocating library routine.
 *   Asynchronous. */
ZQ_API zq_status zq_linear_noalloc(const uint16_t *x, const uint32_t *packed,
                                   const uint16_t *scales, const uint16_t *zeros,
                                   int bits, int group, int M, int N, int K,
                                   uint16_t *out, zq_stream_t stream);

/* One operation of a stack: the arguments of one zq_linear call. */
typedef struct {
    const uint16_t *x;
    const uint32_t *packed;
    const uint16_t *scales;
    const uint16_t *zeros;
    uint16_t *out;
    int bits, group, M, N, K;
} zq_linear_desc;

/* Run n_ops linear layers with the result of calling zq_linear on each, in
 * array order ([wiki] "Оркестратор и GPU-ядра": batched launches, graphs).
 * `ops` is a HOST array, read before the call returns.  An op's x may alias
 * an earlier op's out: the library detects overlapping buffers and keeps
 * such ops ordered; runs of independent ops are fused into one launch per
 * (bits, batch class).  All ops, and the workspace the stack needs
 * (zq_linear_stack_workspace_bytes), are checked before anything is
 * enqueued.  Asynchronous. */
ZQ_API zq_status zq_linear_stack(const zq_linear_desc *ops, int n_ops, zq_stream_t stream);

/* zq_linear_stack with bfloat16 activations and outputs: every op's x and out
 * hold bfloat16 (see zq_linear_bf16); `ops` as zq_linear_stack.  The
 * workspace it needs is zq_linear_stack_bf16_workspace_bytes(ops, n_ops).
 * Asynchronous. */
ZQ_API zq_status zq_linear_stack_bf16(const zq_linear_desc *ops, int n_ops, zq_stream_t stream);
ZQ_API size_t zq_linear_stack_bf16_workspace_bytes(const zq_linear_desc *ops, int n_ops);

/* Test hook: unpack codes with the same device unpack routine zq_linear
 * uses; the inverse of the packing of [wiki] "Формат модели .zse" (code k of
 * a row at stream bits [k*b, k*b+b)).  codes: device uint8 N x K (written).
 * Asynchronous. */
ZQ_API zq_status zq_unpack(const uint32_t *packed, int N, int K, int bits,
                    uint8_t *codes, zq_stream_t stream);

/* Test hook: the tile kernel's dequantization ([wiki] "Формат модели .zse":
 * w_hat = q * scale + zero) over a whole tensor, with the same device routine
 * the tcgen05 kernel uses before its MMAs: w_hat (device, fp16 N x K, written)
 * = fp16(q * s + z) rounded once to nearest even, or 65504 where that rounds
 * to +infinity (groups reaching the top of the fp16 range).  Formats and
 * errors as zq_linear.  Asynchronous. */
ZQ_API zq_status zq_dequant(const uint32_t *packed, const uint16_t *scales, const uint16_t *zeros, int bits,
                            int group, int N, int K, uint16_t *w_hat, zq_stream_t stream);

/* Workspace (see Conventions).  The pages describe no counterpart: these are
 * services of the library, not part of the method.
 *
 * zq_reserve_workspace: gives (current device, stream) a library-allocated
 *   workspace of at least `bytes` (at least 256 KB), replacing a smaller or
 *   attached one.  SYNCHRONOUS when it allocates (waits for `stream` first so
 *   the old buffer is no longer in use); a no-op when the stream already holds
 *   enough.  Call it before capturing the stream into a CUDA graph.
 * zq_attach_workspace: makes the caller's device buffer (256-byte aligned, at
 *   least 256 KB) the workspace of (current device, stream); a library-owned
 *   one is freed (after waiting for the stream).  Its first 256 KB of counters
 *   are cleared by an asynchronous memset on `stream`.  The caller keeps the
 *   buffer alive and unused by anything else until it releases it; no other
 *   stream may share it.
 * zq_release_workspace: waits for `stream`, then frees (library-owned) or
 *   forgets (attached) its workspace.  ZQ_OK if it has none.
 * zq_release_all_workspaces: waits for the current device, then releases the
 *   workspaces of all its streams. */
ZQ_API zq_status zq_reserve_workspace(size_t bytes, zq_stream_t stream);
ZQ_API zq_status zq_attach_workspace(void *buffer, size_t bytes, zq_stream_t stream);
ZQ_API zq_status zq_release_workspace(zq_stream_t stream);
ZQ_API zq_status zq_release_all_workspaces(void);

/* Workspace bytes a zq_linear call with these sizes needs (0 for invalid
 * sizes).  Host only; no device work. */
ZQ_API size_t zq_linear_workspace_bytes(int bits, int M, int N, int K);

/* Workspace bytes zq_linear_stack(ops, n_ops) needs (0 for an invalid op).
 * Host only; reads the HOST array `ops`. */
ZQ_API size_t zq_linear_stack_workspace_bytes(const zq_linear_desc *ops, int n_ops);

/* Test hook: limit, in nanoseconds, of the bounded waits of the linear
 * kernels launched after this call, on every device (default 2000000000, i.e.
 * 2 s; the limit travels with each launch).  A wait that runs out makes its
 * kernel stop and drain and zq_check_device report ZQ_ERR_TIMEOUT; the drain
 * of copies and MMAs already issued keeps its own 2 s bound.  Lets a test make
 * waits run out without any fault.  Host only. */
ZQ_API zq_status zq_set_wait_limit_ns(uint64_t ns);

/* Human-readable name of a status code (static storage). */
ZQ_API const char *zq_status_string(zq_status status);

/* Message of the most recent failure on the calling thread ("" if none). */
ZQ_API const char *zq_last_error(void);

/* Waits for the current device to finish all work, then reports whether any
 * of this library's kernels gave up a bounded wait (ZQ_ERR_TIMEOUT) or a KV
 * append met a NaN or Inf row (ZQ_ERR_NONFINITE, zq_kv.h) since the last call;
 * clears those records.  After a timeout the outputs of the calls involved
 * are unspecified; the workspaces of the device are marked so that the next
 * call on each stream first clears its counters.  Synchronous. */
ZQ_API zq_status zq_check_device(void);

/* Number of kernels this library has launched in this process (all devices).
 * Lets a caller count device work, e.g. inside a timed region. */
ZQ_API uint64_t zq_kernel_launches(void);

/* Library version, major*10000 + minor*100 + patch. */
ZQ_API int zq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ZQ_H */
