/*
 * zq_tp.h — tensor-parallel pieces of the quantized linear layer (C ABI).
 *
 * Source: [wiki] "ZSE - open-source движок для запуска LLM локально на GPU -
 * 2026" (wiki.iphoster.net), section "Тензорный параллелизм": multi-GPU runs
 * go through NCCL collectives (AllReduce, AllGather, Broadcast, ReduceScatter,
 * Barrier); the weights are sharded across processes, column-parallel for the
 * QKV / Gate / Up projections and row-parallel for O / Down.
 *
 * With P shards (one per GPU):
 *   column-parallel  shard r holds output rows [n_r, n_r+1) of W (a row range
 *                    of packed, scales and zeros, no copy) and computes its
 *                    slice of y with an ordinary zq_linear; no exchange unless
 *                    a consumer needs every column.
 *   row-parallel     shard r holds the input columns of whole groups
 *                    [g_r, g_r+1) of 128 (packed words, scales and zeros of
 *                    those groups, copied into their own N x K_r tensors) and
 *                    the matching slice of x; zq_linear_partial gives its fp32
 *                    partial sums of the full M x N output, and the shards'
 *                    partial sums are added (NCCL all-reduce / reduce-scatter,
 *                    or zq_reduce_partials in a fixed order over buffers that
 *                    may be peers' memory) and rounded once to fp16.
 * Conventions (pointers, alignment, streams, workspace, errors) are those of
 * zq.h.
 */
#ifndef ZQ_TP_H
#define ZQ_TP_H

#include "zq.h"

#ifdef __cplusplus
extern "C" {
#endif

/* One operation of a partial-sum stack: a zq_linear_partial call. */
typedef struct {
    const uint16_t *x;
    const uint32_t *packed;
    const uint16_t *scales;
    const uint16_t *zeros;
    float *out; /* device, fp32 M x N (written) */
    int bits, group, M, N, K;
} zq_partial_desc;

/* y = x · dequant(W)^T as zq_linear, but written as fp32 partial sums without
 * the fp16 rounding: the per-shard step of a row-parallel (K-split) layer,
 * whose shards' results are added before rounding.  Same kernels, arguments,
 * workspace and errors as zq_linear, with `out` a 16-byte aligned device
 * fp32 M x N buffer.  Asynchronous. */
ZQ_API zq_status zq_linear_partial(const uint16_t *x, const uint32_t *packed, const uint16_t *scales,
                                   const uint16_t *zeros, int bits, int group, int M, int N, int K, float *out,
                                   zq_stream_t stream);

/* zq_linear_stack for partial-sum operations (`ops` a HOST array; hazards,
 * fusion and checks as zq_linear_stack).  Lets one launch write a shard's
 * partial sums for several output slices, e.g. each slice straight into the
 * buffer of the GPU that owns it.  Asynchronous. */
ZQ_API zq_status zq_linear_partial_stack(const zq_partial_desc *ops, int n_ops, zq_stream_t stream);

/* Workspace bytes zq_linear_partial_stack(ops, n_ops) needs (0 for an invalid
 * op).  Host only. */
ZQ_API size_t zq_linear_partial_stack_workspace_bytes(const zq_partial_desc *ops, int n_ops);

/* out[i] = fp16(parts[0][i] + parts[1][i] + ... + parts[n_parts-1][i]) for
 * i < count, added in that order in fp32 and rounded once (nearest even): the
 * reduction of a row-parallel layer's partial sums, deterministic whatever the
 * number of GPUs.  `parts` is a HOST array of 1..16 device pointers (16-byte
 * aligned; this GPU's memory or peers' memory it can read); `out` device fp16.
 * n_parts = 1 converts one fp32 buffer.  count = 0 does nothing.
 * Asynchronous. */
ZQ_API zq_status zq_reduce_partials(const float *const *parts, int n_parts, size_t count, uint16_t *out,
                                    zq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ZQ_TP_H */
