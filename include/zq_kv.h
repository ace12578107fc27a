/*
 * zq_kv.h — C ABI of zKV, the quantized KV cache with sliding precision.
 *
 * Sources (cited by page title and section):
 *   [pt]    "ZSE: Motor de inferência de LLM de código aberto com
 *           inicializações a frio de 3,9 segundos" (openclawradar, pt),
 *           section "Componentes da arquitetura": zKV, a quantized KV cache
 *           with sliding precision that saves about 4x of memory.
 *   [lavx]  "ZSE: A Memory-Efficient LLM Inference Engine with Smart Resource
 *           Orchestration", section "Technical Architecture": the same.
 *   [wiki]  "ZSE - open-source движок для запуска LLM локально на GPU - 2026",
 *           section "Управление KV-кэшем": token-level eviction and
 *           sliding-window attention in a paged cache; section "Формат
 *           модели .zse": the group codec (zq.h).
 *
 * The pages name the component and its saving, nothing more.  Reading taken
 * (the plainest one that gives "sliding precision" and about 4x):
 *   - A plane is the K (or the V) of one layer for one sequence: token t has
 *     one row of H heads x D fp16 values, D a multiple of 128.
 *   - Precision slides with a token's age.  The newest `window` tokens are
 *     kept exactly, in an fp16 ring (token t in slot t % window).  A token
 *     that leaves the window is quantized, one group per 128 values along D,
 *     with the asymmetric codec of zq_quantize_pack at `bits` (2, 3, 4 or 8),
 *     into the store (row t).  INT4 keeps 64 + 4 bytes per 128 values
 *     against 256 in fp16: 3.76x less.
 *   - Appending n tokens to a plane that holds t0 has the result of appending
 *     them one at a time: token t enters slot t % window, and token
 *     t - window, which held that slot, moves to the store.
 *
 * Layouts (row-major, contiguous, device memory):
 *   ring    fp16 window x H x D
 *   packed  uint32 capacity x H x (D * bits / 32), each (token, head) row a
 *           little-endian bitstream as in zq.h
 *   scales  fp16 capacity x H x (D / 128);   zeros  likewise
 *
 * Conventions as in zq.h: the caller owns every buffer; device pointers must
 * be 16-byte aligned; calls are asynchronous and stream-ordered; a rejected
 * call enqueues nothing.  A row holding NaN or Inf leaves its store group
 * unspecified and is reported by zq_check_device() as ZQ_ERR_NONFINITE.
 */
#ifndef ZQ_KV_H
#define ZQ_KV_H

#include "zq.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    uint16_t *ring;    /* fp16 window x heads x dim */
    uint32_t *packed;  /* capacity x heads x dim*bits/32 */
    uint16_t *scales;  /* fp16 capacity x heads x dim/128 */
    uint16_t *zeros;   /* fp16 capacity x heads x dim/128 */
    int window;        /* tokens kept in fp16, >= 1 */
    int capacity;      /* tokens the store can hold, >= 1 */
    int heads;         /* >= 1 */
    int dim;           /* values per head, a multiple of 128 */
    int bits;          /* 2, 3, 4 or 8 */
} zq_kv_plane;

/* Device bytes of a plane: the ring plus the store (packed codes, scales,
 * zeros), each rounded up to 256 bytes.  0 for an invalid shape. */
ZQ_API size_t zq_kv_plane_bytes(int window, int capacity, int heads, int dim, int bits);

/* Appends n tokens (rows: device fp16 n x heads x dim) to a plane that holds
 * t0 tokens; afterwards it holds t0 + n: the newest min(t0 + n, window) in
 * the ring, every older one quantized in the store.  One kernel launch (none
 * for n = 0).  ZQ_ERR_INVALID_ARG for a bad shape or pointer, t0 < 0, n < 0
 * or t0 + n > capacity; ZQ_ERR_UNSUPPORTED for bits outside {2,3,4,8}.
 * Asynchronous. */
ZQ_API zq_status zq_kv_append(const zq_kv_plane *plane, int t0, const uint16_t *rows, int n,
                              zq_stream_t stream);

/* Writes tokens [a, b) of a plane that holds t_total tokens to out (device
 * fp16 (b - a) x heads x dim): ring rows as stored, store rows dequantized
 * to fp16(q * scale + zero) with one rounding.  One kernel launch (none for
 * a = b).  ZQ_ERR_INVALID_ARG unless 0 <= a <= b <= t_total <= capacity.
 * Asynchronous. */
ZQ_API zq_status zq_kv_gather(const zq_kv_plane *plane, int t_total, int a, int b, uint16_t *out,
                              zq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ZQ_KV_H */
