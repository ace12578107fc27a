/*
 * zq_zse.h — C ABI of the .zse container reader: a single mmap-ready file of
 * pre-quantized weights (plus configuration, tokenizer and kernel cache) and
 * a streaming loader of its weights into device memory.
 *
 * Source (cited by page title and section):
 *   [wiki]  "ZSE - open-source движок для запуска LLM локально на GPU - 2026"
 *           (wiki.iphoster.net).  Section "Формат модели .zse": one binary
 *           file with weights, tokenizer, model configuration and kernel
 *           cache; signature ZSE\x01, version 1; a 64-byte header, a CRC32
 *           and a table of 32-byte section entries; sections CONFIG,
 *           TOKENIZER, WEIGHT_INDEX, WEIGHT_DATA, KERNELS; weights aligned to
 *           the 4096-byte page (ready for mmap), tensors inside the weight
 *           section aligned to 256 bytes; flags HAS_TOKENIZER, HAS_KERNELS,
 *           MMAP_READY; tensors that stay unquantized are stored as fp16.
 *           Section "Оркестратор и GPU-ядра": cold start through pinned host
 *           memory, asynchronous copies, weights streamed in 64 MB chunks,
 *           posix_fadvise(WILLNEED), parallel reads, one device allocation.
 *
 * The pages name the parts but not their byte layout; the layout below is
 * this library's reading of them (all integers little-endian):
 *
 *   [0, 64)       header
 *                   0  char[4]  magic "ZSE\x01"
 *                   4  u32      version = 1
 *                   8  u32      flags: 1 HAS_TOKENIZER, 2 HAS_KERNELS, 4 MMAP_READY
 *                  12  u32      section count S (1..16)
 *                  16  u64      file size in bytes
 *                  24  40 bytes reserved (zero)
 *   [64, 68)      u32 CRC-32 (IEEE 802.3 polynomial, reflected, init and
 *                 final xor 0xFFFFFFFF: the zlib crc32) of bytes [0, 64)
 *                 followed by the section table
 *   [68, 68+32S)  section table, one 32-byte entry per section:
 *                   0  u32  type: 1 CONFIG, 2 TOKENIZER, 3 WEIGHT_INDEX,
 *                           4 WEIGHT_DATA, 5 KERNELS (each at most once)
 *                   4  u32  CRC-32 of the section's bytes
 *                   8  u64  offset of the section in the file
 *                  16  u64  size of the section in bytes
 *                  24  u64  reserved (zero)
 *   WEIGHT_DATA starts on a 4096-byte boundary when MMAP_READY is set, and
 *   every tensor array inside it on a 256-byte boundary.
 *   WEIGHT_INDEX: u32 tensor count T, u32 entry size (128), then T entries:
 *                   0  char[64] name (UTF-8, NUL-padded, NUL-terminated)
 *                  64  u32  kind: 0 fp16 (unquantized), 1 quantized
 *                  68  u32  bits: 2, 3, 4 or 8 (quantized); 16 (fp16)
 *                  72  u32  group: 128 (quantized); 0 (fp16)
 *                  76  u32  reserved (zero)
 *                  80  u64  rows N
 *                  88  u64  cols K
 *                  96  u64  data offset: packed codes (quantized, uint32
 *                           N x K*b/32 as in zq.h) or fp16 N x K values
 *                 104  u64  data bytes
 *                 112  u64  scales offset (quantized: fp16 N x K/group)
 *                 120  u64  zeros offset  (quantized: fp16 N x K/group)
 *                 (offsets are relative to the start of WEIGHT_DATA)
 *   CONFIG, TOKENIZER and KERNELS are opaque bytes to this library.
 *
 * Ownership: a zq_zse handle owns its read-only mapping of the file and its
 * pinned staging buffers; zq_zse_close releases them.  Host pointers returned
 * by zq_zse_section stay valid until then.  One handle must not be used from
 * two threads at once.
 */
#ifndef ZQ_ZSE_H
#define ZQ_ZSE_H

#include "zq.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct zq_zse zq_zse;

enum { ZQ_ZSE_CONFIG = 1, ZQ_ZSE_TOKENIZER = 2, ZQ_ZSE_WEIGHT_INDEX = 3, ZQ_ZSE_WEIGHT_DATA = 4,
       ZQ_ZSE_KERNELS = 5 };
enum { ZQ_ZSE_HAS_TOKENIZER = 1, ZQ_ZSE_HAS_KERNELS = 2, ZQ_ZSE_MMAP_READY = 4 };

typedef struct {
    char name[64];
    int kind;   /* 0 fp16, 1 quantized */
    int bits;   /* 2, 3, 4, 8; 16 for fp16 */
    int group;  /* 128; 0 for fp16 */
    uint64_t rows, cols;
    uint64_t data_offset, data_bytes;    /* relative to WEIGHT_DATA */
    uint64_t scales_offset, zeros_offset;
} zq_zse_tensor;

/* Opens and validates a .zse file: magic, version, header CRC, section table
 * (types, bounds, no overlap), the weight index (names, kinds, sizes and
 * alignment of every tensor inside WEIGHT_DATA).  Maps the file read-only and
 * advises the kernel to read the weight section ahead (posix_fadvise
 * WILLNEED).  Section CRCs are checked by zq_zse_verify, not here.
 * ZQ_ERR_INVALID_ARG for a missing or malformed file (message in
 * zq_last_error), ZQ_ERR_UNSUPPORTED for another version.  No GPU needed. */
ZQ_API zq_status zq_zse_open(const char *path, zq_zse **out);

/* Releases the handle (mapping, staging buffers).  NULL is ignored. */
ZQ_API void zq_zse_close(zq_zse *z);

/* Header flags and the number of tensors in the weight index. */
ZQ_API uint32_t zq_zse_flags(const zq_zse *z);
ZQ_API int zq_zse_tensor_count(const zq_zse *z);

/* Entry i of the weight index.  ZQ_ERR_INVALID_ARG if i is out of range. */
ZQ_API zq_status zq_zse_tensor_info(const zq_zse *z, int i, zq_zse_tensor *out);

/* Index of the tensor called `name`, or -1. */
ZQ_API int zq_zse_find(const zq_zse *z, const char *name);

/* Host pointer to a section's bytes inside the mapping and its size (*size),
 * or NULL if the file has no such section. */
ZQ_API const void *zq_zse_section(const zq_zse *z, int type, uint64_t *size);

/* Size of WEIGHT_DATA: the device bytes zq_zse_load_weights writes. */
ZQ_API uint64_t zq_zse_weight_bytes(const zq_zse *z);

/* Recomputes the CRC-32 of the header and of every section and compares them
 * with the stored values: ZQ_OK, or ZQ_ERR_INVALID_ARG naming the first
 * mismatch.  Reads the whole file. */
ZQ_API zq_status zq_zse_verify(const zq_zse *z);

/* Copies WEIGHT_DATA into device memory `dst` (at least
 * zq_zse_weight_bytes bytes; a tensor's arrays then sit at dst + their
 * offsets, 256-byte aligned if dst is).  The section is streamed in 64 MB
 * chunks: host threads read each chunk from the file into one of two pinned
 * buffers while the previous chunk is copied to the device on `stream`.  The
 * pinned buffers are allocated by the first call and kept with the handle.
 * Returns when the data is on the device (synchronous).
 * ZQ_ERR_INVALID_ARG if dst is NULL or too small or the file cannot be read,
 * ZQ_ERR_CUDA on a CUDA failure. */
ZQ_API zq_status zq_zse_load_weights(zq_zse *z, void *dst, uint64_t dst_bytes, zq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ZQ_ZSE_H */
