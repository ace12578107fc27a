// zq_zse.cu — reader of the .zse container and streaming loader of its weights
// into device memory (host code; the byte layout is documented in zq_zse.h).
//
// [wiki] "ZSE - open-source движок для запуска LLM локально на GPU - 2026",
// section "Формат модели .zse" (one mmap-ready file: header, CRC32, section
// table, page-aligned weights, 256-byte-aligned tensors) and section
// "Оркестратор и GPU-ядра" (cold start: pinned host memory, asynchronous
// copies, 64 MB chunks, posix_fadvise WILLNEED, parallel reads, one device
// allocation).
#include <cuda_runtime.h>
#include <fcntl.h>
#include <sys/mman.h>
#include <sys/stat.h>
#include <unistd.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

#include "zq.h"
#include "zq_internal.h"
#include "zq_zse.h"

namespace {

constexpr size_t kHeaderBytes = 64;
constexpr size_t kTableOffset = 68;  // header, then its CRC-32
constexpr size_t kEntryBytes = 32;
constexpr size_t kIndexEntryBytes = 128;
constexpr size_t kChunkBytes = size_t(64) << 20;  // staging chunk (64 MB)
constexpr uint32_t kMaxSections = 16;

// CRC-32, IEEE 802.3 polynomial in reflected form (0xEDB88320), initial value
// and final xor 0xFFFFFFFF.  Eight tables let the loop consume eight bytes
// per step ("slicing by 8"): table t maps a byte to the CRC of that byte
// followed by t zero bytes.
uint32_t g_crc[8][256];
std::once_flag g_crc_once;

void crc_init() {
    for (uint32_t i = 0; i < 256; ++i) {
        uint32_t c = i;
        for (int k = 0; k < 8; ++k) c = (c & 1u) ? 0xEDB88320u ^ (c >> 1) : c >> 1;
        g_crc[0][i] = c;
    }
    for (uint32_t i = 0; i < 256; ++i)
        for (int t = 1; t < 8; ++t) g_crc[t][i] = (g_crc[t - 1][i] >> 8) ^ g_crc[0][g_crc[t - 1][i] & 0xFFu];
}

// Continues a CRC-32 over n more bytes (crc = 0 to start).
uint32_t crc32_update(uint32_t crc, const uint8_t *p, size_t n) {
    std::call_once(g_crc_once, crc_init);
    uint32_t c = ~crc;
    while (n >= 8) {
        uint32_t lo, hi;
        std::memcpy(&lo, p, 4);
        std::memcpy(&hi, p + 4, 4);
        lo ^= c;
        c = g_crc[7][lo & 0xFFu] ^ g_crc[6][(lo >> 8) & 0xFFu] ^ g_crc[5][(lo >> 16) & 0xFFu] ^ g_crc[4][lo >> 24] ^
            g_crc[3][hi & 0xFFu] ^ g_crc[2][(hi >> 8) & 0xFFu] ^ g_crc[1][(hi >> 16) & 0xFFu] ^ g_crc[0][hi >> 24];
        p += 8;
        n -= 8;
    }
    while (n--) c = (c >> 8) ^ g_crc[0][(c ^ *p++) & 0xFFu];
    return ~c;
}

template <typename T>
T rd(const uint8_t *p) {
    T v;
    std::memcpy(&v, p, sizeof(T));
    return v;
}

// a + b <= limit without overflow
bool fits(uint64_t a, uint64_t b, uint64_t limit) { return a <= limit && b <= limit - a; }

struct Section {
    uint32_t type, crc;
    uint64_t off, size;
};

}  // namespace

struct zq_zse {
    int fd = -1;
    const uint8_t *map = nullptr;
    size_t size = 0;
    uint32_t flags = 0;
    std::vector<Section> sections;
    std::vector<zq_zse_tensor> tensors;
    int weights = -1;  // index of WEIGHT_DATA in `sections`
    void *pinned[2] = {nullptr, nullptr};
    cudaEvent_t done[2] = {nullptr, nullptr};
    int device = -1;  // device the staging resources belong to
};

namespace {

const Section *find_section(const zq_zse *z, uint32_t type) {
    for (const Section &s : z->sections)
        if (s.type == type) return &s;
    return nullptr;
}

zq_status bad(const char *fmt, ...) __attribute__((format(printf, 1, 2)));
zq_status bad(const char *fmt, ...) {
    char buf[256];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    zq::set_last_error(buf);
    return ZQ_ERR_INVALID_ARG;
}

void release_staging(zq_zse *z) {
    for (int i = 0; i < 2; ++i) {
        if (z->done[i]) cudaEventDestroy(z->done[i]);
        if (z->pinned[i]) cudaFreeHost(z->pinned[i]);
        z->done[i] = nullptr;
        z->pinned[i] = nullptr;
    }
    z->device = -1;
}

// Parses and validates everything but the section CRCs.
zq_status parse(zq_zse *z) {
    const uint8_t *m = z->map;
    if (z->size < kTableOffset) return bad("file of %zu bytes is shorter than the header", z->size);
    if (std::memcmp(m, "ZSE\x01", 4) != 0) return bad("bad magic: not a .zse file");
    const uint32_t version = rd<uint32_t>(m + 4);
    if (version != 1) {
        zq::set_last_error(("unsupported .zse version " + std::to_string(version)).c_str());
        return ZQ_ERR_UNSUPPORTED;
    }
    z->flags = rd<uint32_t>(m + 8);
    if (z->flags & ~7u) return bad("unknown header flags 0x%x", z->flags);
    const uint32_t n_sec = rd<uint32_t>(m + 12);
    if (n_sec == 0 || n_sec > kMaxSections) return bad("section count %u not in 1..16", n_sec);
    if (rd<uint64_t>(m + 16) != z->size) return bad("header file size differs from the file (%zu bytes)", z->size);
    for (size_t i = 24; i < kHeaderBytes; ++i)
        if (m[i] != 0) return bad("reserved header byte %zu is not zero", i);
    const size_t table_end = kTableOffset + kEntryBytes * n_sec;
    if (z->size < table_end) return bad("file too short for its section table");
    uint32_t crc = crc32_update(0, m, kHeaderBytes);
    crc = crc32_update(crc, m + kTableOffset, table_end - kTableOffset);
    if (crc != rd<uint32_t>(m + kHeaderBytes)) return bad("header CRC-32 mismatch");

    uint32_t seen = 0;
    for (uint32_t i = 0; i < n_sec; ++i) {
        const uint8_t *e = m + kTableOffset + kEntryBytes * i;
        Section s{rd<uint32_t>(e), rd<uint32_t>(e + 4), rd<uint64_t>(e + 8), rd<uint64_t>(e + 16)};
        if (s.type < 1 || s.type > 5) return bad("section %u has an unknown type", i);
        if (seen & (1u << s.type)) return bad("section type %u appears twice", s.type);
        seen |= 1u << s.type;
        if (rd<uint64_t>(e + 24) != 0) return bad("section %u: reserved field is not zero", i);
        if (s.off < table_end || !fits(s.off, s.size, z->size))
            return bad("section %u lies outside the file", i);
        z->sections.push_back(s);
    }
    std::vector<Section> by_off = z->sections;
    std::sort(by_off.begin(), by_off.end(), [](const Section &a, const Section &b) { return a.off < b.off; });
    for (size_t i = 1; i < by_off.size(); ++i)
        if (by_off[i - 1].off + by_off[i - 1].size > by_off[i].off) return bad("sections overlap");
    if (((z->flags & ZQ_ZSE_HAS_TOKENIZER) != 0) != ((seen >> ZQ_ZSE_TOKENIZER) & 1u))
        return bad("HAS_TOKENIZER flag and TOKENIZER section disagree");
    if (((z->flags & ZQ_ZSE_HAS_KERNELS) != 0) != ((seen >> ZQ_ZSE_KERNELS) & 1u))
        return bad("HAS_KERNELS flag and KERNELS section disagree");

    const Section *idx = find_section(z, ZQ_ZSE_WEIGHT_INDEX);
    const Section *wd = find_section(z, ZQ_ZSE_WEIGHT_DATA);
    if ((idx == nullptr) != (wd == nullptr)) return bad("WEIGHT_INDEX and WEIGHT_DATA must come together");
    if (wd == nullptr) return ZQ_OK;
    z->weights = static_cast<int>(wd - z->sections.data());
    if ((z->flags & ZQ_ZSE_MMAP_READY) && (wd->off % 4096) != 0)
        return bad("MMAP_READY file with WEIGHT_DATA at offset %llu (not page-aligned)", static_cast<unsigned long long>(wd->off));
    if (idx->size < 8) return bad("weight index too short");
    const uint8_t *ip = m + idx->off;
    const uint32_t count = rd<uint32_t>(ip), esize = rd<uint32_t>(ip + 4);
    if (esize != kIndexEntryBytes) return bad("weight index entry size %u (expected 128)", esize);
    if (!fits(8, uint64_t(count) * kIndexEntryBytes, idx->size)) return bad("weight index too short");
    const uint64_t W = wd->size;
    for (uint32_t i = 0; i < count; ++i) {
        const uint8_t *e = ip + 8 + kIndexEntryBytes * i;
        zq_zse_tensor t;
        std::memset(&t, 0, sizeof(t));
        std::memcpy(t.name, e, 64);
        if (t.name[63] != '\0' || t.name[0] == '\0') return bad("tensor %u: name not NUL-terminated or empty", i);
        t.kind = static_cast<int>(rd<uint32_t>(e + 64));
        t.bits = static_cast<int>(rd<uint32_t>(e + 68));
        t.group = static_cast<int>(rd<uint32_t>(e + 72));
        if (rd<uint32_t>(e + 76) != 0) return bad("tensor %s: reserved field is not zero", t.name);
        t.rows = rd<uint64_t>(e + 80);
        t.cols = rd<uint64_t>(e + 88);
        t.data_offset = rd<uint64_t>(e + 96);
        t.data_bytes = rd<uint64_t>(e + 104);
        t.scales_offset = rd<uint64_t>(e + 112);
        t.zeros_offset = rd<uint64_t>(e + 120);
        if (t.rows == 0 || t.cols == 0 || t.rows > (1u << 30) || t.cols > (1u << 30))
            return bad("tensor %s: bad shape", t.name);
        if (t.data_offset % 256 || t.scales_offset % 256 || t.zeros_offset % 256)
            return bad("tensor %s: an array is not 256-byte aligned", t.name);
        if (t.kind == 1) {
            if (!(t.bits == 2 || t.bits == 3 || t.bits == 4 || t.bits == 8) || t.group != zq::kGroup ||
                t.cols % zq::kGroup)
                return bad("tensor %s: bad quantized format", t.name);
            const uint64_t sz = t.rows * (t.cols / zq::kGroup) * 2;
            if (t.data_bytes != t.rows * t.cols * t.bits / 8) return bad("tensor %s: data size mismatch", t.name);
            if (!fits(t.scales_offset, sz, W) || !fits(t.zeros_offset, sz, W))
                return bad("tensor %s: scales or zeros outside WEIGHT_DATA", t.name);
        } else if (t.kind == 0) {
            if (t.bits != 16 || t.group != 0 || t.scales_offset || t.zeros_offset)
                return bad("tensor %s: bad fp16 entry", t.name);
            if (t.data_bytes != t.rows * t.cols * 2) return bad("tensor %s: data size mismatch", t.name);
        } else {
            return bad("tensor %s: unknown kind", t.name);
        }
        if (!fits(t.data_offset, t.data_bytes, W)) return bad("tensor %s: data outside WEIGHT_DATA", t.name);
        for (const zq_zse_tensor &u : z->tensors)
            if (std::strcmp(u.name, t.name) == 0) return bad("tensor name %s appears twice", t.name);
        z->tensors.push_back(t);
    }
    return ZQ_OK;
}

}  // namespace

extern "C" {

zq_status zq_zse_open(const char *path, zq_zse **out) {
    if (out == nullptr || path == nullptr) return bad("null argument");
    *out = nullptr;
    zq_zse *z = new zq_zse;
    z->fd = ::open(path, O_RDONLY | O_CLOEXEC);
    if (z->fd < 0) {
        delete z;
        return bad("cannot open %s", path);
    }
    struct stat sb;
    if (fstat(z->fd, &sb) != 0 || sb.st_size <= 0) {
        zq_zse_close(z);
        return bad("cannot stat %s, or it is empty", path);
    }
    z->size = static_cast<size_t>(sb.st_size);
    void *m = mmap(nullptr, z->size, PROT_READ, MAP_SHARED, z->fd, 0);
    if (m == MAP_FAILED) {
        zq_zse_close(z);
        return bad("cannot map %s", path);
    }
    z->map = static_cast<const uint8_t *>(m);
    zq_status st = parse(z);
    if (st != ZQ_OK) {
        zq_zse_close(z);
        return st;
    }
    if (z->weights >= 0) {
        const Section &w = z->sections[z->weights];
        posix_fadvise(z->fd, static_cast<off_t>(w.off), static_cast<off_t>(w.size), POSIX_FADV_WILLNEED);
        const size_t page = 4096, a = w.off / page * page;
        madvise(const_cast<uint8_t *>(z->map) + a, w.off + w.size - a, MADV_WILLNEED);
    }
    *out = z;
    return ZQ_OK;
}

void zq_zse_close(zq_zse *z) {
    if (z == nullptr) return;
    release_staging(z);
    if (z->map) munmap(const_cast<uint8_t *>(z->map), z->size);
    if (z->fd >= 0) ::close(z->fd);
    delete z;
}

uint32_t zq_zse_flags(const zq_zse *z) { return z ? z->flags : 0u; }

int zq_zse_tensor_count(const zq_zse *z) { return z ? static_cast<int>(z->tensors.size()) : 0; }

zq_status zq_zse_tensor_info(const zq_zse *z, int i, zq_zse_tensor *out) {
    if (z == nullptr || out == nullptr) return bad("null argument");
    if (i < 0 || i >= static_cast<int>(z->tensors.size())) return bad("tensor index %d out of range", i);
    *out = z->tensors[i];
    return ZQ_OK;
}

int zq_zse_find(const zq_zse *z, const char *name) {
    if (z == nullptr || name == nullptr) return -1;
    for (size_t i = 0; i < z->tensors.size(); ++i)
        if (std::strcmp(z->tensors[i].name, name) == 0) return static_cast<int>(i);
    return -1;
}

const void *zq_zse_section(const zq_zse *z, int type, uint64_t *size) {
    if (size) *size = 0;
    if (z == nullptr) return nullptr;
    const Section *s = find_section(z, static_cast<uint32_t>(type));
    if (s == nullptr) return nullptr;
    if (size) *size = s->size;
    return z->map + s->off;
}

uint64_t zq_zse_weight_bytes(const zq_zse *z) {
    return (z && z->weights >= 0) ? z->sections[z->weights].size : 0;
}

zq_status zq_zse_verify(const zq_zse *z) {
    if (z == nullptr) return bad("null argument");
    const uint8_t *m = z->map;
    const size_t table_end = kTableOffset + kEntryBytes * z->sections.size();
    uint32_t crc = crc32_update(0, m, kHeaderBytes);
    crc = crc32_update(crc, m + kTableOffset, table_end - kTableOffset);
    if (crc != rd<uint32_t>(m + kHeaderBytes)) return bad("header CRC-32 mismatch");
    for (const Section &s : z->sections)
        if (crc32_update(0, m + s.off, s.size) != s.crc) return bad("CRC-32 mismatch in the section of type %u", s.type);
    return ZQ_OK;
}

zq_status zq_zse_load_weights(zq_zse *z, void *dst, uint64_t dst_bytes, zq_stream_t stream) {
    if (z == nullptr || dst == nullptr) return bad("null argument");
    const uint64_t total = zq_zse_weight_bytes(z);
    if (dst_bytes < total) return bad("destination of %llu bytes is smaller than the weights", static_cast<unsigned long long>(dst_bytes));
    if (total == 0) return ZQ_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess && z->device != dev) {
        release_staging(z);  // staging buffers and events belong to one device
        for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
            e = cudaHostAlloc(&z->pinned[i], kChunkBytes, cudaHostAllocDefault);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&z->done[i], cudaEventDisableTiming);
        }
        if (e == cudaSuccess) z->device = dev;
    }
    if (e != cudaSuccess) {
        release_staging(z);
        zq::set_last_error((std::string("staging buffers: ") + cudaGetErrorString(e)).c_str());
        return ZQ_ERR_CUDA;
    }
    uint8_t *d = static_cast<uint8_t *>(dst);
    const unsigned hw = std::max(1u, std::min(8u, std::thread::hardware_concurrency()));
    uint64_t chunk = 0;
    bool read_failed = false;
    for (uint64_t off = 0; off < total; off += kChunkBytes, ++chunk) {
        const int b = static_cast<int>(chunk & 1);
        const size_t n = static_cast<size_t>(std::min<uint64_t>(kChunkBytes, total - off));
        if (chunk >= 2 && (e = cudaEventSynchronize(z->done[b])) != cudaSuccess) break;
        // Parallel read of the chunk into pinned memory: each thread preads a
        // slice straight from the file (no page-table work for the mapping).
        uint8_t *pin = static_cast<uint8_t *>(z->pinned[b]);
        const size_t per = (n + hw - 1) / hw;
        const uint64_t file_off = z->sections[z->weights].off + off;
        std::vector<std::thread> th;
        std::vector<int> ok(hw, 1);
        auto slice = [&, pin, per, n, file_off](unsigned t) {
            size_t done = 0, want = std::min(per, n - t * per);
            while (done < want) {
                const ssize_t r = pread(z->fd, pin + t * per + done, want - done,
                                        static_cast<off_t>(file_off + t * per + done));
                if (r <= 0) {
                    ok[t] = 0;
                    return;
                }
                done += static_cast<size_t>(r);
            }
        };
        for (unsigned t = 1; t < hw && t * per < n; ++t) th.emplace_back(slice, t);
        slice(0);
        for (auto &x : th) x.join();
        if (std::find(ok.begin(), ok.end(), 0) != ok.end()) {
            read_failed = true;  // copies in flight are waited for below
            break;
        }
        if ((e = cudaMemcpyAsync(d + off, pin, n, cudaMemcpyHostToDevice, s)) != cudaSuccess) break;
        if ((e = cudaEventRecord(z->done[b], s)) != cudaSuccess) break;
    }
    for (int i = 0; i < 2 && e == cudaSuccess; ++i)
        if (chunk > static_cast<uint64_t>(i)) e = cudaEventSynchronize(z->done[i]);
    if (read_failed && e == cudaSuccess) {
        zq::set_last_error("reading the weight section failed");
        return ZQ_ERR_INVALID_ARG;
    }
    if (e != cudaSuccess) {
        zq::set_last_error((std::string("weight copy: ") + cudaGetErrorString(e)).c_str());
        return ZQ_ERR_CUDA;
    }
    return ZQ_OK;
}

}  // extern "C"
