// zq_api.cu — host side of the C ABI declared in include/zq.h: argument
// validation, the per-(device, stream) workspace, planning of decode launches
// (cost-balanced units, split-K choice, fusion of independent stack ops) and
// dispatch to the kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <utility>
#include <vector>

#include "zq.h"
#include "zq_kv.h"
#include "zq_tp.h"
#include "zq_internal.h"
#include "zq_prefill.h"
#include "zq_quant.h"

using namespace zq;

namespace {

thread_local std::string g_last_error;
std::atomic<unsigned long long> g_quant_call{1};
std::atomic<uint64_t> g_launches{0};
std::atomic<unsigned long long> g_wait_ns{2000000000ull};  // limit of the kernels' bounded waits

zq_status fail(zq_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
zq_status fail(zq_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

zq_status cuda_fail(cudaError_t e, const char *what) {
    return fail(ZQ_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool bits_ok(int bits) { return bits == 2 || bits == 3 || bits == 4 || bits == 8; }

bool group_ok(int group) { return group == 32 || group == 64 || group == 128; }

zq_status check_format(int bits, int group, int N, int K) {
    if (!bits_ok(bits)) return fail(ZQ_ERR_UNSUPPORTED, "bits=%d not in {2,3,4,8}", bits);
    if (!group_ok(group)) return fail(ZQ_ERR_UNSUPPORTED, "group=%d not in {32, 64, 128}", group);
    if (N <= 0 || K <= 0) return fail(ZQ_ERR_INVALID_ARG, "N=%d K=%d must be positive", N, K);
    if (K % kGroup != 0) return fail(ZQ_ERR_INVALID_ARG, "K=%d is not a multiple of 128", K);
    if (static_cast<long long>(N) * K > (1LL << 40))
        return fail(ZQ_ERR_INVALID_ARG, "N*K=%lld too large", static_cast<long long>(N) * K);
    return ZQ_OK;
}

zq_status check_ptr(const void *p, const char *name) {
    if (p == nullptr) return fail(ZQ_ERR_INVALID_ARG, "%s is null", name);
    if (!aligned16(p)) return fail(ZQ_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return ZQ_OK;
}

// bits == 16: fp16 weights (N x K in `packed`), no scales or zeros, group not read.
zq_status check_linear(const zq_linear_desc &d) {
    zq_status st = d.bits == 16 ? check_format(4, kGroup, d.N, d.K) : check_format(d.bits, d.group, d.N, d.K);
    if (st != ZQ_OK) return st;
    if (d.M <= 0) return fail(ZQ_ERR_INVALID_ARG, "M=%d must be positive", d.M);
    if ((st = check_ptr(d.x, "x")) != ZQ_OK) return st;
    if ((st = check_ptr(d.packed, "packed")) != ZQ_OK) return st;
    if (d.bits != 16) {
        if ((st = check_ptr(d.scales, "scales")) != ZQ_OK) return st;
        if ((st = check_ptr(d.zeros, "zeros")) != ZQ_OK) return st;
    }
    if ((st = check_ptr(d.out, "out")) != ZQ_OK) return st;
    return ZQ_OK;
}

// One linear operation inside the library: the arguments of a zq_linear call,
// with the output either fp16 (out) or, for partial sums, fp32 (out32; then
// out is null).
struct Op : zq_linear_desc {
    float *out32 = nullptr;
    int xbf16 = 0;  // x and out hold bfloat16 (out32 must then be null)
};

Op make_op(const zq_linear_desc &d) {
    Op o;
    static_cast<zq_linear_desc &>(o) = d;
    return o;
}

// Validation of an op with an fp32 output.
zq_status check_partial(const zq_linear_desc &d, const float *out32) {
    zq_linear_desc t = d;
    t.out = reinterpret_cast<uint16_t *>(const_cast<float *>(out32));
    return check_linear(t);
}

// ---------------------------------------------------------------- device --

struct DeviceInfo {
    int sms = 0;
    std::map<std::tuple<int, int, size_t>, int> occ;  // (bits, mt, smem) -> decode CTAs per SM
};
std::mutex g_dev_mu;
std::map<int, DeviceInfo> g_dev;

zq_status device_info(DeviceInfo **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lk(g_dev_mu);
    auto it = g_dev.find(dev);
    if (it == g_dev.end()) {
        DeviceInfo info;
        e = cudaDeviceGetAttribute(&info.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        it = g_dev.emplace(dev, info).first;
    }
    *out = &it->second;
    return ZQ_OK;
}

zq_status decode_occupancy(DeviceInfo *info, int bits, int mt, size_t smem, int *ctas) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    int &o = info->occ[std::make_tuple(bits, mt, smem)];
    if (o == 0) {
        cudaError_t e = decode_ctas_per_sm(bits, mt, smem, &o);
        if (e != cudaSuccess) return cuda_fail(e, "occupancy query");
        if (o <= 0) return fail(ZQ_ERR_CUDA, "decode kernel does not fit on an SM");
    }
    *ctas = o;
    return ZQ_OK;
}

// ------------------------------------------------------------- workspace --
// One buffer per (device, stream), keyed by the stream's unique id (so a
// stream handle that CUDA recycles after cudaStreamDestroy never inherits
// another stream's buffer).  Layout: [counters | data].  The counters are
// zeroed when the buffer is reserved or attached, every kernel that uses one
// resets it to zero, and after a kernel gave up a wait (which can leave them
// set) zq_check_device marks the buffers dirty: the next call on the stream
// clears them with an asynchronous memset before its launches.
// Calls never allocate, free or synchronise: a buffer comes from
// zq_reserve_workspace (the library allocates it) or zq_attach_workspace (the
// caller owns it), and a call that needs more than the stream holds fails.

constexpr size_t kCounterBytes = 256 * 1024;
constexpr size_t kMaxCounters = kCounterBytes / sizeof(unsigned int);

struct Workspace {
    void *ptr = nullptr;
    size_t bytes = 0;
    bool owned = false;  // allocated by zq_reserve_workspace (else the caller's)
    bool dirty = false;  // counters must be cleared before the next use
};
std::mutex g_ws_mu;
std::map<std::pair<int, unsigned long long>, Workspace> g_ws;

zq_status stream_key(cudaStream_t stream, std::pair<int, unsigned long long> *key) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    unsigned long long id = 0;
    e = cudaStreamGetId(stream, &id);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamGetId");
    *key = {dev, id};
    return ZQ_OK;
}

// Base of the stream's workspace if it holds kCounterBytes + data_bytes;
// clears dirty counters first (stream-ordered).  Never allocates.
zq_status workspace(cudaStream_t stream, size_t data_bytes, uint8_t **base) {
    std::pair<int, unsigned long long> key;
    zq_status st = stream_key(stream, &key);
    if (st != ZQ_OK) return st;
    const size_t need = kCounterBytes + data_bytes;
    std::lock_guard<std::mutex> lk(g_ws_mu);
    auto it = g_ws.find(key);
    const size_t have = it == g_ws.end() ? 0 : it->second.bytes;
    if (have < need)
        return fail(ZQ_ERR_INVALID_ARG,
                    "this call needs a workspace of %zu bytes on its stream, which holds %zu; reserve it "
                    "beforehand with zq_reserve_workspace (or attach one with zq_attach_workspace)",
                    need, have);
    Workspace &ws = it->second;
    if (ws.dirty) {
        cudaError_t e = cudaMemsetAsync(ws.ptr, 0, kCounterBytes, stream);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the workspace counters");
        ws.dirty = false;
    }
    *base = static_cast<uint8_t *>(ws.ptr);
    return ZQ_OK;
}

// Marks every workspace of `dev` dirty (after a kernel gave up a wait).
void workspaces_dirty(int dev) {
    std::lock_guard<std::mutex> lk(g_ws_mu);
    for (auto &kv : g_ws)
        if (kv.first.first == dev) kv.second.dirty = true;
}

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// ------------------------------------------------------------ decode plan --

struct PrepKey {
    const uint16_t *x;
    int M, K, bits, xbf16;
    bool operator==(const PrepKey &o) const {
        return x == o.x && M == o.M && K == o.K && bits == o.bits && xbf16 == o.xbf16;
    }
};

// Shared memory of one decode CTA: `depth` stages, two mbarriers per stage,
// the producer's scheduling state, and slack to align the ring to 1024 bytes.
size_t decode_smem(int stage_bytes, int depth) { return static_cast<size_t>(depth) * (stage_bytes + 16) + 64 + 1024; }
size_t align16(size_t b) { return (b + 15) & ~size_t(15); }

// Plans and launches one decode launch over ops that share bits and MT and are
// mutually independent.  With `dry_bytes` set, only computes the workspace size.
zq_status run_decode(const std::vector<Op> &ops, int bits, int mt, cudaStream_t stream,
                     size_t *dry_bytes = nullptr, uint8_t *fixed_ws = nullptr, size_t fixed_ws_bytes = 0) {
    DeviceInfo *info = nullptr;
    zq_status st = device_info(&info);
    if (st != ZQ_OK) return st;
    const int rows = decode_cta_rows(bits, mt);
    const int mpad = 8 * mt;
    const int gps = decode_gps(bits, mt);

    // Prep entries (distinct activation buffers).
    std::vector<PrepKey> keys;
    std::vector<int> op_entry(ops.size());
    for (size_t i = 0; i < ops.size(); ++i) {
        PrepKey k{ops[i].x, ops[i].M, ops[i].K, bits, ops[i].xbf16};
        auto it = std::find(keys.begin(), keys.end(), k);
        if (it == keys.end()) {
            keys.push_back(k);
            op_entry[i] = static_cast<int>(keys.size()) - 1;
        } else {
            op_entry[i] = static_cast<int>(it - keys.begin());
        }
    }
    if (keys.size() > static_cast<size_t>(kMaxPrepEntries) || ops.size() > static_cast<size_t>(kMaxDecodeOps))
        return fail(ZQ_ERR_INVALID_ARG, "internal: decode launch too large");

    // Work: CTA steps (op, row block, GPS groups), all of equal cost within
    // a launch (same bits).
    long long total_steps = 0, total_units = 0;
    int max_m = 1;
    std::vector<int> rbs(ops.size()), sus(ops.size());
    for (size_t i = 0; i < ops.size(); ++i) {
        rbs[i] = (ops[i].N + rows - 1) / rows;
        sus[i] = (ops[i].K / kGroup + gps - 1) / gps;
        total_steps += static_cast<long long>(rbs[i]) * sus[i];
        total_units += rbs[i];
        max_m = std::max(max_m, ops[i].M);
    }
    if (total_steps > 0x3FFFFFFFLL) return fail(ZQ_ERR_INVALID_ARG, "decode launch too large (steps)");

    // Stage: codes (the step's rows x the box bytes, a multiple of 1024; all
    // stages' codes first, so each starts 1024-aligned), then a meta part of
    // scales and zeros, group sums, activations and the step descriptor.
    const int codes_bytes = decode_codes_bytes(bits, mt);
    const int off_sz = 0;
    const int off_sx = off_sz + rows * 4 * gps;
    const int x_rows_max = mt == 1 ? max_m : mpad;  // staged token rows (and group records)
    const int off_x = off_sx + decode_rec_stride(bits, mt) * x_rows_max * 16;
    const int off_desc = off_x + gps * x_rows_max * 256;
    const int meta_bytes = static_cast<int>(align16(off_desc + 32));
    const int stage = codes_bytes + meta_bytes;
    // Depth: at least 3 stages with as many CTAs per SM as the registers allow
    // (228 KB of shared memory per SM, 1 KB of it reserved per CTA).
    const int reg_ctas = decode_reg_ctas(bits, mt);
    int depth = 0, want_ctas = reg_ctas;
    for (; want_ctas >= 1; --want_ctas) {
        const long long budget = 228 * 1024 / want_ctas - 1024;
        depth = static_cast<int>(std::min<long long>(6, (budget - 1024 - 64) / (stage + 16)));
        if (depth >= 3) break;
    }
    if (want_ctas < 1) {
        want_ctas = 1;
        depth = static_cast<int>(std::min<long long>(6, (227 * 1024 - 1024 - 64) / (stage + 16)));
        if (depth < 2) return fail(ZQ_ERR_UNSUPPORTED, "decode stage of %d bytes does not fit", stage);
    }
    const size_t smem = decode_smem(stage, depth);
    int occ = 0;
    if ((st = decode_occupancy(info, bits, mt, smem, &occ)) != ZQ_OK) return st;
    const long long max_ctas = static_cast<long long>(occ) * info->sms;

    // Chunks.  Large launches: whole row blocks, taken dynamically, longest
    // row blocks first (so the last ones handed out are short).  Otherwise
    // chunks of 2^log2c steps: dynamic with at least 16 steps per CTA, else
    // one chunk per CTA.
    int log2c = 0, dynamic = 0, units = 0, n_ctas = 0;
    long long n_chunks = 0;
    std::vector<size_t> order(ops.size());
    for (size_t i = 0; i < ops.size(); ++i) order[i] = i;
    if (total_units >= 4 * max_ctas) {
        units = 1;
        dynamic = 1;
        n_chunks = total_units;
        n_ctas = static_cast<int>(max_ctas);
        std::stable_sort(order.begin(), order.end(), [&](size_t a, size_t b) { return sus[a] > sus[b]; });
    } else if (total_steps >= 16 * max_ctas) {
        const long long per = total_steps / (12 * max_ctas);
        log2c = 2;
        while (log2c < 8 && (2LL << log2c) <= per) ++log2c;
        dynamic = 1;
        n_chunks = (total_steps + (1LL << log2c) - 1) >> log2c;
        n_ctas = static_cast<int>(max_ctas);
    } else {
        const long long per = (total_steps + max_ctas - 1) / max_ctas;
        while ((1LL << log2c) < per) ++log2c;
        n_chunks = (total_steps + (1LL << log2c) - 1) >> log2c;
        n_ctas = static_cast<int>(n_chunks);
    }
    if (!units && static_cast<size_t>(n_chunks) + 1 > kMaxCounters - 2)  // the last 2 are the tile kernel's
        return fail(ZQ_ERR_INVALID_ARG, "internal: too many chunks");
    const int slot_floats = rows * mpad;

    // Workspace layout.
    size_t off = 0;
    std::vector<size_t> prep_off(keys.size());
    for (size_t e = 0; e < keys.size(); ++e) {
        prep_off[e] = off;
        const size_t G = keys[e].K / kGroup;
        const size_t xr = mt == 1 ? keys[e].M : mpad;
        const size_t steps = (G + gps - 1) / gps;  // x' and records are stored by step (whole GPS blocks)
        off += align256(steps * gps * xr * kGroup * 2) + align256(steps * decode_rec_stride(bits, mt) * xr * 16);
    }
    const size_t part_off = off;
    if (!units) off += align256(static_cast<size_t>(n_chunks) * 2 * slot_floats * 4);
    if (dry_bytes) {
        *dry_bytes = off + kCounterBytes;
        return ZQ_OK;
    }
    uint8_t *ws = fixed_ws;
    if (ws == nullptr) {
        if ((st = workspace(stream, off, &ws)) != ZQ_OK) return st;
    } else if (kCounterBytes + off > fixed_ws_bytes) {
        return fail(ZQ_ERR_UNSUPPORTED, "call needs %zu bytes of scratch, the fixed scratch holds %zu",
                    kCounterBytes + off, fixed_ws_bytes);
    }
    uint8_t *data = ws + kCounterBytes;

    // The kernels' parameter blocks travel with every launch: launches of few
    // ops and activations use the small blocks.
    auto fill_and_launch = [&](auto &pp, auto &dp) -> zq_status {
        std::memset(&pp, 0, sizeof(pp));
        pp.n_entries = static_cast<int>(keys.size());
        pp.work = reinterpret_cast<unsigned int *>(ws);
        long long wsum = 0;
        for (size_t e = 0; e < keys.size(); ++e) {
            PrepEntry &en = pp.e[e];
            const size_t G = keys[e].K / kGroup;
            en.x = keys[e].x;
            en.xg = reinterpret_cast<uint16_t *>(data + prep_off[e]);
            en.x_rows = mt == 1 ? keys[e].M : mpad;
            const size_t steps = (G + gps - 1) / gps;
            en.sx = reinterpret_cast<float *>(data + prep_off[e] + align256(steps * gps * en.x_rows * kGroup * 2));
            en.M = keys[e].M;
            en.x_bf16 = keys[e].xbf16;
            en.K = keys[e].K;
            en.bits = bits;
            en.gps = gps;
            en.rs = decode_rec_stride(bits, mt);
            pp.warp_prefix[e] = wsum;
            wsum += static_cast<long long>(en.x_rows) * G;
        }
        pp.warp_prefix[keys.size()] = wsum;

        std::memset(&dp, 0, sizeof(dp));
        dp.part = reinterpret_cast<float *>(data + part_off);
        dp.cnt = reinterpret_cast<unsigned int *>(ws);
        dp.total_steps = static_cast<int>(total_steps);
        dp.n_ops = static_cast<int>(ops.size());
        dp.slot_floats = slot_floats;
        dp.log2c = log2c;
        dp.n_chunks = static_cast<int>(n_chunks);
        dp.units = units;
        dp.dynamic = dynamic;
        dp.depth = depth;
        dp.codes_bytes = codes_bytes;
        dp.meta_bytes = meta_bytes;
        dp.off_sz = off_sz;
        dp.off_sx = off_sx;
        dp.off_x = off_x;
        dp.off_desc = off_desc;
        dp.wait_ns = g_wait_ns.load();
        const bool swz = decode_swizzled(bits, mt);
        int step0 = 0, unit0 = 0;
        for (size_t oi = 0; oi < ops.size(); ++oi) {
            const size_t i = order[oi];
            DecodeOp &o = dp.ops[oi];
            const PrepEntry &en = pp.e[op_entry[i]];
            o.scales = ops[i].scales;
            o.zeros = ops[i].zeros;
            o.xg = en.xg;
            o.sx = en.sx;
            o.out = ops[i].out;
            o.out32 = ops[i].out32;
            o.M = ops[i].M;
            o.N = ops[i].N;
            o.K = ops[i].K;
            o.G = ops[i].K / kGroup;
            o.row_blocks = rbs[i];
            o.su = sus[i];
            o.sz_vec = (bits != 16 && (o.G % gps) == 0) ? 1 : 0;  // fp16 weights have no scales or zeros
            o.out_bf16 = ops[i].xbf16;
            const uint64_t row_bytes = static_cast<uint64_t>(o.K) * bits / 8;
            cudaError_t te = encode_tensor_map_2d(&o.tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, ops[i].packed, row_bytes,
                                                  static_cast<uint64_t>(o.N), row_bytes,
                                                  static_cast<uint32_t>(decode_box_w(bits, mt)),
                                                  static_cast<uint32_t>(rows),
                                                  swz ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
            if (te != cudaSuccess) return cuda_fail(te, "tensor map for the packed codes");
            o.step0 = step0;
            o.unit0 = unit0;
            step0 += rbs[i] * sus[i];
            unit0 += rbs[i];
        }

        cudaError_t e = launch_prep(pp, wsum, stream);
        if (e != cudaSuccess) return cuda_fail(e, "prep launch");
        e = launch_decode(dp, bits, mt, n_ctas, smem, stream);
        if (e != cudaSuccess) return cuda_fail(e, "decode launch");
        return ZQ_OK;
    };
    zq_status fs;
    if (keys.size() <= static_cast<size_t>(kSmallLaunchOps) && ops.size() <= static_cast<size_t>(kSmallLaunchOps)) {
        PrepParamsSmall pp;
        DecodeParamsSmall dp;
        fs = fill_and_launch(pp, dp);
    } else {
        PrepParams pp;
        DecodeParams dp;
        fs = fill_and_launch(pp, dp);
    }
    if (fs != ZQ_OK) return fs;
    g_launches += 2;
    return ZQ_OK;
}

// Byte range of each buffer an op touches.
struct Range {
    uintptr_t lo, hi;
};
bool overlap(const Range &a, const Range &b) { return a.lo < b.hi && b.lo < a.hi; }

struct OpRanges {
    Range x, packed, scales, zeros, out;
};

OpRanges ranges_of(const Op &d) {
    const size_t G = d.bits == 16 ? 0 : d.K / d.group;  // fp16 weights have no scales or zeros
    auto r = [](const void *p, size_t n) {
        const uintptr_t a = reinterpret_cast<uintptr_t>(p);
        return Range{a, a + n};
    };
    return OpRanges{r(d.x, static_cast<size_t>(d.M) * d.K * 2),
                    r(d.packed, static_cast<size_t>(d.N) * d.K * d.bits / 8),
                    r(d.scales, static_cast<size_t>(d.N) * G * 2), r(d.zeros, static_cast<size_t>(d.N) * G * 2),
                    d.out32 ? r(d.out32, static_cast<size_t>(d.M) * d.N * 4)
                            : r(d.out, static_cast<size_t>(d.M) * d.N * 2)};
}

// b depends on a (a earlier) if they share memory with at least one write.
bool conflicts(const OpRanges &a, const OpRanges &b) {
    const Range *reads_a[] = {&a.x, &a.packed, &a.scales, &a.zeros};
    const Range *reads_b[] = {&b.x, &b.packed, &b.scales, &b.zeros};
    for (const Range *r : reads_b)
        if (overlap(a.out, *r)) return true;
    for (const Range *r : reads_a)
        if (overlap(b.out, *r)) return true;
    return overlap(a.out, b.out);
}

// One persistent launch over all tiles of independent prefill ops of one bit
// width (at most kMaxPrefillOps), ops with the longest K first so that the
// last tiles handed out are the cheap ones.
// The one-token-half plan (every M <= 128) with b-bit codes reads each x as a
// copy whose 32-value chunks are pair-permuted (the order of its dequant
// routine's fp16 pairs); bf16 activations are copied to fp16 whatever the plan.
bool prefill_perm(const std::vector<Op> &ops) {
    int max_m = 0;
    for (const auto &d : ops) max_m = std::max(max_m, d.M);
    return !ops.empty() && max_m <= kPrefillHalfTokens && ops[0].bits != 16;
}
bool prefill_copies(const Op &d, bool perm) { return d.xbf16 || perm; }
bool same_x(const Op &a, const Op &b) { return a.x == b.x && a.M == b.M && a.K == b.K && a.xbf16 == b.xbf16; }

// Workspace bytes of a tile-kernel launch: the fp16 copies (and, for bf16
// activations, per-token factors) of its distinct activations.
size_t prefill_data_bytes(const std::vector<Op> &ops) {
    const bool perm = prefill_perm(ops);
    size_t b = 0;
    for (size_t i = 0; i < ops.size(); ++i) {
        const Op &d = ops[i];
        if (!prefill_copies(d, perm)) continue;
        bool seen = false;
        for (size_t j = 0; j < i; ++j) seen = seen || same_x(ops[j], d);
        if (seen) continue;
        b += align256(static_cast<size_t>(d.M) * d.K * 2) + (d.xbf16 ? align256(static_cast<size_t>(d.M) * 4) : 0);
    }
    return b;
}

zq_status run_prefill(std::vector<Op> ops, cudaStream_t stream) {
    DeviceInfo *info = nullptr;
    zq_status st = device_info(&info);
    if (st != ZQ_OK) return st;
    std::stable_sort(ops.begin(), ops.end(), [](const Op &a, const Op &b) { return a.K > b.K; });
    uint8_t *ws = nullptr;
    if ((st = workspace(stream, prefill_data_bytes(ops), &ws)) != ZQ_OK) return st;
    // Activation copies in the workspace (see zq_act.cu), one per distinct x;
    // the launch reads the copy: bf16 x scaled per token into fp16, and with
    // the one-token-half plan every 32-value chunk pair-permuted.
    const bool perm = prefill_perm(ops);
    struct Copy {
        const Op *src;
        uint16_t *x16;
        float *f;
    };
    std::vector<Copy> conv;
    uint8_t *at = ws + kCounterBytes;
    for (const auto &d : ops) {
        if (!prefill_copies(d, perm)) continue;
        bool known = false;
        for (const auto &c : conv) known = known || same_x(*c.src, d);
        if (known) continue;
        uint16_t *x16 = reinterpret_cast<uint16_t *>(at);
        at += align256(static_cast<size_t>(d.M) * d.K * 2);
        float *f = nullptr;
        cudaError_t e;
        if (d.xbf16) {
            f = reinterpret_cast<float *>(at);
            at += align256(static_cast<size_t>(d.M) * 4);
            e = launch_bf16_rows_to_f16(d.x, d.M, d.K, perm ? d.bits : 0, x16, f, stream);
        } else {
            e = launch_x_pairperm(d.x, d.M, d.K, d.bits, x16, stream);
        }
        if (e != cudaSuccess) return cuda_fail(e, "activation copy launch");
        g_launches += 1;
        conv.push_back({&d, x16, f});
    }
    PrefillGroup pg;
    std::memset(&pg, 0, sizeof(pg));
    pg.n_ops = static_cast<int>(ops.size());
    for (size_t i = 0; i < ops.size(); ++i) pg.ops[i].M = ops[i].M;
    const int plan = prefill_plan(pg, ops[0].bits);  // the plan the launch will run
    const int box_rows = prefill_box_rows(plan), tok_tile = prefill_tok_tile(plan);
    int tiles = 0;
    for (size_t i = 0; i < ops.size(); ++i) {
        PrefillOp &o = pg.ops[i];
        const uint16_t *xa = ops[i].x;
        for (const auto &c : conv)
            if (same_x(*c.src, ops[i])) {
                xa = c.x16;
                o.xscale = c.f;  // null for fp16 x
            }
        o.out_bf16 = ops[i].xbf16;
        cudaError_t e = prefill_x_map_rows(&o.xmap, xa, ops[i].M, ops[i].K, box_rows);
        if (e != cudaSuccess) return cuda_fail(e, "tensor map for x");
        if (ops[i].bits == 16) {
            e = prefill_w_map(&o.wmap, reinterpret_cast<const uint16_t *>(ops[i].packed), ops[i].N, ops[i].K);
            if (e != cudaSuccess) return cuda_fail(e, "tensor map for the fp16 weights");
        }
        o.packed = ops[i].packed;
        o.scales = ops[i].scales;
        o.zeros = ops[i].zeros;
        o.out = ops[i].out;
        o.out32 = ops[i].out32;
        o.M = ops[i].M;
        o.N = ops[i].N;
        o.K = ops[i].K;
        o.gshift = ops[i].bits == 16 ? 2 : (ops[i].group == 32 ? 0 : ops[i].group == 64 ? 1 : 2);
        o.tok_tiles = (ops[i].M + tok_tile - 1) / tok_tile;
        o.tile0 = tiles;
        tiles += prefill_tiles(ops[i].M, ops[i].N, plan);
    }
    pg.n_tiles = tiles;
    pg.wait_ns = g_wait_ns.load();
    pg.tile_ctr = reinterpret_cast<unsigned int *>(ws) + (kMaxCounters - 2);
    cudaError_t e = launch_prefill_group(pg, ops[0].bits, info->sms, stream);
    if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
    g_launches += 1;
    return ZQ_OK;
}

// Launches a batch of mutually independent ops: one launch per (bits, MT)
// class, each holding at most kMaxDecodeOps ops and kMaxPrepEntries inputs.
// With `dry` set nothing is launched: *dry becomes the largest workspace any
// of the launches needs (at least the counters).
zq_status run_batch(const std::vector<Op> &batch, cudaStream_t stream, size_t *dry = nullptr) {
    std::vector<Op> pieces;
    const int bits_list[5] = {2, 3, 4, 8, 16};
    if (dry) *dry = std::max(*dry, kCounterBytes);
    // The decode kernel applies one scale and zero per 128-code block, so
    // groups of 32 or 64 run on the tile kernel at any M.
    const auto on_tile = [](const Op &d) { return d.M > kDecodeMaxM || (d.bits != 16 && d.group != kGroup); };
    for (int bits : bits_list) {
        std::vector<Op> pre;
        for (const auto &d : batch)
            if (on_tile(d) && d.bits == bits) pre.push_back(d);
        for (size_t i = 0; i < pre.size(); i += kMaxPrefillOps) {
            std::vector<Op> launch(pre.begin() + i,
                                               pre.begin() + std::min(pre.size(), i + kMaxPrefillOps));
            if (dry) {
                *dry = std::max(*dry, kCounterBytes + prefill_data_bytes(launch));
                continue;
            }
            zq_status st = run_prefill(launch, stream);
            if (st != ZQ_OK) return st;
        }
    }
    for (const auto &d : batch)
        if (!on_tile(d)) pieces.push_back(d);
    const int mt_list[3] = {1, 2, 4};
    for (int bits : bits_list)
        for (int mt : mt_list) {
            std::vector<Op> cls;
            for (const auto &d : pieces)
                if (d.bits == bits && mt_for_m(d.M) == mt) cls.push_back(d);
            size_t i = 0;
            while (i < cls.size()) {
                std::vector<Op> launch;
                std::vector<std::pair<const uint16_t *, int>> inputs;
                while (i < cls.size() && launch.size() < static_cast<size_t>(kMaxDecodeOps)) {
                    std::pair<const uint16_t *, int> key{cls[i].x, cls[i].M * 1000003 + cls[i].K};
                    const bool known = std::find(inputs.begin(), inputs.end(), key) != inputs.end();
                    if (!known && inputs.size() == static_cast<size_t>(kMaxPrepEntries)) break;
                    if (!known) inputs.push_back(key);
                    launch.push_back(cls[i++]);
                }
                size_t b = 0;
                zq_status st = run_decode(launch, bits, mt, stream, dry ? &b : nullptr);
                if (st != ZQ_OK) return st;
                if (dry) *dry = std::max(*dry, b);
            }
        }
    return ZQ_OK;
}

// Splits a stack into batches of mutually independent ops (an op that shares
// written memory with an earlier op of the batch starts the next batch) and
// runs them in order; with `dry` set, only sizes the workspace.
zq_status run_stack(const Op *ops, int n_ops, cudaStream_t s, size_t *dry) {
    std::vector<Op> batch;
    std::vector<OpRanges> br;
    constexpr size_t kMaxBatch = 1024;
    for (int i = 0; i < n_ops; ++i) {
        const OpRanges r = ranges_of(ops[i]);
        bool dep = batch.size() >= kMaxBatch;
        for (size_t j = 0; j < br.size() && !dep; ++j) dep = conflicts(br[j], r);
        if (dep) {
            zq_status st = run_batch(batch, s, dry);
            if (st != ZQ_OK) return st;
            batch.clear();
            br.clear();
        }
        batch.push_back(ops[i]);
        br.push_back(r);
    }
    if (!batch.empty()) return run_batch(batch, s, dry);
    return ZQ_OK;
}

// Checks that the stream's workspace covers the stack (nothing is enqueued
// when it does not, apart from clearing counters a failed kernel left set),
// then runs it.
zq_status checked_stack(const Op *ops, int n_ops, cudaStream_t s) {
    if (n_ops == 0) return ZQ_OK;
    size_t need = kCounterBytes;
    zq_status st = run_stack(ops, n_ops, s, &need);
    if (st != ZQ_OK) return st;
    uint8_t *base = nullptr;
    if ((st = workspace(s, need - kCounterBytes, &base)) != ZQ_OK) return st;
    return run_stack(ops, n_ops, s, nullptr);
}

// ------------------------------------------------------ allocation-free path --
// Scratch of zq_linear_noalloc: a fixed device array in this file, so that
// call never allocates.  Every GPU that loads the library holds it until the
// process exits.  Device code could name the array directly; host code needs
// its device address, looked up once per device.

constexpr size_t kNoallocScratchBytes = 4u << 20;  // 4 MiB
constexpr int kNoallocMaxM = 8;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mu;
std::map<std::pair<int, unsigned long long>, uint8_t *> g_noalloc_addr;  // (device, context id) -> address

// Unique id of the calling thread's current CUDA context (0 if none or not
// available).  A context torn down and created again (cudaDeviceReset) gets a
// new id, so an address cached for the old one is never reused.
unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch array in the current device's context, looked
// up once per (device, context) with that device current.
zq_status noalloc_scratch(uint8_t **ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    auto it = g_noalloc_addr.find({dev, ctx});
    if (it == g_noalloc_addr.end() || ctx == 0) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
        const unsigned long long ctx_now = current_context_id();  // the lookup may have created the context
        if (ctx_now == 0) {
            *ptr = static_cast<uint8_t *>(p);
            return ZQ_OK;
        }
        it = g_noalloc_addr.insert_or_assign({dev, ctx_now}, static_cast<uint8_t *>(p)).first;
    }
    *ptr = it->second;
    return ZQ_OK;
}

}  // namespace

// =================================================================== C ABI ==

extern "C" {

size_t zq_packed_words(int N, int K, int bits) {
    if (!bits_ok(bits) || N <= 0 || K <= 0 || K % kGroup != 0) return 0;
    return static_cast<size_t>(N) * K * bits / 32;
}

zq_status zq_quantize_pack(const float *w, int N, int K, int bits, int group, uint32_t *packed,
                           uint16_t *scales, uint16_t *zeros, zq_stream_t stream) {
    zq_status st = check_format(bits, group, N, K);
    if (st != ZQ_OK) return st;
    if ((st = check_ptr(w, "w")) != ZQ_OK) return st;
    if ((st = check_ptr(packed, "packed")) != ZQ_OK) return st;
    if ((st = check_ptr(scales, "scales")) != ZQ_OK) return st;
    if ((st = check_ptr(zeros, "zeros")) != ZQ_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const unsigned long long id = g_quant_call.fetch_add(1);
    const int slot = static_cast<int>(id % kQuantStatusSlots);
    cudaError_t e = launch_quantize_pack(w, N, K, bits, group, packed, scales, zeros, slot, id, s);
    if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
    ++g_launches;
    unsigned long long got = 0;
    e = read_quant_status(slot, &got, s);
    if (e != cudaSuccess) return cuda_fail(e, "quantize status");
    if (got == id) return fail(ZQ_ERR_NONFINITE, "weights contain NaN/Inf or |w| > 65504");
    return ZQ_OK;
}

zq_status zq_quantize_pack_symmetric(const float *w, int N, int K, int bits, int group, uint32_t *packed,
                                     uint16_t *scales, uint16_t *zeros, zq_stream_t stream) {
    zq_status st = check_format(bits, group, N, K);
    if (st != ZQ_OK) return st;
    if ((st = check_ptr(w, "w")) != ZQ_OK) return st;
    if ((st = check_ptr(packed, "packed")) != ZQ_OK) return st;
    if ((st = check_ptr(scales, "scales")) != ZQ_OK) return st;
    if ((st = check_ptr(zeros, "zeros")) != ZQ_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const unsigned long long id = g_quant_call.fetch_add(1);
    const int slot = static_cast<int>(id % kQuantStatusSlots);
    cudaError_t e = launch_quantize_pack_symmetric(w, N, K, bits, group, packed, scales, zeros, slot, id, s);
    if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
    ++g_launches;
    unsigned long long got = 0;
    e = read_quant_status(slot, &got, s);
    if (e != cudaSuccess) return cuda_fail(e, "quantize status");
    if (got == id)
        return fail(ZQ_ERR_NONFINITE,
                    "weights contain NaN/Inf or |w| > 65504, or a group's symmetric zero "
                    "-2^(bits-1)*scale is not a finite fp16");
    return ZQ_OK;
}

zq_status zq_linear(const uint16_t *x, const uint32_t *packed, const uint16_t *scales,
                    const uint16_t *zeros, int bits, int group, int M, int N, int K, uint16_t *out,
                    zq_stream_t stream) {
    zq_linear_desc d{x, packed, scales, zeros, out, bits, group, M, N, K};
    zq_status st = check_linear(d);
    if (st != ZQ_OK) return st;
    const Op op = make_op(d);
    return checked_stack(&op, 1, reinterpret_cast<cudaStream_t>(stream));
}

zq_status zq_linear_partial(const uint16_t *x, const uint32_t *packed, const uint16_t *scales,
                            const uint16_t *zeros, int bits, int group, int M, int N, int K, float *out,
                            zq_stream_t stream) {
    zq_linear_desc d{x, packed, scales, zeros, nullptr, bits, group, M, N, K};
    zq_status st = check_partial(d, out);
    if (st != ZQ_OK) return st;
    Op op = make_op(d);
    op.out32 = out;
    return checked_stack(&op, 1, reinterpret_cast<cudaStream_t>(stream));
}

zq_status zq_linear_noalloc(const uint16_t *x, const uint32_t *packed, const uint16_t *scales,
                            const uint16_t *zeros, int bits, int group, int M, int N, int K, uint16_t *out,
                            zq_stream_t stream) {
    zq_linear_desc d{x, packed, scales, zeros, out, bits, group, M, N, K};
    zq_status st = check_linear(d);
    if (st != ZQ_OK) return st;
    if (M > kNoallocMaxM)
        return fail(ZQ_ERR_UNSUPPORTED, "zq_linear_noalloc supports M <= %d (got M=%d)", kNoallocMaxM, M);
    if (bits != 16 && group != kGroup)
        return fail(ZQ_ERR_UNSUPPORTED, "zq_linear_noalloc supports groups of 128 (got %d)", group);
    uint8_t *ws = nullptr;
    if ((st = noalloc_scratch(&ws)) != ZQ_OK) return st;
    std::vector<Op> one{make_op(d)};
    size_t need = 0;
    if ((st = run_decode(one, bits, mt_for_m(M), nullptr, &need)) != ZQ_OK) return st;
    if (need > kNoallocScratchBytes)
        return fail(ZQ_ERR_UNSUPPORTED, "zq_linear_noalloc: this call needs %zu bytes of scratch, the limit is %zu",
                    need, kNoallocScratchBytes);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // The split-K arrival counters must start at zero; the array keeps what the
    // previous call left, so clear them (a memset, not an allocation).
    cudaError_t e = cudaMemsetAsync(ws, 0, kCounterBytes, s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the scratch counters");
    return run_decode(one, bits, mt_for_m(M), s, nullptr, ws, kNoallocScratchBytes);
}

zq_status zq_linear_bf16(const uint16_t *x, const uint32_t *packed, const uint16_t *scales,
                         const uint16_t *zeros, int bits, int group, int M, int N, int K, uint16_t *out,
                         zq_stream_t stream) {
    zq_linear_desc d{x, packed, scales, zeros, out, bits, group, M, N, K};
    zq_status st = check_linear(d);
    if (st != ZQ_OK) return st;
    Op op = make_op(d);
    op.xbf16 = 1;
    return checked_stack(&op, 1, reinterpret_cast<cudaStream_t>(stream));
}

// Validates the public descriptors of a stack (fp16 outputs, or fp32 partial
// sums when `partial`) into internal ops; reports the first bad op.
zq_status stack_ops(const zq_linear_desc *ops, const zq_partial_desc *pops, int n_ops, std::vector<Op> *out) {
    if (n_ops < 0 || (n_ops > 0 && ops == nullptr && pops == nullptr))
        return fail(ZQ_ERR_INVALID_ARG, "ops is null or n_ops < 0");
    out->clear();
    out->reserve(n_ops);
    for (int i = 0; i < n_ops; ++i) {
        Op op;
        zq_status st;
        if (ops) {
            op = make_op(ops[i]);
            st = check_linear(ops[i]);
        } else {
            const zq_partial_desc &p = pops[i];
            op = make_op(zq_linear_desc{p.x, p.packed, p.scales, p.zeros, nullptr, p.bits, p.group, p.M, p.N, p.K});
            op.out32 = p.out;
            st = check_partial(op, p.out);
        }
        if (st != ZQ_OK) {
            std::string msg = g_last_error;
            return fail(st, "op %d: %s", i, msg.c_str());
        }
        out->push_back(op);
    }
    return ZQ_OK;
}

zq_status zq_linear_stack(const zq_linear_desc *ops, int n_ops, zq_stream_t stream) {
    std::vector<Op> v;
    zq_status st = stack_ops(ops, nullptr, n_ops, &v);
    if (st != ZQ_OK) return st;
    return checked_stack(v.data(), n_ops, reinterpret_cast<cudaStream_t>(stream));
}

zq_status zq_linear_stack_bf16(const zq_linear_desc *ops, int n_ops, zq_stream_t stream) {
    std::vector<Op> v;
    zq_status st = stack_ops(ops, nullptr, n_ops, &v);
    if (st != ZQ_OK) return st;
    for (auto &op : v) op.xbf16 = 1;
    return checked_stack(v.data(), n_ops, reinterpret_cast<cudaStream_t>(stream));
}

size_t zq_linear_stack_bf16_workspace_bytes(const zq_linear_desc *ops, int n_ops) {
    std::vector<Op> v;
    if (stack_ops(ops, nullptr, n_ops, &v) != ZQ_OK) return 0;
    for (auto &op : v) op.xbf16 = 1;
    size_t need = 0;
    if (run_stack(v.data(), n_ops, nullptr, &need) != ZQ_OK) return 0;
    return need;
}

zq_status zq_linear_partial_stack(const zq_partial_desc *ops, int n_ops, zq_stream_t stream) {
    std::vector<Op> v;
    zq_status st = stack_ops(nullptr, ops, n_ops, &v);
    if (st != ZQ_OK) return st;
    return checked_stack(v.data(), n_ops, reinterpret_cast<cudaStream_t>(stream));
}

size_t zq_linear_stack_workspace_bytes(const zq_linear_desc *ops, int n_ops) {
    std::vector<Op> v;
    if (stack_ops(ops, nullptr, n_ops, &v) != ZQ_OK) return 0;
    size_t need = 0;
    if (run_stack(v.data(), n_ops, nullptr, &need) != ZQ_OK) return 0;
    return need;
}

size_t zq_linear_partial_stack_workspace_bytes(const zq_partial_desc *ops, int n_ops) {
    std::vector<Op> v;
    if (stack_ops(nullptr, ops, n_ops, &v) != ZQ_OK) return 0;
    size_t need = 0;
    if (run_stack(v.data(), n_ops, nullptr, &need) != ZQ_OK) return 0;
    return need;
}

zq_status zq_reduce_partials(const float *const *parts, int n_parts, size_t count, uint16_t *out,
                             zq_stream_t stream) {
    if (n_parts < 1 || n_parts > kMaxReduceParts)
        return fail(ZQ_ERR_INVALID_ARG, "n_parts=%d must be in [1, %d]", n_parts, kMaxReduceParts);
    if (parts == nullptr) return fail(ZQ_ERR_INVALID_ARG, "parts is null");
    if (count == 0) return ZQ_OK;
    zq_status st;
    for (int i = 0; i < n_parts; ++i)
        if ((st = check_ptr(parts[i], "parts[i]")) != ZQ_OK) return st;
    if ((st = check_ptr(out, "out")) != ZQ_OK) return st;
    cudaError_t e = launch_reduce_partials(parts, n_parts, count, out, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "reduce launch");
    ++g_launches;
    return ZQ_OK;
}

zq_status zq_unpack(const uint32_t *packed, int N, int K, int bits, uint8_t *codes, zq_stream_t stream) {
    zq_status st = check_format(bits, kGroup, N, K);
    if (st != ZQ_OK) return st;
    if ((st = check_ptr(packed, "packed")) != ZQ_OK) return st;
    if ((st = check_ptr(codes, "codes")) != ZQ_OK) return st;
    cudaError_t e = launch_unpack(packed, N, K, bits, codes, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "unpack launch");
    ++g_launches;
    return ZQ_OK;
}

zq_status zq_dequant(const uint32_t *packed, const uint16_t *scales, const uint16_t *zeros, int bits, int group,
                     int N, int K, uint16_t *w_hat, zq_stream_t stream) {
    zq_status st = check_format(bits, group, N, K);
    if (st != ZQ_OK) return st;
    if ((st = check_ptr(packed, "packed")) != ZQ_OK) return st;
    if ((st = check_ptr(scales, "scales")) != ZQ_OK) return st;
    if ((st = check_ptr(zeros, "zeros")) != ZQ_OK) return st;
    if ((st = check_ptr(w_hat, "w_hat")) != ZQ_OK) return st;
    cudaError_t e = launch_dequant_test(packed, scales, zeros, bits, group, N, K, w_hat,
                                        reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dequant launch");
    ++g_launches;
    return ZQ_OK;
}

zq_status zq_reserve_workspace(size_t bytes, zq_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    std::pair<int, unsigned long long> key;
    zq_status st = stream_key(s, &key);
    if (st != ZQ_OK) return st;
    const size_t need = std::max(bytes, kCounterBytes);
    std::lock_guard<std::mutex> lk(g_ws_mu);
    Workspace &ws = g_ws[key];
    if (ws.bytes >= need) return ZQ_OK;
    // The old buffer may still be in use by work queued on the stream.
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    if (ws.owned && ws.ptr) cudaFree(ws.ptr);
    ws = Workspace{};
    void *p = nullptr;
    e = cudaMalloc(&p, need);
    if (e != cudaSuccess) {
        g_ws.erase(key);
        return cuda_fail(e, "cudaMalloc(workspace)");
    }
    e = cudaMemset(p, 0, kCounterBytes);
    if (e != cudaSuccess) {
        cudaFree(p);
        g_ws.erase(key);
        return cuda_fail(e, "cudaMemset(workspace)");
    }
    ws.ptr = p;
    ws.bytes = need;
    ws.owned = true;
    return ZQ_OK;
}

zq_status zq_attach_workspace(void *buffer, size_t bytes, zq_stream_t stream) {
    if (buffer == nullptr) return fail(ZQ_ERR_INVALID_ARG, "buffer is null");
    if ((reinterpret_cast<uintptr_t>(buffer) & 255u) != 0)
        return fail(ZQ_ERR_INVALID_ARG, "buffer is not 256-byte aligned");
    if (bytes < kCounterBytes)
        return fail(ZQ_ERR_INVALID_ARG, "a workspace needs at least %zu bytes (got %zu)", kCounterBytes, bytes);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    std::pair<int, unsigned long long> key;
    zq_status st = stream_key(s, &key);
    if (st != ZQ_OK) return st;
    std::lock_guard<std::mutex> lk(g_ws_mu);
    Workspace &ws = g_ws[key];
    if (ws.owned && ws.ptr) {
        cudaError_t e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
        cudaFree(ws.ptr);
    }
    ws = Workspace{};
    cudaError_t e = cudaMemsetAsync(buffer, 0, kCounterBytes, s);
    if (e != cudaSuccess) {
        g_ws.erase(key);
        return cuda_fail(e, "clearing the workspace counters");
    }
    ws.ptr = buffer;
    ws.bytes = bytes;
    return ZQ_OK;
}

zq_status zq_release_workspace(zq_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    std::pair<int, unsigned long long> key;
    zq_status st = stream_key(s, &key);
    if (st != ZQ_OK) return st;
    std::lock_guard<std::mutex> lk(g_ws_mu);
    auto it = g_ws.find(key);
    if (it == g_ws.end()) return ZQ_OK;
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    if (it->second.owned && it->second.ptr) {
        e = cudaFree(it->second.ptr);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFree(workspace)");
    }
    g_ws.erase(it);
    return ZQ_OK;
}

zq_status zq_release_all_workspaces(void) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    std::lock_guard<std::mutex> lk(g_ws_mu);
    for (auto it = g_ws.begin(); it != g_ws.end();) {
        if (it->first.first != dev) {
            ++it;
            continue;
        }
        if (it->second.owned && it->second.ptr) cudaFree(it->second.ptr);
        it = g_ws.erase(it);
    }
    return ZQ_OK;
}

size_t zq_linear_workspace_bytes(int bits, int M, int N, int K) {
    if (check_format(bits == 16 ? 4 : bits, kGroup, N, K) != ZQ_OK || M <= 0) return 0;
    // the plan needs only the sizes: any aligned, distinct fake pointers do
    const auto fake = [](uintptr_t i) { return reinterpret_cast<void *>(i << 20); };
    const Op d = make_op(zq_linear_desc{static_cast<const uint16_t *>(fake(1)),
                                        static_cast<const uint32_t *>(fake(2)),
                                        static_cast<const uint16_t *>(fake(3)),
                                        static_cast<const uint16_t *>(fake(4)),
                                        static_cast<uint16_t *>(fake(1 << 20)), bits, kGroup, M, N, K});
    size_t need = 0;
    if (run_stack(&d, 1, nullptr, &need) != ZQ_OK) return 0;
    return need;
}

size_t zq_linear_bf16_workspace_bytes(int bits, int M, int N, int K) {
    if (check_format(bits == 16 ? 4 : bits, kGroup, N, K) != ZQ_OK || M <= 0) return 0;
    const auto fake = [](uintptr_t i) { return reinterpret_cast<void *>(i << 20); };
    Op d = make_op(zq_linear_desc{static_cast<const uint16_t *>(fake(1)), static_cast<const uint32_t *>(fake(2)),
                                  static_cast<const uint16_t *>(fake(3)), static_cast<const uint16_t *>(fake(4)),
                                  static_cast<uint16_t *>(fake(1 << 20)), bits, kGroup, M, N, K});
    d.xbf16 = 1;
    size_t need = 0;
    if (run_stack(&d, 1, nullptr, &need) != ZQ_OK) return 0;
    return need;
}

zq_status zq_set_wait_limit_ns(uint64_t ns) {
    g_wait_ns.store(ns);
    return ZQ_OK;
}

const char *zq_status_string(zq_status status) {
    switch (status) {
        case ZQ_OK: return "ZQ_OK";
        case ZQ_ERR_INVALID_ARG: return "ZQ_ERR_INVALID_ARG";
        case ZQ_ERR_UNSUPPORTED: return "ZQ_ERR_UNSUPPORTED";
        case ZQ_ERR_NONFINITE: return "ZQ_ERR_NONFINITE";
        case ZQ_ERR_CUDA: return "ZQ_ERR_CUDA";
        case ZQ_ERR_TIMEOUT: return "ZQ_ERR_TIMEOUT";
    }
    return "ZQ_UNKNOWN_STATUS";
}

const char *zq_last_error(void) { return g_last_error.c_str(); }

uint64_t zq_kernel_launches(void) { return g_launches.load(); }

zq_status zq_check_device(void) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    int err = 0, err2 = 0, err3 = 0;
    e = read_prefill_error(&err);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
    e = read_decode_error(&err2);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
    e = read_kv_error(&err3);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
    if (err != 0 || err2 != 0) {
        // A kernel that gave up may have left split-K or tile counters set.
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess) workspaces_dirty(dev);
    }
    if (err != 0 || err2 != 0)
        return fail(static_cast<zq_status>(err ? err : err2), "a kernel gave up a bounded wait");
    if (err3 != 0) return fail(static_cast<zq_status>(err3), "a KV-cache row held NaN or Inf");
    return ZQ_OK;
}

// ------------------------------------------------------------------ zKV --

static size_t round256(size_t v) { return (v + 255) / 256 * 256; }

size_t zq_kv_plane_bytes(int window, int capacity, int heads, int dim, int bits) {
    if (window < 1 || capacity < 1 || heads < 1 || dim < 128 || dim % 128 != 0) return 0;
    if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8)) return 0;
    const size_t hr = static_cast<size_t>(capacity) * heads;  // (token, head) rows of the store
    return round256(static_cast<size_t>(window) * heads * dim * 2) + round256(hr * dim * bits / 8) +
           2 * round256(hr * (dim / 128) * 2);
}

static zq_status check_plane(const zq_kv_plane *pl, KvArgs *a) {
    if (pl == nullptr) return fail(ZQ_ERR_INVALID_ARG, "plane is NULL");
    if (!(pl->bits == 2 || pl->bits == 3 || pl->bits == 4 || pl->bits == 8))
        return fail(ZQ_ERR_UNSUPPORTED, "plane bits must be 2, 3, 4 or 8 (got %d)", pl->bits);
    if (pl->window < 1 || pl->capacity < 1 || pl->heads < 1 || pl->dim < 128 || pl->dim % 128 != 0)
        return fail(ZQ_ERR_INVALID_ARG, "plane shape: window=%d capacity=%d heads=%d dim=%d (dim a multiple of 128)",
                    pl->window, pl->capacity, pl->heads, pl->dim);
    zq_status st;
    if ((st = check_ptr(pl->ring, "ring")) != ZQ_OK) return st;
    if ((st = check_ptr(pl->packed, "packed")) != ZQ_OK) return st;
    if ((st = check_ptr(pl->scales, "scales")) != ZQ_OK) return st;
    if ((st = check_ptr(pl->zeros, "zeros")) != ZQ_OK) return st;
    *a = KvArgs{pl->ring, pl->packed, pl->scales, pl->zeros, pl->window, pl->heads, pl->dim, pl->bits};
    return ZQ_OK;
}

zq_status zq_kv_append(const zq_kv_plane *plane, int t0, const uint16_t *rows, int n, zq_stream_t stream) {
    KvArgs a;
    zq_status st = check_plane(plane, &a);
    if (st != ZQ_OK) return st;
    if (t0 < 0 || n < 0 || static_cast<long long>(t0) + n > plane->capacity)
        return fail(ZQ_ERR_INVALID_ARG, "append of %d tokens to %d: capacity is %d", n, t0, plane->capacity);
    if (n == 0) return ZQ_OK;
    if ((st = check_ptr(rows, "rows")) != ZQ_OK) return st;
    cudaError_t e = launch_kv_append(a, rows, t0, n, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kv append launch");
    ++g_launches;
    return ZQ_OK;
}

zq_status zq_kv_gather(const zq_kv_plane *plane, int t_total, int a_tok, int b_tok, uint16_t *out,
                       zq_stream_t stream) {
    KvArgs a;
    zq_status st = check_plane(plane, &a);
    if (st != ZQ_OK) return st;
    if (!(0 <= a_tok && a_tok <= b_tok && b_tok <= t_total && t_total <= plane->capacity))
        return fail(ZQ_ERR_INVALID_ARG, "gather [%d, %d) of %d tokens (capacity %d)", a_tok, b_tok, t_total,
                    plane->capacity);
    if (a_tok == b_tok) return ZQ_OK;
    if ((st = check_ptr(out, "out")) != ZQ_OK) return st;
    cudaError_t e = launch_kv_gather(a, t_total, a_tok, b_tok, out, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kv gather launch");
    ++g_launches;
    return ZQ_OK;
}

int zq_version(void) { return 100; }

}  // extern "C"

void zq::set_last_error(const char *msg) { g_last_error = msg; }

unsigned long long zq::wait_limit_ns() { return g_wait_ns.load(); }
