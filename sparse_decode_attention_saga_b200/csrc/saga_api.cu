// C ABI of libsaga.so (declared in include/saga.h): argument validation,
// workspace carving, TMA descriptor encoding and kernel dispatch.  Every
// check happens before anything is enqueued; nothing here allocates device
// memory or synchronises, except saga_workspace_error which is documented to.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <mutex>

#include "saga.h"
#include "saga_kernels.h"
#include "saga_params.h"

using namespace saga;

namespace {

// Ring shape of the streaming kernels (tuning constants, measured on B200):
// with head_dim 64 and one n-tile of query heads per key head (G <= 8) one
// CTA per SM with a 6 x 32 KB ring of K streams best; with more tensor-core
// and compare work per byte (two n-tiles, or head_dim 128) two CTAs per SM
// with 3 x 32 KB each hide it better.
#ifndef SAGA_STREAM_STAGES_NT1
#define SAGA_STREAM_STAGES_NT1 6
#endif
#ifndef SAGA_STREAM_CTAS_PER_SM_NT1
#define SAGA_STREAM_CTAS_PER_SM_NT1 1
#endif
#ifndef SAGA_STREAM_STAGES_NT2
#define SAGA_STREAM_STAGES_NT2 3
#endif
#ifndef SAGA_STREAM_CTAS_PER_SM_NT2
#define SAGA_STREAM_CTAS_PER_SM_NT2 2
#endif
struct StreamShape {
    int stages, ctas_per_sm;
};
StreamShape stream_shape(const Geometry& g) {
    return g.NT == 1 && g.d == 64 ? StreamShape{SAGA_STREAM_STAGES_NT1, SAGA_STREAM_CTAS_PER_SM_NT1}
                     : StreamShape{SAGA_STREAM_STAGES_NT2, SAGA_STREAM_CTAS_PER_SM_NT2};
}
constexpr long long kMinTilesPerCta = 4;
constexpr int kMaxDevices = 64;
constexpr long long kMaxGatherParts = 32;

std::atomic<uint64_t> g_launches{0};
thread_local cudaEvent_t t_ev_start = nullptr;
thread_local cudaEvent_t t_ev_stop = nullptr;

struct DeviceInfo {
    bool ready = false;
    int sms = 0;
    int major = 0;
    int max_smem = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int device_info(DeviceInfo* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SAGA_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        cudaDeviceProp p;
        if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) return SAGA_ERR_DEVICE;
        d.sms = p.multiProcessorCount;
        d.major = p.major;
        d.max_smem = static_cast<int>(p.sharedMemPerBlockOptin);
        d.ready = true;
    }
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return SAGA_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *out = d;
    return d.major == 10 ? SAGA_OK : SAGA_ERR_DEVICE;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shapes -> Geometry, or a status.
int make_geometry(const saga_dims* d, Geometry* g) {
    if (!d) return SAGA_ERR_INVALID_ARG;
    if (d->batch <= 0 || d->h_q <= 0 || d->h_k <= 0 || d->h_v <= 0 || d->head_dim <= 0 ||
        d->l_kv <= 0 || d->l_cap < d->l_kv)
        return SAGA_ERR_INVALID_ARG;
    if (d->v_head_dim < 0) return SAGA_ERR_INVALID_ARG;
    const int dv = d->v_head_dim ? d->v_head_dim : d->head_dim;
    // key/value head dims: equal and 64 or 128, or 32-dim keys with 64-dim
    // values (two or more key heads, so that a 32 KB tile has <= 256 rows)
    const bool same = (d->head_dim == 64 || d->head_dim == 128) && dv == d->head_dim;
    const bool narrow_keys = d->head_dim == 32 && dv == 64 && d->h_k >= 2;
    if (!same && !narrow_keys) return SAGA_ERR_UNSUPPORTED;
    if (d->h_k != 1 && d->h_k != 2 && d->h_k != 4 && d->h_k != 8) return SAGA_ERR_UNSUPPORTED;
    if (d->h_q % d->h_k != 0 || d->h_q % d->h_v != 0) return SAGA_ERR_UNSUPPORTED;
    if (d->h_q / d->h_k > 16 || d->h_q > 128) return SAGA_ERR_UNSUPPORTED;
    if (static_cast<long long>(d->batch) * d->l_cap >= (1ll << 31)) return SAGA_ERR_UNSUPPORTED;
    if (static_cast<long long>(d->batch) * d->h_q > 65535) return SAGA_ERR_UNSUPPORTED;
    Geometry& x = *g;
    x.b = d->batch;
    x.hq = d->h_q;
    x.hk = d->h_k;
    x.hv = d->h_v;
    x.d = d->head_dim;
    x.dv = dv;
    x.l = d->l_kv;
    x.l_cap = d->l_cap;
    x.G = x.hq / x.hk;
    x.NT = (x.G + 7) / 8;
    x.P = kStageBytes / (x.hk * x.d * 2);
    x.KB = x.d < 64 ? x.d : 64;
    x.WPK = kConsumerWarps / x.hk;
    x.MBW = 128 / x.d;
    x.tiles = (x.l + x.P - 1) / x.P;
    x.l_pad = x.tiles * x.P;
    // A batch row of `tiles` tiles meets at most 2*C/b + 2 CTA ranges when
    // C <= b*tiles (every range holds at least floor(T/C) >= T/(2C) tiles).
    const int per_batch = 2 * ((kMaxCtas + x.b - 1) / x.b) + 2;
    x.S_cap = per_batch < x.tiles ? per_batch : x.tiles;
    x.rec = x.dv + kRecHeader;
    x.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(x.d)));
    return SAGA_OK;
}

// The dense kernel's geometry: the cache's own, or, with more than two value
// heads per key head (or a stage of two that does not fit twice in shared
// memory), one key head per value head, of which each group of *k_group
// reads the same cache key head.
int dense_geometry(const saga_dims* d, Geometry* g, int* k_group) {
    int st = make_geometry(d, g);
    *k_group = 1;
    if (st) return st;
    if (g->hv <= 2 * g->hk && dense_smem_bytes(*g, 2) <= static_cast<size_t>(kMaxDynamicSmem)) return st;
    if (g->hv <= g->hk || g->hv % g->hk) return SAGA_ERR_UNSUPPORTED;
    saga_dims dd = *d;
    dd.h_k = d->h_v;
    if ((st = make_geometry(&dd, g))) return st;
    *k_group = d->h_v / d->h_k;
    return SAGA_OK;
}

int check_ws(const Geometry& g, const void* ws, size_t ws_bytes) {
    if (!ws || !aligned(ws, 256)) return SAGA_ERR_INVALID_ARG;
    if (ws_bytes < workspace_layout(g).total) return SAGA_ERR_WORKSPACE;
    return SAGA_OK;
}

template <typename T>
T* ws_at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// Tensor map of a cache [b * l_cap, heads, dim] bf16: boxes of min(dim, 64)
// elements x 1 head x P positions, each box row swizzled across its width
// (128-byte rows for 64-element boxes, 64-byte rows for 32-dim keys).
int encode_cache_map(CUtensorMap* map, const void* base, const Geometry& g, int heads, int dim) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(dim), static_cast<cuuint64_t>(heads),
                          static_cast<cuuint64_t>(g.b) * g.l_cap};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(dim) * 2,
                             static_cast<cuuint64_t>(heads) * dim * 2};
    const cuuint32_t inner = dim < 64 ? static_cast<cuuint32_t>(dim) : 64u;
    cuuint32_t box[3] = {inner, 1, static_cast<cuuint32_t>(g.P)};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                inner == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? SAGA_OK : SAGA_ERR_CUDA;
}

int max_slots(const Geometry& g, long long T, int C) {
    int m = 0;
    for (int bb = 0; bb < g.b; ++bb) {
        const int s = slots_of_batch(bb, g.tiles, T, C);
        m = s > m ? s : m;
    }
    return m;
}

// Grid of the streaming kernels: `per_sm` CTAs per SM, at most one per tile, and
// never more partial-record slots per batch row than the workspace holds.
int stream_ctas(const Geometry& g, const DeviceInfo& dev, int per_sm) {
    const long long T = static_cast<long long>(g.b) * g.tiles;
    long long c = static_cast<long long>(dev.sms) * per_sm;
    if (c > kMaxCtas) c = kMaxCtas;
    // at least kMinTilesPerCta tiles each: a CTA's pipeline start costs a few
    // microseconds, and every CTA adds a partial-record slot to each row
    const long long by_work = (T + kMinTilesPerCta - 1) / kMinTilesPerCta;
    if (c > by_work) c = by_work;
    if (c > T) c = T;
    int C = static_cast<int>(c < 1 ? 1 : c);
    while (C > 1 && max_slots(g, T, C) > g.S_cap) --C;
    return C;
}

// From this many CTAs per row (few rows) the gather grid is part-major: most
// rows then need only some of their parts, and the needed ones go first
// (measured: Llama-shaped batch 1 at 8K, 23.5 -> 21.5 us per reuse step;
// row-major stays faster at batch 16, 233 -> 229 us).
constexpr int kPartMajorParts = 16;
// A decode step given stored logits streams K instead when it has at most
// this many rows of at least this many positions.
constexpr long long kFusedFewRows = 64;
// Static shared memory of the candidate compaction kernel (its last-digit
// histogram, the stash of its threshold bucket's candidates and block-scan
// scratch), beside the row bitmap.
constexpr size_t kCandStaticSmem = 16 * 1024;
constexpr int kFusedMinPositions = 65536;
// Up to this many rows per SM the compare/compact kernel reads 16 logits per
// thread per sub-round (more bytes in flight per CTA; two CTAs per SM by its
// registers), beyond it 4 (measured on refresh steps: Qwen-shaped batch 16
// at 128K 265 -> 238 us, Sigma-style 271 -> 238 us, Qwen-shaped batch 1 at
// 32K 42.1 -> 39.0 us; the Llama-shaped batch 16, 512 rows, 491 -> 501 us
// in two waves, so it keeps 4).
constexpr long long kSelectWideRowsPerSm = 2;

// CTAs per row of the gather kernel: about 8 per SM over all rows, never more
// than the partial-record slots of a row.
int gather_parts(const Geometry& g, const DeviceInfo& dev) {
    const long long rows = static_cast<long long>(g.b) * g.hq;
    long long parts = (8ll * dev.sms + rows - 1) / rows;
    const long long cap = static_cast<long long>(g.S_cap) * g.WPK;
    if (parts > cap) parts = cap;
    // few rows: each part still wants >= 128 kept entries, so more parts than
    // this only add CTAs that build the list table and exit
    if (parts > kMaxGatherParts) parts = kMaxGatherParts;
    return static_cast<int>(parts < 1 ? 1 : parts);
}

}  // namespace

namespace saga {
// CTAs per row of the radix passes.  Cost model: waves of 8 CTAs per SM, each
// wave as long as one CTA's share of the row plus a fixed per-CTA cost (its
// 2048-bin histogram is cleared and flushed) worth about 3000 logits.
int radix_chunks(long long rows, int l, int sms) {
    const long long slots = 8ll * sms;
    const long long max_chunks = (l + 4095) / 4096;
    long long best = 1;
    double best_cost = 1e300;
    for (long long c = 1; c <= max_chunks && c <= kRadixMaxChunks; ++c) {
        const long long waves = (rows * c + slots - 1) / slots;
        const double cost = static_cast<double>(waves) * (static_cast<double>((l + c - 1) / c) + 3000.0);
        if (cost < best_cost) {
            best_cost = cost;
            best = c;
        }
    }
    return static_cast<int>(best);
}
}  // namespace saga

namespace {

int cuda_status(cudaError_t e) { return e == cudaSuccess ? SAGA_OK : SAGA_ERR_CUDA; }

void ev_start(cudaStream_t s) {
    if (t_ev_start) cudaEventRecord(t_ev_start, s);
}
void ev_stop(cudaStream_t s) {
    if (t_ev_stop) cudaEventRecord(t_ev_stop, s);
}

// Logits of every row into `dst` [b*hq][l] (the refresh path).
int run_logits(const Geometry& g, const DeviceInfo& dev, const void* q, const void* k, float* dst,
               uint32_t* err, cudaStream_t s) {
    CUtensorMap kmap;
    int st = encode_cache_map(&kmap, k, g, g.hk, g.d);
    if (st) return st;
    StreamArgs a{};
    a.g = g;
    a.C = stream_ctas(g, dev, stream_shape(g).ctas_per_sm);
    a.stages = stream_shape(g).stages;
    a.q = q;
    a.logits = dst;
    a.err = err;
    ev_start(s);
    const cudaError_t e = launch_qk_stream(kStreamLogits, kmap, a, s);
    ev_stop(s);
    g_launches += 1;
    return cuda_status(e);
}

}  // namespace

namespace saga {
void note_launches(int n) { g_launches += static_cast<uint64_t>(n); }

namespace {
// The largest dynamic shared-memory limit set so far for each kernel, per device.
struct SmemAttr {
    const void* fn;
    int bytes[kMaxDevices];
};
constexpr int kMaxSmemAttrs = 128;
constexpr int kDefaultDynamicSmem = 48 * 1024;  // needs no attribute
SmemAttr g_smem_attr[kMaxSmemAttrs];
int g_n_smem_attr = 0;
std::mutex g_smem_attr_mu;
}  // namespace

cudaError_t allow_dynamic_smem(const void* fn, int bytes) {
    if (bytes <= kDefaultDynamicSmem) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_smem_attr_mu);
    SmemAttr* rec = nullptr;
    for (int i = 0; i < g_n_smem_attr; ++i)
        if (g_smem_attr[i].fn == fn) rec = &g_smem_attr[i];
    if (rec && rec->bytes[dev] >= bytes) return cudaSuccess;  // never lowered
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    if (!rec && g_n_smem_attr < kMaxSmemAttrs) {
        rec = &g_smem_attr[g_n_smem_attr++];
        rec->fn = fn;
        for (int d = 0; d < kMaxDevices; ++d) rec->bytes[d] = 0;
    }
    if (rec) rec->bytes[dev] = bytes;  // (a full table only means setting it again next time)
    return cudaSuccess;
}
}  // namespace saga

// The workspace header's counter of empty-set rows (the word after the
// sticky error flag).
static uint32_t* ws_empty_rows(void* ws, const WsLayout& L) { return ws_at<uint32_t>(ws, L.err) + 1; }

// Exact thresholds over stored logits, or over logits computed here into
// logits_out (the workspace's logits region when null).  The radix pass 1
// leaves its candidates (every logit at or above the lower edge of the
// threshold's first-digit bucket) in the workspace for the compaction of a
// refresh step (thresholds of -inf and no candidates when N >= l).  With
// two_digits the passes stop there: the compaction over the candidates
// finds the last digit and writes the thresholds.
static int refresh_impl(const Geometry& g, const DeviceInfo& dev, int32_t N, const void* q,
                        const void* k, const float* logits_in, float* logits_out, float* thresh_out,
                        void* ws, cudaStream_t s, bool two_digits = false) {
    const WsLayout L = workspace_layout(g);
    uint32_t* err = ws_at<uint32_t>(ws, L.err);
    const long long rows = static_cast<long long>(g.b) * g.hq;
    int st;
    const float* logits = logits_in;
    if (!logits) {
        float* dst = logits_out ? logits_out : ws_at<float>(ws, L.logits);
        if ((st = run_logits(g, dev, q, k, dst, err, s))) return st;
        logits = dst;
    }
    if (N >= g.l) {
        g_launches += 1;
        return cuda_status(launch_fill(thresh_out, rows, -std::numeric_limits<float>::infinity(), s));
    }
    // tickets (a safety net: they are kept at zero between launches),
    // histograms and radix state
    cudaError_t e = cudaMemsetAsync(ws_at<uint8_t>(ws, L.tickets), 0, L.cnt - L.tickets, s);
    if (e != cudaSuccess) return SAGA_ERR_CUDA;
    RadixArgs r{};
    r.passes = two_digits ? kRadixPasses - 1 : kRadixPasses;
    r.logits = logits;
    r.rows = rows;
    r.l = g.l;
    r.N = N;
    r.chunks = radix_chunks(rows, g.l, dev.sms);
    r.hist = ws_at<uint32_t>(ws, L.hist);
    r.state = ws_at<uint32_t>(ws, L.state);
    r.tickets = ws_at<uint32_t>(ws, L.tickets);
    r.thresh = thresh_out;
    r.err = err;
    // pass 1 copies every logit at or above its bucket's lower edge out, so
    // that pass 2 and the compaction of the refresh step read only those
    r.cand = ws_at<int2>(ws, L.cand);
    r.cand_cnt = ws_at<int32_t>(ws, L.cand_cnt);
    g_launches += r.passes;
    return cuda_status(launch_radix_select(r, s));
}

// Softmax and gathered value rows over contiguous kept lists (idx, s, cnt,
// rowmax per row), the last CTA of each row merging its parts into out (or
// into part's records).
static int gather_contiguous(const Geometry& g, const DeviceInfo& dev, const void* q, const void* k,
                             const void* v, const int32_t* idx, const float* sv, const int32_t* cnt,
                             const float* rowmax, float* out, float* part, int32_t* sel_cnt, void* ws,
                             const WsLayout& L, cudaStream_t s) {
    float* records = ws_at<float>(ws, L.records);
    GatherArgs ga{};
    ga.g = g;
    ga.mode = kListContiguous;
    ga.parts = gather_parts(g, dev);
    ga.part_major = ga.parts >= kPartMajorParts;
    ga.max_lists = 1;
    ga.v = v;
    ga.idx = idx;
    ga.list_s = sv;
    ga.cnt = cnt;
    ga.rowmax = rowmax;
    ga.records = records;
    ga.tickets = ws_at<uint32_t>(ws, L.tickets);
    ga.err = ws_at<uint32_t>(ws, L.err);
    ga.cmb.g = g;
    ga.cmb.mode = kCombineParts;
    ga.cmb.parts = ga.parts;
    ga.cmb.records = records;
    ga.cmb.out = out;
    ga.cmb.part = part;
    ga.cmb.sel_cnt = sel_cnt;
    ga.cmb.empty_rows = part ? nullptr : ws_empty_rows(ws, L);
    if (part) {  // a shard that kept nothing reports its maxima (recomputed from q and k)
        ga.cmb.fallback = 1;
        ga.cmb.q = q;
        ga.cmb.k = k;
        ga.cmb.v = v;
    }
    g_launches += 1;
    return cuda_status(launch_gather_pv(ga, s));
}

extern "C" {

size_t saga_workspace_bytes(const saga_dims* dims, int32_t N) {
    Geometry g, gd;
    int k_group = 1;
    if (N <= 0 || make_geometry(dims, &g) != SAGA_OK) return 0;
    const size_t total = workspace_layout(g).total;
    // the dense kernel's geometry may hold its partial records differently
    if (dense_geometry(dims, &gd, &k_group) != SAGA_OK) return total;
    const size_t dense_total = workspace_layout(gd).total;
    return dense_total > total ? dense_total : total;
}

int saga_topn_refresh(const saga_dims* dims, int32_t N, const void* q, const void* k,
                      const float* logits_in, float* logits_out, float* thresh_out, void* ws,
                      size_t ws_bytes, saga_stream_t stream) {
    Geometry g;
    int st = make_geometry(dims, &g);
    if (st) return st;
    if (N <= 0 || !thresh_out || !aligned(thresh_out, 4)) return SAGA_ERR_INVALID_ARG;
    if (logits_in) {
        if (!aligned(logits_in, 4)) return SAGA_ERR_INVALID_ARG;
    } else {
        if (!q || !k || !aligned(q, 16) || !aligned(k, 16)) return SAGA_ERR_INVALID_ARG;
        if (logits_out && !aligned(logits_out, 4)) return SAGA_ERR_INVALID_ARG;
    }
    if ((st = check_ws(g, ws, ws_bytes))) return st;
    DeviceInfo dev;
    if ((st = device_info(&dev))) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return refresh_impl(g, dev, N, q, k, logits_in, logits_out, thresh_out, ws, s);
}

// Many records per row (few rows, many slots): several CTAs per row merge
// shares of about 64 records into partial records stored past the inputs.
static void set_combine_chunks(const Geometry& g, CombineArgs* ca, void* ws, const WsLayout& L) {
    const int r_max = max_slots(g, static_cast<long long>(g.b) * g.tiles, ca->C) * ca->recs_per_slot;
    const int chunks = r_max > 128 ? std::min(32, (r_max + 63) / 64) : 1;
    if (chunks > 1 && r_max + chunks <= g.S_cap * g.WPK) {
        ca->chunks = chunks;
        ca->partial_slot = r_max;
        ca->tickets = ws_at<uint32_t>(ws, L.tickets);
    }
}

// One decode step; the merged rows go to out (normalised), or with part to
// part as unnormalised per-row records (a sequence shard's contribution).
static int atopn_decode_impl(const saga_dims* dims, const void* q, const void* k, const void* v,
                             const float* thresh, const float* logits_in, float* out, float* part,
                             int32_t* sel_idx, int32_t* sel_cnt, void* ws, size_t ws_bytes,
                             saga_stream_t stream) {
    Geometry g;
    int st = make_geometry(dims, &g);
    if (st) return st;
    if (!v || !aligned(v, 16) || !thresh || !aligned(thresh, 4) ||
        (out ? !aligned(out, 4) : (!part || !aligned(part, 4))))
        return SAGA_ERR_INVALID_ARG;
    if (logits_in ? !aligned(logits_in, 4) : (!q || !k || !aligned(q, 16) || !aligned(k, 16)))
        return SAGA_ERR_INVALID_ARG;
    if ((sel_idx && !aligned(sel_idx, 4)) || (sel_cnt && !aligned(sel_cnt, 4)))
        return SAGA_ERR_INVALID_ARG;
    if ((st = check_ws(g, ws, ws_bytes))) return st;
    DeviceInfo dev;
    if ((st = device_info(&dev))) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const WsLayout L = workspace_layout(g);
    uint32_t* err = ws_at<uint32_t>(ws, L.err);
    const long long rows = static_cast<long long>(g.b) * g.hq;
    float* records = ws_at<float>(ws, L.records);
    // Few long rows: the compare kernel's one CTA per row leaves most SMs
    // idle (Llama-shaped batch 1 at 128K: refresh step 110 us over stored
    // logits, 89 us when the decode streams K again through the fused path,
    // which yields the same logits bit for bit; at 8K to 32K the stored
    // logits stay faster).
    if (logits_in && !sel_idx && rows <= kFusedFewRows && g.l >= kFusedMinPositions && q && k &&
        aligned(q, 16) && aligned(k, 16))
        logits_in = nullptr;

    if (logits_in) {
        // stored logits -> compare/compact -> gathered PV -> combine
        const float* logits = logits_in;
        SelectArgs sa{};
        sa.logits = logits;
        sa.thresh = thresh;
        sa.rows = rows;
        sa.l = g.l;
        sa.idx = sel_idx ? sel_idx : ws_at<int32_t>(ws, L.list_idx);
        sa.s = ws_at<float>(ws, L.list_s);
        sa.cnt = ws_at<int32_t>(ws, L.cnt);
        sa.rowmax = ws_at<float>(ws, L.rowmax);
        // a shard keeps nothing when nothing passes: the whole row's maxima
        // are found when the shards' records are merged
        sa.keep_max = part ? 0 : 1;
        sa.empty_rows = part ? nullptr : ws_empty_rows(ws, L);
        sa.err = err;
        // up to two CTAs per SM of the wide form (its registers) in one wave
        sa.wide = rows <= kSelectWideRowsPerSm * dev.sms;
        cudaError_t e = launch_select_compact(sa, s);
        g_launches += 1;
        if (e != cudaSuccess) return SAGA_ERR_CUDA;

        return gather_contiguous(g, dev, q, k, v, sa.idx, sa.s, sa.cnt, sa.rowmax, out, part, sel_cnt,
                                 ws, L, s);
    }

    // fused: stream K, compare on chip, lists -> gathered PV with the row merge
    const int C = stream_ctas(g, dev, stream_shape(g).ctas_per_sm);
    const int slots = max_slots(g, static_cast<long long>(g.b) * g.tiles, C);
    if (gather_smem_bytes(slots * g.WPK) > static_cast<size_t>(kGatherMaxSmem))
        return SAGA_ERR_UNSUPPORTED;  // checked before anything is enqueued
    CUtensorMap kmap;
    if ((st = encode_cache_map(&kmap, k, g, g.hk, g.d))) return st;
    StreamArgs a{};
    a.g = g;
    a.C = C;
    a.stages = stream_shape(g).stages;
    a.q = q;
    a.thresh = thresh;
    a.list = ws_at<int2>(ws, L.list_idx);  // spans the list_idx and list_s regions
    a.seg_cnt = ws_at<int32_t>(ws, L.seg_cnt);
    a.seg_mall = ws_at<float>(ws, L.seg_mall);
    a.err = err;
    ev_start(s);
    cudaError_t e = launch_qk_stream(kStreamSelect, kmap, a, s);
    ev_stop(s);
    g_launches += 1;
    if (e != cudaSuccess) return SAGA_ERR_CUDA;

    GatherArgs ga{};
    ga.g = g;
    ga.mode = kListSegments;
    ga.C = a.C;
    ga.parts = gather_parts(g, dev);
    ga.part_major = ga.parts >= kPartMajorParts;
    ga.max_lists = slots * g.WPK;
    ga.v = v;
    ga.seg_list = a.list;
    ga.seg_cnt = a.seg_cnt;
    ga.seg_mall = a.seg_mall;
    ga.records = records;
    ga.tickets = ws_at<uint32_t>(ws, L.tickets);
    ga.err = err;
    ga.cmb.g = g;
    ga.cmb.mode = kCombineParts;
    ga.cmb.parts = ga.parts;
    ga.cmb.fallback = 1;
    ga.cmb.q = q;
    ga.cmb.k = k;
    ga.cmb.v = v;
    ga.cmb.records = records;
    ga.cmb.out = out;
    ga.cmb.part = part;
    ga.cmb.sel_cnt = sel_cnt;
    ga.cmb.sel_idx = sel_idx;
    ga.cmb.empty_rows = part ? nullptr : ws_empty_rows(ws, L);
    ga.cmb.C = a.C;              // the fallback recomputes only the lists
    ga.cmb.seg_mall = a.seg_mall;  // that hold the row maximum
    g_launches += 1;
    if ((e = launch_gather_pv(ga, s)) != cudaSuccess || !sel_idx) return cuda_status(e);

    // the kept positions of the on-chip compare, ascending (the logits region
    // of the workspace, unused on this path, holds the per-row bitmaps)
    IndexArgs ia{};
    ia.g = g;
    ia.C = a.C;
    ia.seg_list = a.list;
    ia.seg_cnt = a.seg_cnt;
    ia.bitmap = ws_at<uint32_t>(ws, L.logits);
    ia.idx = sel_idx;
    ia.err = err;
    g_launches += 1;
    return cuda_status(launch_lists_to_index(ia, s));
}

int saga_atopn_decode(const saga_dims* dims, const void* q, const void* k, const void* v,
                      const float* thresh, const float* logits_in, float* out, int32_t* sel_idx,
                      int32_t* sel_cnt, void* ws, size_t ws_bytes, saga_stream_t stream) {
    if (!out) return SAGA_ERR_INVALID_ARG;
    return atopn_decode_impl(dims, q, k, v, thresh, logits_in, out, nullptr, sel_idx, sel_cnt, ws,
                             ws_bytes, stream);
}

int saga_atopn_refresh_step(const saga_dims* dims, int32_t N, const void* q, const void* k,
                            const void* v, float* thresh_out, float* out, int32_t* sel_idx,
                            int32_t* sel_cnt, void* ws, size_t ws_bytes, saga_stream_t stream) {
    Geometry g;
    int st = make_geometry(dims, &g);
    if (st) return st;
    if (N <= 0 || !q || !k || !v || !thresh_out || !out || !aligned(q, 16) || !aligned(k, 16) ||
        !aligned(v, 16) || !aligned(thresh_out, 4) || !aligned(out, 4))
        return SAGA_ERR_INVALID_ARG;
    if ((sel_idx && !aligned(sel_idx, 4)) || (sel_cnt && !aligned(sel_cnt, 4))) return SAGA_ERR_INVALID_ARG;
    if ((st = check_ws(g, ws, ws_bytes))) return st;
    DeviceInfo dev;
    if ((st = device_info(&dev))) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const WsLayout L = workspace_layout(g);
    const long long rows = static_cast<long long>(g.b) * g.hq;
    // few long rows: one compaction CTA per row leaves most SMs idle, and
    // streaming K again through the fused kernel (the same logits bit for
    // bit) is faster
    const bool few_long_rows = rows <= kFusedFewRows && g.l >= kFusedMinPositions;
    // every entry kept, or a row whose bitmap does not fit on chip: the
    // compaction reads the stored logits
    const bool from_candidates = N < g.l && !few_long_rows &&
                                 cand_select_smem(g.l) + kCandStaticSmem <= static_cast<size_t>(dev.max_smem);
    if ((st = refresh_impl(g, dev, N, q, k, nullptr, nullptr, thresh_out, ws, s, from_candidates)))
        return st;
    if (!from_candidates) {
        const float* logits_in = few_long_rows && N < g.l ? nullptr : ws_at<float>(ws, L.logits);
        return atopn_decode_impl(dims, q, k, v, thresh_out, logits_in, out, nullptr, sel_idx, sel_cnt, ws,
                                 ws_bytes, stream);
    }
    CandSelectArgs ca{};
    ca.cand = ws_at<int2>(ws, L.cand);
    ca.cand_cnt = ws_at<int32_t>(ws, L.cand_cnt);
    ca.chunks = radix_chunks(rows, g.l, dev.sms);  // as the radix passes cut the rows
    ca.state = ws_at<uint32_t>(ws, L.state);       // the last digit is found here
    ca.thresh = thresh_out;
    ca.rows = rows;
    ca.l = g.l;
    ca.idx = sel_idx ? sel_idx : ws_at<int32_t>(ws, L.list_idx);
    ca.s = ws_at<float>(ws, L.list_s);
    ca.cnt = ws_at<int32_t>(ws, L.cnt);
    ca.rowmax = ws_at<float>(ws, L.rowmax);
    ca.empty_rows = ws_empty_rows(ws, L);
    ca.err = ws_at<uint32_t>(ws, L.err);
    g_launches += 1;
    if (launch_cand_select(ca, s) != cudaSuccess) return SAGA_ERR_CUDA;
    return gather_contiguous(g, dev, q, k, v, ca.idx, ca.s, ca.cnt, ca.rowmax, out, nullptr, sel_cnt, ws,
                             L, s);
}

int saga_atopn_decode_partial(const saga_dims* dims, const void* q, const void* k, const void* v,
                              const float* thresh, const float* logits_in, float* part, void* ws,
                              size_t ws_bytes, saga_stream_t stream) {
    // q and k are needed even with stored logits: a shard that keeps nothing
    // recomputes its row maxima from them
    if (!part || !q || !k || !aligned(q, 16) || !aligned(k, 16)) return SAGA_ERR_INVALID_ARG;
    return atopn_decode_impl(dims, q, k, v, thresh, logits_in, nullptr, part, nullptr, nullptr, ws,
                             ws_bytes, stream);
}

int saga_merge_partials(const saga_dims* dims, const float* parts, int32_t R, float* out,
                        int32_t* sel_cnt, saga_stream_t stream) {
    Geometry g;
    int st = make_geometry(dims, &g);
    if (st) return st;
    if (R <= 0 || !parts || !aligned(parts, 4) || !out || !aligned(out, 4) ||
        (sel_cnt && !aligned(sel_cnt, 4)))
        return SAGA_ERR_INVALID_ARG;
    DeviceInfo dev;
    if ((st = device_info(&dev))) return st;
    MergeArgs a{};
    a.parts = parts;
    a.R = R;
    a.rows = static_cast<long long>(g.b) * g.hq;
    a.out = out;
    a.sel_cnt = sel_cnt;
    g_launches += 1;
    return cuda_status(launch_merge_parts(g.dv, a, reinterpret_cast<cudaStream_t>(stream)));
}

int saga_qk_logits(const saga_dims* dims, const void* q, const void* k, float* logits_out, void* ws,
                   size_t ws_bytes, saga_stream_t stream) {
    Geometry g;
    int st = make_geometry(dims, &g);
    if (st) return st;
    if (!q || !k || !logits_out || !aligned(q, 16) || !aligned(k, 16) || !aligned(logits_out, 4))
        return SAGA_ERR_INVALID_ARG;
    if ((st = check_ws(g, ws, ws_bytes))) return st;
    DeviceInfo dev;
    if ((st = device_info(&dev))) return st;
    const WsLayout L = workspace_layout(g);
    return run_logits(g, dev, q, k, logits_out, ws_at<uint32_t>(ws, L.err),
                      reinterpret_cast<cudaStream_t>(stream));
}

int saga_topn_histogram(const saga_dims* dims, int32_t pass, const float* logits,
                        const uint32_t* state, uint32_t* hist, saga_stream_t stream) {
    Geometry g;
    int st = make_geometry(dims, &g);
    if (st) return st;
    if (pass < 0 || pass >= kRadixPasses || !logits || !aligned(logits, 4) || !hist ||
        !aligned(hist, 4) || (pass > 0 && (!state || !aligned(state, 4))))
        return SAGA_ERR_INVALID_ARG;
    DeviceInfo dev;
    if ((st = device_info(&dev))) return st;
    ShardHistArgs a{};
    a.logits = logits;
    a.rows = static_cast<long long>(g.b) * g.hq;
    a.l = g.l;
    a.chunks = radix_chunks(a.rows, g.l, dev.sms);
    a.state = state;
    a.hist = hist;
    g_launches += 1;
    return cuda_status(launch_shard_hist(pass, a, reinterpret_cast<cudaStream_t>(stream)));
}

int saga_topn_select_digit(const saga_dims* dims, int32_t N, int32_t pass, const uint32_t* hist,
                           uint32_t* state, float* thresh_out, saga_stream_t stream) {
    Geometry g;
    int st = make_geometry(dims, &g);
    if (st) return st;
    if (N <= 0 || pass < 0 || pass >= kRadixPasses || !hist || !aligned(hist, 4) || !state ||
        !aligned(state, 4) || !thresh_out || !aligned(thresh_out, 4))
        return SAGA_ERR_INVALID_ARG;
    DeviceInfo dev;
    if ((st = device_info(&dev))) return st;
    ShardDigitArgs a{};
    a.hist = hist;
    a.rows = static_cast<long long>(g.b) * g.hq;
    a.N = N;
    a.state = state;
    a.thresh = thresh_out;
    g_launches += 1;
    return cuda_status(launch_shard_digit(pass, a, reinterpret_cast<cudaStream_t>(stream)));
}

int saga_decode_dense(const saga_dims* dims, const void* q, const void* k, const void* v,
                      float* out, void* ws, size_t ws_bytes, saga_stream_t stream) {
    Geometry g;
    int k_group = 1;
    int st = dense_geometry(dims, &g, &k_group);
    if (st) return st;
    if (!dense_supported(g)) return SAGA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !out || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) ||
        !aligned(out, 4))
        return SAGA_ERR_INVALID_ARG;
    if ((st = check_ws(g, ws, ws_bytes))) return st;
    DeviceInfo dev;
    if ((st = device_info(&dev))) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const WsLayout L = workspace_layout(g);

    int stages = 4;
    while (stages > 2 && dense_smem_bytes(g, stages) > static_cast<size_t>(dev.max_smem)) --stages;
    if (dense_smem_bytes(g, stages) > static_cast<size_t>(dev.max_smem)) return SAGA_ERR_UNSUPPORTED;

    CUtensorMap kmap, vmap;
    if ((st = encode_cache_map(&kmap, k, g, g.hk / k_group, g.d))) return st;
    if ((st = encode_cache_map(&vmap, v, g, g.hv, g.dv))) return st;
    DenseArgs a{};
    a.g = g;
    a.k_group = k_group;
    a.C = stream_ctas(g, dev, 1);
    a.stages = stages;
    a.q = q;
    a.records = ws_at<float>(ws, L.records);
    a.err = ws_at<uint32_t>(ws, L.err);
    ev_start(s);
    cudaError_t e = launch_dense(kmap, vmap, a, s);
    ev_stop(s);
    g_launches += 1;
    if (e != cudaSuccess) return SAGA_ERR_CUDA;

    CombineArgs ca{};
    ca.g = g;
    ca.mode = kCombineSlots;
    ca.C = a.C;
    ca.recs_per_slot = g.WPK;
    ca.records = a.records;
    ca.out = out;
    set_combine_chunks(g, &ca, ws, L);
    g_launches += 1;
    return cuda_status(launch_combine(ca, s));
}

int saga_cache_append(const saga_dims* dims, const void* k_new, const void* v_new, void* k,
                      void* v, saga_stream_t stream) {
    Geometry g;
    int st = make_geometry(dims, &g);
    if (st) return st;
    if (g.l >= g.l_cap) return SAGA_ERR_INVALID_ARG;  // no room for the new row
    if (!k_new || !v_new || !k || !v || !aligned(k_new, 16) || !aligned(v_new, 16) ||
        !aligned(k, 16) || !aligned(v, 16))
        return SAGA_ERR_INVALID_ARG;
    DeviceInfo dev;
    if ((st = device_info(&dev))) return st;
    AppendArgs a{};
    a.b = g.b;
    a.hk = g.hk;
    a.hv = g.hv;
    a.d = g.d;
    a.dv = g.dv;
    a.l_cap = g.l_cap;
    a.pos = g.l;
    a.k_new = k_new;
    a.v_new = v_new;
    a.k = k;
    a.v = v;
    g_launches += 1;
    return cuda_status(launch_cache_append(a, reinterpret_cast<cudaStream_t>(stream)));
}

int saga_workspace_reset(void* ws, size_t ws_bytes, saga_stream_t stream) {
    if (!ws) return SAGA_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, reinterpret_cast<cudaStream_t>(stream)));
}

int saga_workspace_error(void* ws, size_t ws_bytes, saga_stream_t stream) {
    if (!ws || ws_bytes < 256) return SAGA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SAGA_ERR_CUDA;
    if (cudaMemcpy(&word, ws, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess)
        return SAGA_ERR_CUDA;
    if (word && cudaMemset(ws, 0, sizeof word) != cudaSuccess) return SAGA_ERR_CUDA;
    if (word & kErrTimeout) return SAGA_ERR_TIMEOUT;
    return (word & kErrBounds) ? SAGA_ERR_BOUNDS : SAGA_OK;
}

int saga_workspace_empty_rows(void* ws, size_t ws_bytes, uint64_t* count_out, saga_stream_t stream) {
    if (!ws || ws_bytes < 256 || !count_out) return SAGA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    uint32_t* counter = reinterpret_cast<uint32_t*>(ws) + 1;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SAGA_ERR_CUDA;
    if (cudaMemcpy(&word, counter, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess)
        return SAGA_ERR_CUDA;
    if (word && cudaMemset(counter, 0, sizeof word) != cudaSuccess) return SAGA_ERR_CUDA;
    *count_out = word;
    return SAGA_OK;
}

const char* saga_status_string(int status) {
    switch (status) {
        case SAGA_OK: return "ok";
        case SAGA_ERR_INVALID_ARG: return "invalid argument";
        case SAGA_ERR_UNSUPPORTED: return "unsupported shape";
        case SAGA_ERR_WORKSPACE: return "workspace too small";
        case SAGA_ERR_CUDA: return "CUDA error";
        case SAGA_ERR_DEVICE: return "no sm_100 device";
        case SAGA_ERR_TIMEOUT: return "a bounded device wait timed out";
        case SAGA_ERR_BOUNDS: return "an index out of range (debug build check)";
        default: return "unknown status";
    }
}

uint64_t saga_launch_count(void) { return g_launches.load(); }

void saga_set_kernel_events(void* start_event, void* stop_event) {
    t_ev_start = static_cast<cudaEvent_t>(start_event);
    t_ev_stop = static_cast<cudaEvent_t>(stop_event);
}

int saga_version(void) { return 100; }

}  // extern "C"
