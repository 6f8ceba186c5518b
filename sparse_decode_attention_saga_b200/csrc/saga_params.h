// Shapes, tiling constants, the CTA/tile partition and the workspace layout,
// shared by the host dispatcher and the kernels.
#pragma once

#include <stddef.h>
#include <stdint.h>

#ifdef __CUDACC__
#define SAGA_HD __host__ __device__ __forceinline__
#else
#define SAGA_HD inline
#endif

namespace saga {

// Streaming kernels: 8 consumer warps (the mma/compare work) + 1 producer
// warp that issues the TMA loads.
constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kStreamThreads = kConsumerThreads + 32;
// Bytes of K per pipeline stage: P positions x h_k heads x d x 2 B.
constexpr int kStageBytes = 32768;
// Upper bound on the grid of every streaming kernel (sizes the workspace).
constexpr int kMaxCtas = 512;
// Dynamic shared memory a streaming CTA may use (sm_100 opt-in limit: 227 KB).
constexpr int kMaxDynamicSmem = 227 * 1024;
// Dynamic shared memory of the gather kernel's list table.
constexpr int kGatherMaxSmem = 96 * 1024;
// Bounded device waits give up after this long and raise kErrTimeout.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;
constexpr uint32_t kErrTimeout = 1u;
// Debug builds (SAGA_DEBUG): an index read from another kernel's output was
// out of range (the access was skipped).
constexpr uint32_t kErrBounds = 2u;
// Radix select: 32-bit keys in digits of 11, 11 and 10 bits.
constexpr int kRadixBins = 2048;
constexpr int kRadixPasses = 3;
// CTAs per row of a radix pass at most (sizes the candidate counts).
constexpr int kRadixMaxChunks = 64;
// Partial record: m (kept max), l (sum of exp), count, m_all, o[d].
constexpr int kRecHeader = 4;

struct Geometry {
    int b, hq, hk, hv, d, l, l_cap;
    int dv;     // value head dim (d is the key and query head dim)
    int G;      // query heads per key head
    int NT;     // n-tiles of 8 query heads per key head (1 or 2)
    int P;      // positions per tile: kStageBytes / (h_k * d * 2)
    int KB;     // key TMA box / shared-memory row: min(d, 64) elements
    int WPK;    // consumer warps per key head: 8 / h_k
    int MBW;    // 16-position m-blocks per warp per tile: 128 / d (4 for d = 32)
    int tiles;  // tiles per batch row: ceil(l / P)
    int l_pad;  // tiles * P (row stride of the kept-entry lists)
    int S_cap;  // partial-record slots per (batch, query head)
    int rec;    // floats per partial record: dv + kRecHeader
    float scale;
};

// The streaming kernels cut the flattened (batch, tile) space of T tiles into
// C contiguous ranges, one per CTA: CTA c owns tiles [T*c/C, T*(c+1)/C).
SAGA_HD long long cta_tile_begin(long long T, int C, int c) { return T * c / C; }
// The CTA whose range holds tile x: max c with T*c/C <= x.
SAGA_HD int cta_of_tile(long long x, long long T, int C) {
    return static_cast<int>(((x + 1) * C + T - 1) / T) - 1;
}
// Number of CTAs whose range meets batch row bb (its partial-record slots).
SAGA_HD int slots_of_batch(int bb, int tiles, long long T, int C) {
    const long long x0 = static_cast<long long>(bb) * tiles;
    return cta_of_tile(x0 + tiles - 1, T, C) - cta_of_tile(x0, T, C) + 1;
}

// List j (= slot * WPK + warp) of batch row bb in the fused kernel's kept
// lists: the offset of its first entry in the row's list region and the
// number of entries it can hold (the warp's share of the slot's positions).
struct SegList {
    int start, cap;
};
SAGA_HD SegList seg_list_of(int P, int MBW, int WPK, int tiles, int bb, int j, long long T, int C) {
    const long long x0 = static_cast<long long>(bb) * tiles;
    const int sl = j / WPK, sub = j - sl * WPK;
    const int c = cta_of_tile(x0, T, C) + sl;
    const long long t0 = cta_tile_begin(T, C, c), t1 = cta_tile_begin(T, C, c + 1);
    const long long s0 = t0 > x0 ? t0 : x0;
    const long long s1 = t1 < x0 + tiles ? t1 : x0 + tiles;
    const int cap = static_cast<int>((s1 - s0) * MBW * 16);
    return SegList{static_cast<int>((s0 - x0) * P) + sub * cap, cap};
}

// The regions up to `rowmax` depend only on the batch and head counts, so
// their offsets do not move when the cached length changes (decode with a
// growing cache); the per-row tickets, which must be zero on entry, live
// there.
struct WsLayout {
    size_t err;       // uint32 sticky flag, then the uint32 empty-set row counter (256-byte header)
    size_t tickets;   // uint32 [b*hq]  last-CTA tickets (zero on entry, left at zero)
    size_t hist;      // uint32 [kRadixPasses][b*hq][kRadixBins]
    size_t state;     // uint32 [b*hq][2]  (prefix, rank)
    size_t cnt;       // int32  [b*hq]
    size_t cand_cnt;  // int32  [b*hq][kRadixMaxChunks]  radix pass-1 candidates per chunk
    size_t rowmax;    // float  [b*hq]
    size_t records;   // float  [b*hq][S_cap * WPK][rec]
    size_t seg_cnt;   // int32  [b*hq][S_cap][WPK]
    size_t seg_mall;  // float  [b*hq][S_cap][WPK]
    size_t list_idx;  // int32  [b*hq][l_pad]; with list_s also the int2 [b*hq][l_pad]
    size_t list_s;    // float  [b*hq][l_pad]   (position, logit) pairs of the fused path
    size_t logits;    // float  [b*hq][l]
    size_t cand;      // int2   [b*hq][l]  radix pass-1 candidates (position, logit bits)
    size_t total;
};

SAGA_HD size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline WsLayout workspace_layout(const Geometry& g) {
    const size_t rows = static_cast<size_t>(g.b) * g.hq;
    WsLayout w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + bytes, 256);
        return at;
    };
    w.err = take(256);
    w.tickets = take(rows * sizeof(uint32_t));
    w.hist = take(static_cast<size_t>(kRadixPasses) * rows * kRadixBins * sizeof(uint32_t));
    w.state = take(rows * 2 * sizeof(uint32_t));
    w.cnt = take(rows * sizeof(int32_t));
    w.cand_cnt = take(rows * kRadixMaxChunks * sizeof(int32_t));
    w.rowmax = take(rows * sizeof(float));
    w.records = take(rows * g.S_cap * g.WPK * g.rec * sizeof(float));
    w.seg_cnt = take(rows * g.S_cap * g.WPK * sizeof(int32_t));
    w.seg_mall = take(rows * g.S_cap * g.WPK * sizeof(float));
    w.list_idx = take(rows * g.l_pad * sizeof(int32_t));
    w.list_s = take(rows * g.l_pad * sizeof(float));
    w.logits = take(rows * g.l * sizeof(float));
    w.cand = take(rows * g.l * 2 * sizeof(int32_t));
    w.total = off;
    return w;
}

}  // namespace saga
