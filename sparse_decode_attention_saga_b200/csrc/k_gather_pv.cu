// Softmax over the kept logits and the gathered probability-value product.
//
// Method: "More Value per Key" (ai.info summary, Main Findings, "Bottleneck
// shift"): with top-N sparsity the probability-value product touches only
// h_q x N value vectors per decoded token, so this kernel reads only the
// value rows of kept positions, from value head vh(i) = i*h_v/h_q (SAGA,
// Key Contributions #3).
//
// A row's kept entries live in one or more ascending lists of (position,
// logit) pairs: one contiguous list from a compaction kernel
// (kListContiguous), or one list per
// (streaming CTA slot, consumer warp) from the fused kernel (kListSegments).
// Grid (parts, rows), or (rows, parts) with part_major: every CTA builds the
// row's list table (counts and exclusive prefix) in shared memory and takes
// an equal share of the row's flattened entries, so the work is balanced
// whatever the lists' lengths.  Parts past what the row's entry count needs
// return without a record; with few rows (many parts per row) the grid is
// part-major, so part p of every row is scheduled before part p + 1 of any
// row and no row waits for a second wave of CTAs that turn out to be empty.
// Each warp then works through its own contiguous part of that share without
// block barriers: 32 entries at a time, one (position, logit) per lane read
// with coalesced loads, and each value row handled by a lane group (8 or 16
// lanes, 16 bytes each), weighted by exp(s - m) and accumulated in fp32.
// With long rows and many of them (STAGED) the 32 value rows are copied
// with cp.async into a two-stage per-warp ring in shared memory (the next
// 32 rows' loads in flight while these are summed); otherwise they are
// loaded into registers, a few per lane at a time.  m is the row's largest logit, which is always kept when anything is
// (tau_eff <= max), so no running max is needed.  The share's (m, sum of
// weights, count, row max, unnormalised output) record is merged across
// shares by the last CTA of the row; all shares used the same reference m,
// so the merge is a plain sum of the records in one pass.
#include "combine_row.cuh"

namespace saga {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMinShare = 128;  // kept entries per CTA at least
#ifndef SAGA_GATHER_STAGED_SHARE
#define SAGA_GATHER_STAGED_SHARE 1024
#endif
// ... with the stage ring, whose stages only overlap when a warp has
// several rounds of 32 entries (a tuning constant: 1024 against 128 took
// the Llama-shaped batch-16 gather from 45.1 to 43.8 us and the Sigma-style
// one from 32.9 to 29.6 us)
constexpr int kMinShareStaged = SAGA_GATHER_STAGED_SHARE;
#ifndef SAGA_GATHER_STAGES
#define SAGA_GATHER_STAGES 2
#endif
#ifndef SAGA_GATHER_MINBLOCKS
#define SAGA_GATHER_MINBLOCKS 3
#endif
// CTAs per SM the register budget is sized for with the stage ring (a
// tuning constant; its shared memory allows three with two stages), four
// without
template <bool STAGED>
constexpr int gather_min_blocks() { return STAGED ? SAGA_GATHER_MINBLOCKS : 4; }

static_assert(kThreads == kCombineThreads, "the last CTA of a row runs the row merge");

// Per-warp ring of value-row stages (cp.async, 64-dim value heads): 32 rows
// of the value head dim, then the 32 entries' weights.  128-dim value heads
// load their rows into registers, kGatherInflight per lane at a time.
constexpr int kGatherStages = SAGA_GATHER_STAGES;
constexpr int kGatherInflight = 2;
template <int D>
struct GatherStage {
    static constexpr int kRowsBytes = 32 * D * 2;
    static constexpr int kBytes = kRowsBytes + 32 * 4;
};
__host__ __device__ inline size_t gather_ring_offset(int max_lists) {
    return ((2 * static_cast<size_t>(max_lists) + 1) * sizeof(int) + 127) / 128 * 128;
}

// D: value head dim, DK: key/query head dim, PM: part-major grid (rows, parts)
// STAGED: the value rows go through the cp.async ring (64-dim value heads).
template <int D, int DK, int NT, bool PM, bool STAGED>
__global__ void __launch_bounds__(kThreads, gather_min_blocks<STAGED>()) gather_pv_kernel(const GatherArgs a) {
    constexpr int LPR = D * 2 / 16;    // lanes per value row (16 B each)
    constexpr int RPI = 32 / LPR;      // value rows per warp instruction
    constexpr bool kStaged = STAGED && D == 64;  // value rows through the cp.async ring

    extern __shared__ int table[];     // pre, start
    __shared__ float red_m[kWarps];
    __shared__ float red_l[kWarps];
    __shared__ float red_o[kWarps][D];
    __shared__ int red_i[kWarps];
    __shared__ long long row_base;
    __shared__ int is_last;

    pdl_wait();     // lists, counts and maxima come from the previous kernel
    pdl_trigger();
    const Geometry& g = a.g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long row = PM ? blockIdx.x : blockIdx.y;
    const int part = PM ? blockIdx.y : blockIdx.x;
    const int bb = static_cast<int>(row / g.hq);
    const int i = static_cast<int>(row - static_cast<long long>(bb) * g.hq);
    const int vh = i * g.hv / g.hq;
    int* pre = table;                      // exclusive prefix of list counts; pre[nl] = total
    int* start = table + a.max_lists + 1;  // list start inside the row's list region

    // ---- list table of the row
    float m_all = -kInf;
    int nl = 1;
    if (a.mode == kListContiguous) {
        if (tid == 0) {
            pre[0] = 0;
            const int c = __ldg(a.cnt + row);
            in_bounds(c >= 0 && c <= g.l, a.err);
            pre[1] = min(max(c, 0), g.l);
            start[0] = 0;
            row_base = row * g.l;
        }
        m_all = __ldg(a.rowmax + row);
        __syncthreads();
    } else {
        const long long T = static_cast<long long>(g.b) * g.tiles;
        const long long x0 = static_cast<long long>(bb) * g.tiles;
        const int c_first = cta_of_tile(x0, T, a.C);
        const int slots = cta_of_tile(x0 + g.tiles - 1, T, a.C) - c_first + 1;
        nl = slots * g.WPK;  // <= max_lists (checked by the host)
        // Each thread owns a run of consecutive lists: it requests their counts
        // and maxima all at once, works out where each list starts (the
        // streaming CTA's segment of the row, split evenly over its warps)
        // while they are in flight, and keeps the clamped counts for the scan.
        const size_t rbase = static_cast<size_t>(row) * g.S_cap * g.WPK;
        const int per = (nl + kThreads - 1) / kThreads;
        const int j0 = min(nl, tid * per), j1 = min(nl, j0 + per);
        float mloc = -kInf;
        int run = 0;
        constexpr int kRun = 4;  // counts in flight per thread
        for (int jb = j0; jb < j1; jb += kRun) {
            int cu[kRun];
            float mm[kRun];
#pragma unroll
            for (int u = 0; u < kRun; ++u) {
                cu[u] = jb + u < j1 ? a.seg_cnt[rbase + jb + u] : 0;
                mm[u] = jb + u < j1 ? a.seg_mall[rbase + jb + u] : -kInf;
            }
            int sl_prev = -1, pos = 0, cap = 0;
#pragma unroll
            for (int u = 0; u < kRun; ++u) {
                const int j = jb + u;
                if (j < j1) {
                    const int sl = j / g.WPK;
                    if (sl != sl_prev) {
                        const int c = c_first + sl;
                        const long long t0 = cta_tile_begin(T, a.C, c), t1 = cta_tile_begin(T, a.C, c + 1);
                        const long long s0 = t0 > x0 ? t0 : x0;
                        const long long s1 = t1 < x0 + g.tiles ? t1 : x0 + g.tiles;
                        pos = static_cast<int>((s0 - x0) * g.P);
                        cap = static_cast<int>((s1 - s0) * g.MBW * 16);  // entries a warp can hold
                        sl_prev = sl;
                    }
                    start[j] = pos + (j - sl * g.WPK) * cap;
                    in_bounds(cu[u] >= 0 && cu[u] <= cap, a.err);
                    const int cnt_j = cu[u] < 0 ? 0 : (cu[u] > cap ? cap : cu[u]);
                    pre[j] = cnt_j;
                    run += cnt_j;
                    mloc = fmaxf(mloc, mm[u]);
                }
            }
        }
        int inc = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        mloc = warp_max(mloc);
        if (lane == 31) red_i[warp] = inc;
        if (lane == 0) red_m[warp] = mloc;
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            before += w < warp ? red_i[w] : 0;
            total += red_i[w];
            m_all = fmaxf(m_all, red_m[w]);
        }
        int acc = before + inc - run;
        for (int j = j0; j < j1; ++j) {
            const int c = pre[j];
            pre[j] = acc;
            acc += c;
        }
        if (tid == 0) {
            pre[nl] = total;
            row_base = row * g.l_pad;
        }
        __syncthreads();
    }
    const int total = pre[nl];
    // Shares of at least kMinShare entries: with few kept entries per row the
    // parts past `parts` return here instead of each paying a CTA's fixed cost
    // for a handful of rows.
    constexpr int kShare = kStaged ? kMinShareStaged : kMinShare;
    const int parts = max(1, min(a.parts, (total + kShare - 1) / kShare));
    if (part >= parts) return;  // not needed for this row: no record, no ticket
    const int e0 = static_cast<int>(static_cast<long long>(total) * part / parts);
    const int e1 = static_cast<int>(static_cast<long long>(total) * (part + 1) / parts);
    const int n = e1 - e0;
    // each warp owns a contiguous sub-share and needs no block barrier
    const int w0 = e0 + static_cast<int>(static_cast<long long>(n) * warp / kWarps);
    const int w1 = e0 + static_cast<int>(static_cast<long long>(n) * (warp + 1) / kWarps);
    // Softmax reference: whenever a row keeps anything its largest kept logit
    // is the row's largest logit (tau_eff <= max), so exp(s - m) needs no
    // running max and no rescaling.
    const float m = m_all;

    const int grp = lane / LPR, col0 = (lane % LPR) * 8;
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;
    float lsum = 0.f;
    const char* vrow0 = reinterpret_cast<const char*>(a.v) +
                        (static_cast<size_t>(bb) * g.l_cap * g.hv + vh) * D * 2;
    const size_t vstride = static_cast<size_t>(g.hv) * D * 2;  // bytes between positions
    constexpr int ROUNDS = 32 / RPI;   // value rows per lane group per 32 entries

    // entry e -> (position, logit); out-of-range entries give (0, -inf)
    // The list holding entry e is the last j with pre[j] <= e.  Each lane's
    // entries only move forward (by 32 per round); with d = 64 a cursor `lo`
    // stays put while the entry is still inside its list (one compare) and
    // otherwise moves by binary search over the later lists; with d = 128 the
    // extra live register costs more than it saves (measured), so every
    // lookup is a binary search.
    int lo = 0;
    auto fetch = [&](int e, int& pos, float& s) {
        pos = 0;
        s = -kInf;
        if (e < w1) {
            if (D != 64) lo = 0;
            if (lo + 1 < nl && pre[lo + 1] <= e) {
                int l2 = lo + 1, hi = nl - 1;
                while (l2 < hi) {
                    const int mid = (l2 + hi + 1) >> 1;
                    if (pre[mid] <= e) l2 = mid; else hi = mid - 1;
                }
                lo = l2;
            }
            const long long at = row_base + start[lo] + (e - pre[lo]);
            if (a.mode == kListContiguous) {
                pos = __ldg(a.idx + at);
                s = __ldg(a.list_s + at);
            } else {
                const int2 ps = __ldg(a.seg_list + at);
                pos = ps.x;
                s = __int_as_float(ps.y);
            }
            if (!in_bounds(pos >= 0 && pos < g.l, a.err)) {
                pos = 0;
                s = -kInf;
            }
        }
    };

    const int grp_col = (lane % LPR) * 16;  // this lane's 16 bytes of a value row
    if constexpr (kStaged) {
        // Value rows of 32 entries at a time go to a per-warp ring of
        // kGatherStages stages in shared memory with cp.async (16 bytes per
        // lane and copy, zeros for entries past the share), so that the
        // loads of the next stage are in flight while this one is summed;
        // each stage also holds its entries' weights exp(s - m).  The
        // entries of the next stage to issue are fetched one issue ahead.
        uint8_t* ring = reinterpret_cast<uint8_t*>(table) + gather_ring_offset(a.max_lists) +
                        static_cast<size_t>(warp) * kGatherStages * GatherStage<D>::kBytes;
        int nxt_pos;
        float nxt_s;
        fetch(w0 + lane, nxt_pos, nxt_s);
        auto issue = [&](int st, int e_base) {
            const int pos = nxt_pos;
            const float s = nxt_s;
            uint8_t* rows = ring + st * GatherStage<D>::kBytes;
            reinterpret_cast<float*>(rows + GatherStage<D>::kRowsBytes)[lane] =
                e_base + lane < w1 ? __expf(s - m) : 0.f;
            const uint32_t rows_a = smem_addr(rows);
#pragma unroll
            for (int i = 0; i < LPR; ++i) {
                const int q = i * 32 + lane;  // 16-byte chunk q: row q / LPR, column chunk q % LPR
                const int r = q / LPR, cc = q % LPR;
                const int pr = __shfl_sync(0xffffffffu, pos, r);
                cp_async_16(rows_a + r * (D * 2) + cc * 16, vrow0 + static_cast<size_t>(pr) * vstride + cc * 16,
                            e_base + r < w1 ? 16u : 0u);
            }
            cp_async_commit();
            fetch(e_base + 32 + lane, nxt_pos, nxt_s);
        };
        auto consume = [&](int st) {
            const uint8_t* rows = ring + st * GatherStage<D>::kBytes;
            const float* pw = reinterpret_cast<const float*>(rows + GatherStage<D>::kRowsBytes);
            lsum += pw[lane];
#pragma unroll
            for (int r0 = 0; r0 < ROUNDS; ++r0) {
                const int r = r0 * RPI + grp;
                const uint4 raw = *reinterpret_cast<const uint4*>(rows + r * (D * 2) + grp_col);
                const float p = pw[r];
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    acc[2 * c] = fmaf(p, bf16_lo(w4[c]), acc[2 * c]);
                    acc[2 * c + 1] = fmaf(p, bf16_hi(w4[c]), acc[2 * c + 1]);
                }
            }
        };
        const int nr = (w1 - w0 + 31) / 32;  // rounds of this warp
#pragma unroll
        for (int st = 0; st < kGatherStages; ++st) {
            if (st < nr) issue(st, w0 + st * 32);
            else cp_async_commit();  // empty groups keep the count of pending groups uniform
        }
        for (int it = 0; it < nr; ++it) {
            const int st = it % kGatherStages;
            cp_async_wait<kGatherStages - 1>();  // this lane's copies of round it are done
            __syncwarp();                        // and every lane's
            consume(st);
            __syncwarp();                        // the stage is free again
            if (it + kGatherStages < nr) issue(st, w0 + (it + kGatherStages) * 32);
            else cp_async_commit();
        }
        cp_async_wait<0>();
    } else {
        // Few entries per warp, or 128-dim value rows (the ring would leave
        // one CTA per SM): the rows are loaded into registers,
        // kGatherInflight per lane at a time, with the next round's entries
        // in flight.
        int nxt_pos;
        float nxt_s;
        fetch(w0 + lane, nxt_pos, nxt_s);
        constexpr int INFLIGHT = ROUNDS < kGatherInflight ? ROUNDS : kGatherInflight;
        for (int base = w0; base < w1; base += 32) {
            const int pos = nxt_pos;
            const float s = nxt_s;
            fetch(base + 32 + lane, nxt_pos, nxt_s);
            const float p_lane = base + lane < w1 ? __expf(s - m) : 0.f;
            lsum += p_lane;
            // lane group grp gathers entries grp, grp+RPI, ... of the 32
#pragma unroll
            for (int r0 = 0; r0 < ROUNDS; r0 += INFLIGHT) {
                uint4 raw[INFLIGHT];
#pragma unroll
                for (int u = 0; u < INFLIGHT; ++u) {
                    const int k = (r0 + u) * RPI + grp;
                    const int pk = __shfl_sync(0xffffffffu, pos, k);
                    raw[u] = base + k < w1 ? __ldg(reinterpret_cast<const uint4*>(
                                                 vrow0 + static_cast<size_t>(pk) * vstride + grp_col))
                                           : make_uint4(0u, 0u, 0u, 0u);
                }
                float pu[INFLIGHT];
#pragma unroll
                for (int u = 0; u < INFLIGHT; ++u)
                    pu[u] = __shfl_sync(0xffffffffu, p_lane, (r0 + u) * RPI + grp);
#pragma unroll
                for (int u = 0; u < INFLIGHT; ++u) {
                    const uint32_t w4[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        acc[2 * c] = fmaf(pu[u], bf16_lo(w4[c]), acc[2 * c]);
                        acc[2 * c + 1] = fmaf(pu[u], bf16_hi(w4[c]), acc[2 * c + 1]);
                    }
                }
            }
        }
    }

    // reduce the row groups of the warp (lanes with equal col0), then merge the
    // warps' (max, sum, output) with log-sum-exp weights
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) {
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], o);
    }
    lsum = warp_sum(lsum);
    if (grp == 0) {
#pragma unroll
        for (int c = 0; c < 8; ++c) red_o[warp][col0 + c] = acc[c];
    }
    if (lane == 0) red_l[warp] = lsum;
    __syncthreads();
    float* rec = a.records + (static_cast<size_t>(row) * g.S_cap * g.WPK + part) * g.rec;
    for (int c = tid; c < D; c += kThreads) {
        float o = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) o += red_o[w][c];
        rec[kRecHeader + c] = o;
    }
    if (tid == 0) {
        float l = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) l += red_l[w];
        rec[0] = n > 0 ? m : -kInf;
        rec[1] = l;
        rec[2] = __int_as_float(n);
        rec[3] = m_all;
    }

    // the row's last CTA to finish merges the row's `parts` records
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = atomicAdd(a.tickets + row, 1u) == static_cast<unsigned>(parts - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    if (tid == 0) a.tickets[row] = 0u;
    merge_same_reference<D, DK, NT>(a.cmb, row, parts, m_all);
}

}  // namespace

size_t gather_smem_bytes(int max_lists) {
    return (2 * static_cast<size_t>(max_lists) + 1) * sizeof(int);
}

static size_t gather_total_smem(int max_lists, bool staged) {
    if (!staged) return gather_smem_bytes(max_lists);  // no ring
    return gather_ring_offset(max_lists) + static_cast<size_t>(kWarps) * kGatherStages * GatherStage<64>::kBytes;
}

// The ring pays where each warp has many rounds of 32 entries (long rows,
// many of them: Llama-shaped batch 16 at 128K, 44.7 against 52.9 us for the
// gather with its merge); with few entries per warp its extra latency and
// the lower occupancy cost more (batch 1 at 128K: 12.3 against 7.1 us;
// batch 16 at 8K: 26.1 against 22.8 us).
static bool gather_staged(const Geometry& g) {
    return g.dv == 64 && g.l >= 65536 && static_cast<long long>(g.b) * g.hq >= 128;
}


cudaError_t launch_gather_pv(const GatherArgs& a, cudaStream_t stream) {
    const long long rows = static_cast<long long>(a.g.b) * a.g.hq;
    if (a.parts < 1 || a.parts > 65535 || rows > (a.part_major ? 0x7fffffffll : 65535ll))
        return cudaErrorInvalidValue;
    const dim3 grid = a.part_major ? dim3(static_cast<unsigned>(rows), static_cast<unsigned>(a.parts))
                                   : dim3(static_cast<unsigned>(a.parts), static_cast<unsigned>(rows));
    if (gather_smem_bytes(a.max_lists) > static_cast<size_t>(kGatherMaxSmem) || a.cmb.parts != a.parts)
        return cudaErrorInvalidValue;
    const bool staged = gather_staged(a.g);
    const size_t smem = gather_total_smem(a.max_lists, staged);
#define SAGA_GATHER_CASE(D_, DK_, NT_, ST_)                                                    \
    if (a.g.dv == D_ && a.g.d == DK_ && a.g.NT == NT_ && staged == ST_) {                      \
        auto k_rows = gather_pv_kernel<D_, DK_, NT_, false, ST_>;                              \
        auto k_parts = gather_pv_kernel<D_, DK_, NT_, true, ST_>;                              \
        auto kern = a.part_major ? k_parts : k_rows;                                           \
        const cudaError_t attr = allow_dynamic_smem(kern, static_cast<int>(smem));            \
        if (attr != cudaSuccess) return attr;                                                  \
        return launch_dependent(kern, grid, dim3(kThreads), smem, stream, a);                  \
    }
    SAGA_GATHER_CASE(64, 64, 1, false)
    SAGA_GATHER_CASE(64, 64, 2, false)
    SAGA_GATHER_CASE(64, 64, 1, true)
    SAGA_GATHER_CASE(64, 64, 2, true)
    SAGA_GATHER_CASE(128, 128, 1, false)
    SAGA_GATHER_CASE(128, 128, 2, false)
    SAGA_GATHER_CASE(64, 32, 1, false)
    SAGA_GATHER_CASE(64, 32, 2, false)
    SAGA_GATHER_CASE(64, 32, 1, true)
    SAGA_GATHER_CASE(64, 32, 2, true)
#undef SAGA_GATHER_CASE
    return cudaErrorInvalidValue;
}

}  // namespace saga
