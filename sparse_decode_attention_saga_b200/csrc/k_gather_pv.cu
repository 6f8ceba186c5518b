// Softmax over the kept logits and the gathered probability-value product.
//
// Method: "More Value per Key" (ai.info summary, Main Findings, "Bottleneck
// shift"): with top-N sparsity the probability-value product touches only
// h_q x N value vectors per decoded token, so this kernel reads only the
// value rows of kept positions, from value head vh(i) = i*h_v/h_q (SAGA,
// Key Contributions #3).
//
// A row's kept entries live in one or more ascending lists of (position,
// logit) pairs: one contiguous list from the compare/compact kernel
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
// with coalesced loads one round ahead, and 16-byte value-row loads by lane
// groups (8 or 16 lanes per row), weighted by exp(s - m) and accumulated in
// fp32.  m is the row's largest logit, which is always kept when anything is
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
#ifndef SAGA_GATHER_INFLIGHT
#define SAGA_GATHER_INFLIGHT 2
#endif
#ifndef SAGA_GATHER_MINBLOCKS
#define SAGA_GATHER_MINBLOCKS 4
#endif
// value-row loads in flight per lane group, and CTAs per SM the register
// budget is sized for (tuning constants)
constexpr int kGatherInflight = SAGA_GATHER_INFLIGHT;
constexpr int kGatherMinBlocks = SAGA_GATHER_MINBLOCKS;

static_assert(kThreads == kCombineThreads, "the last CTA of a row runs the row merge");

// D: value head dim, DK: key/query head dim, PM: part-major grid (rows, parts)
template <int D, int DK, int NT, bool PM>
__global__ void __launch_bounds__(kThreads, kGatherMinBlocks) gather_pv_kernel(const GatherArgs a) {
    constexpr int LPR = D * 2 / 16;    // lanes per value row (16 B each)
    constexpr int RPI = 32 / LPR;      // value rows per warp instruction

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
    const int parts = max(1, min(a.parts, (total + kMinShare - 1) / kMinShare));
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
    const __nv_bfloat16* vbase = reinterpret_cast<const __nv_bfloat16*>(a.v) +
                                 (static_cast<size_t>(bb) * g.l_cap * g.hv + vh) * D + col0;
    const size_t vstride = static_cast<size_t>(g.hv) * D;
    constexpr int ROUNDS = 32 / RPI;   // value-row loads per lane per 32 entries
    constexpr int INFLIGHT = ROUNDS < kGatherInflight ? ROUNDS : kGatherInflight;

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
    int nxt_pos;
    float nxt_s;
    fetch(w0 + lane, nxt_pos, nxt_s);
    for (int base = w0; base < w1; base += 32) {
        // one entry per lane; the next round's entries are already in flight
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
                raw[u] = base + k < w1 ? __ldg(reinterpret_cast<const uint4*>(vbase + pk * vstride))
                                       : make_uint4(0u, 0u, 0u, 0u);
            }
            float p[INFLIGHT];
#pragma unroll
            for (int u = 0; u < INFLIGHT; ++u)
                p[u] = __shfl_sync(0xffffffffu, p_lane, (r0 + u) * RPI + grp);
#pragma unroll
            for (int u = 0; u < INFLIGHT; ++u) {
                const uint32_t w4[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    acc[2 * c] = fmaf(p[u], bf16_lo(w4[c]), acc[2 * c]);
                    acc[2 * c + 1] = fmaf(p[u], bf16_hi(w4[c]), acc[2 * c + 1]);
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


cudaError_t launch_gather_pv(const GatherArgs& a, cudaStream_t stream) {
    const long long rows = static_cast<long long>(a.g.b) * a.g.hq;
    if (a.parts < 1 || a.parts > 65535 || rows > (a.part_major ? 0x7fffffffll : 65535ll))
        return cudaErrorInvalidValue;
    const dim3 grid = a.part_major ? dim3(static_cast<unsigned>(rows), static_cast<unsigned>(a.parts))
                                   : dim3(static_cast<unsigned>(a.parts), static_cast<unsigned>(rows));
    const size_t smem = gather_smem_bytes(a.max_lists);
    if (smem > static_cast<size_t>(kGatherMaxSmem) || a.cmb.parts != a.parts) return cudaErrorInvalidValue;
#define SAGA_GATHER_CASE(D_, DK_, NT_)                                                         \
    if (a.g.dv == D_ && a.g.d == DK_ && a.g.NT == NT_) {                                       \
        auto k_rows = gather_pv_kernel<D_, DK_, NT_, false>;                                   \
        auto k_parts = gather_pv_kernel<D_, DK_, NT_, true>;                                   \
        auto kern = a.part_major ? k_parts : k_rows;                                           \
        const cudaError_t attr = allow_dynamic_smem(kern, kGatherMaxSmem);                     \
        if (attr != cudaSuccess) return attr;                                                  \
        return launch_dependent(kern, grid, dim3(kThreads), smem, stream, a);                  \
    }
    SAGA_GATHER_CASE(64, 64, 1)
    SAGA_GATHER_CASE(64, 64, 2)
    SAGA_GATHER_CASE(128, 128, 1)
    SAGA_GATHER_CASE(128, 128, 2)
    SAGA_GATHER_CASE(64, 32, 1)
    SAGA_GATHER_CASE(64, 32, 2)
#undef SAGA_GATHER_CASE
    return cudaErrorInvalidValue;
}

}  // namespace saga
