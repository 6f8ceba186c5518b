// Log-sum-exp merge of the partial records of one (batch, query head) row,
// and the empty-set fallback, shared by the combine kernel and by the last
// gather CTA of a row.
//
// Each partial record holds (m, l, count, m_all, o[d]) with
// o = sum_j exp(s_j - m) V_j and l = sum_j exp(s_j - m) over the part's kept
// entries.  The merge is M = max m_r, out = sum_r exp(m_r - M) o_r /
// sum_r exp(m_r - M) l_r (split-K / flash-decoding combine).
//
// Empty-set reading (the pages are silent): when a stale threshold lies above
// every logit of the row, nothing was kept and the row keeps its maximal
// entries instead (tau_eff = min(tau, max_j s_j)).  The streaming kernel
// recorded the maximum logit each part saw; here the row's logits are
// recomputed with the same tensor-core routine (bit-identical values), the
// positions equal to that maximum are found, and their value rows averaged
// (equal logits give equal softmax weights).
#pragma once

#include "qk_tile.cuh"
#include "saga_kernels.h"

namespace saga {

constexpr int kCombineThreads = 256;

// The empty-set rule's row, by one warp: the positions whose logit equals
// the row maximum m_star (recomputed bit for bit with the streaming
// kernel's tensor-core routine), their count, and the mean of their value
// rows into out_row.  With the fused kernel's per-list maxima (a.seg_mall)
// only the lists holding m_star are recomputed, otherwise the whole row.
// raw: out_row gets the sum of the value rows at m_star instead of their
// mean.  idx_out (nullable): their positions, ascending.  Returns their
// number (all lanes).
template <int DV, int D, int NT>  // D: key/query head dim, DV: value head dim
__device__ int fallback_row(const CombineArgs& a, long long row, float m_star, float* out_row,
                            int32_t* cnt_out, uint8_t* kbuf, bool raw = false,
                            int32_t* idx_out = nullptr) {
    const Geometry& g = a.g;
    const int lane = threadIdx.x & 31;
    const int bb = static_cast<int>(row / g.hq);
    const int i = static_cast<int>(row - static_cast<long long>(bb) * g.hq);
    const int kh = i / g.G, hl = i - kh * g.G;
    const int vh = i * g.hv / g.hq;
    const int nti = hl >> 3, col = hl & 7;
    const int gq = lane >> 2, tq = lane & 3;
    constexpr int CPL = DV / 32;  // value columns per lane

    QFrag<D, NT> qf;
    load_q_frag<D, NT>(qf, reinterpret_cast<const __nv_bfloat16*>(a.q), g.hq, g.G, bb, kh, lane);
    const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(a.k);
    const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(a.v);
    float osum[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) osum[c] = 0.f;
    int count = 0;
    // positions j0 .. j0+15: their logits recomputed, those equal to m_star
    // (ascending: h, then lane) counted and their value rows summed
    auto block = [&](int j0) {
        // 16 key rows of head kh into the swizzled tile layout of qk_mma
        for (int q8 = lane; q8 < 16 * D / 8; q8 += 32) {
            const int r = q8 / (D / 8), cc = q8 - r * (D / 8);
            const int dh = cc / KTile<D>::CPR, c8 = cc % KTile<D>::CPR;
            const int pos = j0 + r;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (pos < g.l)
                v = *reinterpret_cast<const uint4*>(
                    K + ((static_cast<size_t>(bb) * g.l_cap + pos) * g.hk + kh) * D + cc * 8);
            *reinterpret_cast<uint4*>(kbuf + KTile<D>::offset(dh, 16, r, c8)) = v;
        }
        __syncwarp();
        float acc[1][NT][4];
        qk_mma<D, NT, 1>(smem_addr(kbuf), 16, 0, 0, qf, acc, lane);
        __syncwarp();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            bool match = false;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float s = __fmul_rn(acc[0][nt][2 * h + e], g.scale);
                    const int pos = j0 + gq + 8 * h;
                    if (nt == nti && 2 * tq + e == col && pos < g.l && s == m_star) match = true;
                }
            uint32_t ball = __ballot_sync(0xffffffffu, match);
            while (ball) {
                const int src = __ffs(ball) - 1;
                ball &= ball - 1;
                const int pos = j0 + (src >> 2) + 8 * h;
                if (idx_out && lane == 0) idx_out[count] = pos;
                const __nv_bfloat16* vr =
                    V + ((static_cast<size_t>(bb) * g.l_cap + pos) * g.hv + vh) * DV + lane * CPL;
#pragma unroll
                for (int c = 0; c < CPL; ++c) osum[c] += __bfloat162float(vr[c]);
                ++count;
            }
        }
    };
    // (64-dim values with at most 8 query heads per key head only: in the
    // other instantiations the extra loop state spills registers of the
    // gather kernel that inlines this)
    bool lists_only = false;
    if constexpr (DV == 64 && NT == 1) lists_only = a.seg_mall != nullptr;
    if (lists_only) {
        // The fused kernel's per-(slot, warp) maxima say which of its lists
        // hold the row maximum: only their positions are recomputed (for each
        // slot in order, its tiles in order, in each tile the warps' 16-row
        // blocks in order, so positions stay ascending).
        const long long T = static_cast<long long>(g.b) * g.tiles;
        const long long x0 = static_cast<long long>(bb) * g.tiles;
        const int c_first = cta_of_tile(x0, T, a.C);
        const int slots = cta_of_tile(x0 + g.tiles - 1, T, a.C) - c_first + 1;
        const float* mall_row = a.seg_mall + static_cast<size_t>(row) * g.S_cap * g.WPK;
        for (int sl = 0; sl < slots; ++sl) {
            const uint32_t subs =
                __ballot_sync(0xffffffffu, lane < g.WPK && __ldcg(mall_row + sl * g.WPK + lane) == m_star);
            if (!subs) continue;
            // the slot's tiles of this batch row, as offsets in the row
            const int c = c_first + sl;
            const int r0 = static_cast<int>(max(cta_tile_begin(T, a.C, c) - x0, 0ll));
            const int r1 = static_cast<int>(min(cta_tile_begin(T, a.C, c + 1) - x0,
                                                static_cast<long long>(g.tiles)));
            for (int tl = r0; tl < r1; ++tl)
                for (uint32_t sm = subs; sm; sm &= sm - 1u) {
                    const int sub = __ffs(sm) - 1;
                    for (int mbi = 0; mbi < g.MBW; ++mbi) block(tl * g.P + (sub * g.MBW + mbi) * 16);
                }
        }
    } else {
        for (int j0 = 0; j0 < g.l; j0 += 16) block(j0);
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) out_row[lane * CPL + c] = raw ? osum[c] : osum[c] / static_cast<float>(count);
    if (lane == 0 && cnt_out) *cnt_out = count;
    return count;
}

// Number of partial records of row (of batch element bb).
__device__ __forceinline__ int row_records(const CombineArgs& a, int bb) {
    if (a.mode == kCombineParts) return a.parts;
    const Geometry& g = a.g;
    const long long T = static_cast<long long>(g.b) * g.tiles;
    return slots_of_batch(bb, g.tiles, T, a.C) * a.recs_per_slot;
}

// Merges records r_begin .. r_begin + R - 1 of row `row` (R < 0: all the
// row's records) into out, or, with partial_out, into one partial record
// (m, l, count, m_all, o) without normalising.  All kCombineThreads threads
// of the block take part (block barriers).  Records are read through L2, so
// a CTA of the kernel that wrote them may merge them.
template <int D, int DK, int NT>  // D: value head dim, DK: key/query head dim
__device__ void combine_row(const CombineArgs& a, long long row, int r_begin = 0, int R = -1,
                            float* partial_out = nullptr) {
    constexpr int kWarps = kCombineThreads / 32;
    constexpr int kThreads = kCombineThreads;
    __shared__ float red[3][kWarps];
    __shared__ int red_c[kWarps];
    __shared__ float red_o[kWarps][D];
    __shared__ __align__(1024) uint8_t kbuf[16 * DK * 2];

    const Geometry& g = a.g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bb = static_cast<int>(row / g.hq);
    if (R < 0) R = row_records(a, bb);
    const float* recs =
        a.records + (static_cast<size_t>(row) * g.S_cap * g.WPK + r_begin) * g.rec;

    float M = -kInf, mall = -kInf;
    int cnt = 0;
    for (int r = tid; r < R; r += kThreads) {
        const float* rec = recs + static_cast<size_t>(r) * g.rec;
        M = fmaxf(M, __ldcg(rec));
        mall = fmaxf(mall, __ldcg(rec + 3));
        cnt += __float_as_int(__ldcg(rec + 2));
    }
    M = warp_max(M);
    mall = warp_max(mall);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) {
        red[0][warp] = M;
        red[1][warp] = mall;
        red_c[warp] = cnt;
    }
    __syncthreads();
    M = red[0][0];
    mall = red[1][0];
    cnt = red_c[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
        M = fmaxf(M, red[0][w]);
        mall = fmaxf(mall, red[1][w]);
        cnt += red_c[w];
    }

    float* out_row = a.out + static_cast<size_t>(row) * D;
    if (cnt == 0 && a.fallback && !partial_out) {
        if (warp == 0) {
            fallback_row<D, DK, NT>(a, row, mall, out_row, a.sel_cnt ? a.sel_cnt + row : nullptr, kbuf,
                                    false, a.sel_idx ? a.sel_idx + static_cast<size_t>(row) * g.l : nullptr);
            if (lane == 0 && a.empty_rows) atomicAdd(a.empty_rows, 1u);
        }
        return;
    }

    float lsum = 0.f;
    for (int r = tid; r < R; r += kThreads) {
        const float* rec = recs + static_cast<size_t>(r) * g.rec;
        const float m = __ldcg(rec);
        if (m > -kInf) lsum += __ldcg(rec + 1) * __expf(m - M);
    }
    lsum = warp_sum(lsum);
    __syncthreads();
    if (lane == 0) red[2][warp] = lsum;
    __syncthreads();
    lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) lsum += red[2][w];
    const float inv = partial_out ? 1.f : 1.f / lsum;

    // Records are spread over the warps (warp w sums records w, w+8, ...;
    // lane owns D/32 columns), so the loads of different records are in
    // flight together; the warps' partial sums are then added in a fixed order.
    constexpr int CPL = D / 32;
    float o[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[c] = 0.f;
    // eight records per warp in flight: their loads are issued before any is used
    constexpr int U = 8;
    for (int r0 = warp; r0 < R; r0 += U * kWarps) {
        float mv[U], ov[U][CPL];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = r0 + u * kWarps;
            const float* rec = recs + static_cast<size_t>(r < R ? r : 0) * g.rec;
            mv[u] = r < R ? __ldcg(rec) : -kInf;
#pragma unroll
            for (int c = 0; c < CPL; ++c) ov[u][c] = __ldcg(rec + kRecHeader + lane * CPL + c);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (mv[u] > -kInf) {
                const float wgt = __expf(mv[u] - M);
#pragma unroll
                for (int c = 0; c < CPL; ++c) o[c] = fmaf(ov[u][c], wgt, o[c]);
            }
        }
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) red_o[warp][lane * CPL + c] = o[c];
    __syncthreads();
    float* dst = partial_out ? partial_out + kRecHeader : out_row;
    for (int c = tid; c < D; c += kThreads) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += red_o[w][c];
        dst[c] = v * inv;
    }
    if (tid == 0) {
        if (partial_out) {
            partial_out[0] = M;
            partial_out[1] = lsum;
            partial_out[2] = __int_as_float(cnt);
            partial_out[3] = mall;
        } else if (a.sel_cnt) {
            a.sel_cnt[row] = cnt;
        }
    }
}

// Merge of R partial records that were all weighted with the same
// reference (the row's largest logit m_all; empty records hold l = 0 and
// o = 0): out = sum_r o_r / sum_r l_r, with every record load in flight at
// once (one L2 round trip instead of the three dependent passes of
// combine_row).  Rows that kept nothing take the empty-set fallback.
template <int D, int DK, int NT>
__device__ void merge_same_reference(const CombineArgs& a, long long row, int R, float m_all) {
    constexpr int kWarps = kCombineThreads / 32;
    constexpr int U = 4;  // records per warp
    constexpr int CPL = D / 32;
    __shared__ float red_o[kWarps][D];
    __shared__ float red_l[kWarps];
    __shared__ int red_c[kWarps];
    __shared__ __align__(1024) uint8_t kbuf[16 * DK * 2];

    const Geometry& g = a.g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float* recs = a.records + static_cast<size_t>(row) * g.S_cap * g.WPK * g.rec;
    float lw = 0.f, osum[CPL];
    int cw = 0;
#pragma unroll
    for (int k = 0; k < CPL; ++k) osum[k] = 0.f;
    for (int r0 = warp; r0 < R; r0 += U * kWarps) {  // one pass when R <= 32
        float o[U][CPL], l[U];
        int c[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = r0 + u * kWarps;
            const float* rec = recs + static_cast<size_t>(r < R ? r : 0) * g.rec;
#pragma unroll
            for (int k = 0; k < CPL; ++k) o[u][k] = r < R ? __ldcg(rec + kRecHeader + lane * CPL + k) : 0.f;
            l[u] = r < R ? __ldcg(rec + 1) : 0.f;
            c[u] = r < R ? __float_as_int(__ldcg(rec + 2)) : 0;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            lw += l[u];
            cw += c[u];
#pragma unroll
            for (int k = 0; k < CPL; ++k) osum[k] += o[u][k];
        }
    }
#pragma unroll
    for (int k = 0; k < CPL; ++k) red_o[warp][lane * CPL + k] = osum[k];
    if (lane == 0) {
        red_l[warp] = lw;
        red_c[warp] = cw;
    }
    __syncthreads();
    float lsum = 0.f;
    int cnt = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        lsum += red_l[w];
        cnt += red_c[w];
    }
    float* part = a.part ? a.part + static_cast<size_t>(row) * (D + kRecHeader) : nullptr;
    float* out_row = part ? part + kRecHeader : a.out + static_cast<size_t>(row) * D;
    if (cnt == 0) {
        if (a.fallback) {
            if (warp == 0) {
                const int c = fallback_row<D, DK, NT>(
                    a, row, m_all, out_row, part || !a.sel_cnt ? nullptr : a.sel_cnt + row, kbuf,
                    part != nullptr,
                    part || !a.sel_idx ? nullptr : a.sel_idx + static_cast<size_t>(row) * g.l);
                if (part && lane == 0) {
                    part[0] = -kInf;
                    part[1] = static_cast<float>(c);
                    part[2] = __int_as_float(0);
                    part[3] = m_all;
                }
                if (!part && lane == 0 && a.empty_rows) atomicAdd(a.empty_rows, 1u);
            }
        } else {
            for (int k = tid; k < D; k += kCombineThreads) out_row[k] = 0.f;
            if (tid == 0 && part) {
                part[0] = -kInf;
                part[1] = 0.f;
                part[2] = __int_as_float(0);
                part[3] = m_all;
            }
            if (tid == 0 && !part && a.sel_cnt) a.sel_cnt[row] = 0;
        }
        return;
    }
    const float inv = part ? 1.f : 1.f / lsum;
    for (int k = tid; k < D; k += kCombineThreads) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += red_o[w][k];
        out_row[k] = v * inv;
    }
    if (tid == 0) {
        if (part) {
            part[0] = m_all;  // every share was weighted with exp(s - m_all)
            part[1] = lsum;
            part[2] = __int_as_float(cnt);
            part[3] = m_all;
        } else if (a.sel_cnt) {
            a.sel_cnt[row] = cnt;
        }
    }
}

}  // namespace saga
