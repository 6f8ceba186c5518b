// Softmax over the kept logits and the gathered probability-value product.
//
// Method: "More Value per Key" (ai.info summary, Main Findings, "Bottleneck
// shift"): with top-N sparsity the probability-value product touches only
// h_q x N value vectors per decoded token, so this kernel reads only the
// value rows of kept positions, from value head vh(i) = i*h_v/h_q (SAGA,
// Key Contributions #3).
//
// A row's kept entries live in one or more ascending lists: one contiguous
// list from the compare/compact kernel (kListContiguous), or one list per
// (streaming CTA slot, consumer warp) from the fused kernel (kListSegments).
// Grid (parts, rows): every CTA builds the row's list table (counts and
// exclusive prefix) in shared memory and takes an equal share of the row's
// flattened entries, so the work is balanced whatever the lists' lengths.
// The share is processed in batches: the batch's (position, logit) pairs are
// copied to shared memory with coalesced loads, its largest logit updates
// the running max (online rescaling between batches), and then every lane
// group gathers value rows with 16-byte loads, many rows in flight per lane,
// weights them by exp(s - m) and accumulates in fp32.  The share's (m, sum of
// weights, count, row max, unnormalised output) goes to a partial record
// that the combine kernel merges.
#include "saga_device.cuh"
#include "saga_kernels.h"

namespace saga {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 2048;  // entries staged in shared memory at a time

template <int D>
__global__ void __launch_bounds__(kThreads, 3) gather_pv_kernel(const GatherArgs a) {
    constexpr int LPR = D * 2 / 16;    // lanes per value row (16 B each)
    constexpr int RPI = 32 / LPR;      // value rows per warp instruction
    constexpr int UNROLL = 8;
    constexpr int MBW = 128 / D;

    extern __shared__ int table[];     // pre[max_lists + 1], start[max_lists]
    __shared__ int ent_pos[kBatch];
    __shared__ float ent_s[kBatch];
    __shared__ float red_m[kWarps];
    __shared__ float red_l[kWarps];
    __shared__ float red_o[kWarps][D];
    __shared__ int red_i[kWarps];
    __shared__ long long row_base;

    const Geometry& g = a.g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long row = blockIdx.y;
    const int part = blockIdx.x;
    const int bb = static_cast<int>(row / g.hq);
    const int i = static_cast<int>(row - static_cast<long long>(bb) * g.hq);
    const int vh = i * g.hv / g.hq;
    int* pre = table;                       // exclusive prefix of list counts; pre[nl] = total
    int* start = table + a.max_lists + 1;   // list start inside the row's list region

    // ---- list table of the row
    float m_all = -kInf;
    int nl = 1;
    if (a.mode == kListContiguous) {
        if (tid == 0) {
            pre[0] = 0;
            pre[1] = min(max(__ldg(a.cnt + row), 0), g.l);
            start[0] = 0;
            row_base = row * g.l;
        }
        __syncthreads();
    } else {
        const long long T = static_cast<long long>(g.b) * g.tiles;
        const long long x0 = static_cast<long long>(bb) * g.tiles;
        const int c_first = cta_of_tile(x0, T, a.C);
        const int slots = cta_of_tile(x0 + g.tiles - 1, T, a.C) - c_first + 1;
        nl = slots * g.WPK;  // <= max_lists (checked by the host)
        const int per = (nl + kThreads - 1) / kThreads;
        const int j0 = min(nl, tid * per), j1 = min(nl, j0 + per);
        int run = 0;
        float mloc = -kInf;
        for (int j = j0; j < j1; ++j) {
            const int slot = j / g.WPK, u = j - slot * g.WPK;
            const int c = c_first + slot;
            const long long t0 = cta_tile_begin(T, a.C, c), t1 = cta_tile_begin(T, a.C, c + 1);
            const long long s0 = t0 > x0 ? t0 : x0;
            const long long s1 = t1 < x0 + g.tiles ? t1 : x0 + g.tiles;
            // a list never holds more entries than its warp's positions
            const int cap = static_cast<int>((s1 - s0) * MBW * 16);
            const size_t at = (static_cast<size_t>(row) * g.S_cap + slot) * g.WPK + u;
            const int cu = a.seg_cnt[at];
            start[j] = static_cast<int>((s0 - x0) * g.P +
                                        static_cast<long long>(u) * (s1 - s0) * MBW * 16);
            pre[j] = cu < 0 ? 0 : (cu > cap ? cap : cu);  // counts for now
            run += pre[j];
            mloc = fmaxf(mloc, a.seg_mall[at]);
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
    const int e0 = static_cast<int>(static_cast<long long>(total) * part / a.parts);
    const int e1 = static_cast<int>(static_cast<long long>(total) * (part + 1) / a.parts);
    const int n = e1 - e0;

    const int grp = lane / LPR, col0 = (lane % LPR) * 8;
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;
    float lsum = 0.f;
    float m = -kInf;
    const __nv_bfloat16* vbase = reinterpret_cast<const __nv_bfloat16*>(a.v) +
                                 (static_cast<size_t>(bb) * g.l_cap * g.hv + vh) * D + col0;
    const size_t vstride = static_cast<size_t>(g.hv) * D;
    constexpr int step = kWarps * RPI;

    // first list that holds entry e0
    int jl = 0;
    while (jl + 1 < nl && pre[jl + 1] <= e0) ++jl;

    for (int b0 = e0; b0 < e1; b0 += kBatch) {
        const int b1 = min(e1, b0 + kBatch);
        // ---- stage the batch's (position, logit) pairs, list by list
        float mloc = -kInf;
        for (int j = jl; j < nl && pre[j] < b1; ++j) {
            const int lo = max(b0, pre[j]), hi = min(b1, pre[j + 1]);
            const long long src = row_base + start[j] - pre[j];
            for (int e = lo + tid; e < hi; e += kThreads) {
                int pos;
                float s;
                if (a.mode == kListContiguous) {
                    pos = __ldg(a.idx + src + e);
                    s = __ldg(a.logits + row * g.l + pos);
                } else {
                    pos = __ldg(a.list_idx + src + e);
                    s = __ldg(a.list_s + src + e);
                }
                ent_pos[e - b0] = pos;
                ent_s[e - b0] = s;
                mloc = fmaxf(mloc, s);
            }
        }
        while (jl + 1 < nl && pre[jl + 1] <= b1) ++jl;
        mloc = warp_max(mloc);
        if (lane == 0) red_m[warp] = mloc;
        __syncthreads();
        float m_new = m;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) m_new = fmaxf(m_new, red_m[w]);
        const float alpha = m > -kInf ? __expf(m - m_new) : 0.f;
        lsum *= alpha;
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] *= alpha;
        m = m_new;

        // ---- gather the batch's value rows
        const int nb = b1 - b0;
        for (int e = warp * RPI + grp; e < nb; e += step * UNROLL) {
            uint4 raw[UNROLL];
            float p[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int eu = e + u * step;
                const bool ok = eu < nb;
                const int pos = ok ? ent_pos[eu] : 0;
                p[u] = ok ? __expf(ent_s[eu] - m) : 0.f;
                raw[u] = ok ? __ldg(reinterpret_cast<const uint4*>(vbase + pos * vstride))
                            : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                lsum += p[u];
                const uint32_t w4[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    acc[2 * c] = fmaf(p[u], bf16_lo(w4[c]), acc[2 * c]);
                    acc[2 * c + 1] = fmaf(p[u], bf16_hi(w4[c]), acc[2 * c + 1]);
                }
            }
        }
        __syncthreads();  // the next batch overwrites the staged entries
    }

    // every lane of a row group saw each of the group's weights: count once
    lsum = (lane % LPR == 0) ? lsum : 0.f;
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
        rec[3] = a.mode == kListContiguous ? (n > 0 ? m : -kInf) : m_all;
    }
}

}  // namespace

size_t gather_smem_bytes(int max_lists) {
    return (2 * static_cast<size_t>(max_lists) + 1) * sizeof(int);
}

cudaError_t launch_gather_pv(const GatherArgs& a, cudaStream_t stream) {
    const dim3 grid(a.parts, static_cast<unsigned>(static_cast<long long>(a.g.b) * a.g.hq));
    const size_t smem = gather_smem_bytes(a.max_lists);
    if (smem > static_cast<size_t>(kGatherMaxSmem)) return cudaErrorInvalidValue;
    if (a.g.d == 64) {
        static const cudaError_t attr = cudaFuncSetAttribute(
            gather_pv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGatherMaxSmem);
        if (attr != cudaSuccess) return attr;
        gather_pv_kernel<64><<<grid, kThreads, smem, stream>>>(a);
    } else {
        static const cudaError_t attr = cudaFuncSetAttribute(
            gather_pv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGatherMaxSmem);
        if (attr != cudaSuccess) return attr;
        gather_pv_kernel<128><<<grid, kThreads, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace saga
