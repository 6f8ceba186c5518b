// Compare + ordered compaction over stored logits (refresh steps, and any
// step whose logits the caller supplies).
//
// Method: "More Value per Key" (ai.info summary, Key Contributions #2,
// Methodology ¶2): the kept entries are found by a per-element comparison
// with the threshold, not by sorting.  Reading for the empty set (the pages
// are silent): tau_eff = min(tau, row max), i.e. when a stale threshold lies
// above every logit the row's maximal entries are kept.
//
// One CTA of 256 threads per (batch, query head) row.  A round covers
// 4 x 256 x VEC positions: each thread reads VEC consecutive logits per
// sub-round (16-byte loads when rows are 16-byte aligned; VEC = 16 when the
// rows are few, so that the few CTAs keep 64 KB of loads in flight between
// the round's barriers, VEC = 4 otherwise, which keeps four CTAs per SM and
// the whole grid in one wave), counts its kept
// ones, the counts are prefix-summed inside the warp (shuffles) and across
// the 8 warps x 4 sub-rounds (warp 0), and every kept position (and its
// logit, for the gather kernel) is written at its rank, so the output is
// ascending.  The row's largest logit is stored for the gather kernel's
// softmax.  If nothing passed (only possible when tau > row max) the row is
// compacted again against its max, unless keep_max is 0 (a sequence shard,
// whose empty-set rule belongs to the whole row).
#include "saga_device.cuh"
#include "saga_kernels.h"

namespace saga {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSub = 4;  // sub-rounds per round; kSub * kWarps == 32 counts per round

template <int VEC>
__global__ void __launch_bounds__(kThreads) select_compact_kernel(const SelectArgs a) {
    constexpr int kRound = kSub * kThreads * VEC;  // positions per round
    __shared__ int counts[kSub * kWarps];
    __shared__ int offsets[kSub * kWarps];
    __shared__ int round_total;
    __shared__ float red[kWarps];

    pdl_wait();  // the logits and thresholds come from earlier kernels
    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long row = blockIdx.x;
    const float* src = a.logits + row * a.l;
    int32_t* dst = a.idx + row * a.l;
    float* sdst = a.s + row * a.l;
    const float tau = __ldg(a.thresh + row);

    float tmax = -kInf;
    int total = 0;
    for (int pass = 0; pass < 2; ++pass) {
        float t_eff = tau;
        if (pass == 1) t_eff = red[0];  // only reached when nothing was kept: keep the max
        total = 0;
        for (int base = 0; base < a.l; base += kRound) {
            float v[kSub][VEC];
#pragma unroll
            for (int k = 0; k < kSub; ++k) {
                const int j = base + (k * kThreads + tid) * VEC;
                if (VEC >= 4 && j + VEC <= a.l) {
#pragma unroll
                    for (int h = 0; h < VEC / 4; ++h) {
                        const float4 x = __ldg(reinterpret_cast<const float4*>(src + j) + h);
                        v[k][4 * h] = x.x;
                        v[k][4 * h + 1] = x.y;
                        v[k][4 * h + 2] = x.z;
                        v[k][4 * h + 3] = x.w;
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < VEC; ++c) v[k][c] = j + c < a.l ? __ldg(src + j + c) : -kInf;
                }
            }
            uint32_t kb[kSub];
            int lane_off[kSub];
#pragma unroll
            for (int k = 0; k < kSub; ++k) {
                const int j = base + (k * kThreads + tid) * VEC;
                kb[k] = 0u;
#pragma unroll
                for (int c = 0; c < VEC; ++c) {
                    if (pass == 0) tmax = fmaxf(tmax, v[k][c]);
                    if (j + c < a.l && v[k][c] >= t_eff) kb[k] |= 1u << c;
                }
                const int mine = __popc(kb[k]);
                int inc = mine;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int x = __shfl_up_sync(0xffffffffu, inc, o);
                    if (lane >= o) inc += x;
                }
                lane_off[k] = inc - mine;
                if (lane == 31) counts[k * kWarps + warp] = inc;
            }
            __syncthreads();
            if (warp == 0) {
                // exclusive scan of the 32 counts in position order (k major, warp minor)
                const int c = counts[lane];
                int inc = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int x = __shfl_up_sync(0xffffffffu, inc, o);
                    if (lane >= o) inc += x;
                }
                offsets[lane] = inc - c;
                if (lane == 31) round_total = inc;
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < kSub; ++k) {
                if (!kb[k]) continue;
                int at = total + offsets[k * kWarps + warp] + lane_off[k];
                const int j = base + (k * kThreads + tid) * VEC;
#pragma unroll
                for (int c = 0; c < VEC; ++c) {
                    if (kb[k] & (1u << c)) {
                        dst[at] = j + c;
                        sdst[at] = v[k][c];
                        ++at;
                    }
                }
            }
            total += round_total;
            __syncthreads();
        }
        if (pass == 0) {
            tmax = warp_max(tmax);
            if (lane == 0) red[warp] = tmax;
            __syncthreads();
            if (tid == 0) {
                float m = red[0];
                for (int w = 1; w < kWarps; ++w) m = fmaxf(m, red[w]);
                red[0] = m;
                a.rowmax[row] = m;
            }
            __syncthreads();
        }
        if (total > 0 || !a.keep_max) break;
    }
    if (tid == 0) a.cnt[row] = total;
}

}  // namespace

cudaError_t launch_select_compact(const SelectArgs& a, cudaStream_t stream) {
    const bool vec = (a.l % 4 == 0) && ((reinterpret_cast<uintptr_t>(a.logits) & 15u) == 0);
    const dim3 grid(static_cast<unsigned>(a.rows)), block(kThreads);
    if (!vec) return launch_dependent(select_compact_kernel<1>, grid, block, 0, stream, a);
    return a.wide ? launch_dependent(select_compact_kernel<16>, grid, block, 0, stream, a)
                  : launch_dependent(select_compact_kernel<4>, grid, block, 0, stream, a);
}

}  // namespace saga
