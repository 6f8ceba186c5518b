// Compare + ordered compaction over stored logits (refresh steps, and any
// step whose logits the caller supplies).
//
// Method: "More Value per Key" (ai.info summary, Key Contributions #2,
// Methodology ¶2): the kept entries are found by a per-element comparison
// with the threshold, not by sorting.  Reading for the empty set (the pages
// are silent): tau_eff = min(tau, row max), i.e. when a stale threshold lies
// above every logit the row's maximal entries are kept.
//
// One CTA per (batch, query head) row.  Each round covers 16 x 256 positions:
// every warp ballots its 32 positions per sub-round, the 128 warp counts are
// prefix-summed by warp 0, and each kept lane writes its position at the
// scanned offset, so the output is ascending.  If nothing passed (only
// possible when tau > row max) the row is compacted again against its max.
#include "saga_device.cuh"
#include "saga_kernels.h"

namespace saga {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSub = 16;                    // sub-rounds per round
constexpr int kRound = kSub * kThreads;     // positions per round

__global__ void __launch_bounds__(kThreads) select_compact_kernel(const SelectArgs a) {
    __shared__ int counts[kSub * kWarps];
    __shared__ int offsets[kSub * kWarps];
    __shared__ int round_total;
    __shared__ float warp_max_s[kWarps];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long row = blockIdx.x;
    const float* src = a.logits + row * a.l;
    int32_t* dst = a.idx + row * a.l;
    const float tau = __ldg(a.thresh + row);
    constexpr float kNegInf = -kInf;

    float tmax = kNegInf;
    int total = 0;
    for (int pass = 0; pass < 2; ++pass) {
        float t_eff = tau;
        if (pass == 1) {
            // Only reached when nothing was kept: keep the row's maximum.
            tmax = warp_max(tmax);
            if (lane == 0) warp_max_s[warp] = tmax;
            __syncthreads();
            float m = warp_max_s[0];
            for (int w = 1; w < kWarps; ++w) m = fmaxf(m, warp_max_s[w]);
            t_eff = m;
        }
        total = 0;
        for (int base = 0; base < a.l; base += kRound) {
            float v[kSub];
#pragma unroll
            for (int k = 0; k < kSub; ++k) {
                const int j = base + k * kThreads + tid;
                v[k] = j < a.l ? __ldg(src + j) : kNegInf;
            }
            uint32_t ball[kSub];
#pragma unroll
            for (int k = 0; k < kSub; ++k) {
                const int j = base + k * kThreads + tid;
                if (pass == 0) tmax = fmaxf(tmax, v[k]);
                ball[k] = __ballot_sync(0xffffffffu, j < a.l && v[k] >= t_eff);
                if (lane == 0) counts[k * kWarps + warp] = __popc(ball[k]);
            }
            __syncthreads();
            if (warp == 0) {
                // exclusive scan of the 128 counts in position order (k major, warp minor)
                int c[4], s = 0;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    c[u] = counts[lane * 4 + u];
                    s += c[u];
                }
                int inc = s;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int n = __shfl_up_sync(0xffffffffu, inc, o);
                    if (lane >= o) inc += n;
                }
                int run = inc - s;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    offsets[lane * 4 + u] = run;
                    run += c[u];
                }
                if (lane == 31) round_total = inc;
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < kSub; ++k) {
                if (ball[k] & (1u << lane)) {
                    const int at = total + offsets[k * kWarps + warp] + __popc(ball[k] & lanemask_lt());
                    dst[at] = base + k * kThreads + tid;
                }
            }
            total += round_total;
            __syncthreads();
        }
        if (total > 0) break;
    }
    if (tid == 0) a.cnt[row] = total;
}

}  // namespace

cudaError_t launch_select_compact(const SelectArgs& a, cudaStream_t stream) {
    select_compact_kernel<<<static_cast<unsigned>(a.rows), kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace saga
