// Kernels for a decode whose cached sequence is split into contiguous shards
// (one per rank): the exact threshold from per-shard digit histograms that
// the caller sums across ranks, and the merge of the per-shard partial
// records.
//
// Method: "More Value per Key" (ai.info summary, Key Contributions #2): the
// threshold is the exact N-th largest logit of the whole row, and the kept
// set is every entry at or above it.  Over shards both stay exact: a digit
// histogram of the whole row is the sum of the shards' histograms, so every
// rank takes the same radix digits as a single GPU would (same 11/11/10-bit
// digits of the same order-preserving key), and the softmax over the kept
// entries of all shards is the log-sum-exp merge of the shards' partial
// records (split-K / flash-decoding combine).  Empty-set reading as on one
// GPU: when nothing is kept anywhere, the row's maximal entries are.
#include "saga_device.cuh"
#include "saga_kernels.h"

namespace saga {

namespace {

constexpr int kThreads = 256;

template <int PASS>
struct Digit {
    static constexpr int shift = PASS == 0 ? 21 : (PASS == 1 ? 10 : 0);
    static constexpr int width = PASS == 2 ? 10 : 11;
    static constexpr int nb = 1 << width;
    static constexpr int high = (shift + width) & 31;  // bits above the digit
};

// Grid (chunks, rows): histogram of digit PASS over the keys of the chunk
// that carry the prefix fixed by the earlier passes, added to hist[row].
template <int PASS>
__global__ void __launch_bounds__(kThreads) shard_hist_kernel(const ShardHistArgs a) {
    using Dg = Digit<PASS>;
    __shared__ uint32_t h[Dg::nb];
    const long long row = blockIdx.y;
    for (int i = threadIdx.x; i < Dg::nb; i += kThreads) h[i] = 0u;
    __syncthreads();
    const uint32_t prefix = PASS == 0 ? 0u : a.state[row * 2];
    const bool done = PASS > 0 && a.state[row * 2 + 1] == 0u;  // threshold already known
    const int per = (a.l + a.chunks - 1) / a.chunks;
    const int j0 = blockIdx.x * per, j1 = min(a.l, j0 + per);
    const float* src = a.logits + row * a.l;
    if (!done)
        for (int j = j0 + threadIdx.x; j < j1; j += kThreads) {
            const uint32_t key = float_to_key(__ldg(src + j));
            if (PASS == 0 || (key >> Dg::high) == prefix) atomicAdd(&h[(key >> Dg::shift) & (Dg::nb - 1)], 1u);
        }
    __syncthreads();
    uint32_t* out = a.hist + row * kRadixBins;
    for (int i = threadIdx.x; i < Dg::nb; i += kThreads)
        if (h[i]) atomicAdd(out + i, h[i]);
}

// One CTA per row: the digit that holds rank `rank` counted from the top of
// the summed histogram.  State (prefix, rank) for the next pass, or the
// threshold after the last; rank 0 marks a row whose threshold is known.
template <int PASS>
__global__ void __launch_bounds__(kThreads) shard_digit_kernel(const ShardDigitArgs a) {
    using Dg = Digit<PASS>;
    constexpr int per_thread = Dg::nb / kThreads;
    __shared__ uint32_t warp_tot[kThreads / 32];
    const long long row = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t prefix = PASS == 0 ? 0u : a.state[row * 2];
    const uint32_t rank = PASS == 0 ? static_cast<uint32_t>(a.N) : a.state[row * 2 + 1];
    if (PASS > 0 && rank == 0u) return;
    const uint32_t* hist = a.hist + row * kRadixBins;
    uint32_t cnt[per_thread];
    uint32_t sum = 0;
    const int top = Dg::nb - tid * per_thread;  // exclusive upper bin of this thread
#pragma unroll
    for (int k = 0; k < per_thread; ++k) {
        cnt[k] = hist[top - 1 - k];  // descending bins
        sum += cnt[k];
    }
    // block-wide exclusive scan of the per-thread sums (descending bins)
    uint32_t inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    uint32_t before_w = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
        before_w += w < warp ? warp_tot[w] : 0u;
        total += warp_tot[w];
    }
    const uint32_t excl = before_w + inc - sum;
    if (PASS == 0 && static_cast<uint32_t>(a.N) >= total) {  // N >= l: every position is kept
        if (tid == 0) {
            a.thresh[row] = -kInf;
            a.state[row * 2] = 0u;
            a.state[row * 2 + 1] = 0u;
        }
        return;
    }
    if (excl < rank && rank <= excl + sum) {
        uint32_t before = excl;
        int digit = top - 1;
#pragma unroll
        for (int k = 0; k < per_thread; ++k) {
            if (before + cnt[k] >= rank) {
                digit = top - 1 - k;
                break;
            }
            before += cnt[k];
        }
        const uint32_t key = (prefix << Dg::width) | static_cast<uint32_t>(digit);
        if (PASS < kRadixPasses - 1) {
            a.state[row * 2] = key;
            a.state[row * 2 + 1] = rank - before;
        } else {
            a.thresh[row] = key_to_float(key);
            a.state[row * 2 + 1] = 0u;
        }
    }
}

// One warp per row: log-sum-exp merge of the R shards' partial records.
template <int DV>
__global__ void __launch_bounds__(kThreads) merge_parts_kernel(const MergeArgs a) {
    constexpr int CPL = DV / 32;
    const long long row = static_cast<long long>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= a.rows) return;
    const size_t rec = DV + kRecHeader;
    auto part = [&](int r) { return a.parts + (static_cast<size_t>(r) * a.rows + row) * rec; };
    long long total = 0;
    float M = -kInf, MX = -kInf;
    for (int r = 0; r < a.R; ++r) {
        const float* p = part(r);
        const int c = __float_as_int(p[2]);
        total += c;
        if (c > 0) M = fmaxf(M, p[0]);
        MX = fmaxf(MX, p[3]);
    }
    float o[CPL], den = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[c] = 0.f;
    long long at_max = 0;
    for (int r = 0; r < a.R; ++r) {
        const float* p = part(r);
        const int c = __float_as_int(p[2]);
        float w;
        if (total > 0) {
            if (c <= 0) continue;
            w = __expf(p[0] - M);  // the shard's softmax reference against the row's
        } else {
            if (!(p[3] == MX)) continue;  // nothing kept anywhere: the shards at the row max
            w = 1.f;
            at_max += static_cast<long long>(p[1]);
        }
        den = fmaf(w, p[1], den);
#pragma unroll
        for (int k = 0; k < CPL; ++k) o[k] = fmaf(w, p[kRecHeader + lane * CPL + k], o[k]);
    }
    const float inv = 1.f / den;
    float* dst = a.out + row * DV;
#pragma unroll
    for (int k = 0; k < CPL; ++k) dst[lane * CPL + k] = o[k] * inv;
    if (lane == 0 && a.sel_cnt) a.sel_cnt[row] = static_cast<int32_t>(total > 0 ? total : at_max);
}

}  // namespace

cudaError_t launch_shard_hist(int pass, const ShardHistArgs& a, cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>(a.chunks), static_cast<unsigned>(a.rows));
    cudaError_t e = cudaMemsetAsync(a.hist, 0, static_cast<size_t>(a.rows) * kRadixBins * sizeof(uint32_t), stream);
    if (e != cudaSuccess) return e;
    if (pass == 0) shard_hist_kernel<0><<<grid, kThreads, 0, stream>>>(a);
    else if (pass == 1) shard_hist_kernel<1><<<grid, kThreads, 0, stream>>>(a);
    else shard_hist_kernel<2><<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_shard_digit(int pass, const ShardDigitArgs& a, cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>(a.rows));
    if (pass == 0) shard_digit_kernel<0><<<grid, kThreads, 0, stream>>>(a);
    else if (pass == 1) shard_digit_kernel<1><<<grid, kThreads, 0, stream>>>(a);
    else shard_digit_kernel<2><<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_merge_parts(int dv, const MergeArgs& a, cudaStream_t stream) {
    const unsigned blocks = static_cast<unsigned>((a.rows + kThreads / 32 - 1) / (kThreads / 32));
    if (dv == 64) merge_parts_kernel<64><<<blocks, kThreads, 0, stream>>>(a);
    else if (dv == 128) merge_parts_kernel<128><<<blocks, kThreads, 0, stream>>>(a);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace saga
