// Exact threshold refresh: the N-th largest logit of every (batch, query
// head) row, counting duplicates.
//
// Method: "More Value per Key" (ai.info summary, Key Contributions #2): Atop-N
// finds the exact N-th largest logit only on every n-th token and reuses
// that threshold on the tokens in between.  The pages do
// not say how the exact threshold is found; this is an MSB-first radix select
// on order-preserving 32-bit keys (digits of 11, 11 and 10 bits), which is
// exact and needs no sort.
//
// Pass p, grid (chunks, rows): each CTA histograms the digit of the keys of
// its chunk that match the prefix fixed by the earlier passes (shared-memory
// atomics), adds its histogram to the row's global one,
// and takes a ticket; the CTA that takes the last ticket scans the histogram
// from the top bin, fixes the digit that holds the rank, and stores
// (prefix, rank) for the next pass, or the threshold after the last pass.
// No CTA waits for another.  With a candidate buffer, pass 1 also copies the
// (position, logit) of every key at or above the lower edge of pass 0's
// bucket into its chunk's part of the buffer (each warp lists a round's
// members in shared memory and stores them together at a place reserved
// from a per-CTA counter; the order inside a chunk is not fixed), and pass 2
// reads only those candidates, each CTA its own chunk's.  The kept set
// (logit >= threshold) lies among them, so a refresh step stops after pass
// 1 and one kernel finds the last digit and compacts the kept entries from
// the candidates alone (k_select.cu).
#include <type_traits>

#include "saga_device.cuh"
#include "saga_kernels.h"

namespace saga {

namespace {

constexpr int kThreads = 256;
constexpr int kWarpsR = kThreads / 32;
constexpr int kLoads = 16;
constexpr int kMemberBuf = 64;  // pass 1: members a warp lists at a time

// Block-wide exclusive scan of one value per thread; returns the block total.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t& excl,
                                                         uint32_t* warp_tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    uint32_t before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
        const uint32_t x = warp_tot[w];
        before += (w < warp) ? x : 0u;
        total += x;
    }
    excl = before + inc - v;
    return total;
}

// Eight CTAs per SM on the vectorised path: the grid sizing (radix_chunks)
// counts on them (the scalar path keeps its registers).
template <int PASS, int VEC>
__global__ void __launch_bounds__(kThreads, VEC == 4 ? 8 : 4) radix_pass_kernel(const RadixArgs a) {
    constexpr int kLoadsV = kLoads / VEC;        // VEC-wide loads per thread per round
    constexpr int kRound = kLoads * kThreads;    // positions per round
    constexpr int shift = PASS == 0 ? 21 : (PASS == 1 ? 10 : 0);
    constexpr int width = PASS == 2 ? 10 : 11;
    constexpr int nb = 1 << width;
    constexpr int per_thread = nb / kThreads;
    constexpr int high = (shift + width) & 31;  // bits above this digit (unused in pass 0)

    __shared__ uint32_t hist[nb];
    __shared__ uint32_t warp_tot[kThreads / 32];
    __shared__ int is_last;
    __shared__ int s_cand;  // pass 1: candidates this CTA has copied out
    // pass 1: each warp's members of the round (positions), kMemberBuf at a time
    __shared__ int s_members[PASS == 1 ? kWarpsR * kMemberBuf : 1];

    pdl_wait();  // logits, histograms and the previous pass's state
    pdl_trigger();
    const int tid = threadIdx.x;
    const long long row = blockIdx.y;
    const int chunk = blockIdx.x;
    for (int i = tid; i < nb; i += kThreads) hist[i] = 0;
    if (tid == 0) s_cand = 0;
    const uint32_t prefix = PASS == 0 ? 0u : __ldcg(a.state + row * 2);
    __syncthreads();
    const bool from_cand = PASS == 2 && a.cand != nullptr;
    const int lane = tid & 31, warp = tid >> 5;

    const float* src = a.logits + row * a.l;
    const int per = radix_chunk_len(a.l, a.chunks);
    const int j0 = from_cand ? 0 : chunk * per;
    const int j1 = from_cand ? 0 : min(a.l, j0 + per);
    int2* cdst = PASS == 1 && a.cand ? a.cand + row * a.l + static_cast<long long>(chunk) * per : nullptr;
    // pass 1 copies out every logit at or above the lower edge of pass 0's
    // bucket: the bucket's members (pass 2 reads them) and every larger
    // one, so that the kept set (logit >= threshold) lies among them.
    // The test is a float compare against the bucket's lower edge (the
    // order of the keys is the order of the floats), so that the key is
    // computed for members only.  The lowest buckets (-inf and negative
    // NaNs) have a NaN for an edge: every logit is a member then, a superset
    // that pass 2 and the compaction filter.  (Logits are finite: a NaN
    // would take its key's place in pass 0 but not in this compare.)
    const float lo_f = key_to_float(prefix << 21);
    const bool all_members = isnan(lo_f);
    // 64 bytes of independent coalesced loads per thread per round (16-byte
    // loads when the rows are 16-byte aligned) keep enough bytes in flight to
    // stream the logits at HBM speed; whole rounds skip the bounds checks.
    auto round = [&](int base, auto whole) {
        constexpr bool kWhole = decltype(whole)::value;
        float v[kLoadsV][VEC];
#pragma unroll
        for (int k = 0; k < kLoadsV; ++k) {
            const int j = base + (k * kThreads + tid) * VEC;
            if (VEC == 4 && (kWhole || j + VEC <= j1)) {
                const float4 x = __ldg(reinterpret_cast<const float4*>(src + j));
                const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int c = 0; c < VEC; ++c) v[k][c] = xs[c];
            } else {
#pragma unroll
                for (int c = 0; c < VEC; ++c) v[k][c] = kWhole || j + c < j1 ? __ldg(src + j + c) : 0.f;
            }
        }
        if constexpr (PASS == 1) {
            // Members are a few percent of the logits: a bitmask of this
            // thread's members (branch-free) first.
            uint32_t m = 0u;
#pragma unroll
            for (int k = 0; k < kLoadsV; ++k)
#pragma unroll
                for (int c = 0; c < VEC; ++c) {
                    const int j = base + (k * kThreads + tid) * VEC + c;
                    const bool in = (kWhole || j < j1) && (v[k][c] >= lo_f || all_members);
                    m |= static_cast<uint32_t>(in) << (k * VEC + c);
                }
            // The warp's members of the round in one list (a warp scan of the
            // per-thread counts; positions only), then one pass of the warp's
            // lanes over the list: each member's logit read again (L2), its
            // key into the histogram, and the candidates stored together.
            const int cnt_t = __popc(m);
            int incl = cnt_t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int x = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += x;
            }
            const int wtot = __shfl_sync(0xffffffffu, incl, 31);
            if (wtot) {
                int* wbuf = s_members + warp * kMemberBuf;
                int wbase = 0;
                if (cdst && lane == 0) wbase = atomicAdd(&s_cand, wtot);
                wbase = __shfl_sync(0xffffffffu, wbase, 0);
                // (more members than the buffer holds: several batches)
                for (int b0 = 0; b0 < wtot; b0 += kMemberBuf) {
                    int at = incl - cnt_t;
                    for (uint32_t mm = m; mm; mm &= mm - 1u, ++at) {
                        const int e = __ffs(mm) - 1;
                        if (at >= b0 && at < b0 + kMemberBuf)
                            wbuf[at - b0] = base + ((e / VEC) * kThreads + tid) * VEC + e % VEC;
                    }
                    __syncwarp();
                    const int nbatch = min(kMemberBuf, wtot - b0);
                    for (int i = lane; i < nbatch; i += 32) {
                        const int j = wbuf[i];
                        const float x = __ldg(src + j);
                        const uint32_t key = float_to_key(x);
                        if ((key >> high) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
                        if (cdst) cdst[wbase + b0 + i] = make_int2(j, __float_as_int(x));
                    }
                    __syncwarp();
                }
            }
        } else {
#pragma unroll
            for (int k = 0; k < kLoadsV; ++k)
#pragma unroll
                for (int c = 0; c < VEC; ++c) {
                    const int j = base + (k * kThreads + tid) * VEC + c;
                    if (kWhole || j < j1) {
                        const uint32_t key = float_to_key(v[k][c]);
                        if (PASS == 0) {
                            atomicAdd(&hist[key >> shift], 1u);
                        } else if ((key >> high) == prefix) {
                            atomicAdd(&hist[key & (nb - 1)], 1u);
                        }
                    }
                }
        }
    };
    if (!from_cand) {
        int base = j0;
        for (; base + kRound <= j1; base += kRound) round(base, std::true_type{});
        if (base < j1) round(base, std::false_type{});
    } else {
        // pass 2 over the candidates pass 1 copied out of this chunk
        const int nc = __ldcg(a.cand_cnt + row * kRadixMaxChunks + chunk);
        in_bounds(nc >= 0 && nc <= per, a.err);
        const int n = min(max(nc, 0), per);
        const int2* cs = a.cand + row * a.l + static_cast<long long>(chunk) * per;
        for (int j = tid; j < n; j += kThreads) {
            const uint32_t key = float_to_key(__int_as_float(__ldcg(cs + j).y));
            if ((key >> high) == prefix) atomicAdd(&hist[key & (nb - 1)], 1u);
        }
    }
    __syncthreads();
    if (PASS == 1 && cdst && tid == 0) a.cand_cnt[row * kRadixMaxChunks + chunk] = s_cand;

    uint32_t* ghist = a.hist + (static_cast<long long>(PASS) * a.rows + row) * kRadixBins;
    for (int i = tid; i < nb; i += kThreads)
        if (hist[i]) atomicAdd(ghist + i, hist[i]);
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(a.tickets + row, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    // Last CTA of the row: find the bin holding rank `rank` counted from the
    // top.  Thread tid owns bins [nb - (tid+1)*per_thread, nb - tid*per_thread).
    const uint32_t rank = PASS == 0 ? static_cast<uint32_t>(a.N) : __ldcg(a.state + row * 2 + 1);
    uint32_t cnt[per_thread];
    uint32_t sum = 0;
    const int top = nb - tid * per_thread;  // exclusive upper bin of this thread
#pragma unroll
    for (int k = 0; k < per_thread; ++k) {
        cnt[k] = __ldcg(ghist + top - 1 - k);  // descending bins
        sum += cnt[k];
    }
    uint32_t excl;
    block_exclusive_scan(sum, excl, warp_tot);
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
        const uint32_t new_prefix = (prefix << width) | static_cast<uint32_t>(digit);
        if (PASS < kRadixPasses - 1) {
            a.state[row * 2] = new_prefix;
            a.state[row * 2 + 1] = rank - before;
        } else {
            a.thresh[row] = key_to_float(new_prefix);
        }
    }
    if (tid == 0) a.tickets[row] = 0u;
}

__global__ void fill_kernel(float* p, long long n, float value) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x)
        p[i] = value;
}

}  // namespace

cudaError_t launch_radix_select(const RadixArgs& a, cudaStream_t stream) {
    const dim3 grid(a.chunks, static_cast<unsigned>(a.rows));
    const bool vec = (a.l % 4 == 0) && ((reinterpret_cast<uintptr_t>(a.logits) & 15u) == 0);
    const dim3 block(kThreads);
    // pass 0 follows the histogram clear (an ordinary launch); passes 1 and 2
    // may be scheduled while the pass before them drains
    if (vec) {
        radix_pass_kernel<0, 4><<<grid, block, 0, stream>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e == cudaSuccess) e = launch_dependent(radix_pass_kernel<1, 4>, grid, block, 0, stream, a);
        if (e == cudaSuccess && a.passes > 2)
            e = launch_dependent(radix_pass_kernel<2, 4>, grid, block, 0, stream, a);
        return e;
    }
    radix_pass_kernel<0, 1><<<grid, block, 0, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = launch_dependent(radix_pass_kernel<1, 1>, grid, block, 0, stream, a);
    if (e == cudaSuccess && a.passes > 2)
        e = launch_dependent(radix_pass_kernel<2, 1>, grid, block, 0, stream, a);
    return e;
}

cudaError_t launch_fill(float* p, long long n, float value, cudaStream_t stream) {
    const int blocks = static_cast<int>((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
    fill_kernel<<<blocks > 0 ? blocks : 1, 256, 0, stream>>>(p, n, value);
    return cudaGetLastError();
}

}  // namespace saga
