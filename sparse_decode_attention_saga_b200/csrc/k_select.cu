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
                    if ((kb[k] & (1u << c)) && in_bounds(at < a.l, a.err)) {
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
        if (tid == 0 && a.empty_rows) atomicAdd(a.empty_rows, 1u);  // the empty-set rule fires
    }
    if (tid == 0) a.cnt[row] = total;
}

// One CTA per row: clear the row's bitmap, set the bit of every listed
// position (a position is listed at most once per row), then each thread
// takes a contiguous run of bitmap words and writes their set positions at
// its offset from a block scan of the runs' counts, which yields the row's
// kept positions in ascending order.
__global__ void __launch_bounds__(kThreads) lists_to_index_kernel(const IndexArgs a) {
    __shared__ int warp_tot[kWarps];
    pdl_wait();  // the lists come from the fused kernel, two launches back
    const Geometry& g = a.g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long row = blockIdx.x;
    const int bb = static_cast<int>(row / g.hq);
    const long long T = static_cast<long long>(g.b) * g.tiles;
    const int nl = slots_of_batch(bb, g.tiles, T, a.C) * g.WPK;
    const int32_t* cnt = a.seg_cnt + static_cast<size_t>(row) * g.S_cap * g.WPK;
    auto clamped = [&](int j, SegList& sl) {
        sl = seg_list_of(g.P, g.MBW, g.WPK, g.tiles, bb, j, T, a.C);
        const int c = __ldg(cnt + j);
        in_bounds(c >= 0 && c <= sl.cap, a.err);
        return min(max(c, 0), sl.cap);
    };
    int mine = 0;
    for (int j = tid; j < nl; j += kThreads) {
        SegList sl;
        mine += clamped(j, sl);
    }
    mine = __reduce_add_sync(0xffffffffu, mine);
    if (lane == 0) warp_tot[warp] = mine;
    __syncthreads();
    int total = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) total += warp_tot[w];
    if (total == 0) return;  // the empty-set fallback of the row merge writes this row

    const int words = (g.l + 31) >> 5;
    uint32_t* bm = a.bitmap + static_cast<size_t>(row) * words;
    for (int w = tid; w < words; w += kThreads) bm[w] = 0u;
    __syncthreads();
    const int2* lists = a.seg_list + static_cast<size_t>(row) * g.l_pad;
    for (int j = warp; j < nl; j += kWarps) {
        SegList sl;
        const int n = clamped(j, sl);
        for (int e = lane; e < n; e += 32) {
            const int pos = __ldg(&lists[sl.start + e].x);
            if (in_bounds(pos >= 0 && pos < g.l, a.err)) atomicOr(bm + (pos >> 5), 1u << (pos & 31));
        }
    }
    __syncthreads();

    const int per = (words + kThreads - 1) / kThreads;
    const int w0 = min(words, tid * per), w1 = min(words, w0 + per);
    int c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(__ldcg(bm + w));
    int inc = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += x;
    }
    __syncthreads();
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    int at = inc - c;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) at += w < warp ? warp_tot[w] : 0;
    int32_t* dst = a.idx + static_cast<size_t>(row) * g.l;
    for (int w = w0; w < w1; ++w) {
        uint32_t bits = __ldcg(bm + w);
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1u;
            dst[at++] = (w << 5) + b;
        }
    }
}

// One CTA per row over the radix candidates.  With the radix state of the
// first two digits (a.state) the threshold's 22-bit prefix is known: one
// pass over the candidates sets the bit of every position above that bucket
// in a shared bitmap of the row (kept whatever the last digit), counts the
// bucket's candidates by their last 10 bits in a shared histogram and
// stashes them (a few per row); a block scan picks the bin holding the rank
// still sought, which completes the exact N-th largest logit (written to
// a.thresh; the third radix pass is not needed), and only the stashed
// candidates are compared with it.  Without the state the thresholds are
// given and every candidate is compared.  Then each thread takes a
// contiguous run of bitmap words, a block scan of the runs' counts gives
// every word's rank, and each kept candidate is written at its word's rank
// plus the set bits below it, so the output is ascending whatever order the
// candidates came in (a position is a candidate at most once).  The row's
// largest logit is the largest candidate.  Nothing kept (only when the
// threshold lies above every logit) keeps the row's maxima, as the
// compaction over stored logits does.
// Dynamic shared memory (cand_select_smem): bitmap [words] | word ranks [words].
constexpr int kCandThreads = 512;
constexpr int kCandWarps = kCandThreads / 32;
constexpr int kCandStash = 1024;

__device__ __forceinline__ uint32_t cand_block_scan(uint32_t v, uint32_t& excl, uint32_t* warp_tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += x;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    uint32_t before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kCandWarps; ++w) {
        before += w < warp ? warp_tot[w] : 0u;
        total += warp_tot[w];
    }
    excl = before + inc - v;
    return total;
}

__global__ void __launch_bounds__(kCandThreads) cand_select_kernel(const CandSelectArgs a) {
    extern __shared__ uint32_t bm[];
    __shared__ uint32_t warp_tot[kCandWarps];
    __shared__ float red[kCandWarps];
    __shared__ uint32_t hist[1024];
    __shared__ float s_tau;
    __shared__ int s_nstash;
    __shared__ int2 stash[kCandStash];  // the candidates of the threshold's 22-bit bucket
    pdl_wait();  // candidates and radix state (or thresholds) from the radix passes
    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long row = blockIdx.x;
    const int words = (a.l + 31) >> 5;
    uint32_t* wrank = bm + words;
    const int per = radix_chunk_len(a.l, a.chunks);
    const int2* cand = a.cand + row * a.l;
    const int32_t* ccnt = a.cand_cnt + row * kRadixMaxChunks;
    // every candidate of the row, chunk by chunk: fn(position, logit), four
    // independent loads per thread in flight
    auto each = [&](auto fn) {
        for (int c = 0; c < a.chunks; ++c) {
            const int nc = __ldcg(ccnt + c);
            in_bounds(nc >= 0 && nc <= per, a.err);
            const int n = min(max(nc, 0), per);
            const int2* cs = cand + static_cast<long long>(c) * per;
            for (int e0 = 0; e0 < n; e0 += 4 * kCandThreads) {
                int2 p[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = e0 + u * kCandThreads + tid;
                    p[u] = e < n ? __ldcg(cs + e) : make_int2(-1, 0);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (e0 + u * kCandThreads + tid < n && in_bounds(p[u].x >= 0 && p[u].x < a.l, a.err))
                        fn(p[u].x, __int_as_float(p[u].y));
            }
        }
    };

    // Kept bits: with the radix state the row's 22-bit threshold prefix is
    // known, so one pass sets the bit of every candidate above that bucket
    // (kept whatever the last digit), counts the bucket's candidates by their
    // last 10 bits and stashes them; the digit holding the rank gives the
    // threshold, and only the stashed ones are compared with it (a second
    // pass over the candidates only when the bucket overflows the stash).
    float tau;
    float m = -kInf;
    for (int w = tid; w < words; w += kCandThreads) bm[w] = 0u;
    if (a.state) {
        for (int i = tid; i < 1024; i += kCandThreads) hist[i] = 0u;
        if (tid == 0) s_nstash = 0;
    }
    __syncthreads();
    if (a.state) {
        const uint32_t prefix = __ldcg(a.state + row * 2), rank = __ldcg(a.state + row * 2 + 1);
        each([&](int pos, float x) {
            m = fmaxf(m, x);
            const uint32_t key = float_to_key(x);
            if ((key >> 10) > prefix) {
                atomicOr(bm + (pos >> 5), 1u << (pos & 31));
            } else if ((key >> 10) == prefix) {
                atomicAdd(&hist[key & 1023u], 1u);
                const int at = atomicAdd(&s_nstash, 1);
                if (at < kCandStash) stash[at] = make_int2(pos, __float_as_int(x));
            }
        });
        // (the bucket's lower edge stands if no bin holds the rank, which the
        // radix state of finite logits rules out)
        if (tid == 0) s_tau = key_to_float(prefix << 10);
        __syncthreads();
        constexpr int kPer = 1024 / kCandThreads;  // bins per thread, from the top
        const int top = 1024 - tid * kPer;
        uint32_t cnt[kPer], sum = 0;
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            cnt[k] = hist[top - 1 - k];
            sum += cnt[k];
        }
        uint32_t excl;
        cand_block_scan(sum, excl, warp_tot);
        if (excl < rank && rank <= excl + sum) {
            uint32_t before = excl;
            int digit = top - 1;
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                if (before + cnt[k] >= rank) {
                    digit = top - 1 - k;
                    break;
                }
                before += cnt[k];
            }
            const float t = key_to_float((prefix << 10) | static_cast<uint32_t>(digit));
            s_tau = t;
            a.thresh[row] = t;
        }
        __syncthreads();
        tau = s_tau;
        const int nst = s_nstash;
        if (nst <= kCandStash) {
            for (int i = tid; i < nst; i += kCandThreads) {
                const int2 p = stash[i];
                if (__int_as_float(p.y) >= tau) atomicOr(bm + (p.x >> 5), 1u << (p.x & 31));
            }
        } else {
            each([&](int pos, float x) {
                if ((float_to_key(x) >> 10) == prefix && x >= tau) atomicOr(bm + (pos >> 5), 1u << (pos & 31));
            });
        }
    } else {
        tau = __ldg(a.thresh + row);
        each([&](int pos, float x) {
            m = fmaxf(m, x);
            if (x >= tau) atomicOr(bm + (pos >> 5), 1u << (pos & 31));
        });
    }
    m = warp_max(m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = red[0];
#pragma unroll
    for (int w = 1; w < kCandWarps; ++w) m = fmaxf(m, red[w]);

    // word ranks; nothing kept (only when the threshold lies above every
    // logit) keeps the row's maxima, as the compaction over stored logits does
    const int run = (words + kCandThreads - 1) / kCandThreads;
    const int w0 = min(words, tid * run), w1 = min(words, w0 + run);
    uint32_t total = 0;
    for (int pass = 0; pass < 2; ++pass) {
        uint32_t c = 0;
        for (int w = w0; w < w1; ++w) c += __popc(bm[w]);
        uint32_t at;
        total = cand_block_scan(c, at, warp_tot);
        for (int w = w0; w < w1; ++w) {
            wrank[w] = at;
            at += __popc(bm[w]);
        }
        if (total > 0 || pass == 1) break;
        if (tid == 0 && a.empty_rows) atomicAdd(a.empty_rows, 1u);
        __syncthreads();
        each([&](int pos, float x) {
            if (x >= m) atomicOr(bm + (pos >> 5), 1u << (pos & 31));
        });
        __syncthreads();
    }
    __syncthreads();
    int32_t* dst = a.idx + row * a.l;
    float* sdst = a.s + row * a.l;
    each([&](int pos, float x) {
        const int w = pos >> 5;
        const uint32_t bits = bm[w], bit = 1u << (pos & 31);
        if (!(bits & bit)) return;
        const uint32_t r = wrank[w] + __popc(bits & (bit - 1u));
        dst[r] = pos;
        sdst[r] = x;
    });
    if (tid == 0) {
        a.cnt[row] = static_cast<int32_t>(total);
        a.rowmax[row] = m;
    }
}

}  // namespace

size_t cand_select_smem(int l) { return 2 * ((static_cast<size_t>(l) + 31) / 32) * sizeof(uint32_t); }

cudaError_t launch_cand_select(const CandSelectArgs& a, cudaStream_t stream) {
    const size_t smem = cand_select_smem(a.l);
    const cudaError_t e = allow_dynamic_smem(cand_select_kernel, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return launch_dependent(cand_select_kernel, dim3(static_cast<unsigned>(a.rows)), dim3(kCandThreads),
                            smem, stream, a);
}

cudaError_t launch_lists_to_index(const IndexArgs& a, cudaStream_t stream) {
    const long long rows = static_cast<long long>(a.g.b) * a.g.hq;
    return launch_dependent(lists_to_index_kernel, dim3(static_cast<unsigned>(rows)), dim3(kThreads), 0,
                            stream, a);
}

cudaError_t launch_select_compact(const SelectArgs& a, cudaStream_t stream) {
    const bool vec = (a.l % 4 == 0) && ((reinterpret_cast<uintptr_t>(a.logits) & 15u) == 0);
    const dim3 grid(static_cast<unsigned>(a.rows)), block(kThreads);
    if (!vec) return launch_dependent(select_compact_kernel<1>, grid, block, 0, stream, a);
    return a.wide ? launch_dependent(select_compact_kernel<16>, grid, block, 0, stream, a)
                  : launch_dependent(select_compact_kernel<4>, grid, block, 0, stream, a);
}

}  // namespace saga
