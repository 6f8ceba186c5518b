// Streaming query-key kernel over the K cache.
//
// Method: "More Value per Key" (ai.info summary).  Main Findings, "Bottleneck
// shift": once the probability-value product is sparse, the query-key
// product over every cached position is the dominant cost, so this kernel is
// built to stream K at HBM speed.  Key Contributions #2 / Methodology ¶2:
// selection is a per-element comparison against the stored thresholds, not a
// sort.
//
// One CTA owns a contiguous range of (batch, 32 KB tile) units.  Warp 8 is
// the producer: it issues one TMA box per (key head, 64-dim half) into a
// multi-stage shared-memory ring (full/empty mbarriers).  Warps 0-7 consume:
// warp w handles key head w / (8/h_k) and a fixed slice of each tile's
// positions, computing the logits of all G query heads of that key head on
// tensor cores (qk_tile.cuh), then
//   kStreamLogits: stores them to the logits array (refresh steps), or
//   kStreamSelect: compares them with the per-(batch, query head) thresholds,
//     appends the kept (position, logit) pairs to per-(row, CTA slot, warp)
//     lists (offsets from a shuffle scan over the lanes sharing a head), and
//     records the count and the maximum logit seen (for the empty-set
//     fallback).
// Logits never reach device memory on the select path.
#include "qk_tile.cuh"
#include "saga_kernels.h"

#ifndef SAGA_STREAM_K_HINT
#define SAGA_STREAM_K_HINT 1
#endif

namespace saga {

namespace {

template <int D, int NT, int MODE>
__global__ void __launch_bounds__(kStreamThreads, 2)
    qk_stream_kernel(const __grid_constant__ CUtensorMap kmap, const StreamArgs a) {
    constexpr int MBW = 128 / D;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const int stages = a.stages;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(stages) * kStageBytes);
    uint64_t* empty = full + stages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);

    const Geometry& g = a.g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    pdl_trigger();  // the gather kernel may be scheduled behind this grid

    const long long T = static_cast<long long>(g.b) * g.tiles;
    const int C = a.C, c = blockIdx.x;
    const long long t0 = cta_tile_begin(T, C, c), t1 = cta_tile_begin(T, C, c + 1);
    const int ntile = static_cast<int>(t1 - t0);
    const uint32_t stage0 = smem_addr(smem);

    if (warp == kConsumerWarps) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensor_map(&kmap);
            // K is read once per step: its lines go first, so that the kept
            // lists and logits written meanwhile stay in L2 for the next kernel
            const uint64_t k_policy = l2_policy_evict_first();
            (void)k_policy;
            int issued = 0;
            int bb = static_cast<int>(t0 / g.tiles);
            int tl = static_cast<int>(t0 - static_cast<long long>(bb) * g.tiles);
            int st = 0;
            uint32_t phase = 0;
            for (int k = 0; k < ntile; ++k) {
                if (!mbar_wait(&empty[st], phase ^ 1, abort_flag)) break;
                const int z = bb * g.l_cap + tl * g.P;
                mbar_arrive_expect_tx(&full[st], kStageBytes);
                uint8_t* dst = smem + static_cast<size_t>(st) * kStageBytes;
                for (int kh = 0; kh < g.hk; ++kh)
                    for (int dh = 0; dh < KTile<D>::NBOX; ++dh)
#if SAGA_STREAM_K_HINT
                        tma_load_3d_hint(dst + (kh * KTile<D>::NBOX + dh) * g.P * KTile<D>::ROWB,
                                         &kmap, &full[st], dh * 64, kh, z, k_policy);
#else
                        tma_load_3d(dst + (kh * KTile<D>::NBOX + dh) * g.P * KTile<D>::ROWB,
                                    &kmap, &full[st], dh * 64, kh, z);
#endif
                issued = k + 1;
                if (++tl == g.tiles) {
                    tl = 0;
                    ++bb;
                }
                if (++st == stages) {
                    st = 0;
                    phase ^= 1;
                }
            }
            // Drain: the last load armed on each stage must land before exit.
            int dummy = 0;
            for (int k = (issued > stages ? issued - stages : 0); k < issued; ++k)
                if (!mbar_wait(&full[k % stages], (k / stages) & 1, &dummy))
                    raise_device_error(a.err, kErrTimeout);
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    const int kh = warp / g.WPK, sub = warp % g.WPK;
    const int mb0 = sub * MBW;
    const int gq = lane >> 2, tq = lane & 3;
    const int G = g.G;
    const float scale = g.scale;

    QFrag<D, NT> qf;
    float tau[NT][2], mall[NT][2];
    int cnt[NT][2];
    int2* lst[NT][2];  // this warp's kept (position, logit) list of each head column
    int cur_bb = -1, slot = 0;
    long long sub_base = 0;

    auto begin_segment = [&](int bb) {
        load_q_frag<D, NT>(qf, reinterpret_cast<const __nv_bfloat16*>(a.q), g.hq, G, bb, kh, lane);
        if (MODE == kStreamSelect) {
            const long long x0 = static_cast<long long>(bb) * g.tiles;
            const long long s0 = t0 > x0 ? t0 : x0;
            const long long s1 = t1 < x0 + g.tiles ? t1 : x0 + g.tiles;
            slot = c - cta_of_tile(x0, T, C);
            sub_base = (s0 - x0) * g.P + static_cast<long long>(sub) * (s1 - s0) * MBW * 16;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int hl = nt * 8 + 2 * tq + e;
                    const int hc = hl < G ? hl : 0;
                    const size_t row = static_cast<size_t>(bb) * g.hq + kh * G + hc;
                    tau[nt][e] = hl < G ? raw_threshold(__ldg(a.thresh + row), scale) : kInf;
                    mall[nt][e] = -kInf;
                    cnt[nt][e] = 0;
                    lst[nt][e] = a.list + row * g.l_pad + sub_base;
                }
        }
    };

    auto end_segment = [&](int bb) {
        if constexpr (MODE == kStreamSelect) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float m = mall[nt][e];  // raw accumulator max; scaling is monotone
                    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
                    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
                    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
                    m = __fmul_rn(m, scale);
                    const int hl = nt * 8 + 2 * tq + e;
                    if (gq == 0 && hl < G) {
                        const size_t row = static_cast<size_t>(bb) * g.hq + kh * G + hl;
                        const size_t at = (row * g.S_cap + slot) * g.WPK + sub;
                        a.seg_cnt[at] = cnt[nt][e];
                        a.seg_mall[at] = m;
                    }
                }
        }
        (void)bb;
    };

    // Tile epilogue: logits store, or compare + list append, for the tile
    // whose (unscaled) accumulators are x, in the current segment.
    auto epilogue = [&](float (&x)[MBW][NT][4], int tl_e) {
            const int pos0 = tl_e * g.P + mb0 * 16 + gq;
            const bool full_tile = (tl_e + 1) * g.P <= g.l;  // every position of the tile is valid
            if (MODE == kStreamLogits) {
#pragma unroll
                for (int mbi = 0; mbi < MBW; ++mbi)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int pos = pos0 + mbi * 16 + 8 * h;
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int hl = nt * 8 + 2 * tq + e;
                                if ((full_tile || pos < g.l) && hl < G)
                                    a.logits[(static_cast<size_t>(cur_bb) * g.hq + kh * G + hl) * g.l + pos] =
                                        __fmul_rn(x[mbi][nt][2 * h + e], scale);
                            }
                    }
            } else {
                // Per n-tile: a bitmask of this thread's kept values (2 heads x
                // 2*MBW positions), then one segmented scan over the 8 lanes that
                // share each head (lanes tq, tq+4, ...) gives every thread its
                // offset in the (row, slot, warp) lists; both heads' counts travel
                // packed in one word.  The list order is (tile, lane, value):
                // deterministic, which is all the gather kernel needs.
                constexpr int HB = 2 * MBW;  // values per head per thread and tile
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    uint32_t km = 0u;
#pragma unroll
                    for (int mbi = 0; mbi < MBW; ++mbi)
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int pos = pos0 + mbi * 16 + 8 * h;
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                // raw compare (tau holds the raw threshold); head
                                // columns past G have tau = +inf and are never
                                // reported, so only the position needs checking
                                const float v = x[mbi][nt][2 * h + e];
                                if (full_tile || pos < g.l) {
                                    mall[nt][e] = fmaxf(mall[nt][e], v);
                                    if (v >= tau[nt][e]) km |= 1u << (e * HB + mbi * 2 + h);
                                }
                            }
                        }
                    if (__any_sync(0xffffffffu, km != 0u)) {
                        const uint32_t mine = static_cast<uint32_t>(__popc(km & ((1u << HB) - 1u))) |
                                              (static_cast<uint32_t>(__popc(km >> HB)) << 16);
                        uint32_t inc = mine;
#pragma unroll
                        for (int d = 4; d < 32; d <<= 1) {
                            const uint32_t x = __shfl_up_sync(0xffffffffu, inc, d);
                            if (lane >= d) inc += x;
                        }
                        const uint32_t tot = __shfl_sync(0xffffffffu, inc, 28 + tq);
                        if (km) {
                            const uint32_t excl = inc - mine;
                            int o0 = cnt[nt][0] + static_cast<int>(excl & 0xffffu);
                            int o1 = cnt[nt][1] + static_cast<int>(excl >> 16);
#pragma unroll
                            for (int mbi = 0; mbi < MBW; ++mbi)
#pragma unroll
                                for (int h = 0; h < 2; ++h) {
                                    const int pos = pos0 + mbi * 16 + 8 * h;
                                    if (km & (1u << (mbi * 2 + h))) {
                                        lst[nt][0][o0] = make_int2(
                                            pos, __float_as_int(__fmul_rn(x[mbi][nt][2 * h], scale)));
                                        ++o0;
                                    }
                                    if (km & (1u << (HB + mbi * 2 + h))) {
                                        lst[nt][1][o1] = make_int2(
                                            pos, __float_as_int(__fmul_rn(x[mbi][nt][2 * h + 1], scale)));
                                        ++o1;
                                    }
                                }
                        }
                        cnt[nt][0] += static_cast<int>(tot & 0xffffu);
                        cnt[nt][1] += static_cast<int>(tot >> 16);
                    }
                }
            }
    };

    // Software pipeline: tile k's mma runs (and its stage is released) before
    // tile k-1's epilogue, so a stage is handed back as soon as its data has
    // been read and the epilogue never delays the ring.
    bool ok = true;
    int bb = static_cast<int>(t0 / g.tiles);
    int tl = static_cast<int>(t0 - static_cast<long long>(bb) * g.tiles);
    int st = 0;
    uint32_t phase = 0;
    float acc_prev[MBW][NT][4];
    int tl_prev = 0;
    bool have_prev = false;
    for (int k = 0; k < ntile; ++k) {
        if (bb != cur_bb) {
            if (have_prev) epilogue(acc_prev, tl_prev);
            have_prev = false;
            if (cur_bb >= 0) end_segment(cur_bb);
            begin_segment(bb);
            cur_bb = bb;
        }
        const bool got = mbar_wait(&full[st], phase, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
        }
        float acc[MBW][NT][4];
        qk_mma<D, NT, MBW>(stage0 + st * kStageBytes, g.P, kh, mb0, qf, acc, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
        if (++st == stages) {
            st = 0;
            phase ^= 1;
        }
        if (have_prev) epilogue(acc_prev, tl_prev);
#pragma unroll
        for (int mbi = 0; mbi < MBW; ++mbi)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc_prev[mbi][nt][e] = acc[mbi][nt][e];
        tl_prev = tl;
        have_prev = true;
        if (++tl == g.tiles) {
            tl = 0;
            ++bb;
        }
    }
    if (have_prev && ok) epilogue(acc_prev, tl_prev);
    if (cur_bb >= 0) end_segment(cur_bb);
    if (!ok && lane == 0) raise_device_error(a.err, kErrTimeout);
}

template <int D, int NT, int MODE>
cudaError_t launch_t(const CUtensorMap& kmap, const StreamArgs& a, cudaStream_t stream) {
    const size_t smem = stream_smem_bytes(a.stages);
    auto kern = qk_stream_kernel<D, NT, MODE>;
    const cudaError_t attr = allow_dynamic_smem(kern, kMaxDynamicSmem);
    if (attr != cudaSuccess) return attr;
    kern<<<a.C, kStreamThreads, smem, stream>>>(kmap, a);
    return cudaGetLastError();
}

}  // namespace

size_t stream_smem_bytes(int stages) {
    return 1024 + static_cast<size_t>(stages) * kStageBytes + 2 * stages * sizeof(uint64_t) + 16;
}

cudaError_t launch_qk_stream(int mode, const CUtensorMap& kmap, const StreamArgs& a,
                             cudaStream_t stream) {
    const int d = a.g.d, nt = a.g.NT;
#define SAGA_QK_CASE(D_, NT_)                                                         \
    if (d == D_ && nt == NT_)                                                         \
        return mode == kStreamLogits ? launch_t<D_, NT_, kStreamLogits>(kmap, a, stream) \
                                     : launch_t<D_, NT_, kStreamSelect>(kmap, a, stream);
    SAGA_QK_CASE(64, 1)
    SAGA_QK_CASE(64, 2)
    SAGA_QK_CASE(128, 1)
    SAGA_QK_CASE(128, 2)
    SAGA_QK_CASE(32, 1)
    SAGA_QK_CASE(32, 2)
#undef SAGA_QK_CASE
    return cudaErrorInvalidValue;
}

}  // namespace saga
