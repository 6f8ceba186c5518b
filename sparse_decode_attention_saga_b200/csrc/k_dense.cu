// Dense grouped-query decode attention: the full-attention baseline the
// speedups are measured against ("More Value per Key", ai.info summary, Main
// Findings: the end-to-end speedups compare against full attention).
//
// Split-K (flash-decoding) over the flattened (batch, tile) space, same
// partition as the streaming kernel.  The producer warp loads each tile's K
// and V boxes with TMA (128-byte swizzle).  Each consumer warp owns one key
// head and a slice of the tile's positions:
//   logits of its G query heads on tensor cores (the same routine as the
//   sparse path), online softmax per head (running max / sum), and the
//   weights written to a per-warp scratch as bf16 hi + lo parts
//   (p = hi + lo to about 16 bits);
//   the probability-value product also on tensor cores, swap-AB:
//   O^T (16 head dims x 8 query heads) += V^T (16 dims x 16 positions,
//   ldmatrix.trans from the swizzled V box) x P^T (16 positions x 8 heads),
//   once with the hi and once with the lo weights, fp32 accumulators in
//   registers.  The query heads of one column tile share one value head.
// Every warp writes one partial record per (row, CTA slot); the combine
// kernel merges them.
// More than two value heads per key head (SAGA's (h_k, h_v) = (1, 8), or
// 32-dim keys with h_v = 4 h_k): the kernel runs on a geometry with one key
// head per value head, each loading its cache key head (k_group of them
// share one), so that every warp's query heads use a single value head.
// The shared key rows then come from HBM once and from L2 k_group times.
#include "qk_tile.cuh"
#include "saga_kernels.h"

namespace saga {

namespace {

// bf16 entries per head row of the weight scratch: a warp's positions + 8
// (the B-fragment reads of the eight heads then hit distinct banks)
__host__ __device__ constexpr int weight_stride(int d) { return (128 / d) * 16 + 8; }

template <int D, int DV, int NT, int NCT>  // D: key/query head dim, DV: value head dim
__global__ void __launch_bounds__(kStreamThreads, 1)
    dense_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                 const DenseArgs a) {
    constexpr int MBW = 128 / D;
    constexpr int DVH = DV / 64;       // 64-wide value boxes per value head
    constexpr int HS = NT * 8;         // head slots per key head
    constexpr int ROWS = MBW * 16;     // positions per warp per tile
    constexpr int PS = weight_stride(D);
    constexpr int MT = DV / 16;        // 16-dim row tiles of O^T

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const Geometry& g = a.g;
    const int stages = a.stages;
    const int vbytes = g.P * g.hv * DV * 2;
    const int stage_bytes = kStageBytes + vbytes;
    uint16_t* pbuf_all = reinterpret_cast<uint16_t*>(smem + static_cast<size_t>(stages) * stage_bytes);
    float* abuf_all = reinterpret_cast<float*>(pbuf_all + kConsumerWarps * 2 * HS * PS);
    uint64_t* full = reinterpret_cast<uint64_t*>(abuf_all + kConsumerWarps * HS);
    uint64_t* empty = full + stages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);

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
    pdl_trigger();  // the combine kernel may be scheduled behind this grid

    const long long T = static_cast<long long>(g.b) * g.tiles;
    const int C = a.C, c = blockIdx.x;
    const long long t0 = cta_tile_begin(T, C, c), t1 = cta_tile_begin(T, C, c + 1);
    const int ntile = static_cast<int>(t1 - t0);

    if (warp == kConsumerWarps) {
        if (lane == 0) {
            prefetch_tensor_map(&kmap);
            prefetch_tensor_map(&vmap);
            int issued = 0;
            for (int k = 0; k < ntile; ++k) {
                const int st = k % stages;
                if (!mbar_wait(&empty[st], ((k / stages) & 1) ^ 1, abort_flag)) break;
                const long long t = t0 + k;
                const int bb = static_cast<int>(t / g.tiles);
                const int tl = static_cast<int>(t - static_cast<long long>(bb) * g.tiles);
                const int z = bb * g.l_cap + tl * g.P;
                mbar_arrive_expect_tx(&full[st], stage_bytes);
                uint8_t* dst = smem + static_cast<size_t>(st) * stage_bytes;
                // key head kh of the geometry reads cache key head kh / k_group
                // (a counter: a division here sits on the ring's turnaround)
                if (a.k_group == 1) {
                    for (int kh = 0; kh < g.hk; ++kh)
                        for (int dh = 0; dh < KTile<D>::NBOX; ++dh)
                            tma_load_3d(dst + (kh * KTile<D>::NBOX + dh) * g.P * KTile<D>::ROWB, &kmap,
                                        &full[st], dh * 64, kh, z);
                } else {
                    for (int kh = 0, src = 0, r = 0; kh < g.hk; ++kh) {
                        for (int dh = 0; dh < KTile<D>::NBOX; ++dh)
                            tma_load_3d(dst + (kh * KTile<D>::NBOX + dh) * g.P * KTile<D>::ROWB, &kmap,
                                        &full[st], dh * 64, src, z);
                        if (++r == a.k_group) {
                            r = 0;
                            ++src;
                        }
                    }
                }
                for (int vh = 0; vh < g.hv; ++vh)
                    for (int dh = 0; dh < DVH; ++dh)
                        tma_load_3d(dst + kStageBytes + (vh * DVH + dh) * g.P * 128, &vmap,
                                    &full[st], dh * 64, vh, z);
                issued = k + 1;
            }
            int dummy = 0;
            for (int k = (issued > stages ? issued - stages : 0); k < issued; ++k)
                if (!mbar_wait(&full[k % stages], (k / stages) & 1, &dummy))
                    raise_device_error(a.err, kErrTimeout);
        }
        return;
    }

    const int kh = warp / g.WPK, sub = warp % g.WPK;
    const int mb0 = sub * MBW;
    const int gq = lane >> 2, tq = lane & 3;
    const int G = g.G;
    uint16_t* pb_hi = pbuf_all + warp * 2 * HS * PS;
    uint16_t* pb_lo = pb_hi + HS * PS;
    float* abuf = abuf_all + warp * HS;

    // Column tiles of O^T: NCT tiles of 8 head slots.  With VPK = 2 value
    // heads per key head, tile ct holds the GV = G / 2 <= 8 query heads of
    // value head kh*2 + ct; otherwise the G heads of the group's one value
    // head fill tiles of 8.
    const int VPK = g.hv > g.hk ? g.hv / g.hk : 1;
    const int GV = G / VPK;
    auto head_of = [&](int ct, int n) { return VPK > 1 ? ct * GV + n : ct * 8 + n; };
    auto head_ok = [&](int ct, int n) { return VPK > 1 ? n < GV : ct * 8 + n < G; };
    int vh_ct[NCT];
#pragma unroll
    for (int ct = 0; ct < NCT; ++ct) vh_ct[ct] = (kh * G + head_of(ct, 0)) * g.hv / g.hq;

    QFrag<D, NT> qf;
    float m_run[NT][2], l_run[NT][2];
    float o[MT][NCT][4];  // O^T fragments: dims mt*16 + gq (+8), heads 2tq (+1) of tile ct
    int cur_bb = -1, slot = 0;

    auto begin_segment = [&](int bb) {
        load_q_frag<D, NT>(qf, reinterpret_cast<const __nv_bfloat16*>(a.q), g.hq, G, bb, kh, lane);
        slot = c - cta_of_tile(static_cast<long long>(bb) * g.tiles, T, C);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                m_run[nt][e] = -kInf;
                l_run[nt][e] = 0.f;
            }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int ct = 0; ct < NCT; ++ct)
#pragma unroll
                for (int e = 0; e < 4; ++e) o[mt][ct][e] = 0.f;
    };

    auto end_segment = [&](int bb) {
        // header by the lanes that own each head's softmax state
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int hl = nt * 8 + 2 * tq + e;
                if (gq == 0 && hl < G) {
                    const size_t row = static_cast<size_t>(bb) * g.hq + kh * G + hl;
                    float* rec = a.records +
                                 ((row * g.S_cap + slot) * g.WPK + sub) * static_cast<size_t>(g.rec);
                    rec[0] = m_run[nt][e];
                    rec[1] = l_run[nt][e];
                    rec[2] = __int_as_float(0);
                    rec[3] = m_run[nt][e];
                }
            }
        // output columns from the O^T fragments
#pragma unroll
        for (int ct = 0; ct < NCT; ++ct)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                if (!head_ok(ct, 2 * tq + e)) continue;
                const size_t row = static_cast<size_t>(bb) * g.hq + kh * G + head_of(ct, 2 * tq + e);
                float* rec = a.records +
                             ((row * g.S_cap + slot) * g.WPK + sub) * static_cast<size_t>(g.rec) + kRecHeader;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    rec[mt * 16 + gq] = o[mt][ct][e];
                    rec[mt * 16 + gq + 8] = o[mt][ct][2 + e];
                }
            }
    };

    const uint32_t stage0 = smem_addr(smem);
    const uint32_t pb_hi_a = smem_addr(pb_hi), pb_lo_a = smem_addr(pb_lo);
    // ldmatrix.trans addressing: lane -> matrix mi = lane/8 (dims +8 for odd mi,
    // positions +8 for mi >= 2), row = lane%8 (one position per row)
    const int ld_pos = (lane >> 4) * 8 + (lane & 7);
    const int ld_dim = ((lane >> 3) & 1) * 8;
    bool ok = true;
    for (int k = 0; k < ntile; ++k) {
        const long long t = t0 + k;
        const int bb = static_cast<int>(t / g.tiles);
        const int tl = static_cast<int>(t - static_cast<long long>(bb) * g.tiles);
        if (bb != cur_bb) {
            if (cur_bb >= 0) end_segment(cur_bb);
            begin_segment(bb);
            cur_bb = bb;
        }
        const int st = k % stages;
        const bool got = mbar_wait(&full[st], (k / stages) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
        }
        const uint32_t sbase = stage0 + static_cast<uint32_t>(st * stage_bytes);
        float acc[MBW][NT][4];
        qk_mma<D, NT, MBW>(sbase, g.P, kh, mb0, qf, acc, lane);

        // online softmax per head column (2t+e of n-tile nt); weights -> scratch
        const int pos0 = tl * g.P + mb0 * 16 + gq;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int hl = nt * 8 + 2 * tq + e;
                float mt_ = -kInf;
#pragma unroll
                for (int mbi = 0; mbi < MBW; ++mbi)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int pos = pos0 + mbi * 16 + 8 * h;
                        const bool valid = pos < g.l && hl < G;
                        const float s = valid ? acc[mbi][nt][2 * h + e] * g.scale : -kInf;
                        acc[mbi][nt][2 * h + e] = s;
                        mt_ = fmaxf(mt_, s);
                    }
                mt_ = fmaxf(mt_, __shfl_xor_sync(0xffffffffu, mt_, 4));
                mt_ = fmaxf(mt_, __shfl_xor_sync(0xffffffffu, mt_, 8));
                mt_ = fmaxf(mt_, __shfl_xor_sync(0xffffffffu, mt_, 16));
                const float m_new = fmaxf(m_run[nt][e], mt_);
                const bool live = m_new > -kInf;
                const float alpha = live ? __expf(m_run[nt][e] - m_new) : 1.f;
                float psum = 0.f;
#pragma unroll
                for (int mbi = 0; mbi < MBW; ++mbi)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float s = acc[mbi][nt][2 * h + e];
                        const float p = live ? __expf(s - m_new) : 0.f;
                        psum += p;
                        const __nv_bfloat16 hi = __float2bfloat16_rn(p);
                        const __nv_bfloat16 lo = __float2bfloat16_rn(p - __bfloat162float(hi));
                        const int at = hl * PS + mbi * 16 + 8 * h + gq;
                        pb_hi[at] = __bfloat16_as_ushort(hi);
                        pb_lo[at] = __bfloat16_as_ushort(lo);
                    }
                psum += __shfl_xor_sync(0xffffffffu, psum, 4);
                psum += __shfl_xor_sync(0xffffffffu, psum, 8);
                psum += __shfl_xor_sync(0xffffffffu, psum, 16);
                l_run[nt][e] = l_run[nt][e] * alpha + psum;
                m_run[nt][e] = m_new;
                if (gq == 0) abuf[hl] = alpha;
            }
        __syncwarp();

        // rescale O^T by each head's alpha, then O^T += V^T P^T (hi and lo)
#pragma unroll
        for (int ct = 0; ct < NCT; ++ct)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float al = head_ok(ct, 2 * tq + e) ? abuf[head_of(ct, 2 * tq + e)] : 1.f;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    o[mt][ct][e] *= al;
                    o[mt][ct][2 + e] *= al;
                }
            }
        const int lim = g.l - (tl * g.P + mb0 * 16);  // valid positions of this warp's slice
#pragma unroll
        for (int ks = 0; ks < MBW; ++ks) {
            uint32_t bh[NCT][2], bl[NCT][2];
#pragma unroll
            for (int ct = 0; ct < NCT; ++ct) {
                const bool hv_ok = head_ok(ct, gq);
                const uint32_t off = static_cast<uint32_t>((head_of(ct, hv_ok ? gq : 0) * PS + ks * 16 + 2 * tq) * 2);
                uint32_t h0 = 0u, h1 = 0u, l0 = 0u, l1 = 0u;
                if (hv_ok) {
                    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(h0) : "r"(pb_hi_a + off));
                    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(h1) : "r"(pb_hi_a + off + 16));
                    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(l0) : "r"(pb_lo_a + off));
                    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(l1) : "r"(pb_lo_a + off + 16));
                }
                bh[ct][0] = h0;
                bh[ct][1] = h1;
                bl[ct][0] = l0;
                bl[ct][1] = l1;
            }
            const int pos = mb0 * 16 + ks * 16 + ld_pos;  // position row (in the tile) of this lane
            // this thread's A elements cover positions ks*16 + 2tq (+1, +8, +9) of the slice
            const int pa = ks * 16 + 2 * tq;
            const bool ragged = lim < ROWS;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int dim = mt * 16 + ld_dim;
                const int dh = dim >> 6, chunk = (dim & 63) >> 3;
                uint32_t a0 = 0u, a1 = 0u, a2 = 0u, a3 = 0u;
#pragma unroll
                for (int ct = 0; ct < NCT; ++ct) {
                    if (ct == 0 || VPK > 1) {
                        const uint32_t addr = sbase + kStageBytes +
                                              static_cast<uint32_t>((vh_ct[ct] * DVH + dh) * g.P * 128 + pos * 128 +
                                                                    ((chunk ^ (pos & 7)) << 4));
                        ldmatrix_x4_trans(addr, a0, a1, a2, a3);
                        if (ragged) {
                            // positions past l: zero the value elements so that
                            // whatever the cache holds there cannot reach the sum
                            const uint32_t m0 = (pa < lim ? 0xffffu : 0u) | (pa + 1 < lim ? 0xffff0000u : 0u);
                            const uint32_t m8 = (pa + 8 < lim ? 0xffffu : 0u) | (pa + 9 < lim ? 0xffff0000u : 0u);
                            a0 &= m0;
                            a1 &= m0;
                            a2 &= m8;
                            a3 &= m8;
                        }
                    }
                    mma_16816(o[mt][ct], a0, a1, a2, a3, bh[ct][0], bh[ct][1]);
                    mma_16816(o[mt][ct], a0, a1, a2, a3, bl[ct][0], bl[ct][1]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }
    if (cur_bb >= 0) end_segment(cur_bb);
    if (!ok && lane == 0) raise_device_error(a.err, kErrTimeout);
}

template <int D, int DV, int NT, int NCT>
cudaError_t launch_t(const CUtensorMap& kmap, const CUtensorMap& vmap, const DenseArgs& a,
                     cudaStream_t stream) {
    const size_t smem = dense_smem_bytes(a.g, a.stages);
    auto kern = dense_kernel<D, DV, NT, NCT>;
    const cudaError_t attr = allow_dynamic_smem(kern, kMaxDynamicSmem);
    if (attr != cudaSuccess) return attr;
    if (smem > static_cast<size_t>(kMaxDynamicSmem)) return cudaErrorInvalidValue;
    kern<<<a.C, kStreamThreads, smem, stream>>>(kmap, vmap, a);
    return cudaGetLastError();
}

}  // namespace

bool dense_supported(const Geometry& g) {
    // each key head's query heads use one value head, or two whole ones
    // (more value heads per key head would also not fit a stage: its value
    // rows are the K tile's bytes times h_v*d_v / (h_k*d))
    return g.hv <= 2 * g.hk && (g.hv % g.hk == 0 || g.hk % g.hv == 0);
}

size_t dense_stage_bytes(const Geometry& g) {
    return static_cast<size_t>(kStageBytes) + static_cast<size_t>(g.P) * g.hv * g.dv * 2;
}

size_t dense_smem_bytes(const Geometry& g, int stages) {
    const size_t hs = static_cast<size_t>(g.NT) * 8;
    return 1024 + stages * dense_stage_bytes(g) +
           kConsumerWarps * hs * (2 * weight_stride(g.d) * sizeof(uint16_t) + sizeof(float)) +
           2 * stages * sizeof(uint64_t) + 16;
}

cudaError_t launch_dense(const CUtensorMap& kmap, const CUtensorMap& vmap, const DenseArgs& a,
                         cudaStream_t stream) {
    if (!dense_supported(a.g)) return cudaErrorInvalidValue;
    const int d = a.g.d, dv = a.g.dv, nt = a.g.NT;
    const int vpk = a.g.hv > a.g.hk ? a.g.hv / a.g.hk : 1;
    const int nct = vpk > 1 ? vpk : nt;  // column tiles of query heads: 1 or 2
#define SAGA_DENSE_CASE(DK_, DV_, NT_, NCT_)                                   \
    if (d == DK_ && dv == DV_ && nt == NT_ && nct == NCT_)                     \
        return launch_t<DK_, DV_, NT_, NCT_>(kmap, vmap, a, stream);
    SAGA_DENSE_CASE(64, 64, 1, 1)
    SAGA_DENSE_CASE(64, 64, 1, 2)
    SAGA_DENSE_CASE(64, 64, 2, 2)
    SAGA_DENSE_CASE(128, 128, 1, 1)
    SAGA_DENSE_CASE(128, 128, 1, 2)
    SAGA_DENSE_CASE(128, 128, 2, 2)
    SAGA_DENSE_CASE(32, 64, 1, 1)
    SAGA_DENSE_CASE(32, 64, 1, 2)
    SAGA_DENSE_CASE(32, 64, 2, 2)
#undef SAGA_DENSE_CASE
    return cudaErrorInvalidValue;
}

}  // namespace saga
