// Dense grouped-query decode attention: the full-attention baseline the
// speedups are measured against ("More Value per Key", ai.info summary, Main
// Findings, end-to-end decoding speedups over baseline full attention).
//
// Split-K (flash-decoding) over the flattened (batch, tile) space, same
// partition as the streaming kernel.  The producer warp loads each tile's K
// boxes (128-byte swizzle, read by ldmatrix) and V boxes (plain rows) with
// TMA; each consumer warp computes the logits of its key head's G query heads
// for its slice of the tile on tensor cores (the same routine as the sparse
// path), keeps a running max / sum per head (online softmax), writes the
// weights to a per-warp scratch, and accumulates weight x value in fp32 on
// the CUDA cores, each lane owning d/32 output columns.  Every warp writes
// one partial record per (row, CTA slot); the combine kernel merges them.
#include "qk_tile.cuh"
#include "saga_kernels.h"

namespace saga {

namespace {

constexpr int kPStride = 36;  // floats per head row of the weight scratch (bank spread)

template <int D, int NT>
__global__ void __launch_bounds__(kStreamThreads, 1)
    dense_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                 const DenseArgs a) {
    constexpr int MBW = 128 / D;
    constexpr int DH = D / 64;
    constexpr int HS = NT * 8;        // head slots per key head
    constexpr int CPL = D / 32;       // output columns per lane
    constexpr int ROWS = MBW * 16;    // positions per warp per tile

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const Geometry& g = a.g;
    const int stages = a.stages;
    const int vbytes = g.P * g.hv * D * 2;
    const int stage_bytes = kStageBytes + vbytes;
    float* pbuf_all = reinterpret_cast<float*>(smem + static_cast<size_t>(stages) * stage_bytes);
    float* abuf_all = pbuf_all + kConsumerWarps * HS * kPStride;
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
                for (int kh = 0; kh < g.hk; ++kh)
                    for (int dh = 0; dh < DH; ++dh)
                        tma_load_3d(dst + (kh * DH + dh) * g.P * 128, &kmap, &full[st], dh * 64,
                                    kh, z);
                for (int vh = 0; vh < g.hv; ++vh)
                    for (int dh = 0; dh < DH; ++dh)
                        tma_load_3d(dst + kStageBytes + (vh * DH + dh) * g.P * 128, &vmap,
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
    float* pbuf = pbuf_all + warp * HS * kPStride;
    float* abuf = abuf_all + warp * HS;
    // value-row byte offset of this lane's columns inside a (vh, dh) box row
    const int vcol_dh = (lane * CPL) / 64;
    const int vcol_off = ((lane * CPL) % 64) * 2;
    int vbox[HS];
#pragma unroll
    for (int hl = 0; hl < HS; ++hl) {
        const int vh = hl < G ? (kh * G + hl) * g.hv / g.hq : 0;
        vbox[hl] = kStageBytes + (vh * DH + vcol_dh) * g.P * 128 + vcol_off;
    }

    QFrag<D, NT> qf;
    float m_run[NT][2], l_run[NT][2];
    float o[HS][CPL];
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
        for (int hl = 0; hl < HS; ++hl)
#pragma unroll
            for (int cc = 0; cc < CPL; ++cc) o[hl][cc] = 0.f;
    };

    auto end_segment = [&](int bb) {
        // header by the lanes that own each head's softmax state, o by all lanes
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
#pragma unroll
        for (int hl = 0; hl < HS; ++hl) {
            if (hl >= G) break;
            const size_t row = static_cast<size_t>(bb) * g.hq + kh * G + hl;
            float* rec =
                a.records + ((row * g.S_cap + slot) * g.WPK + sub) * static_cast<size_t>(g.rec);
#pragma unroll
            for (int cc = 0; cc < CPL; ++cc) rec[kRecHeader + lane * CPL + cc] = o[hl][cc];
        }
    };

    const uint32_t stage0 = smem_addr(smem);
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

        // online softmax per head column (2t+e of n-tile nt)
        const int pos0 = tl * g.P + mb0 * 16 + gq;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int hl = nt * 8 + 2 * tq + e;
                float mt = -kInf;
#pragma unroll
                for (int mbi = 0; mbi < MBW; ++mbi)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int pos = pos0 + mbi * 16 + 8 * h;
                        const bool valid = pos < g.l && hl < G;
                        const float s = valid ? acc[mbi][nt][2 * h + e] * g.scale : -kInf;
                        acc[mbi][nt][2 * h + e] = s;
                        mt = fmaxf(mt, s);
                    }
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
                const float m_new = fmaxf(m_run[nt][e], mt);
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
                        pbuf[hl * kPStride + mbi * 16 + 8 * h + gq] = p;
                    }
                psum += __shfl_xor_sync(0xffffffffu, psum, 4);
                psum += __shfl_xor_sync(0xffffffffu, psum, 8);
                psum += __shfl_xor_sync(0xffffffffu, psum, 16);
                l_run[nt][e] = l_run[nt][e] * alpha + psum;
                m_run[nt][e] = m_new;
                if (gq == 0) abuf[hl] = alpha;
            }
        __syncwarp();

        // o[hl] = alpha * o[hl] + sum_j p[hl][j] * V[j, vh(hl)]
        const uint8_t* stage_ptr = smem + static_cast<size_t>(st) * stage_bytes;
#pragma unroll
        for (int hl = 0; hl < HS; ++hl) {
            if (hl >= G) break;
            const float alpha = abuf[hl];
#pragma unroll
            for (int cc = 0; cc < CPL; ++cc) o[hl][cc] *= alpha;
            const uint8_t* vrow = stage_ptr + vbox[hl] + (mb0 * 16) * 128;
#pragma unroll
            for (int j = 0; j < ROWS; j += 4) {
                const float4 p4 = *reinterpret_cast<const float4*>(pbuf + hl * kPStride + j);
                const float pj[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const uint8_t* vp = vrow + (j + jj) * 128;
                    if (CPL == 2) {
                        const uint32_t w = *reinterpret_cast<const uint32_t*>(vp);
                        o[hl][0] = fmaf(pj[jj], bf16_lo(w), o[hl][0]);
                        o[hl][1] = fmaf(pj[jj], bf16_hi(w), o[hl][1]);
                    } else {
                        const uint2 w = *reinterpret_cast<const uint2*>(vp);
                        o[hl][0] = fmaf(pj[jj], bf16_lo(w.x), o[hl][0]);
                        o[hl][1] = fmaf(pj[jj], bf16_hi(w.x), o[hl][1]);
                        o[hl][CPL > 2 ? 2 : 0] = fmaf(pj[jj], bf16_lo(w.y), o[hl][CPL > 2 ? 2 : 0]);
                        o[hl][CPL > 3 ? 3 : 0] = fmaf(pj[jj], bf16_hi(w.y), o[hl][CPL > 3 ? 3 : 0]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }
    if (cur_bb >= 0) end_segment(cur_bb);
    if (!ok && lane == 0) raise_device_error(a.err, kErrTimeout);
}

template <int D, int NT>
cudaError_t launch_t(const CUtensorMap& kmap, const CUtensorMap& vmap, const DenseArgs& a,
                     cudaStream_t stream) {
    const size_t smem = dense_smem_bytes(a.g, a.stages);
    auto kern = dense_kernel<D, NT>;
    static const cudaError_t attr = cudaFuncSetAttribute(
        kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynamicSmem);
    if (attr != cudaSuccess) return attr;
    if (smem > static_cast<size_t>(kMaxDynamicSmem)) return cudaErrorInvalidValue;
    kern<<<a.C, kStreamThreads, smem, stream>>>(kmap, vmap, a);
    return cudaGetLastError();
}

}  // namespace

size_t dense_stage_bytes(const Geometry& g) {
    return static_cast<size_t>(kStageBytes) + static_cast<size_t>(g.P) * g.hv * g.d * 2;
}

size_t dense_smem_bytes(const Geometry& g, int stages) {
    const size_t hs = static_cast<size_t>(g.NT) * 8;
    return 1024 + stages * dense_stage_bytes(g) +
           kConsumerWarps * hs * (kPStride + 1) * sizeof(float) + 2 * stages * sizeof(uint64_t) + 16;
}

cudaError_t launch_dense(const CUtensorMap& kmap, const CUtensorMap& vmap, const DenseArgs& a,
                         cudaStream_t stream) {
    const int d = a.g.d, nt = a.g.NT;
    if (d == 64 && nt == 1) return launch_t<64, 1>(kmap, vmap, a, stream);
    if (d == 64 && nt == 2) return launch_t<64, 2>(kmap, vmap, a, stream);
    if (d == 128 && nt == 1) return launch_t<128, 1>(kmap, vmap, a, stream);
    if (d == 128 && nt == 2) return launch_t<128, 2>(kmap, vmap, a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace saga
