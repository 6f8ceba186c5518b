// The grouped query-key product on tensor cores, shared by every kernel that
// produces logits (the logits kernel, the fused compare kernel, the dense
// kernel and the combine kernel's empty-set fallback), so that all of them
// produce bit-identical logits for the same query and key rows.
//
// Swap-AB mapping of the decode GEMV onto mma.m16n8k16 (bf16 in, fp32 acc):
//   A (16 x 16, row-major) = 16 cached positions x 16 head-dim elements,
//   B (16 x 8,  col-major) = 16 head-dim elements x 8 query heads of one key
//                            head's group (zero-padded past G),
//   C (16 x 8)             = logits of 16 positions x 8 query heads.
// C fragment of lane (g = lane/4, t = lane%4): c[0], c[1] = rows g, columns
// 2t, 2t+1; c[2], c[3] = row g+8, same columns.
//
// Shared-memory K tile: one TMA box per (key head kh, 64-wide part dh of the
// head dim), [rows = positions][128 B], written with the 128-byte swizzle
// (16-byte chunk c of row r lands at chunk c ^ (r & 7)); 32-dim keys use
// one box per head with 64-byte rows and the 64-byte swizzle (chunk c of
// row r at c ^ ((r >> 1) & 3)).  Either way the eight row addresses of every
// ldmatrix phase hit distinct banks.
#pragma once

#include "saga_device.cuh"

namespace saga {

// Shared-memory layout of the K boxes for head dim D.
template <int D>
struct KTile {
    static constexpr int ROWB = D >= 64 ? 128 : D * 2;  // bytes per box row
    static constexpr int NBOX = D >= 64 ? D / 64 : 1;   // boxes per key head
    static constexpr int CPR = ROWB / 16;               // 16-byte chunks per row
    static constexpr int BOXW = ROWB / 2;               // elements per box row
    // byte offset of 16-byte chunk `chunk` (logical) of row r of box `box`
    static __host__ __device__ __forceinline__ int offset(int box, int rows_per_box, int r,
                                                          int chunk) {
        const int swz = ROWB == 128 ? (r & 7) : ((r >> 1) & 3);
        return box * rows_per_box * ROWB + r * ROWB + ((chunk ^ swz) << 4);
    }
};

// q fragments of one key head's group: qf[nt][ks][0..1] for n-tile nt
// (query heads nt*8 .. nt*8+7 of the group) and k-step ks (16 dims).
template <int D, int NT>
struct QFrag {
    uint32_t r[NT][D / 16][2];
};

// Loads the B fragments for batch bb, key head kh from q [b, hq, D] bf16.
template <int D, int NT>
__device__ __forceinline__ void load_q_frag(QFrag<D, NT>& qf, const __nv_bfloat16* q, int hq,
                                            int G, int bb, int kh, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int hl = nt * 8 + g;
        const bool valid = hl < G;
        const uint32_t* row = reinterpret_cast<const uint32_t*>(
            q + (static_cast<size_t>(bb) * hq + kh * G + (valid ? hl : 0)) * D);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            qf.r[nt][ks][0] = valid ? __ldg(row + (ks * 16 + 2 * t) / 2) : 0u;
            qf.r[nt][ks][1] = valid ? __ldg(row + (ks * 16 + 8 + 2 * t) / 2) : 0u;
        }
    }
}

// acc[mbi][nt][*] = logits (unscaled) of m-block mb0+mbi of the tile for key
// head kh.  `tile` is the shared address of the stage, `rows_per_box` the
// number of position rows in each (kh, dh) box.
template <int D, int NT, int MB>
__device__ __forceinline__ void qk_mma(uint32_t tile, int rows_per_box, int kh, int mb0,
                                       const QFrag<D, NT>& qf, float (&acc)[MB][NT][4],
                                       int lane) {
    using L = KTile<D>;
    const int chunk_hi = lane >> 4;
#pragma unroll
    for (int mbi = 0; mbi < MB; ++mbi) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mbi][nt][e] = 0.f;
        const int r = (mb0 + mbi) * 16 + (lane & 15);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const int dh = ks / (L::CPR / 2);  // 16 dims = two chunks per k-step
            const int chunk = ((ks % (L::CPR / 2)) << 1) | chunk_hi;
            const uint32_t addr =
                tile + static_cast<uint32_t>(L::offset(kh * L::NBOX + dh, rows_per_box, r, chunk));
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(addr, a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                mma_16816(acc[mbi][nt], a0, a1, a2, a3, qf.r[nt][ks][0], qf.r[nt][ks][1]);
        }
    }
}

// Smallest fp32 x with fl(x * scale) >= tau.  fl(x * scale) is monotone in x,
// so "x >= raw_threshold(tau, scale)" decides exactly what "fl(x * scale) >=
// tau" decides, with one compare on the raw tensor-core accumulator.  The
// start fl(tau / scale) is within two ulps of the boundary.
__device__ __forceinline__ float raw_threshold(float tau, float scale) {
    float x = __fdiv_rn(tau, scale);
    if (!(x == x)) return x;  // NaN threshold: nothing compares >= it
    for (int i = 0; i < 4 && __fmul_rn(x, scale) >= tau; ++i) {
        const float below = nextafterf(x, -kInf);
        if (__fmul_rn(below, scale) < tau) break;
        x = below;
    }
    for (int i = 0; i < 4 && __fmul_rn(x, scale) < tau; ++i) x = nextafterf(x, kInf);
    return x;
}

}  // namespace saga
