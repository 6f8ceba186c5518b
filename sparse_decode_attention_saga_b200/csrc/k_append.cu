// Cache growth: the decode step's new key and value rows written at position
// l_kv of every batch element's cache.
//
// Method: "More Value per Key" (ai.info summary, Main Findings: latency over
// 32 generated tokens).  Each generated token appends its own key and value
// rows to the cache before it attends, so the cached length grows by one per
// step; the thresholds carried between refreshes then also meet positions
// that did not exist when they were computed, which the element-wise compare
// handles like any other position.
//
// One grid-stride pass of 16-byte copies over the b*(h_k + h_v) new rows.
#include "saga_device.cuh"
#include "saga_kernels.h"

namespace saga {

namespace {

__global__ void __launch_bounds__(256) append_kernel(const AppendArgs a) {
    pdl_wait();  // the cache may still be read by the previous step's kernels
    pdl_trigger();
    const int ck = a.d / 8, cv = a.dv / 8;  // 16-byte chunks per key / value head row
    const long long nk = static_cast<long long>(a.b) * a.hk * ck;
    const long long nv = static_cast<long long>(a.b) * a.hv * cv;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < nk + nv;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const bool is_k = i < nk;
        const long long j = is_k ? i : i - nk;
        const int heads = is_k ? a.hk : a.hv;
        const long long per_b = static_cast<long long>(heads) * (is_k ? ck : cv);
        const long long bb = j / per_b;
        const long long rem = j - bb * per_b;  // (head, chunk) inside the new row
        const uint4* src = reinterpret_cast<const uint4*>(is_k ? a.k_new : a.v_new) + j;
        uint4* dst = reinterpret_cast<uint4*>(is_k ? a.k : a.v) +
                     (bb * a.l_cap + a.pos) * per_b + rem;
        *dst = __ldg(src);
    }
}

}  // namespace

cudaError_t launch_cache_append(const AppendArgs& a, cudaStream_t stream) {
    const long long chunks = static_cast<long long>(a.b) * (a.hk * (a.d / 8) + a.hv * (a.dv / 8));
    const unsigned blocks = static_cast<unsigned>((chunks + 255) / 256 < 1024 ? (chunks + 255) / 256 : 1024);
    return launch_dependent(append_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, stream, a);
}

}  // namespace saga
