// The combine kernel: one CTA per (batch, query head) row merges the row's
// partial records (combine_row.cuh).  Used after the dense kernel; the
// sparse paths merge in the gather kernel's last CTA of each row.
#include "combine_row.cuh"

namespace saga {

namespace {

template <int D, int NT>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineArgs a) {
    pdl_wait();  // the partial records come from the previous kernel
    combine_row<D, NT>(a, blockIdx.x);
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
    const unsigned rows = static_cast<unsigned>(static_cast<long long>(a.g.b) * a.g.hq);
    const int d = a.g.d, nt = a.g.NT;
    const dim3 grid(rows), block(kCombineThreads);
    if (d == 64 && nt == 1) return launch_dependent(combine_kernel<64, 1>, grid, block, 0, stream, a);
    if (d == 64 && nt == 2) return launch_dependent(combine_kernel<64, 2>, grid, block, 0, stream, a);
    if (d == 128 && nt == 1) return launch_dependent(combine_kernel<128, 1>, grid, block, 0, stream, a);
    if (d == 128 && nt == 2) return launch_dependent(combine_kernel<128, 2>, grid, block, 0, stream, a);
    return cudaErrorInvalidValue;
}

}  // namespace saga
