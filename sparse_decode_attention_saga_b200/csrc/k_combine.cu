// The combine kernel: one CTA per (batch, query head) row merges the row's
// partial records (combine_row.cuh).  Used after the dense kernel; the
// sparse paths merge in the gather kernel's last CTA of each row.
#include "combine_row.cuh"

namespace saga {

namespace {

// Grid (chunks, rows).  One chunk: the CTA merges the row.  Several: CTA c
// merges its share of the row's records into a partial record at slot
// partial_slot + c (past every input record), and the row's last CTA to
// finish (per-row ticket, no spin) merges the chunks' partial records.
template <int D, int DK, int NT>  // D: value head dim, DK: key/query head dim
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineArgs a) {
    __shared__ int is_last;
    pdl_wait();  // the partial records come from the previous kernel
    const long long row = blockIdx.y;
    if (a.chunks <= 1) {
        combine_row<D, DK, NT>(a, row);
        return;
    }
    const Geometry& g = a.g;
    const int bb = static_cast<int>(row / g.hq);
    const int R = row_records(a, bb), c = blockIdx.x;
    const int r0 = static_cast<int>(static_cast<long long>(R) * c / a.chunks);
    const int r1 = static_cast<int>(static_cast<long long>(R) * (c + 1) / a.chunks);
    // the record area is workspace memory: chunk partials go past the inputs
    float* part = const_cast<float*>(a.records) +
                  (static_cast<size_t>(row) * g.S_cap * g.WPK + a.partial_slot + c) * g.rec;
    combine_row<D, DK, NT>(a, row, r0, r1 - r0, part);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomicAdd(a.tickets + row, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    if (threadIdx.x == 0) a.tickets[row] = 0u;
    combine_row<D, DK, NT>(a, row, a.partial_slot, a.chunks);
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
    const unsigned rows = static_cast<unsigned>(static_cast<long long>(a.g.b) * a.g.hq);
    const dim3 grid(a.chunks > 1 ? a.chunks : 1, rows), block(kCombineThreads);
#define SAGA_COMBINE_CASE(DV_, DK_, NT_)                                                       \
    if (a.g.dv == DV_ && a.g.d == DK_ && a.g.NT == NT_)                                        \
        return launch_dependent(combine_kernel<DV_, DK_, NT_>, grid, block, 0, stream, a);
    SAGA_COMBINE_CASE(64, 64, 1)
    SAGA_COMBINE_CASE(64, 64, 2)
    SAGA_COMBINE_CASE(128, 128, 1)
    SAGA_COMBINE_CASE(128, 128, 2)
    SAGA_COMBINE_CASE(64, 32, 1)
    SAGA_COMBINE_CASE(64, 32, 2)
#undef SAGA_COMBINE_CASE
    return cudaErrorInvalidValue;
}

}  // namespace saga
