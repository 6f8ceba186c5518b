// saga_topn_refresh_noalloc: the exact-threshold refresh (radix select over
// caller-supplied logits) for callers that cannot allocate device memory.
//
// Who needs it: a caller that cannot hand this library a workspace, because
// it may not call cudaMalloc (or any allocator) on the decode path -- for
// example a plugin inside a host engine that owns all device memory and
// offers its plugins no allocator, or a latency-critical loop that must not
// allocate after start-up since allocation can synchronise the device and can
// fail under memory pressure.  Such a caller passes only its inputs and
// outputs; the scratch the radix select needs (per row: three 2048-bin
// histograms, the (prefix, rank) state and a completion ticket) lives in the
// file-scope device array below instead of a caller workspace.
//
// The array is a fixed 16 MiB: every GPU that loads this library holds it
// until the process exits.  That covers batch * h_q <= 682 rows (the largest
// workload here has 512).  Larger shapes are rejected with
// SAGA_ERR_WORKSPACE before anything is enqueued.
#include <cuda_runtime.h>

#include <limits>
#include <mutex>

#include "saga.h"
#include "saga_kernels.h"
#include "saga_params.h"

using namespace saga;

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;
// histograms [kRadixPasses][rows][kRadixBins], state [rows][2], tickets [rows]
constexpr size_t kRowBytes = (size_t(kRadixPasses) * kRadixBins + 2 + 1) * sizeof(uint32_t);
constexpr long long kMaxRows = static_cast<long long>(kScratchBytes / kRowBytes);
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_refresh_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};  // device address of g_refresh_scratch, per device
int g_sms[kMaxDevices] = {};

// Once per device, with that device current: look up the array's device
// address (the host-side symbol is only a stand-in and must never be handed
// to a kernel) and the SM count.
int scratch_of_current_device(uint8_t** scratch, int* sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return SAGA_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
        int major = 0, n = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            major != 10)
            return SAGA_ERR_DEVICE;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            return SAGA_ERR_CUDA;
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_refresh_scratch) != cudaSuccess || !p) return SAGA_ERR_CUDA;
        g_scratch[dev] = p;
        g_sms[dev] = n;
    }
    *scratch = static_cast<uint8_t*>(g_scratch[dev]);
    *sms = g_sms[dev];
    return SAGA_OK;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" int saga_topn_refresh_noalloc(const saga_dims* dims, int32_t N, const float* logits_in,
                                         float* thresh_out, saga_stream_t stream) {
    if (!dims || dims->batch <= 0 || dims->h_q <= 0 || dims->l_kv <= 0 || N <= 0)
        return SAGA_ERR_INVALID_ARG;
    if (!logits_in || !thresh_out || !aligned4(logits_in) || !aligned4(thresh_out))
        return SAGA_ERR_INVALID_ARG;
    const long long rows = static_cast<long long>(dims->batch) * dims->h_q;
    if (rows > kMaxRows) return SAGA_ERR_WORKSPACE;
    uint8_t* scratch = nullptr;
    int sms = 0;
    int st = scratch_of_current_device(&scratch, &sms);
    if (st) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int l = dims->l_kv;

    if (N >= l) {
        note_launches(1);
        return launch_fill(thresh_out, rows, -std::numeric_limits<float>::infinity(), s) ==
                       cudaSuccess
                   ? SAGA_OK
                   : SAGA_ERR_CUDA;
    }
    uint32_t* hist = reinterpret_cast<uint32_t*>(scratch);
    uint32_t* state = hist + static_cast<size_t>(kRadixPasses) * rows * kRadixBins;
    uint32_t* tickets = state + rows * 2;
    // Every call shares the array: the histograms and tickets must start at
    // zero, so clear them on the call's stream before the passes run.
    if (cudaMemsetAsync(scratch, 0, static_cast<size_t>(rows) * kRowBytes, s) != cudaSuccess)
        return SAGA_ERR_CUDA;
    RadixArgs r{};
    r.passes = kRadixPasses;
    r.logits = logits_in;
    r.rows = rows;
    r.l = l;
    r.N = N;
    r.chunks = radix_chunks(rows, l, sms);
    r.hist = hist;
    r.state = state;
    r.tickets = tickets;
    r.thresh = thresh_out;
    r.err = nullptr;
    note_launches(kRadixPasses);
    return launch_radix_select(r, s) == cudaSuccess ? SAGA_OK : SAGA_ERR_CUDA;
}
