// diag.cu -- self-test of the bounded wait (mbar_wait) that every TMA and
// tensor-core pipeline of the library relies on to turn a stalled pipeline
// into CF_ERR_TIMEOUT instead of a hung GPU.  One CTA initialises two
// mbarriers, completes the phase of the first itself and leaves the second
// untouched; it then waits on both with a small poll limit and reports what
// each wait returned.  Nothing faults, traps or spins without bound: the
// unsignalled wait gives up after `polls` polls.
#include <cuda_runtime.h>

#include "bounds.cuh"
#include "cf.h"
#include "cf_diag.h"
#include "cf_trace.h"
#include "mbar.cuh"

namespace {

constexpr int32_t kMaxDiagPolls = 1 << 16;

__global__ void diag_wait_kernel(uint32_t polls, int32_t *out) {
    __shared__ __align__(8) uint64_t bars[2];
    const uint32_t done = static_cast<uint32_t>(__cvta_generic_to_shared(&bars[0]));
    const uint32_t never = static_cast<uint32_t>(__cvta_generic_to_shared(&bars[1]));
    if (threadIdx.x != 0) return;
    cf::mbar_init(done, 1);
    cf::mbar_init(never, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    cf::mbar_arrive(done);   // phase 0 of `done` completes
    // out[0]: the signalled barrier's wait completed (1)
    out[0] = cf::mbar_wait(done, 0, polls) ? 1 : 0;
    // out[1]: the unsignalled barrier's wait gave up, and the caller records
    // CF_ERR_TIMEOUT as the pipelines do
    out[1] = cf::mbar_wait(never, 0, polls) ? (int32_t)CF_OK : (int32_t)CF_ERR_TIMEOUT;
}

}  // namespace

// Positive control of the debug build's index checks: writes out[i] = i for
// every i < n, each write guarded by a check that declares an extent of n / 2.
// Every write the check lets through stays inside out[0, n).
__global__ void diag_bounds_kernel(int32_t *out, int n) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        if (CF_IN(i < n / 2)) out[i] = i;
}

// Bounds-checked debug build: this translation unit's first failed index
// check, read and cleared (synchronises the device).
#ifdef CF_DEBUG_BOUNDS
int32_t cf_bounds_take_diag() {
    int32_t v = 0;
    const int32_t z = 0;
    if (cudaMemcpyFromSymbol(&v, cf::g_bounds_hit, sizeof v) != cudaSuccess ||
        cudaMemcpyToSymbol(cf::g_bounds_hit, &z, sizeof z) != cudaSuccess) {
        (void)cudaGetLastError();
        return -1;
    }
    return v;
}
#endif

extern "C" cf_status cf_diag_bounds_selftest(int32_t *out_dev, int32_t n, void *stream) {
    if (!cf::kBoundsChecked) return CF_ERR_UNSUPPORTED;
    if (!out_dev || n < 2 || n > (1 << 20)) return CF_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out_dev) & 3u) != 0) return CF_ERR_ALIGNMENT;
    diag_bounds_kernel<<<1, 256, 0, (cudaStream_t)stream>>>(out_dev, n);
    return cudaGetLastError() == cudaSuccess ? CF_OK : CF_ERR_CUDA;
}

extern "C" cf_status cf_diag_bounded_wait(int32_t polls, int32_t *out_dev, void *stream) {
    cf::TraceRange trace_("cf_diag_bounded_wait");
    if (polls < 1 || polls > kMaxDiagPolls || !out_dev) return CF_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out_dev) & 3u) != 0) return CF_ERR_ALIGNMENT;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, out_dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return CF_ERR_INVALID_ARG;
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return CF_ERR_INVALID_ARG;
    diag_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint32_t)polls, out_dev);
    return cudaGetLastError() == cudaSuccess ? CF_OK : CF_ERR_CUDA;
}
