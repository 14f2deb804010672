// diag.cu -- self-test of the bounded wait (mbar_wait) that every TMA and
// tensor-core pipeline of the library relies on to turn a stalled pipeline
// into CF_ERR_TIMEOUT instead of a hung GPU.  One CTA initialises two
// mbarriers, completes the phase of the first itself and leaves the second
// untouched; it then waits on both with a small poll limit and reports what
// each wait returned.  Nothing faults, traps or spins without bound: the
// unsignalled wait gives up after `polls` polls.
#include <cuda_runtime.h>

#include "cf.h"
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
