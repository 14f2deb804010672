// lowrank_noalloc.cu -- the low-rank sender for callers that cannot allocate
// device memory.
//
// cf_lowrank_encode needs a scratch workspace that its caller allocates.
// Some callers have no way to do that at the point where they compress: a
// plug-in or hook that runs inside a host framework which owns every device
// allocation through its own pool and hands the plug-in no allocator; a
// serving loop that must not call cudaMalloc mid-step because the call can
// synchronise the device and stall every stream; a small C host that links
// only this library.  For them this file keeps the scratch in one
// file-scope device array of fixed size and passes its device address to the
// same implementation cf_lowrank_encode uses, so nothing is allocated per
// call and no allocating routine is called.
//
// Host code must not pass the array's name to a kernel: on the host that
// name is only a stand-in for the symbol, not a device address.  The device
// address is looked up once per device with cudaGetSymbolAddress, with that
// device current, on the first call made on it, and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "cf.h"
#include "lowrank_api.cuh"

namespace {

// Shared by every call on a device; holds the previous call's contents.
static __device__ __align__(256) unsigned char g_noalloc_scratch[CF_LOWRANK_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

cf_status noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return CF_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return CF_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            (void)cudaGetLastError();
            return CF_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return CF_OK;
}

}  // namespace

extern "C" cf_status cf_lowrank_encode_noalloc(const cf_desc *d, const uint16_t *x,
                                               float *recon_s, float *err, const float *omega,
                                               uint8_t *p_codes, float *p_scales,
                                               uint8_t *q_codes, float *q_scales, void *stream) {
    const cf_status ds = cf_lowrank::check_desc(d);
    if (ds != CF_OK) return ds;
    if (!omega) return CF_ERR_INVALID_ARG;
    const int64_t need = cf_lowrank_workspace_bytes(d);
    if (need <= 0 || (uint64_t)need > (uint64_t)CF_LOWRANK_NOALLOC_SCRATCH_BYTES)
        return CF_ERR_WORKSPACE;
    void *ws = nullptr;
    const cf_status ss = noalloc_scratch(&ws);
    if (ss != CF_OK) return ss;
    return cf_lowrank_encode(d, x, recon_s, err, omega, p_codes, p_scales, q_codes, q_scales, ws,
                             (size_t)CF_LOWRANK_NOALLOC_SCRATCH_BYTES, stream);
}
