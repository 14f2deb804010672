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
#include "cf_common.cuh"
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

// A reference for the encode's byte mix: a plain streaming pass that
// reads a bf16 array x and an fp32 array r and writes two fp32 arrays,
// a = (float)x - r and r = (float)x + r (6 bytes read, 8 written per
// element, as the encode reads x and recon and writes err and recon).
// Each thread takes kMixUnroll groups of 8 elements a grid stride apart and
// issues all their loads before any store.
constexpr int kMixUnroll = 4;

__global__ void __launch_bounds__(128) diag_stream_mix_kernel(const uint4 *x, float4 *r, float4 *a,
                                                              int64_t n8) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < n8; i0 += stride * kMixUnroll) {
        uint4 xv[kMixUnroll];
        float4 r0[kMixUnroll], r1[kMixUnroll];
#pragma unroll
        for (int k = 0; k < kMixUnroll; ++k) {
            const int64_t i = i0 + k * stride;
            if (i < n8 && CF_IN(2 * i + 1 < 2 * n8)) {
                xv[k] = cf::ld_ro_v4(x + i);
                r0[k] = cf::ld_state_v4(reinterpret_cast<const float *>(r + 2 * i));
                r1[k] = cf::ld_state_v4(reinterpret_cast<const float *>(r + 2 * i + 1));
            }
        }
#pragma unroll
        for (int k = 0; k < kMixUnroll; ++k) {
            const int64_t i = i0 + k * stride;
            if (i >= n8 || !CF_IN(2 * i + 1 < 2 * n8)) break;
            const uint32_t w[4] = {xv[k].x, xv[k].y, xv[k].z, xv[k].w};
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = cf::bf16_bits_to_f32((w[e >> 1] >> ((e & 1) * 16)) & 0xffffu);
            const float rr[8] = {r0[k].x, r0[k].y, r0[k].z, r0[k].w, r1[k].x, r1[k].y, r1[k].z, r1[k].w};
            float d[8], s[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                d[e] = __fsub_rn(f[e], rr[e]);
                s[e] = __fadd_rn(f[e], rr[e]);
            }
            cf::st_stream_v4(reinterpret_cast<float *>(a + 2 * i), make_float4(d[0], d[1], d[2], d[3]));
            cf::st_stream_v4(reinterpret_cast<float *>(a + 2 * i + 1), make_float4(d[4], d[5], d[6], d[7]));
            cf::st_state_v4(reinterpret_cast<float *>(r + 2 * i), make_float4(s[0], s[1], s[2], s[3]));
            cf::st_state_v4(reinterpret_cast<float *>(r + 2 * i + 1), make_float4(s[4], s[5], s[6], s[7]));
        }
    }
}

}  // namespace

extern "C" cf_status cf_diag_stream_mix(const uint16_t *x, float *r, float *a, int64_t n, void *stream) {
    cf::TraceRange trace_("cf_diag_stream_mix");
    if (n < 0 || n % 8 != 0) return CF_ERR_INVALID_ARG;
    if (n == 0) return CF_OK;
    if (!x || !r || !a) return CF_ERR_INVALID_ARG;
    if (((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(r) | reinterpret_cast<uintptr_t>(a)) &
         15u) != 0)
        return CF_ERR_ALIGNMENT;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // 16 CTAs of 128 threads per SM (the best of the launch shapes measured
    // on B200 for this pass), capped by the work
    int64_t blocks = (int64_t)sms * 16;
    const int64_t need = (n / 8 + 127) / 128;
    if (blocks > need) blocks = need;
    diag_stream_mix_kernel<<<(unsigned)blocks, 128, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const uint4 *>(x), reinterpret_cast<float4 *>(r), reinterpret_cast<float4 *>(a), n / 8);
    return cudaGetLastError() == cudaSuccess ? CF_OK : CF_ERR_CUDA;
}

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
