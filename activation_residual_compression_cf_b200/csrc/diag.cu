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
// Longest row the staged reference accepts (two 6C-byte slots fit in
// shared memory; rows longer than 15360 channels need more than 480
// consumer threads and are refused as unsupported).
constexpr int64_t kMixTmaMaxC = 16384;

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

// 1-D bulk copy global -> shared (no multicast) completing on an mbarrier;
// both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void mix_bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void mix_bulk_s2g(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}

// The same byte mix moved by the encode's own memory pipeline: a producer
// lane bulk-copies each row's x (bf16, 2C bytes) and r (fp32, 4C bytes) into
// a ring of shared-memory slots (no multicast); consumer warps read the row
// from shared memory, release the slot and form a = (float)x - r and
// r = (float)x + r, GPT groups of 8 channels per thread.  BULK = false:
// they write a and r with streaming 16-byte stores.  BULK = true (the
// standard encode's store path): they write them into one of two
// shared-memory output rows, and one thread has the copy engine store the
// row after the next row's barrier (every consumer passes a barrier per
// row, as the encode's do for the scale); before that barrier it waits
// until the previous store has read its output row.  None of the encode's
// per-row work (scale, quantisation, codes).  Every mbarrier wait is
// bounded: on expiry the status word gets CF_ERR_TIMEOUT and the CTA's
// consumers leave together at the next barrier (BULK) or each warp leaves
// (otherwise).
template <int GPT, bool BULK>
__global__ void __launch_bounds__(512) diag_stream_mix_tma_kernel(const uint16_t *x, float *r, float *a,
                                                                  int64_t rows, int64_t C, int stages,
                                                                  int32_t *status) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int abort_row[2];   // BULK: set before a row's barrier, read after it
    const int64_t G = C >> 3;
    const uint32_t slot = (uint32_t)(6 * C);
    const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const uint32_t obytes = BULK ? (uint32_t)(8 * C) : 0u;   // output row: a (4C) then r (4C)
    const uint32_t obase = base + (uint32_t)stages * slot;
    const uint32_t bars = obase + 2u * obytes;
    const int tid = threadIdx.x;
    const int nc = blockDim.x - 32;
    if (tid == 0) {
        abort_row[0] = abort_row[1] = 0;
        for (int s = 0; s < stages; ++s) {
            cf::mbar_init(bars + 8u * s, 1);
            cf::mbar_init(bars + 8u * (stages + s), (uint32_t)(nc / 32));
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (tid < 32) {
        if (tid != 0) return;
        int i = 0;
        for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
            const int s = i % stages;
            const uint32_t ph = (uint32_t)(i / stages) & 1u;
            if (!cf::mbar_wait(bars + 8u * (stages + s), ph ^ 1u)) {
                if (status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
                return;
            }
            if (!CF_IN(row < rows && s < stages)) continue;
            const uint32_t dst = base + (uint32_t)s * slot;
            cf::mbar_expect_tx(bars + 8u * s, slot);
            mix_bulk_g2s(dst, x + row * C, (uint32_t)(2 * C), bars + 8u * s);
            mix_bulk_g2s(dst + (uint32_t)(2 * C), r + row * C, (uint32_t)(4 * C), bars + 8u * s);
            ++i;
        }
        return;
    }
    const int ct = tid - 32, lane = ct & 31;
    int i = 0, par = 0, orow = 0;
    float *pend_a = nullptr, *pend_r = nullptr;   // BULK, thread ct 0: the row waiting in output row pend_o
    int pend_o = 0;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        const int s = i % stages;
        const uint32_t ph = (uint32_t)(i / stages) & 1u;
        bool ok = true;
        if (lane == 0) ok = cf::mbar_wait(bars + 8u * s, ph);
        ok = __shfl_sync(cf::kFullMask, ok ? 1 : 0, 0) != 0;
        if (!ok) {
            if (lane == 0 && status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
            if constexpr (!BULK) return;
            if (lane == 0) abort_row[par] = 1;   // acted on after the barrier
        }
        const uint8_t *sx = smem + (size_t)s * slot;
        const float *sr = reinterpret_cast<const float *>(sx + 2 * C);
        float f[GPT][8], rr[GPT][8];
#pragma unroll
        for (int j = 0; j < GPT; ++j) {
            const int64_t g = (int64_t)j * nc + ct;
            if (ok && g < G && CF_IN(8 * g + 8 <= C)) {
                const uint4 xw = *reinterpret_cast<const uint4 *>(sx + 16 * g);
                const float4 p0 = *reinterpret_cast<const float4 *>(sr + 8 * g);
                const float4 p1 = *reinterpret_cast<const float4 *>(sr + 8 * g + 4);
                const uint32_t w[4] = {xw.x, xw.y, xw.z, xw.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) f[j][e] = cf::bf16_bits_to_f32((w[e >> 1] >> ((e & 1) * 16)) & 0xffffu);
                rr[j][0] = p0.x; rr[j][1] = p0.y; rr[j][2] = p0.z; rr[j][3] = p0.w;
                rr[j][4] = p1.x; rr[j][5] = p1.y; rr[j][6] = p1.z; rr[j][7] = p1.w;
            }
        }
        // the slot is no longer read (generic-proxy reads before the next
        // async-proxy bulk write into it)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0 && ok) cf::mbar_arrive(bars + 8u * (stages + s));
        ++i;
        float *ar = a + row * C, *rw = r + row * C;
        float *oa = nullptr, *orr = nullptr;
        if constexpr (BULK) {
            if (ct == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            asm volatile("bar.sync 1, %0;" ::"r"(nc) : "memory");
            if (*(volatile int *)&abort_row[par]) {
                if (ct == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
                return;   // every consumer warp sees the same flag here
            }
            par ^= 1;
            if (ct == 0 && pend_a) {
                const uint32_t ob = obase + (uint32_t)(pend_o & 1) * obytes;
                mix_bulk_s2g(pend_a, ob, (uint32_t)(4 * C));
                mix_bulk_s2g(pend_r, ob + (uint32_t)(4 * C), (uint32_t)(4 * C));
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
            oa = reinterpret_cast<float *>(smem + (size_t)stages * slot + (size_t)(orow & 1) * obytes);
            orr = oa + C;
        }
#pragma unroll
        for (int j = 0; j < GPT; ++j) {
            const int64_t g = (int64_t)j * nc + ct;
            if (g >= G || !CF_IN(8 * g + 8 <= C)) continue;
            float d[8], t[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                d[e] = __fsub_rn(f[j][e], rr[j][e]);
                t[e] = __fadd_rn(f[j][e], rr[j][e]);
            }
            if constexpr (BULK) {
                *reinterpret_cast<float4 *>(oa + 8 * g) = make_float4(d[0], d[1], d[2], d[3]);
                *reinterpret_cast<float4 *>(oa + 8 * g + 4) = make_float4(d[4], d[5], d[6], d[7]);
                *reinterpret_cast<float4 *>(orr + 8 * g) = make_float4(t[0], t[1], t[2], t[3]);
                *reinterpret_cast<float4 *>(orr + 8 * g + 4) = make_float4(t[4], t[5], t[6], t[7]);
            } else {
                cf::st_stream_v4(ar + 8 * g, make_float4(d[0], d[1], d[2], d[3]));
                cf::st_stream_v4(ar + 8 * g + 4, make_float4(d[4], d[5], d[6], d[7]));
                cf::st_stream_v4(rw + 8 * g, make_float4(t[0], t[1], t[2], t[3]));
                cf::st_stream_v4(rw + 8 * g + 4, make_float4(t[4], t[5], t[6], t[7]));
            }
        }
        if constexpr (BULK) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            if (ct == 0) {
                pend_a = ar;
                pend_r = rw;
                pend_o = orow;
            }
            ++orow;
        }
    }
    if constexpr (BULK) {
        // the last row's outputs: every consumer has written its part
        asm volatile("bar.sync 1, %0;" ::"r"(nc) : "memory");
        if (ct == 0) {
            if (pend_a) {
                const uint32_t ob = obase + (uint32_t)(pend_o & 1) * obytes;
                mix_bulk_s2g(pend_a, ob, (uint32_t)(4 * C));
                mix_bulk_s2g(pend_r, ob + (uint32_t)(4 * C), (uint32_t)(4 * C));
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
            asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
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

extern "C" cf_status cf_diag_stream_mix_tma(const uint16_t *x, float *r, float *a, int64_t rows, int64_t C,
                                             int32_t bulk, int32_t *status_dev, void *stream) {
    cf::TraceRange trace_("cf_diag_stream_mix_tma");
    if (rows < 0 || C < 8 || C % 8 != 0 || C > kMixTmaMaxC || (bulk != 0 && bulk != 1)) return CF_ERR_INVALID_ARG;
    if (rows == 0) return CF_OK;
    if (!x || !r || !a) return CF_ERR_INVALID_ARG;
    if (((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(r) | reinterpret_cast<uintptr_t>(a)) &
         15u) != 0 ||
        (reinterpret_cast<uintptr_t>(status_dev) & 3u) != 0)
        return CF_ERR_ALIGNMENT;
    // the encode's launch shapes: per-thread stores with 2 groups of 8
    // channels per consumer thread (4 where that keeps the CTA within 512
    // threads) and a ring of up to 4 slots of 6C bytes; bulk stores with 4
    // groups, 2 slots and two 8C-byte output rows
    const int64_t G = C / 8;
    int gpt = bulk ? 4 : 2;
    int64_t nc = ((G + gpt - 1) / gpt + 31) / 32 * 32;
    if (nc > 480) {
        gpt = 4;
        nc = ((G + gpt - 1) / gpt + 31) / 32 * 32;
    }
    if (nc > 480) return CF_ERR_UNSUPPORTED;
    const int64_t slot = 6 * C;
    int stages = bulk ? 2 : (int)(120000 / slot);
    if (stages > 4) stages = 4;
    if (stages < 2) stages = 2;
    const size_t smem = (size_t)stages * slot + (bulk ? 16 * (size_t)C : 0) + 16 * (size_t)stages;
    if (smem > 227 * 1024) return CF_ERR_UNSUPPORTED;
    void (*k)(const uint16_t *, float *, float *, int64_t, int64_t, int, int32_t *) =
        bulk ? (gpt == 2 ? diag_stream_mix_tma_kernel<2, true> : diag_stream_mix_tma_kernel<4, true>)
             : (gpt == 2 ? diag_stream_mix_tma_kernel<2, false> : diag_stream_mix_tma_kernel<4, false>);
    const int threads = (int)nc + 32;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return CF_ERR_CUDA;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, threads, smem) != cudaSuccess || occ < 1) {
        (void)cudaGetLastError();
        occ = 1;
    }
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t grid = (int64_t)sms * occ;
    if (grid > rows) grid = rows;
    k<<<(unsigned)grid, threads, smem, (cudaStream_t)stream>>>(x, r, a, rows, C, stages, status_dev);
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
