// lowrank_umma.cuh -- tcgen05 (5th-generation tensor core) kernels for the two
// dense products of subspace iteration:
//   project:     Yp[s] = Vb[tok block, channel split s] . Qt[:, split s]^T
//                M = 128 tokens, N = rp, K = channels (K-major A and B)
//   backproject: Zp[s] = Vb[token split s, ch block]^T . Pt[:, split s]^T
//                M = 128 channels, N = rp, K = tokens (A is MN-major: V is
//                stored token-major and the reduction runs over tokens)
//
// One CTA of 4 warps per output tile and K split:
//   warp 0, one lane : TMA producer (cp.async.bulk.tensor, no multicast) into
//                      a 4-stage ring of 128-byte-swizzled shared tiles
//   warp 1           : allocates TMEM; one lane issues tcgen05.mma
//                      (kind::f16, bf16 in, fp32 accumulate in TMEM) and
//                      tcgen05.commit releases each stage
//   all 4 warps      : epilogue, tcgen05.ld 32 lanes x rp columns per warp,
//                      one output row per thread, 16-byte stores
// Every mbarrier wait is bounded; on expiry the kernel records
// CF_ERR_TIMEOUT in the status word, stops issuing work, frees its TMEM and
// returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "cf.h"
#include "lowrank_api.cuh"

namespace cf {
namespace umma {

constexpr int kStages = 4;
constexpr int kBK = 64;                 // K elements per stage (128 B of bf16)
constexpr int kTileBytesA = 128 * kBK * 2;  // 16 KB
constexpr uint32_t kWaitLimit = 1u << 22;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the completion of phase `parity`; false on expiry.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// 3-D tile load: coordinates (x, y) inside buffer z of a [buffers][rows][cols]
// map whose buffer stride is the per-buffer workspace stride.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int32_t x, int32_t y, int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor (sm_100 layout): start address, leading and
// stride byte offsets (all >> 4), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo_bytes,
                                               uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;   // version
    d |= (uint64_t)2 << 61;   // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool a_mn_major) {
    return (1u << 4)                       // D format f32
           | (1u << 7)                     // A format bf16
           | (1u << 10)                    // B format bf16
           | ((a_mn_major ? 1u : 0u) << 15)  // A major
           | ((uint32_t)(n >> 3) << 17)    // N / 8
           | ((uint32_t)(128 >> 4) << 24);  // M / 16
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 TMEM lanes x 16 columns of fp32 into 16 registers of this thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    // the wait takes the destination registers as operands, so no use of
    // them can be scheduled above it
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared tile geometry of one stage.  A: 16 KB; B: rp rows x 128 B.
template <int BN>
struct StageGeom {
    static constexpr int kBytesB = BN * kBK * 2;
    static constexpr int kBytes = kTileBytesA + kBytesB;
    static constexpr int kSmem = kStages * kBytes + 1024 /*align slack*/ + 256 /*barriers*/;
    static constexpr uint32_t kTmemCols = BN <= 32 ? 32 : 64;
};

// Common CTA skeleton.  A_MN: A operand is MN-major (backproject).
//   rows0      : first output row of this tile (token for project, channel
//                for backproject); TMA y (project) / x (backproject) base
//   kbeg, nkb  : first K element of this split and number of 64-wide blocks
template <int BN, bool A_MN>
__device__ __forceinline__ void gemm_tile(const CUtensorMap *mapA, const CUtensorMap *mapB,
                                          int32_t rows0, int32_t kbeg, int nkb, int32_t zb,
                                          float *out, int64_t out_rows, int32_t *status) {
    using G = StageGeom<BN>;
    extern __shared__ uint8_t dsmem[];
    const uint32_t base = (smem_u32(dsmem) + 1023u) & ~1023u;
    uint8_t *gbase = dsmem + (base - smem_u32(dsmem));
    const uint32_t bars = base + kStages * G::kBytes;  // full[S], empty[S], done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + kStages * G::kBytes + 8 * (2 * kStages + 1));
    __shared__ int failed;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto full = [&](int s) { return bars + 8u * s; };
    auto empty = [&](int s) { return bars + 8u * (kStages + s); };
    const uint32_t done = bars + 8u * (2 * kStages);

    if (threadIdx.x == 0) {
        failed = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(G::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // producer
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % kStages;
            const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
            if (!mbar_wait(empty(s), ph ^ 1u)) {
                atomicExch(&failed, 1);
                break;
            }
            if (*(volatile int *)&failed) break;
            const uint32_t sa = base + s * G::kBytes;
            const uint32_t sb = sa + kTileBytesA;
            mbar_expect_tx(full(s), (uint32_t)G::kBytes);
            const int32_t k = kbeg + kb * kBK;
            if (!A_MN) {
                tma_load_3d(sa, mapA, full(s), k, rows0, zb);      // box {64 ch, 128 tok, 1}
            } else {
                tma_load_3d(sa, mapA, full(s), rows0, k, zb);      // box {64 ch, 64 tok, 1}
                tma_load_3d(sa + kTileBytesA / 2, mapA, full(s), rows0 + 64, k, zb);
            }
            tma_load_3d(sb, mapB, full(s), k, 0, zb);              // box {64 k, BN rows, 1}
        }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer
        constexpr uint32_t idesc = idesc_bf16(BN, A_MN);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % kStages;
            const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
            if (!mbar_wait(full(s), ph)) {
                atomicExch(&failed, 1);
                ok = false;
                break;
            }
            fence_after_sync();
            const uint32_t sa = base + s * G::kBytes;
            const uint32_t sb = sa + kTileBytesA;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
                // K-major: 16 elements = 32 B further along the swizzled row.
                // MN-major: 16 K rows = two 8-row atoms of 1 KB.
                const uint64_t da = A_MN ? sw128_desc(sa + kk * 2048u, kTileBytesA / 2, 1024)
                                         : sw128_desc(sa + kk * 32u, 16, 1024);
                const uint64_t db = sw128_desc(sb + kk * 32u, 16, 1024);
                mma_bf16(tmem, da, db, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(empty(s));
        }
        if (ok) mma_commit(done);
    }

    // Epilogue: TMEM lane i of warp w holds output row rows0 + 32 w + i.
    __syncwarp();
    bool have = false;
    if (lane == 0) have = mbar_wait(done, 0) && !*(volatile int *)&failed;
    have = __shfl_sync(0xffffffffu, have ? 1 : 0, 0) != 0;
    if (nkb > 0 && have) {
        fence_after_sync();
        const int64_t row = (int64_t)rows0 + warp * 32 + lane;
        const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll
        for (int c = 0; c < BN; c += 16) {
            float v[16];
            tmem_ld16(taddr + c, v);
            if (row < out_rows) {
                float4 *dst = reinterpret_cast<float4 *>(out + row * BN + c);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
    } else if (nkb > 0 && lane == 0 && status) {
        atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(G::kTmemCols)
                     : "memory");
    }
}

// Yp[split][t][0..BN) of buffer blockIdx.z for the token block blockIdx.x and
// channel split blockIdx.y.
template <int BN>
__global__ void __launch_bounds__(128, 1)
project_kernel(const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapQt,
               const cf_lowrank::LrBatch B, const cf_lowrank::Layout L) {
    const int bz = blockIdx.z;
    if (B.at<int32_t>(bz, L.off_status)[cf_lowrank::kSkipWord]) return;
    const int32_t t0 = blockIdx.x * 128;
    const int64_t kb = (int64_t)blockIdx.y * cf_lowrank::kChunkA;
    const int64_t ke = (kb + cf_lowrank::kChunkA < L.C) ? kb + cf_lowrank::kChunkA : L.C;
    const int nkb = (int)((ke - kb + kBK - 1) / kBK);
    float *yp = B.at<float>(bz, L.off_yp) + (int64_t)blockIdx.y * L.T * BN;
    gemm_tile<BN, false>(&mapV, &mapQt, t0, (int32_t)kb, nkb, bz, yp, L.T,
                         B.at<int32_t>(bz, L.off_status) + cf_lowrank::kStatusWord);
}

// Zp[split][c][0..BN) of buffer blockIdx.z for the channel block blockIdx.x
// and token split blockIdx.y.
template <int BN>
__global__ void __launch_bounds__(128, 1)
backproject_kernel(const __grid_constant__ CUtensorMap mapVt, const __grid_constant__ CUtensorMap mapPt,
                   const cf_lowrank::LrBatch B, const cf_lowrank::Layout L) {
    const int bz = blockIdx.z;
    if (B.at<int32_t>(bz, L.off_status)[cf_lowrank::kSkipWord]) return;
    const int32_t c0 = blockIdx.x * 128;
    const int64_t kb = (int64_t)blockIdx.y * cf_lowrank::kChunkB;
    const int64_t ke = (kb + cf_lowrank::kChunkB < L.T) ? kb + cf_lowrank::kChunkB : L.T;
    const int nkb = (int)((ke - kb + kBK - 1) / kBK);
    float *zp = B.at<float>(bz, L.off_zp) + (int64_t)blockIdx.y * L.C * BN;
    gemm_tile<BN, true>(&mapVt, &mapPt, c0, (int32_t)kb, nkb, bz, zp, L.C,
                        B.at<int32_t>(bz, L.off_status) + cf_lowrank::kStatusWord);
}

}  // namespace umma
}  // namespace cf
