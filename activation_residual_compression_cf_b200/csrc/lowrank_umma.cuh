// lowrank_umma.cuh -- tcgen05 (5th-generation tensor core) kernels for the two
// dense products of subspace iteration:
//   project:     Y[tok tile] = Vb[tok tile, :] . Qt^T
//                M = 128 tokens, N = rp, K = all channels (K-major A and B)
//   backproject: Q[ch block] = Vb[:, ch block]^T . Pt^T
//                M = 128 channels, N = rp, K = all tokens (A is MN-major: V
//                is stored token-major and the reduction runs over tokens)
// Each CTA accumulates its whole K range in TMEM (no split-K), so its rows
// are final when the MMAs end: the projection's tail forms the tile's
// partial Gram and the buffer's last tile factors G; the back-projection's
// tail writes the bf16 transpose and the column maxima.
//
// One CTA of 4 warps per output tile:
//   warp 0, one lane : TMA producer (cp.async.bulk.tensor, no multicast) into
//                      a 3-stage ring of 128-byte-swizzled shared tiles
//                      (three CTAs per SM: measured on B200, 3 stages beat
//                      4 at two CTAs per SM and 6-8 at one)
//   warp 1           : allocates TMEM; one lane issues tcgen05.mma
//                      (kind::f16, bf16 in, fp32 accumulate in TMEM) and
//                      tcgen05.commit releases each stage
//   all 4 warps      : epilogue, tcgen05.ld 32 lanes x rp columns per warp,
//                      one output row per thread, 16-byte stores
// The first projection of an encode has its own kernel
// (project_residual_kernel, below) that forms Vb from x and recon itself.
// Every mbarrier wait is bounded; on expiry the kernel records
// CF_ERR_TIMEOUT in the status word, stops issuing work, frees its TMEM and
// returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "bounds.cuh"
#include "cf.h"
#include "lowrank_api.cuh"
#include "lowrank_kernels.cuh"
#include "mbar.cuh"

namespace cf {
namespace umma {

constexpr int kStages = 3;               // ring depth of the plain projections
constexpr int kBK = 64;                 // K elements per stage (128 B of bf16)
constexpr int kTileBytesA = 128 * kBK * 2;  // 16 KB

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
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
//   kbeg, nkb  : first K element and number of 64-wide K blocks
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
            if (row < out_rows && CF_IN(row >= 0 && c + 16 <= BN)) {
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

// Tail of the projection Y = Vb Q, run after a CTA has written the complete
// Y rows of token tile `tile` (all channels in one accumulation): the
// tile's fp64 partial Gram Y_tile^T Y_tile (upper triangle, rows in order);
// the last tile of the buffer to finish (per-buffer ticket) sums the partial
// Grams in tile order and factors G = R^T R.  Every sum runs in a fixed
// order, so the result does not depend on which CTA finishes last.  (A
// reduction whose order varied from run to run would be amplified by the
// bf16 operand roundings of later iterations into visible differences.)
// A pivot not above 1e-10 of its original diagonal entry marks the column
// dead: its row of R and its inverse diagonal are zero (P gets a zero
// column) and CF_ERR_NUMERIC is recorded.  Output: R (fp32 [rp][rp], upper)
// and 1/diag(R) (fp32 [rp], 0 where dead).  The ticket is reset by its last
// user.  The pipeline's shared memory is reused: every stage has been
// consumed once the tile's product is done.
// The tail runs on the first 128 threads of the CTA (all of them in the
// plain projection, the four converter warps in the fused one).
__device__ __forceinline__ void tail_sync() {
    asm volatile("bar.sync 3, 128;" ::: "memory");
}

template <int BN>
__device__ __forceinline__ void project_tail(const cf_lowrank::LrBatch &B, const cf_lowrank::Layout &L,
                                             int bz, int tile) {
    extern __shared__ uint8_t dsmem[];
    const uint32_t base = (smem_u32(dsmem) + 1023u) & ~1023u;
    uint8_t *gbase = dsmem + (base - smem_u32(dsmem));
    // Y tile in shared memory, fp32, row pitch BN + 8 words so that the
    // 4 x 8 fragment reads below fall in 32 distinct banks
    constexpr int LDY = BN + 8;
    constexpr int kYsBytes = (128 * LDY * 4 + 255) & ~255;
    static_assert(kYsBytes + BN * (BN + 1) * 8 <= kStages * StageGeom<BN>::kBytes, "tail scratch");
    float *ys = reinterpret_cast<float *>(gbase);                 // [128][LDY] Y of the tile
    double *A = reinterpret_cast<double *>(gbase + kYsBytes);     // [BN][BN + 1] G, then R
    __shared__ double gdiag[64], invd[64];
    __shared__ double rowbuf[2][33];
    __shared__ int dead[64];
    __shared__ int is_last;
    const int tid = threadIdx.x;

    // this thread's Y row (written by this thread in the epilogue)
    const int64_t T = L.T;
    const int64_t t = (int64_t)tile * 128 + tid;
    if (t < T) {
        const float4 *yr = reinterpret_cast<const float4 *>(B.at<float>(bz, L.off_y) + t * BN);
#pragma unroll
        for (int q = 0; q < BN / 4; ++q)
            *reinterpret_cast<float4 *>(ys + tid * LDY + 4 * q) = yr[q];
    } else {
#pragma unroll
        for (int q = 0; q < BN / 4; ++q)
            *reinterpret_cast<float4 *>(ys + tid * LDY + 4 * q) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    tail_sync();

    // The tile's partial Gram Y^T Y on the fp64 tensor path (mma.sync
    // m8n8k4 f64; tcgen05 has no fp64 kind): 8 x 8 output blocks (I, J),
    // I <= J, dealt to the 4 warps round robin; each warp runs its blocks'
    // accumulators side by side over the 128 rows, 4 rows per step.  The
    // fp32 values are exact in fp64, so every product is exact and only the
    // fp64 sums round.  A fragment: A[i][k] = Y[k][8I + i] (i = lane / 4,
    // k = lane % 4); B fragment: B[k][j] = Y[k][8J + j] (k = lane % 4,
    // j = lane / 4); D: row lane / 4, columns 2 (lane % 4) + {0, 1}.
    {
        constexpr int NB = BN / 8;
        constexpr int NU = NB * (NB + 1) / 2;
        constexpr int MT = (NU + 3) / 4;               // blocks per warp, at most
        const int warp = tid >> 5, lane = tid & 31;
        const int fr = lane >> 2, fk = lane & 3;
        int bi[MT], bj[MT];
        double acc[MT][2];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            int u = warp + 4 * m, I = 0;
            while (u >= NB - I && I < NB) { u -= NB - I; ++I; }  // u-th upper block, row-major
            bi[m] = I < NB ? I : -1;
            bj[m] = I < NB ? I + u : -1;
            acc[m][0] = acc[m][1] = 0.0;
        }
#pragma unroll 2
        for (int k0 = 0; k0 < 128; k0 += 4) {
            const float *row = ys + (k0 + fk) * LDY;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (bi[m] < 0) continue;
                const double a = (double)row[8 * bi[m] + fr];
                const double b = (double)row[8 * bj[m] + fr];
                asm volatile(
                    "mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                    : "+d"(acc[m][0]), "+d"(acc[m][1])
                    : "d"(a), "d"(b));
            }
        }
        double *gpt = B.at<double>(bz, L.off_gp) + (int64_t)tile * BN * BN;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (bi[m] < 0) continue;
            const int i = 8 * bi[m] + fr;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int j = 8 * bj[m] + 2 * fk + c;
                if (i <= j) gpt[i * BN + j] = acc[m][c];
            }
        }
    }
    double *gp = B.at<double>(bz, L.off_gp);
    __threadfence();
    tail_sync();
    uint32_t *fin = B.at<uint32_t>(bz, L.off_status) + cf_lowrank::kTicketWord;
    if (tid == 0) is_last = atomicAdd(fin, 1u) == (uint32_t)(L.nTileT - 1) ? 1 : 0;
    tail_sync();
    if (!is_last) return;
    __threadfence();

    // G = sum of the tiles' partial Grams in tile order (8 loads in flight)
    const int ld = BN + 1, r = L.r, ntile = L.nTileT;
    for (int e = tid; e < BN * BN; e += 128) {
        const int i = e / BN, j = e - (e / BN) * BN;
        if (i > j) continue;
        double a[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
        int g = 0;
        for (; g + 8 <= ntile; g += 8) {
#pragma unroll
            for (int u = 0; u < 8; ++u) a[u] += __ldcg(gp + (int64_t)(g + u) * BN * BN + e);
        }
        for (; g < ntile; ++g) a[0] += __ldcg(gp + (int64_t)g * BN * BN + e);
        const double v = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
        A[i * ld + j] = v;
        if (i == j) gdiag[i] = v;
    }
    tail_sync();
    if (BN <= 32) {
        quad_cholesky(A, ld, r, gdiag, dead, invd, rowbuf);   // all 128 threads
    } else if (tid < 32) {
        warp_cholesky_smem(A, ld, r, gdiag, dead, invd);
    }
    tail_sync();
    float *rmat = B.at<float>(bz, L.off_rmat);
    float *rinvd = rmat + BN * BN;
    int nd = 0;
    for (int e = tid; e < BN * BN; e += 128) {
        const int i = e / BN, c = e - (e / BN) * BN;
        rmat[e] = (i <= c && c < r) ? (float)A[i * ld + c] : 0.0f;
    }
    for (int j = tid; j < BN; j += 128) {
        const bool live = j < r && !dead[j];
        rinvd[j] = live ? (float)invd[j] : 0.0f;
        nd += (j < r && dead[j]) ? 1 : 0;
    }
    if (nd) atomicCAS(B.at<int32_t>(bz, L.off_status) + cf_lowrank::kStatusWord, (int32_t)CF_OK,
                      (int32_t)CF_ERR_NUMERIC);
    if (tid == 0) *fin = 0u;
}

// Tail of the back-projection Q = Vb^T P for channel block `cblk`, run after
// the CTA has written the block's complete Q rows (all tokens in one
// accumulation): the bf16 transpose Qt [rp][C] for the next projection and,
// on the last iteration, max |Q[:, k]| folded into the column maxima (float
// bits, atomicMax).
template <int BN>
__device__ __forceinline__ void backproject_tail(const cf_lowrank::LrBatch &B, const cf_lowrank::Layout &L,
                                                 int bz, int cblk, int want_amax) {
    __shared__ float Wm[4][BN];
    const int tid = threadIdx.x;
    const int64_t C = L.C;
    const int64_t c = (int64_t)cblk * 128 + tid;
    float v[BN];
    if (c < C) {
        const float4 *qr = reinterpret_cast<const float4 *>(B.at<float>(bz, L.off_q) + c * BN);
#pragma unroll
        for (int q = 0; q < BN / 4; ++q) {
            const float4 z = qr[q];
            v[4 * q] = z.x;
            v[4 * q + 1] = z.y;
            v[4 * q + 2] = z.z;
            v[4 * q + 3] = z.w;
        }
        bf16 *qt = B.at<bf16>(bz, L.off_qt);
#pragma unroll
        for (int k = 0; k < BN; ++k)
            if (CF_IN((int64_t)k * C + c < (int64_t)L.rp * C)) qt[(int64_t)k * C + c] = __float2bfloat16_rn(v[k]);
    } else {
#pragma unroll
        for (int k = 0; k < BN; ++k) v[k] = 0.0f;
    }
    if (want_amax) {
        const int warp = tid >> 5, lane = tid & 31;
#pragma unroll
        for (int k = 0; k < BN; ++k) {
            float m = fabsf(v[k]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) Wm[warp][k] = m;
        }
        __syncthreads();
        uint32_t *amax = B.at<uint32_t>(bz, L.off_amax) + BN;
        for (int k = tid; k < BN; k += 128) {
            const float m = fmaxf(fmaxf(Wm[0][k], Wm[1][k]), fmaxf(Wm[2][k], Wm[3][k]));
            atomicMax(amax + k, __float_as_uint(m));
        }
    }
}

// Y[t][0..BN) of buffer blockIdx.z for the token tile blockIdx.x, over all
// channels, then the tile's share of G and R (above).
template <int BN>
__global__ void __launch_bounds__(128, 1)
project_kernel(const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapQt,
               const cf_lowrank::LrBatch B, const cf_lowrank::Layout L) {
    const int bz = blockIdx.z;
    if (B.at<int32_t>(bz, L.off_status)[cf_lowrank::kSkipWord]) return;
    const int32_t t0 = blockIdx.x * 128;
    const int nkb = (int)((L.C + kBK - 1) / kBK);
    gemm_tile<BN, false>(&mapV, &mapQt, t0, 0, nkb, bz, B.at<float>(bz, L.off_y), L.T,
                         B.at<int32_t>(bz, L.off_status) + cf_lowrank::kStatusWord);
    project_tail<BN>(B, L, bz, blockIdx.x);
}

// Q[c][0..BN) of buffer blockIdx.z for the channel block blockIdx.x, over
// all tokens, then the block's Qt and column maxima (above).
template <int BN>
__global__ void __launch_bounds__(128, 1)
backproject_kernel(const __grid_constant__ CUtensorMap mapVt, const __grid_constant__ CUtensorMap mapPt,
                   const cf_lowrank::LrBatch B, const cf_lowrank::Layout L, int want_amax) {
    const int bz = blockIdx.z;
    if (B.at<int32_t>(bz, L.off_status)[cf_lowrank::kSkipWord]) return;
    const int32_t c0 = blockIdx.x * 128;
    const int nkb = (int)((L.T + kBK - 1) / kBK);
    gemm_tile<BN, true>(&mapVt, &mapPt, c0, 0, nkb, bz, B.at<float>(bz, L.off_q), L.C,
                        B.at<int32_t>(bz, L.off_status) + cf_lowrank::kStatusWord);
    backproject_tail<BN>(B, L, bz, blockIdx.x, want_amax);
}

// First projection of an encode, fused with the residual: Y = Vb Q with
// Vb = bf16((float)x - recon) formed here from the caller's x and recon
// instead of being read back from the workspace.  One CTA per 128-token tile
// over all channels (no split-K), 288 threads, one CTA per SM:
//   warps 0-7 (converters): warp w owns rows 16 w .. 16 w + 15 of the tile.
//     For each 64-channel k-block it copies its rows' x (bf16) and recon
//     (fp32) segments into a stage of a 4-deep shared ring with 16-byte
//     asynchronous copies (cp.async, zero-filled past T and C), issued four
//     k-blocks ahead so the loads never wait on the arithmetic; then it forms
//     v = x - recon (rounded once to fp32, once to bf16: the residual
//     kernel's arithmetic) and writes it in place over the stage's x rows in
//     the 128-byte-swizzled layout the tensor cores read (a row's 16-byte
//     chunks only permute within that row, and the warp owns its rows), and
//     to the workspace copy Vb for the later passes.  Warps 0-3 then run the
//     epilogue (Y rows from TMEM) and the tile's Gram / the buffer's Cholesky
//     (project_tail);
//   warp 8: allocates TMEM; one lane TMA-loads the Qt tiles (no multicast)
//     and issues tcgen05.mma (kind::f16) per k-block; commits release stages.
// Every wait is bounded; on expiry CF_ERR_TIMEOUT goes to the buffer's status
// word, the loops end, and TMEM is freed.
constexpr int kFusedConverters = 8;                        // warps 0-7
constexpr int kFusedThreads = 32 * kFusedConverters + 32;  // + warp 8
constexpr int kFusedStages = 4;
constexpr int kFusedX = 128 * 128;                         // x / A tile: 128 rows x 128 B
constexpr int kFusedR = 128 * 256;                         // recon tile: 128 rows x 256 B

template <int BN>
struct FusedGeom {
    static constexpr int kBytesB = BN * kBK * 2;
    static constexpr int kStage = kFusedX + kFusedR + kBytesB;   // multiple of 1 KB
    static constexpr int kSmem = kFusedStages * kStage + 1024 + 256;
    static constexpr uint32_t kTmemCols = BN <= 32 ? 32 : 64;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    // src-size 0 writes 16 zero bytes and reads nothing
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
// wait until at most kFusedStages - 1 groups of this thread are in flight
__device__ __forceinline__ void cp_async_wait_oldest() {
    asm volatile("cp.async.wait_group %0;" ::"n"(kFusedStages - 1) : "memory");
}

template <int BN>
__global__ void __launch_bounds__(kFusedThreads, 1)
project_residual_kernel(const __grid_constant__ CUtensorMap mapQt, const cf_lowrank::LrBatch B,
                        const cf_lowrank::Layout L) {
    using G = FusedGeom<BN>;
    constexpr int S = kFusedStages;
    static_assert(((128 * (BN + 8) * 4 + 255) & ~255) + BN * (BN + 1) * 8 <= S * G::kStage,
                  "tail scratch");
    const int bz = blockIdx.z;
    if (B.at<int32_t>(bz, L.off_status)[cf_lowrank::kSkipWord]) return;
    const cf_lowrank::LrPtrs pp = B.get(bz);
    const int64_t T = L.T, C = L.C;
    const int64_t t0 = (int64_t)blockIdx.x * 128;
    const int nkb = (int)((C + kBK - 1) / kBK);
    int32_t *status = B.at<int32_t>(bz, L.off_status) + cf_lowrank::kStatusWord;
    bf16 *vb = B.at<bf16>(bz, L.off_vb);

    extern __shared__ uint8_t dsmem[];
    const uint32_t base = (smem_u32(dsmem) + 1023u) & ~1023u;
    uint8_t *gbase = dsmem + (base - smem_u32(dsmem));
    // barriers: a_full[S] (8 converter warps), b_full[S] (tx), empty[S]
    // (commit), done (commit)
    const uint32_t bars = base + S * G::kStage;
    auto a_full = [&](int q) { return bars + 8u * q; };
    auto b_full = [&](int q) { return bars + 8u * (S + q); };
    auto empty = [&](int q) { return bars + 8u * (2 * S + q); };
    const uint32_t done = bars + 8u * (3 * S);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + S * G::kStage + 8 * (3 * S + 1));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int q = 0; q < S; ++q) {
            mbar_init(a_full(q), kFusedConverters);
            mbar_init(b_full(q), 1);
            mbar_init(empty(q), 1);
        }
        mbar_init(done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kFusedConverters) {
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

    bool have = false;
    if (warp == kFusedConverters) {
        if (lane == 0) {
            auto load_b = [&](int kb) {
                const int q = kb % S;
                mbar_expect_tx(b_full(q), (uint32_t)G::kBytesB);
                tma_load_3d(base + q * G::kStage + kFusedX + kFusedR, &mapQt, b_full(q), kb * kBK, 0, bz);
            };
            for (int kb = 0; kb < nkb && kb < S; ++kb) load_b(kb);
            constexpr uint32_t idesc = idesc_bf16(BN, false);
            bool ok = true;
            for (int kb = 0; kb < nkb; ++kb) {
                const int q = kb % S;
                const uint32_t ph = (uint32_t)(kb / S) & 1u;
                if (!mbar_wait(a_full(q), ph) || !mbar_wait(b_full(q), ph)) {
                    ok = false;
                    break;
                }
                fence_after_sync();
                const uint32_t sa = base + q * G::kStage, sb = sa + kFusedX + kFusedR;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)
                    mma_bf16(tmem, sw128_desc(sa + kk * 32u, 16, 1024), sw128_desc(sb + kk * 32u, 16, 1024),
                             idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                mma_commit(empty(q));
                if (kb + S < nkb) {
                    // this stage's B is read once its product is done
                    if (!mbar_wait(empty(q), ph)) {
                        ok = false;
                        break;
                    }
                    load_b(kb + S);
                }
            }
            if (ok)
                mma_commit(done);
            else
                atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
        }
        __syncwarp();
    } else {
        const int r0 = 16 * warp;   // this warp's first row in the tile
        // Stage kb's copies of this warp's rows: 16 rows x (8 x-chunks + 16
        // recon-chunks) of 16 bytes = 384 chunks, 12 per lane.
        auto issue = [&](int kb) {
            const int q = kb % S;
            const uint32_t sx = base + q * G::kStage, sr = sx + kFusedX;
            const int64_t cbase = (int64_t)kb * kBK;
#pragma unroll
            for (int j = 0; j < 12; ++j) {
                const int ci = lane + 32 * j;
                if (ci < 128) {
                    const int row = r0 + (ci >> 3), cc = ci & 7;
                    const int64_t t = t0 + row, c = cbase + 8 * cc;
                    const bool ok = t < T && c < C;
                    cp_async16(sx + row * 128 + cc * 16, ok ? (const void *)(pp.x + t * C + c) : pp.x, ok);
                } else {
                    const int cr = ci - 128;
                    const int row = r0 + (cr >> 4), cc = cr & 15;
                    const int64_t t = t0 + row, c = cbase + 4 * cc;
                    const bool ok = t < T && c < C;
                    cp_async16(sr + row * 256 + cc * 16, ok ? (const void *)(pp.recon + t * C + c) : pp.recon,
                               ok);
                }
            }
            cp_async_commit();
        };
        for (int kb = 0; kb < S; ++kb) {
            if (kb < nkb)
                issue(kb);
            else
                cp_async_commit();   // keep one group per k-block
        }
        const int sub = lane >> 4, cl = (lane & 15) * 4;   // row within a pair, channel offset
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
            const int q = kb % S;
            cp_async_wait_oldest();
            __syncwarp();
            uint8_t *sx = gbase + q * G::kStage;
            const uint8_t *sr = sx + kFusedX;
            const int64_t c = (int64_t)kb * kBK + cl;
            const bool cok = c < C;                  // C % 8 == 0: all 4 channels or none
            uint2 w[8];
#pragma unroll
            for (int pr = 0; pr < 8; ++pr) {
                const int row = r0 + 2 * pr + sub;
                const uint2 xv = *reinterpret_cast<const uint2 *>(sx + row * 128 + cl * 2);
                const float4 rv = *reinterpret_cast<const float4 *>(sr + row * 256 + cl * 4);
                const float v0 = __fsub_rn(bf16_bits_to_f32(xv.x & 0xffffu), rv.x);
                const float v1 = __fsub_rn(bf16_bits_to_f32(xv.x >> 16), rv.y);
                const float v2 = __fsub_rn(bf16_bits_to_f32(xv.y & 0xffffu), rv.z);
                const float v3 = __fsub_rn(bf16_bits_to_f32(xv.y >> 16), rv.w);
                const __nv_bfloat162 h0 = __floats2bfloat162_rn(v0, v1);
                const __nv_bfloat162 h1 = __floats2bfloat162_rn(v2, v3);
                w[pr] = make_uint2(*reinterpret_cast<const uint32_t *>(&h0),
                                   *reinterpret_cast<const uint32_t *>(&h1));
            }
            __syncwarp();   // every lane has read its rows' x before any is overwritten
#pragma unroll
            for (int pr = 0; pr < 8; ++pr) {
                const int row = r0 + 2 * pr + sub;
                // 128-byte swizzle: 16-byte chunk j of row `row` sits at
                // chunk j ^ (row & 7); this lane's 8 bytes are half a chunk
                const int chunk = (cl >> 3) ^ (row & 7);
                *reinterpret_cast<uint2 *>(sx + row * 128 + chunk * 16 + (cl & 4) * 2) = w[pr];
                const int64_t t = t0 + row;
                if (cok && t < T) *reinterpret_cast<uint2 *>(vb + t * C + c) = w[pr];
            }
            // generic writes of the A tile before the tensor cores read it
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(a_full(q));
            // refill this stage with k-block kb + S once its product is done
            if (kb + S < nkb) {
                ok = __all_sync(kFullMask, mbar_wait(empty(q), (uint32_t)((kb / S) & 1)));
                if (!ok) break;
                issue(kb + S);
            } else {
                cp_async_commit();
            }
        }
        // no copy may land after this CTA's shared memory is reused
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (!ok && lane == 0) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
        // epilogue (warps 0-3): TMEM lane 32 w + i holds Y row t0 + 32 w + i
        if (warp < 4) have = __all_sync(kFullMask, ok && mbar_wait(done, 0));
        if (have) {
            fence_after_sync();
            const int64_t row = t0 + 32 * warp + lane;
            const uint32_t taddr = tmem + ((uint32_t)(32 * warp) << 16);
            float *y = B.at<float>(bz, L.off_y);
#pragma unroll
            for (int cc = 0; cc < BN; cc += 16) {
                float v[16];
                tmem_ld16(taddr + cc, v);
                if (row < T && CF_IN(row >= 0 && cc + 16 <= BN)) {
                    float4 *dst = reinterpret_cast<float4 *>(y + row * BN + cc);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        dst[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                }
            }
        }
    }
    // every TMEM read is done: free it (the tail below uses only shared and
    // global memory)
    fence_before_sync();
    __syncthreads();
    if (warp == kFusedConverters) {
        fence_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(G::kTmemCols)
                     : "memory");
        return;
    }
    if (warp >= 4) return;   // the tail runs on warps 0-3
    project_tail<BN>(B, L, bz, blockIdx.x);
}

}  // namespace umma
}  // namespace cf
