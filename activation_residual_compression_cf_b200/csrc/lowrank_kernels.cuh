// lowrank_kernels.cuh -- device kernels of the low-rank mode (CUDA cores).
//
// The two dense products of subspace iteration (Y = V Q and Q = V^T P) have
// tensor-core versions in lowrank_umma.cuh; the SIMT versions here are the
// straightforward form, used for shapes the tensor-core tiles do not cover
// and as an on-device cross-check of them.
#pragma once

#include <cuda_bf16.h>
#include <math.h>

#include "bounds.cuh"
#include "cf.h"
#include "cf_common.cuh"
#include "lowrank_api.cuh"

namespace cf {

using bf16 = __nv_bfloat16;
using cf_lowrank::Layout;
using cf_lowrank::LrBatch;
using cf_lowrank::LrPtrs;

// Every kernel of a (batched) low-rank call handles buffer blockIdx.z.  A
// buffer whose pointers failed validation in lr_prep_kernel is skipped by all.
__device__ __forceinline__ bool lr_skipped(const LrBatch &B, const Layout &L, int b) {
    return B.ws != nullptr && B.at<int32_t>(b, L.off_status)[cf_lowrank::kSkipWord] != 0;
}

// Per-buffer set-up of a low-rank encode: zero the status word, the Gram
// tickets and the column maxima of this buffer's workspace slice, then check
// its pointers (x, recon, err: 16-byte aligned; omega, scales: 4-byte; all
// non-null except omega, whose null means a warm start and needs the warm
// tag of an earlier encode of this shape) and mark the buffer skipped with
// the error in its status word.
__global__ void lr_prep_kernel(const LrBatch B, const Layout L) {
    const int b = blockIdx.x;
    int32_t *st = B.at<int32_t>(b, L.off_status);
    uint32_t *gt = B.at<uint32_t>(b, L.off_gt);
    uint32_t *amax = B.at<uint32_t>(b, L.off_amax);
    for (int i = threadIdx.x; i < 4; i += blockDim.x) st[i] = 0;
    for (int i = threadIdx.x; i < L.nGroups; i += blockDim.x) gt[i] = 0u;
    for (int i = threadIdx.x; i < 2 * L.rp; i += blockDim.x) amax[i] = 0u;
    __syncthreads();
    if (threadIdx.x == 0) {
        const LrPtrs p = B.get(b);
        int code = CF_OK;
        const uint32_t *wt = reinterpret_cast<const uint32_t *>(st);
        const bool warm_ok = wt[cf_lowrank::kWarmTag] == (cf_lowrank::kWarmMagic | (uint32_t)L.r) &&
                             wt[cf_lowrank::kWarmC] == (uint32_t)L.C;
        if (!p.x || !p.recon || !p.err || !p.pc_out || !p.ps_out || !p.qc_out || !p.qs_out)
            code = CF_ERR_INVALID_ARG;
        else if (!p.omega && !warm_ok)
            code = CF_ERR_INVALID_ARG;   // warm start without an earlier encode
        else if (misaligned16(p.x) || misaligned16(p.recon) || misaligned16(p.err) ||
                 (reinterpret_cast<uintptr_t>(p.omega) & 3u) || (reinterpret_cast<uintptr_t>(p.ps_out) & 3u) ||
                 (reinterpret_cast<uintptr_t>(p.qs_out) & 3u))
            code = CF_ERR_ALIGNMENT;
        st[cf_lowrank::kStatusWord] = code;
        st[cf_lowrank::kSkipWord] = code != CF_OK ? 1 : 0;
    }
}

// Vb = bf16_rn((float)x - recon): the residual the projections read.
__global__ void lr_residual_kernel(const LrBatch B, const Layout L) {
    const int bz = blockIdx.z;
    if (lr_skipped(B, L, bz)) return;
    const LrPtrs pp = B.get(bz);
    const uint16_t *x = pp.x;
    const float *recon = pp.recon;
    bf16 *vb = B.at<bf16>(bz, L.off_vb);
    const int64_t n = L.T * L.C;
    const int64_t groups = n >> 3;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += stride) {
        if (!CF_IN(8 * g + 8 <= n)) continue;
        const uint4 xv = ld_ro_v4(x + 8 * g);
        const float4 a = ld_state_v4(recon + 8 * g);
        const float4 b = ld_state_v4(recon + 8 * g + 4);
        const float rr[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        const uint32_t w4[4] = {xv.x, xv.y, xv.z, xv.w};
        uint32_t out[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const float v0 = __fsub_rn(bf16_bits_to_f32(w4[e >> 1] & 0xffffu), rr[e]);
            const float v1 = __fsub_rn(bf16_bits_to_f32(w4[e >> 1] >> 16), rr[e + 1]);
            const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
            out[e >> 1] = *reinterpret_cast<const uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(vb + 8 * g) = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

// Qt[k][c] = bf16(omega[c][k]) for k < r, 0 for the padding rows.
constexpr int kOmegaTilesPerBlock = 4;

__global__ void lr_omega_kernel(const LrBatch B, const Layout L) {
    // Qt[k][c] = bf16(Omega[c][k]) (0 for k >= r), 32 x 32 tiles (32 x 8
    // threads), kOmegaTilesPerBlock of them a grid stride apart along the
    // channels: coalesced reads of Omega's rows, transposed through shared
    // memory, coalesced writes of Qt's rows.
    const int bz = blockIdx.z;
    if (lr_skipped(B, L, bz)) return;
    const float *omega = B.get(bz).omega;
    if (!omega) return;   // warm start: Qt still holds the previous encode's Q
    bf16 *qt = B.at<bf16>(bz, L.off_qt);
    const int64_t C = L.C;
    const int r = L.r;
    __shared__ float tile[32][33];
    const int k0 = blockIdx.y * 32;
    const int tx = threadIdx.x, ty = threadIdx.y;
    for (int64_t c0 = (int64_t)blockIdx.x * 32; c0 < C; c0 += (int64_t)gridDim.x * 32) {
        for (int j = ty; j < 32; j += 8) {
            const int64_t c = c0 + j;
            const int k = k0 + tx;
            tile[j][tx] = (c < C && k < r && CF_IN(c * r + k < C * r)) ? omega[c * r + k] : 0.0f;
        }
        __syncthreads();
        for (int j = ty; j < 32; j += 8) {
            const int k = k0 + j;
            const int64_t c = c0 + tx;
            if (k < L.rp && c < C && CF_IN((int64_t)k * C + c < (int64_t)L.rp * C))
                qt[(int64_t)k * C + c] = __float2bfloat16_rn(tile[tx][j]);
        }
        __syncthreads();   // the tile is refilled by the next pass
    }
}

// Yp[s][t][k] = sum over the channels of split s of Vb[t][c] * Qt[k][c].
// Block: 64 tokens; thread (tok = tid/4, kg = tid%4) owns k = kg + 4j.
__global__ void __launch_bounds__(256)
lr_project_simt(const LrBatch B, const Layout L) {
    const int bz = blockIdx.z;
    if (lr_skipped(B, L, bz)) return;
    const bf16 *vb = B.at<bf16>(bz, L.off_vb);
    const bf16 *qt = B.at<bf16>(bz, L.off_qt);
    float *yp = B.at<float>(bz, L.off_yp);
    const int64_t T = L.T, C = L.C;
    const int rp = L.rp;
    __shared__ float Vs[64][65];
    __shared__ float Qs[64][65];
    const int tid = threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.x * 64;
    const int s = blockIdx.y;
    const int64_t cb = (int64_t)s * cf_lowrank::kChunkA;
    const int64_t ce = min(C, cb + cf_lowrank::kChunkA);
    const int tok = tid >> 2, kg = tid & 3;
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
    for (int64_t c0 = cb; c0 < ce; c0 += 64) {
        for (int i = tid; i < 64 * 64; i += 256) {
            const int tt = i >> 6, cc = i & 63;
            const int64_t t = t0 + tt, c = c0 + cc;
            Vs[tt][cc] = (t < T && c < ce) ? __bfloat162float(vb[t * C + c]) : 0.0f;
        }
        for (int i = tid; i < rp * 64; i += 256) {
            const int k = i >> 6, cc = i & 63;
            const int64_t c = c0 + cc;
            Qs[k][cc] = (c < ce) ? __bfloat162float(qt[(int64_t)k * C + c]) : 0.0f;
        }
        __syncthreads();
        for (int cc = 0; cc < 64; ++cc) {
            const float v = Vs[tok][cc];
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (kg + 4 * j < rp) acc[j] = fmaf(v, Qs[kg + 4 * j][cc], acc[j]);
        }
        __syncthreads();
    }
    const int64_t t = t0 + tok;
    if (t < T) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (kg + 4 * j < rp) yp[((int64_t)s * T + t) * rp + kg + 4 * j] = acc[j];
    }
}

// Cholesky G = R^T R of the rp x rp matrix in shared memory A (leading
// dimension ld, upper triangle valid), in one warp, for r up to 64 (lane l
// owns columns l and l + 32).  A pivot not above 1e-10 of its original
// diagonal entry gdiag[j] is dead: its row of R and invd[j] become zero and
// dead[j] is set.  On return A's upper triangle holds R and invd[j] =
// 1/R[j][j] (0 where dead); one reciprocal square root gives both.
__device__ __forceinline__ void warp_cholesky_smem(double *A, int ld, int r, const double *gdiag,
                                                   int *dead, double *invd) {
    const int lane = threadIdx.x & 31;
    for (int j = 0; j < r; ++j) {
        const double ajj = A[j * ld + j];
        const bool bad = !(ajj > 1e-10 * gdiag[j]);
        const double inv = bad ? 0.0 : rsqrt(ajj);
        const double rjj = ajj * inv;
        for (int c = lane; c < r; c += 32)
            if (c > j) A[j * ld + c] *= inv;
        __syncwarp();
        if (lane == 0) {
            A[j * ld + j] = rjj;
            dead[j] = bad ? 1 : 0;
            invd[j] = inv;
        }
        for (int c = lane; c < r; c += 32) {
            if (c <= j) continue;
            const double rjc = A[j * ld + c];
            for (int i = j + 1; i <= c; ++i) A[i * ld + c] = fma(-A[j * ld + i], rjc, A[i * ld + c]);
        }
        __syncwarp();
    }
}

// Cholesky of the upper triangle of A (leading dimension ld, r <= 32) by
// the first 128 threads of the block: thread (w, c) = (tid / 32, tid % 32)
// owns column c and the rows i = w, w + 4, ... of it in registers, so every
// warp (one per SM sub-partition) shares the fp64 update work of a step.
// Row j of R is broadcast through shared memory (double-buffered, one
// barrier per step among the 128 threads).  Results as warp_cholesky_smem.
__device__ __forceinline__ void quad_cholesky(double *A, int ld, int r, const double *gdiag,
                                              int *dead, double *invd, double (*rowbuf)[33]) {
    const int tid = threadIdx.x;
    const int w = tid >> 5, c = tid & 31;
    double a[8];  // A[w + 4m][c]
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int i = w + 4 * m;
        a[m] = (c < r && i <= c) ? A[i * ld + c] : 0.0;
    }
    for (int j = 0; j < r; ++j) {
        const int wj = j & 3, mj = j >> 2;
        double *row = rowbuf[j & 1];
        if (w == wj) {
            // this warp holds row j: finish it and publish it
            double ajj = 0.0;
#pragma unroll
            for (int m = 0; m < 8; ++m)
                if (m == mj) ajj = a[m];
            ajj = __shfl_sync(kFullMask, ajj, j);
            const bool bad = !(ajj > 1e-10 * gdiag[j]);
            const double inv = bad ? 0.0 : rsqrt(ajj);
#pragma unroll
            for (int m = 0; m < 8; ++m)
                if (m == mj) {
                    if (c > j) a[m] *= inv;
                    if (c == j) a[m] = ajj * inv;
                    row[c] = (c >= j && c < r) ? a[m] : 0.0;
                }
            if (c == 0) {
                dead[j] = bad ? 1 : 0;
                invd[j] = inv;
            }
        }
        asm volatile("bar.sync 2, 128;" ::: "memory");
        // trailing update of this thread's rows i > j: A[i][c] -= R[j][i] R[j][c]
        if (c > j) {
            const double rjc = row[c];
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int i = w + 4 * m;
                if (i > j && i <= c) a[m] = fma(-row[i], rjc, a[m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int i = w + 4 * m;
        if (c < r && i <= c) A[i * ld + c] = a[m];
    }
}

// Fused Gram + Cholesky, deterministic.  CTA b owns 32 tokens:
//  1. Y = sum of the split partials for its tokens (float4 rows; the loads
//     of up to 8 splits are issued before any is summed; summed in split
//     order), written to y and to shared memory;
//  2. its fp64 partial Gram Gp[b] = Y_b^T Y_b (upper triangle).
// Reduction in two ticketed levels, each summing in a fixed order: the last
// CTA to finish in each group of 16 blocks sums the group's partials into
// Gg[group]; the last group to finish sums the groups in order into G and
// factors G = R^T R in one warp.  (A reduction whose order varied from run
// to run would be amplified by the bf16 operand roundings of later
// iterations into visible differences.)  A pivot not above 1e-10 of its
// original diagonal entry marks the column dead: its row of R and its
// inverse diagonal are zero (P gets a zero column) and CF_ERR_NUMERIC is
// recorded.  Output: R (fp32 [rp][rp], upper) and 1/diag(R) (fp32 [rp], 0
// where dead).  All tickets are reset by their last user.
__global__ void __launch_bounds__(256)
lr_gram_chol_kernel(const LrBatch B, const Layout L) {
    const int bz = blockIdx.z;
    if (lr_skipped(B, L, bz)) return;
    const float *yp = B.at<float>(bz, L.off_yp);
    float *y = B.at<float>(bz, L.off_y);
    double *gp = B.at<double>(bz, L.off_gp);
    double *gg = B.at<double>(bz, L.off_gg);
    const int64_t T = L.T;
    const int r = L.r, rp = L.rp, splits = L.splitsA;
    float *rmat = B.at<float>(bz, L.off_rmat);
    float *rinvd = rmat + rp * rp;
    uint32_t *gticket = B.at<uint32_t>(bz, L.off_gt);
    int32_t *status = B.at<int32_t>(bz, L.off_status) + cf_lowrank::kStatusWord;
    uint32_t *ticket = B.at<uint32_t>(bz, L.off_status) + cf_lowrank::kTicketWord;
    constexpr int TOK = cf_lowrank::kGramTok;
    // one buffer: the fp32 Y block in phases 1-2, the fp64 matrix afterwards
    __shared__ double buf[64 * 65];
    static_assert(TOK * 65 * sizeof(float) <= sizeof(buf), "Y block does not fit");
    float *ys = reinterpret_cast<float *>(buf);
    double *A = buf;
    __shared__ double gdiag[64];
    __shared__ double invd[64];
    __shared__ double rowbuf[2][33];
    __shared__ int dead[64];
    __shared__ int is_last;
    const int tid = threadIdx.x;
    const int ldy = rp + 1;
    const int64_t t0 = (int64_t)blockIdx.x * TOK;
    const int q4 = rp / 4;
    for (int idx = tid; idx < TOK * q4; idx += blockDim.x) {
        const int tt = idx / q4, k = (idx - tt * q4) * 4;
        const int64_t t = t0 + tt;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t < T) {
            const float4 *src = reinterpret_cast<const float4 *>(yp + t * rp + k);
            const int64_t sstride = T * rp / 4;
            // batches of 8 splits: all 8 loads issued before any is summed
            for (int s0 = 0; s0 < splits; s0 += 8) {
                float4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (s0 + u < splits) v[u] = __ldcg(src + (s0 + u) * sstride);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (s0 + u < splits) {
                        acc.x += v[u].x; acc.y += v[u].y; acc.z += v[u].z; acc.w += v[u].w;
                    }
            }
            *reinterpret_cast<float4 *>(y + t * rp + k) = acc;
        }
        float *row = ys + tt * ldy + k;
        row[0] = acc.x; row[1] = acc.y; row[2] = acc.z; row[3] = acc.w;
    }
    __syncthreads();
    const int ne = rp * rp;
    for (int e = tid; e < ne; e += blockDim.x) {
        const int i = e / rp, j = e - (e / rp) * rp;
        if (i > j) continue;
        double a0 = 0.0, a1 = 0.0;
#pragma unroll 4
        for (int tt = 0; tt < TOK; tt += 2) {
            a0 = fma((double)ys[tt * ldy + i], (double)ys[tt * ldy + j], a0);
            a1 = fma((double)ys[(tt + 1) * ldy + i], (double)ys[(tt + 1) * ldy + j], a1);
        }
        gp[(int64_t)blockIdx.x * ne + e] = a0 + a1;
    }
    // level 1: the last CTA of each group of kGramGroup blocks sums them
    const int nblk = gridDim.x;
    const int grp = blockIdx.x / cf_lowrank::kGramGroup;
    const int gb0 = grp * cf_lowrank::kGramGroup;
    const int gn = min(cf_lowrank::kGramGroup, nblk - gb0);
    const int ngrp = (nblk + cf_lowrank::kGramGroup - 1) / cf_lowrank::kGramGroup;
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(gticket + grp, 1u) == (uint32_t)(gn - 1)) ? 1 : 0;
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    for (int e = tid; e < ne; e += blockDim.x) {
        const int i = e / rp, j = e - (e / rp) * rp;
        if (i > j) continue;
        // batches of 16 loads in flight, summed in block order
        double acc = 0.0;
        for (int u0 = 0; u0 < gn; u0 += 16) {
            double v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
                v[u] = (u0 + u < gn) ? __ldcg(gp + (int64_t)(gb0 + u0 + u) * ne + e) : 0.0;
#pragma unroll
            for (int u = 0; u < 16; ++u) acc += v[u];
        }
        gg[(int64_t)grp * ne + e] = acc;
    }
    if (tid == 0) gticket[grp] = 0u;
    // level 2: the last group sums the groups in order
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(ticket, 1u) == (uint32_t)(ngrp - 1)) ? 1 : 0;
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    const int ld = rp + 1;
    for (int e = tid; e < ne; e += blockDim.x) {
        const int i = e / rp, j = e - (e / rp) * rp;
        if (i > j) continue;
        double a[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
        int g = 0;
        for (; g + 8 <= ngrp; g += 8) {
#pragma unroll
            for (int u = 0; u < 8; ++u) a[u] += __ldcg(gg + (int64_t)(g + u) * ne + e);
        }
        for (; g < ngrp; ++g) a[0] += __ldcg(gg + (int64_t)g * ne + e);
        const double v = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
        A[i * ld + j] = v;
        if (i == j) gdiag[i] = v;
    }
    __syncthreads();
    if (r <= 32) {
        if (tid < 128) quad_cholesky(A, ld, r, gdiag, dead, invd, rowbuf);
    } else if (tid < 32) {
        warp_cholesky_smem(A, ld, r, gdiag, dead, invd);
    }
    __syncthreads();
    int nd = 0;
    for (int e = tid; e < ne; e += blockDim.x) {
        const int i = e / rp, c = e - (e / rp) * rp;
        rmat[e] = (i <= c && c < r) ? (float)A[i * ld + c] : 0.0f;
    }
    for (int j = tid; j < rp; j += blockDim.x) {
        const bool live = j < r && !dead[j];
        rinvd[j] = live ? (float)invd[j] : 0.0f;
        nd += (j < r && dead[j]) ? 1 : 0;
    }
    if (nd) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_NUMERIC);
    if (tid == 0) *ticket = 0u;
}

// Row staging for the one-row-per-thread kernels below: a warp copies the
// RP-float rows row0 .. row0 + 31 of a row-major [rows][RP] fp32 array into
// its shared-memory tile [32][RP + 4] with coalesced 16-byte loads (rows past
// `rows` read as 0), so that afterwards lane l holds row row0 + l in the
// tile's row l.  The 4-float pad keeps the lanes' 16-byte row reads free of
// bank conflicts.
template <int RP>
__device__ __forceinline__ void warp_stage_rows(const float *src, int64_t row0, int64_t rows, float *tile,
                                                int lane) {
    constexpr int Q = RP / 4;   // float4 per row
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
#pragma unroll
    for (int i = 0; i < Q; ++i) {
        const int idx = i * 32 + lane;   // float4 index within the warp's 32 rows
        const int rr = idx / Q, c4 = idx - (idx / Q) * Q;
        float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (row0 + rr < rows) v = __ldcg(s4 + row0 * Q + idx);
        *reinterpret_cast<float4 *>(tile + rr * (RP + 4) + 4 * c4) = v;
    }
    __syncwarp();
}

// P = Y R^-1 by forward substitution, one token row per thread:
//   P[t][k] = (Y[t][k] - sum_{j<k} P[t][j] R[j][k]) / R[k][k]
// written as fp32 P [T][rp] and as the bf16 transpose Pt [rp][Tp] (zero
// past T) that the back-projection reads.  On the last iteration (amax !=
// null) it also folds max |P[:, k]| into amax[k] (float bits, atomicMax once
// per CTA and column).
//
// Each warp moves its 32 rows of Y in and of P out through a shared-memory
// tile with coalesced 16-byte accesses.  The substitution runs column by
// column: once P[t][j] is final, it is taken out of every later column,
// reading row j of R as 16-byte shared-memory loads (a row-at-a-time sweep
// needs one scalar load per product).  Each column k still receives its
// products in ascending j, so the sums are exactly those of the row-at-a-time
// form.
// Threads per block: 4 warps, 2 at rank 64 (the R matrix and the staging
// tiles stay within 48 KB of static shared memory).
template <int RP>
__host__ __device__ constexpr int orth_threads() {
    return RP > 48 ? 64 : 128;
}

template <int RP>
__global__ void __launch_bounds__(orth_threads<RP>())
lr_orth_kernel(const LrBatch B, const Layout L, int want_amax) {
    constexpr int kOrthThreads = orth_threads<RP>();
    const int bz = blockIdx.z;
    if (lr_skipped(B, L, bz)) return;
    const float *y = B.at<float>(bz, L.off_y);
    const float *rmat = B.at<float>(bz, L.off_rmat);
    const float *rinvd = rmat + RP * RP;
    float *p = B.at<float>(bz, L.off_p);
    bf16 *pt = B.at<bf16>(bz, L.off_pt);
    const int64_t T = L.T, Tp = L.Tp;
    uint32_t *amax = want_amax ? B.at<uint32_t>(bz, L.off_amax) : nullptr;
    constexpr int NW = kOrthThreads / 32;
    constexpr int Q = RP / 4;
    __shared__ __align__(16) float Rs[RP * RP];
    __shared__ __align__(16) float tiles[NW][32 * (RP + 4)];
    __shared__ float Id[RP];
    __shared__ float Wm[NW][RP];
    for (int i = threadIdx.x; i < RP * RP; i += kOrthThreads) Rs[i] = rmat[i];
    for (int i = threadIdx.x; i < RP; i += kOrthThreads) Id[i] = rinvd[i];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row0 = (int64_t)blockIdx.x * kOrthThreads + 32 * warp;
    float *tile = tiles[warp];
    warp_stage_rows<RP>(y, row0, T, tile, lane);
    __syncthreads();
    const float4 *R4 = reinterpret_cast<const float4 *>(Rs);
    float4 *mine = reinterpret_cast<float4 *>(tile + lane * (RP + 4));
    const int64_t t = row0 + lane;
    float pv[RP];
#pragma unroll
    for (int q = 0; q < Q; ++q) {
        const float4 v = mine[q];
        pv[4 * q] = v.x;
        pv[4 * q + 1] = v.y;
        pv[4 * q + 2] = v.z;
        pv[4 * q + 3] = v.w;
    }
    if (t < T) {
#pragma unroll
        for (int j = 0; j < RP; ++j) {
            pv[j] = pv[j] * Id[j];
            const float nj = -pv[j];
#pragma unroll
            for (int q = (j + 1) / 4; q < Q; ++q) {
                const float4 rv = R4[(j * RP) / 4 + q];
                const float re[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (4 * q + e > j) pv[4 * q + e] = fmaf(nj, re[e], pv[4 * q + e]);
            }
        }
    }   // rows past T stay 0 (the staging read them as 0)
#pragma unroll
    for (int q = 0; q < Q; ++q) mine[q] = make_float4(pv[4 * q], pv[4 * q + 1], pv[4 * q + 2], pv[4 * q + 3]);
    __syncwarp();
    float4 *p4 = reinterpret_cast<float4 *>(p);
#pragma unroll
    for (int i = 0; i < Q; ++i) {
        const int idx = i * 32 + lane;
        const int rr = idx / Q, c4 = idx - (idx / Q) * Q;
        if (row0 + rr < T) p4[row0 * Q + idx] = *reinterpret_cast<const float4 *>(tile + rr * (RP + 4) + 4 * c4);
    }
    if (t < Tp) {
#pragma unroll
        for (int k = 0; k < RP; ++k) pt[(int64_t)k * Tp + t] = __float2bfloat16_rn(pv[k]);
    }
    if (amax) {
#pragma unroll
        for (int k = 0; k < RP; ++k) {
            float m = fabsf(pv[k]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
            if (lane == 0) Wm[warp][k] = m;
        }
        __syncthreads();
        for (int k = threadIdx.x; k < RP; k += kOrthThreads) {
            float m = 0.0f;
            for (int w = 0; w < NW; ++w) m = fmaxf(m, Wm[w][k]);
            atomicMax(amax + k, __float_as_uint(m));
        }
    }
}

// Zp[s][c][k] = sum over the tokens of split s of Vb[t][c] * Pt[k][t].
__global__ void __launch_bounds__(256)
lr_backproject_simt(const LrBatch B, const Layout L) {
    const int bz = blockIdx.z;
    if (lr_skipped(B, L, bz)) return;
    const bf16 *vb = B.at<bf16>(bz, L.off_vb);
    const bf16 *pt = B.at<bf16>(bz, L.off_pt);
    float *zp = B.at<float>(bz, L.off_zp);
    const int64_t T = L.T, Tp = L.Tp, C = L.C;
    const int rp = L.rp;
    __shared__ float Vs[64][65];
    __shared__ float Ps[64][65];
    const int tid = threadIdx.x;
    const int64_t c0 = (int64_t)blockIdx.x * 64;
    const int s = blockIdx.y;
    const int64_t tb = (int64_t)s * cf_lowrank::kChunkB;
    const int64_t te = min(T, tb + cf_lowrank::kChunkB);
    const int ch = tid >> 2, kg = tid & 3;
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
    for (int64_t t0 = tb; t0 < te; t0 += 64) {
        for (int i = tid; i < 64 * 64; i += 256) {
            const int tt = i >> 6, cc = i & 63;
            const int64_t t = t0 + tt, c = c0 + cc;
            Vs[tt][cc] = (t < te && c < C) ? __bfloat162float(vb[t * C + c]) : 0.0f;
        }
        for (int i = tid; i < rp * 64; i += 256) {
            const int k = i >> 6, tt = i & 63;
            const int64_t t = t0 + tt;
            Ps[k][tt] = (t < te) ? __bfloat162float(pt[(int64_t)k * Tp + t]) : 0.0f;
        }
        __syncthreads();
        for (int tt = 0; tt < 64; ++tt) {
            const float v = Vs[tt][ch];
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (kg + 4 * j < rp) acc[j] = fmaf(v, Ps[kg + 4 * j][tt], acc[j]);
        }
        __syncthreads();
    }
    const int64_t c = c0 + ch;
    if (c < C) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (kg + 4 * j < rp) zp[((int64_t)s * C + c) * rp + kg + 4 * j] = acc[j];
    }
}

// Q = sum of the split partials (fixed order), one channel per thread:
// fp32 Q [C][rp] and the bf16 transpose Qt [rp][C] for the next projection.
// On the last iteration (amax != null) it folds max |Q[:, k]| into amax[k].
template <int RP>
__global__ void __launch_bounds__(128)
lr_reduce_q_kernel(const LrBatch B, const Layout L, int want_amax) {
    const int bz = blockIdx.z;
    if (lr_skipped(B, L, bz)) return;
    const float *zp = B.at<float>(bz, L.off_zp);
    float *q = B.at<float>(bz, L.off_q);
    bf16 *qt = B.at<bf16>(bz, L.off_qt);
    const int64_t C = L.C;
    const int splits = L.splitsB;
    uint32_t *amax = want_amax ? B.at<uint32_t>(bz, L.off_amax) + RP : nullptr;
    __shared__ float Wm[4][RP];
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    float v[RP];
#pragma unroll
    for (int k = 0; k < RP; ++k) v[k] = 0.0f;
    if (c < C) {
        // splits in pairs: two rows of loads in flight per step, fixed order
        int s = 0;
        for (; s + 1 < splits; s += 2) {
            const float4 *z0 = reinterpret_cast<const float4 *>(zp + ((int64_t)s * C + c) * RP);
            const float4 *z1 = reinterpret_cast<const float4 *>(zp + ((int64_t)(s + 1) * C + c) * RP);
#pragma unroll
            for (int qd = 0; qd < RP / 4; ++qd) {
                const float4 a = __ldcg(z0 + qd), b = __ldcg(z1 + qd);
                v[4 * qd] += a.x + b.x;
                v[4 * qd + 1] += a.y + b.y;
                v[4 * qd + 2] += a.z + b.z;
                v[4 * qd + 3] += a.w + b.w;
            }
        }
        for (; s < splits; ++s) {
            const float4 *zr = reinterpret_cast<const float4 *>(zp + ((int64_t)s * C + c) * RP);
#pragma unroll
            for (int qd = 0; qd < RP / 4; ++qd) {
                const float4 z = __ldcg(zr + qd);
                v[4 * qd] += z.x;
                v[4 * qd + 1] += z.y;
                v[4 * qd + 2] += z.z;
                v[4 * qd + 3] += z.w;
            }
        }
        float4 *qr = reinterpret_cast<float4 *>(q + c * RP);
#pragma unroll
        for (int qd = 0; qd < RP / 4; ++qd)
            qr[qd] = make_float4(v[4 * qd], v[4 * qd + 1], v[4 * qd + 2], v[4 * qd + 3]);
#pragma unroll
        for (int k = 0; k < RP; ++k) qt[(int64_t)k * C + c] = __float2bfloat16_rn(v[k]);
    }
    if (amax) {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
        for (int k = 0; k < RP; ++k) {
            float m = fabsf(v[k]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
            if (lane == 0) Wm[warp][k] = m;
        }
        __syncthreads();
        for (int k = threadIdx.x; k < RP; k += blockDim.x) {
            float m = 0.0f;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, Wm[w][k]);
            atomicMax(amax + k, __float_as_uint(m));
        }
    }
}

__device__ __forceinline__ int int4_code(float v, float s) {
    if (!(s > 0.0f)) return 0;
    float q = rintf(__fdiv_rn(v, s));
    q = fminf(fmaxf(q, -7.0f), 7.0f);
    return (int)q;
}

// INT4 per column: s_k = amax_k / 7; codes packed two per byte, the even
// column in the low nibble.  One launch packs both factors: blockIdx.y = 0
// packs P (T rows), 1 packs Q (C rows).  Each warp stages its 32 rows through
// shared memory with coalesced loads; a thread then codes one row and writes
// the row's nb bytes, as one 16-byte store per 32 columns when the row's
// codes are 16-byte aligned, else byte by byte (same bytes either way).
// Block 0 of each factor writes the column scales.
constexpr int kPackThreads = 128;

template <int RP>
__global__ void __launch_bounds__(kPackThreads) lr_int4_pack_kernel(const LrBatch B, const Layout L) {
    const int bz = blockIdx.z;
    if (lr_skipped(B, L, bz)) return;
    const int which = blockIdx.y;
    const int64_t rows = which == 0 ? L.T : L.C;
    const int64_t blk0 = (int64_t)blockIdx.x * kPackThreads;
    if (blk0 >= rows) return;   // the shorter factor's grid tail (never block 0)
    const LrPtrs pp = B.get(bz);
    const int r = L.r;
    const float *f = B.at<float>(bz, which == 0 ? L.off_p : L.off_q);
    const uint32_t *amax = B.at<uint32_t>(bz, L.off_amax) + (which == 0 ? 0 : RP);
    uint8_t *codes = which == 0 ? pp.pc_out : pp.qc_out;
    float *scales = which == 0 ? pp.ps_out : pp.qs_out;
    const int nb = (r + 1) / 2;
    constexpr int NW = kPackThreads / 32;
    // the column scales, once per block (the same division every element
    // would otherwise repeat); zero past r, so padded columns code to 0
    __shared__ float sc[RP];
    __shared__ __align__(16) float tiles[NW][32 * (RP + 4)];
    for (int k = threadIdx.x; k < RP; k += kPackThreads)
        sc[k] = k < r ? __fdiv_rn(__uint_as_float(amax[k]), 7.0f) : 0.0f;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row0 = blk0 + 32 * warp;
    float *tile = tiles[warp];
    warp_stage_rows<RP>(f, row0, rows, tile, lane);
    __syncthreads();
    if (blockIdx.x == 0) {
        for (int k = threadIdx.x; k < r; k += kPackThreads) scales[k] = sc[k];
        if (which == 1 && threadIdx.x == 0) {
            // the workspace now holds this encode's final Q (Qt): a later
            // encode of this shape may start from it
            uint32_t *wt = B.at<uint32_t>(bz, L.off_status);
            wt[cf_lowrank::kWarmTag] = cf_lowrank::kWarmMagic | (uint32_t)r;
            wt[cf_lowrank::kWarmC] = (uint32_t)L.C;
        }
    }
    const int64_t row = row0 + lane;
    if (row >= rows) return;
    const float4 *fr = reinterpret_cast<const float4 *>(tile + lane * (RP + 4));
    uint8_t *cr = codes + row * nb;
    const bool vec = (nb % 16) == 0 && (reinterpret_cast<uintptr_t>(cr) & 15u) == 0;
    // 32 columns (16 bytes) at a time; RP is a multiple of 16, so the last
    // block may hold 16 columns (8 bytes)
#pragma unroll
    for (int k0 = 0; k0 < RP; k0 += 32) {
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        constexpr int kMax = 8;
#pragma unroll
        for (int q4 = 0; q4 < kMax; ++q4) {
            if (k0 + 4 * q4 >= RP) break;
            const float4 v = fr[k0 / 4 + q4];
            const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int k = k0 + 4 * q4 + j;
                const uint32_t nib = (uint32_t)int4_code(e[j], sc[k]) & 0xFu;
                const int c = 4 * q4 + j;   // column within the 32-column block
                w[c >> 3] |= nib << (4 * (c & 7));
            }
        }
        const int bytes = (nb - k0 / 2) < 16 ? (nb - k0 / 2) : 16;
        if (bytes <= 0) break;
        if (vec && bytes == 16) {
            *reinterpret_cast<uint4 *>(cr + k0 / 2) = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
#pragma unroll
            for (int bi = 0; bi < 16; ++bi)
                if (bi < bytes && CF_IN(k0 / 2 + bi < nb)) cr[k0 / 2 + bi] = (uint8_t)(w[bi >> 2] >> (8 * (bi & 3)));
        }
    }
}

__device__ __forceinline__ float int4_dequant(const uint8_t *row_codes, int k, const float *scales) {
    const uint32_t byte = row_codes[k >> 1];
    int q = (int)((byte >> ((k & 1) * 4)) & 0xFu);
    q = q >= 8 ? q - 16 : q;
    return __fmul_rn((float)q, __ldg(scales + k));
}

// Batched decode: the caller's pointers of buffer b (no workspace to hold a
// per-buffer status); a bad buffer is skipped and reported once.
__device__ __forceinline__ bool lr_dec_ptrs_ok(const LrBatch &B, const LrPtrs &p) {
    int code = CF_OK;
    if (!p.pc || !p.ps || !p.qc || !p.qs || !p.recon)
        code = CF_ERR_INVALID_ARG;
    else if (misaligned16(p.recon) || (reinterpret_cast<uintptr_t>(p.ps) & 3u) ||
             (reinterpret_cast<uintptr_t>(p.qs) & 3u))
        code = CF_ERR_ALIGNMENT;
    if (code != CF_OK && B.dec_status && threadIdx.x == 0)
        atomicCAS(B.dec_status, (int32_t)CF_OK, (int32_t)code);
    return code == CF_OK;
}

// D = (qP sP)(qQ sQ)^T, then
//   sender:   v = x - recon ; err = v - D ; recon = recon + D
//   receiver: recon = recon + D
// A CTA owns one 256-channel slice (blockIdx.x): it dequantises that slice
// of Q once into shared memory, then walks 32-token tiles (blockIdx.y,
// stride gridDim.y).  Thread (w, l) owns tokens 4w..4w+3 x channels
// 8l..8l+7 of a tile; its x/recon loads are issued before the rank-r FMA
// loop so the HBM traffic overlaps the arithmetic.  D is a fixed chain of
// fused multiply-adds in k order, so sender and receiver form bit-identical
// values from the same payload.
template <bool SENDER>
__global__ void __launch_bounds__(256, 2)
lr_apply_kernel(const LrBatch B, const Layout L) {
    const int bz = blockIdx.z;
    if (lr_skipped(B, L, bz)) return;
    const LrPtrs pp = B.get(bz);
    if (!SENDER && B.dec && !lr_dec_ptrs_ok(B, pp)) return;
    const uint16_t *x = pp.x;
    float *recon = pp.recon, *err = pp.err;
    const uint8_t *pc = pp.pc, *qc = pp.qc;
    const float *ps = pp.ps, *qs = pp.qs;
    const int64_t T = L.T, C = L.C;
    const int r = L.r;
    constexpr int TM = cf_lowrank::kApplyTok, TN = cf_lowrank::kApplyCh;
    extern __shared__ float sm[];
    float *Bs = sm;                   // [r][TN]
    float *As = sm + (size_t)r * TN;  // [r][TM]
    const int tid = threadIdx.x;
    const int64_t c0 = (int64_t)blockIdx.x * TN;
    const int nb = (r + 1) / 2;
    for (int i = tid; i < TN * r; i += blockDim.x) {
        const int cc = i / r, k = i - (i / r) * r;
        const int64_t c = c0 + cc;
        Bs[k * TN + cc] = (c < C) ? int4_dequant(qc + c * nb, k, qs) : 0.0f;
    }
    const int w = tid >> 5, l = tid & 31;
    const int64_t c = c0 + 8 * l;
    const bool col_ok = c < C;  // C % 8 == 0: 8 channels are all in or all out
    const int64_t ntiles = (T + TM - 1) / TM;
    for (int64_t tile = blockIdx.y; tile < ntiles; tile += gridDim.y) {
        const int64_t t0 = tile * TM;
        float ro[4][8];
        uint4 xv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t t = t0 + 4 * w + i;
            if (col_ok && t < T) {
                const float4 a = ld_state_v4(recon + t * C + c);
                const float4 b = ld_state_v4(recon + t * C + c + 4);
                ro[i][0] = a.x; ro[i][1] = a.y; ro[i][2] = a.z; ro[i][3] = a.w;
                ro[i][4] = b.x; ro[i][5] = b.y; ro[i][6] = b.z; ro[i][7] = b.w;
                xv[i] = SENDER ? ld_ro_v4(x + t * C + c) : make_uint4(0, 0, 0, 0);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) ro[i][j] = 0.0f;
                xv[i] = make_uint4(0, 0, 0, 0);
            }
        }
        __syncthreads();  // the previous tile's reads of As are done
        for (int i = tid; i < TM * r; i += blockDim.x) {
            const int tt = i / r, k = i - (i / r) * r;
            const int64_t t = t0 + tt;
            As[k * TM + tt] = (t < T) ? int4_dequant(pc + t * nb, k, ps) : 0.0f;
        }
        __syncthreads();
        float acc[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
        for (int k = 0; k < r; ++k) {
            const float4 a = *reinterpret_cast<const float4 *>(As + k * TM + 4 * w);
            const float4 b0 = *reinterpret_cast<const float4 *>(Bs + k * TN + 8 * l);
            const float4 b1 = *reinterpret_cast<const float4 *>(Bs + k * TN + 8 * l + 4);
            const float av[4] = {a.x, a.y, a.z, a.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = __fmaf_rn(av[i], bv[j], acc[i][j]);
        }
        if (!col_ok) continue;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t t = t0 + 4 * w + i;
            if (t >= T) break;
            float rn[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) rn[j] = __fadd_rn(ro[i][j], acc[i][j]);
            if (SENDER) {
                const uint32_t w4[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
                float eo[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float xf = bf16_bits_to_f32((w4[j >> 1] >> ((j & 1) * 16)) & 0xffffu);
                    eo[j] = __fsub_rn(__fsub_rn(xf, ro[i][j]), acc[i][j]);
                }
                st_stream_v4(err + t * C + c, make_float4(eo[0], eo[1], eo[2], eo[3]));
                st_stream_v4(err + t * C + c + 4, make_float4(eo[4], eo[5], eo[6], eo[7]));
            }
            st_state_v4(recon + t * C + c, make_float4(rn[0], rn[1], rn[2], rn[3]));
            st_state_v4(recon + t * C + c + 4, make_float4(rn[4], rn[5], rn[6], rn[7]));
        }
    }
}

}  // namespace cf
