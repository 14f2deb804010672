// lowrank_kernels.cuh -- device kernels of the low-rank mode (CUDA cores).
//
// The two dense products of subspace iteration (Y = V Q and Q = V^T P) have
// tensor-core versions in lowrank_umma.cuh; the SIMT versions here are the
// straightforward form, used for shapes the tensor-core tiles do not cover
// and as an on-device cross-check of them.
#pragma once

#include <cuda_bf16.h>
#include <math.h>

#include "cf.h"
#include "cf_common.cuh"
#include "lowrank_api.cuh"

namespace cf {

using bf16 = __nv_bfloat16;

// Vb = bf16_rn((float)x - recon): the residual the projections read.
__global__ void lr_residual_kernel(const uint16_t *x, const float *recon, bf16 *vb, int64_t n) {
    const int64_t groups = n >> 3;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += stride) {
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
__global__ void lr_omega_kernel(const float *omega, bf16 *qt, int64_t C, int r, int rp) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)rp * C) return;
    const int k = (int)(i / C);
    const int64_t c = i - (int64_t)k * C;
    qt[i] = __float2bfloat16_rn(k < r ? omega[c * r + k] : 0.0f);
}

// Yp[s][t][k] = sum over the channels of split s of Vb[t][c] * Qt[k][c].
// Block: 64 tokens; thread (tok = tid/4, kg = tid%4) owns k = kg + 4j.
__global__ void __launch_bounds__(256)
lr_project_simt(const bf16 *vb, const bf16 *qt, float *yp, int64_t T, int64_t C, int rp) {
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

// Y = sum of the split partials (fixed order), and this block's partial Gram
// matrix Gp[blk] = Y_blk^T Y_blk in fp64 over its 64 tokens.
__global__ void __launch_bounds__(256)
lr_reduce_gram_kernel(const float *yp, float *y, double *gp, int64_t T, int rp, int splits) {
    __shared__ float Ys[64][65];
    const int tid = threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.x * cf_lowrank::kGramTok;
    for (int i = tid; i < 64 * rp; i += 256) {
        const int tt = i / rp, k = i - (i / rp) * rp;
        const int64_t t = t0 + tt;
        float v = 0.0f;
        if (t < T) {
            for (int s = 0; s < splits; ++s) v += yp[((int64_t)s * T + t) * rp + k];
            y[t * rp + k] = v;
        }
        Ys[tt][k] = v;
    }
    __syncthreads();
    double *g = gp + (int64_t)blockIdx.x * rp * rp;
    for (int e = tid; e < rp * rp; e += 256) {
        const int i = e / rp, j = e - (e / rp) * rp;
        double acc = 0.0;
        for (int tt = 0; tt < 64; ++tt) acc += (double)Ys[tt][i] * (double)Ys[tt][j];
        g[e] = acc;
    }
}

// One CTA: G = sum of the partial Grams; upper Cholesky G = R^T R in fp64;
// Rinv = R^-1 (fp32, zero padded to rp x rp).  A pivot that is not positive,
// or below 1e-10 of its diagonal entry (the column is numerically in the
// span of the earlier ones), marks the column dead: its row of R and its
// column of Rinv are zero, so P gets a zero column, and CF_ERR_NUMERIC is
// recorded in the status word.
__global__ void __launch_bounds__(256)
lr_chol_kernel(const double *gp, int nblk, float *rinv, int r, int rp, int32_t *status) {
    // dynamic shared memory: G, R, X as [rp][rp+1] fp64, then dead flags
    extern __shared__ double dsm[];
    const int ld = rp + 1;
    double *G = dsm;
    double *R = G + rp * ld;
    double *X = R + rp * ld;
    int *dead = reinterpret_cast<int *>(X + rp * ld);
    __shared__ int any_dead;
    const int tid = threadIdx.x;
    for (int e = tid; e < rp * rp; e += blockDim.x) {
        double acc = 0.0;
        for (int b = 0; b < nblk; ++b) acc += gp[(int64_t)b * rp * rp + e];
        G[(e / rp) * ld + e % rp] = acc;
    }
    for (int e = tid; e < rp * ld; e += blockDim.x) {
        R[e] = 0.0;
        X[e] = 0.0;
    }
    if (tid == 0) any_dead = 0;
    __syncthreads();
    for (int j = 0; j < r; ++j) {
        if (tid == 0) {
            double d = G[j * ld + j];
            for (int k = 0; k < j; ++k) d -= R[k * ld + j] * R[k * ld + j];
            const bool bad = !(d > 0.0) || !(d > 1e-10 * G[j * ld + j]);
            dead[j] = bad ? 1 : 0;
            R[j * ld + j] = bad ? 0.0 : sqrt(d);
            if (bad) any_dead = 1;
        }
        __syncthreads();
        for (int i = j + 1 + tid; i < r; i += blockDim.x) {
            double s = G[j * ld + i];
            for (int k = 0; k < j; ++k) s -= R[k * ld + j] * R[k * ld + i];
            R[j * ld + i] = dead[j] ? 0.0 : s / R[j * ld + j];
        }
        __syncthreads();
    }
    // X = R^-1 by back substitution, one column per thread.
    if (tid < r) {
        const int c = tid;
        if (!dead[c]) {
            X[c * ld + c] = 1.0 / R[c * ld + c];
            for (int i = c - 1; i >= 0; --i) {
                if (dead[i]) continue;
                double s = 0.0;
                for (int k = i + 1; k <= c; ++k) s += R[i * ld + k] * X[k * ld + c];
                X[i * ld + c] = -s / R[i * ld + i];
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < rp * rp; e += blockDim.x) {
        const int i = e / rp, c = e % rp;
        rinv[e] = (i < r && c < r) ? (float)X[i * ld + c] : 0.0f;
    }
    if (tid == 0 && any_dead) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_NUMERIC);
}

inline size_t lr_chol_smem_bytes(int rp) {
    return (size_t)3 * rp * (rp + 1) * sizeof(double) + (size_t)rp * sizeof(int);
}

// P = Y Rinv (fp32 [T][rp]) and its bf16 transpose Pt [rp][Tp] (zero past T).
__global__ void lr_orth_kernel(const float *y, const float *rinv, float *p, bf16 *pt, int64_t T,
                               int64_t Tp, int r, int rp) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= Tp * rp) return;
    const int64_t t = i / rp;
    const int k = (int)(i - t * rp);
    float v = 0.0f;
    if (t < T && k < r) {
        const float *yr = y + t * rp;
        for (int j = 0; j <= k; ++j) v = fmaf(yr[j], rinv[j * rp + k], v);
    }
    if (t < T) p[t * rp + k] = v;
    pt[(int64_t)k * Tp + t] = __float2bfloat16_rn(v);
}

// Zp[s][c][k] = sum over the tokens of split s of Vb[t][c] * Pt[k][t].
__global__ void __launch_bounds__(256)
lr_backproject_simt(const bf16 *vb, const bf16 *pt, float *zp, int64_t T, int64_t Tp, int64_t C,
                    int rp) {
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

// Q = sum of the split partials (fixed order): fp32 [C][rp] and bf16 Qt.
__global__ void lr_reduce_q_kernel(const float *zp, float *q, bf16 *qt, int64_t C, int rp,
                                   int splits) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= C * rp) return;
    const int64_t c = i / rp;
    const int k = (int)(i - c * rp);
    float v = 0.0f;
    for (int s = 0; s < splits; ++s) v += zp[(int64_t)s * C * rp + i];
    q[i] = v;
    qt[(int64_t)k * C + c] = __float2bfloat16_rn(v);
}

// amax[k] = max over rows of |f[row][k]| as float bits (non-negative floats
// order like their bit patterns).
__global__ void lr_absmax_kernel(const float *f, int64_t rows, int r, int rp, uint32_t *amax) {
    const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int k = 0; k < r; ++k) {
        float m = (row < rows) ? fabsf(f[row * rp + k]) : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
        if ((threadIdx.x & 31) == 0) atomicMax(amax + k, __float_as_uint(m));
    }
}

__device__ __forceinline__ int int4_code(float v, float s) {
    if (!(s > 0.0f)) return 0;
    float q = rintf(__fdiv_rn(v, s));
    q = fminf(fmaxf(q, -7.0f), 7.0f);
    return (int)q;
}

// INT4 per column: s_k = amax_k / 7; codes packed two per byte, the even
// column in the low nibble; the scales are written by the first r threads.
__global__ void lr_int4_pack_kernel(const float *f, int64_t rows, int r, int rp,
                                    const uint32_t *amax, uint8_t *codes, float *scales) {
    const int nb = (r + 1) / 2;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < r) scales[i] = __fdiv_rn(__uint_as_float(amax[i]), 7.0f);
    if (i >= rows * nb) return;
    const int64_t row = i / nb;
    const int b = (int)(i - row * nb);
    const int k0 = 2 * b, k1 = 2 * b + 1;
    const int q0 = int4_code(f[row * rp + k0], __fdiv_rn(__uint_as_float(amax[k0]), 7.0f));
    const int q1 = (k1 < r) ? int4_code(f[row * rp + k1], __fdiv_rn(__uint_as_float(amax[k1]), 7.0f)) : 0;
    codes[i] = (uint8_t)((q0 & 0xF) | ((q1 & 0xF) << 4));
}

__device__ __forceinline__ float int4_dequant(const uint8_t *row_codes, int k, const float *scales) {
    const uint32_t byte = row_codes[k >> 1];
    int q = (int)((byte >> ((k & 1) * 4)) & 0xFu);
    q = q >= 8 ? q - 16 : q;
    return __fmul_rn((float)q, __ldg(scales + k));
}

// D = (qP sP)(qQ sQ)^T on a 32-token x 256-channel tile, then
//   sender:   v = x - recon ; err = v - D ; recon = recon + D
//   receiver: recon = recon + D
// D is a fixed chain of fused multiply-adds in k order, so sender and
// receiver form bit-identical values from the same payload.
template <bool SENDER>
__global__ void __launch_bounds__(256)
lr_apply_kernel(const uint16_t *x, float *recon, float *err, const uint8_t *pc, const float *ps,
                const uint8_t *qc, const float *qs, int64_t T, int64_t C, int r) {
    extern __shared__ float sm[];
    float *As = sm;                                // [r][32]
    float *Bs = sm + (size_t)r * cf_lowrank::kApplyTok;  // [r][256]
    const int tid = threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.y * cf_lowrank::kApplyTok;
    const int64_t c0 = (int64_t)blockIdx.x * cf_lowrank::kApplyCh;
    const int nb = (r + 1) / 2;
    for (int i = tid; i < cf_lowrank::kApplyTok * r; i += blockDim.x) {
        const int tt = i / r, k = i - (i / r) * r;
        const int64_t t = t0 + tt;
        As[k * cf_lowrank::kApplyTok + tt] = (t < T) ? int4_dequant(pc + t * nb, k, ps) : 0.0f;
    }
    for (int i = tid; i < cf_lowrank::kApplyCh * r; i += blockDim.x) {
        const int cc = i / r, k = i - (i / r) * r;
        const int64_t c = c0 + cc;
        Bs[k * cf_lowrank::kApplyCh + cc] = (c < C) ? int4_dequant(qc + c * nb, k, qs) : 0.0f;
    }
    __syncthreads();
    const int w = tid >> 5, l = tid & 31;
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
    for (int k = 0; k < r; ++k) {
        const float4 a = *reinterpret_cast<const float4 *>(As + k * cf_lowrank::kApplyTok + 4 * w);
        const float4 b0 = *reinterpret_cast<const float4 *>(Bs + k * cf_lowrank::kApplyCh + 8 * l);
        const float4 b1 = *reinterpret_cast<const float4 *>(Bs + k * cf_lowrank::kApplyCh + 8 * l + 4);
        const float av[4] = {a.x, a.y, a.z, a.w};
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = __fmaf_rn(av[i], bv[j], acc[i][j]);
    }
    const int64_t c = c0 + 8 * l;
    if (c >= C) return;  // C % 8 == 0: a group of 8 channels is all in or all out
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t t = t0 + 4 * w + i;
        if (t >= T) break;
        float *rr = recon + t * C + c;
        const float4 ra = ld_state_v4(rr), rb = ld_state_v4(rr + 4);
        const float ro[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
        float rn[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) rn[j] = __fadd_rn(ro[j], acc[i][j]);
        if (SENDER) {
            const uint4 xv = ld_ro_v4(x + t * C + c);
            const uint32_t w4[4] = {xv.x, xv.y, xv.z, xv.w};
            float eo[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float v = __fsub_rn(bf16_bits_to_f32((w4[j >> 1] >> ((j & 1) * 16)) & 0xffffu), ro[j]);
                eo[j] = __fsub_rn(v, acc[i][j]);
            }
            st_stream_v4(err + t * C + c, make_float4(eo[0], eo[1], eo[2], eo[3]));
            st_stream_v4(err + t * C + c + 4, make_float4(eo[4], eo[5], eo[6], eo[7]));
        }
        st_state_v4(rr, make_float4(rn[0], rn[1], rn[2], rn[3]));
        st_state_v4(rr + 4, make_float4(rn[4], rn[5], rn[6], rn[7]));
    }
}

}  // namespace cf
