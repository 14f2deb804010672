// quant_kernels.cuh -- fused quantize-mode encode and decode kernels.
//
// Method: "Accelerating Parallel Diffusion Model Serving with Residual
// Compression" (CompactFusion summary), "Approach": the sender compresses
// the residual against the previous reconstruction and keeps an error
// feedback buffer; the "Measured effects" table names the 1-bit and 2-bit
// quantisers.  The per-row arithmetic is the one documented in cf.h.
//
// Design (B200, HBM bound: 14.1-14.3 B/element encode, 8.1-8.3 decode):
//  * One CTA owns one token row at a time and walks rows in a grid-stride
//    loop over ALL buffers of a batched call (row = buffer * T + token), so a
//    step of 114 buffers is one launch with no tail per buffer.
//  * A thread owns GPT groups of 8 consecutive channels; group g of the row
//    goes to thread g % blockDim, so each warp-wide access is contiguous.
//    x is read with one 16-byte load per group, recon with two, and the
//    whole row stays in registers between the scale reduction and the
//    quantise/update phase: every state byte crosses HBM once.
//  * Scale reduction: warp shuffles, then one shared-memory slot per warp
//    (double-buffered by row parity so one __syncthreads per row suffices),
//    combined by every thread in the same fixed order.  The 1-bit mean-abs
//    sum is accumulated in fp64 like the definition, so the fp32 scale
//    agrees with a sequential fp64 sum except in the rare case where the
//    two fp64 sums straddle an fp32 rounding boundary.
//  * Packing: a group yields 8*BITS code bits; the 4/BITS lanes that share a
//    32-bit word OR their fields together with xor-shuffles and the first of
//    them stores the word.
//  * All state arithmetic uses __fadd_rn/__fsub_rn/__fmul_rn so nothing is
//    contracted into an FMA: sender mirror and receiver update compute the
//    identical rounded value.
#pragma once

#include <cuda_bf16.h>

#include "bounds.cuh"
#include "cf.h"
#include "cf_common.cuh"

namespace cf {

struct EncPtrs {
    const uint16_t *x;
    float *recon;             // standard sender: the reconstruction copy
    float *err;
    uint32_t *codes;
    float *scales;
    const uint16_t *xprev;    // delta-state sender: the previous activation
    int64_t codes_off = 0;    // publishing sender: byte offsets in a payload slot
    int64_t scales_off = 0;
};

struct DecPtrs {
    const uint32_t *codes;
    const float *scales;
    float *recon;
    uint16_t *out;  // bf16 copy of the new reconstruction (emitting decode only)
    const uint64_t *ready = nullptr;  // waiting decode: the sender's ready counter
};

template <class P>
__device__ __forceinline__ P ldg_ptr(P const *field) {
    return reinterpret_cast<P>(
        __ldg(reinterpret_cast<const unsigned long long *>(field)));
}

// Pointer sources: a single buffer passed by value (validated on the host)
// or a device array of buffers (validated per buffer on the device).
struct EncSingle {
    EncPtrs p;
    static constexpr bool kChecked = false;
    static constexpr bool kDelta = false;
    static constexpr bool kPublish = false, kWait = false;
    __device__ __forceinline__ EncPtrs get(int64_t) const { return p; }
};
struct EncDeltaSingle {
    EncPtrs p;
    static constexpr bool kChecked = false;
    static constexpr bool kDelta = true;
    static constexpr bool kPublish = false, kWait = false;
    __device__ __forceinline__ EncPtrs get(int64_t) const { return p; }
};
struct EncDeltaArray {
    const cf_enc_delta_buffer *a;
    static constexpr bool kChecked = true;
    static constexpr bool kDelta = true;
    static constexpr bool kPublish = false, kWait = false;
    __device__ __forceinline__ EncPtrs get(int64_t i) const {
        const cf_enc_delta_buffer *e = a + i;
        EncPtrs p;
        p.x = ldg_ptr(&e->x);
        p.xprev = ldg_ptr(&e->x_prev);
        p.recon = nullptr;
        p.err = ldg_ptr(&e->err);
        p.codes = ldg_ptr(&e->codes);
        p.scales = ldg_ptr(&e->scales);
        return p;
    }
};
struct EncArray {
    const cf_enc_buffer *a;
    static constexpr bool kChecked = true;
    static constexpr bool kDelta = false;
    static constexpr bool kPublish = false, kWait = false;
    __device__ __forceinline__ EncPtrs get(int64_t i) const {
        const cf_enc_buffer *e = a + i;
        EncPtrs p;
        p.x = ldg_ptr(&e->x);
        p.recon = ldg_ptr(&e->recon_s);
        p.err = ldg_ptr(&e->err);
        p.codes = ldg_ptr(&e->codes);
        p.scales = ldg_ptr(&e->scales);
        p.xprev = nullptr;
        return p;
    }
};
template <bool EMIT>
struct DecSingleT {
    DecPtrs p;
    static constexpr bool kChecked = false;
    static constexpr bool kEmit = EMIT;
    static constexpr bool kPublish = false, kWait = false;
    __device__ __forceinline__ DecPtrs get(int64_t) const { return p; }
};
using DecSingle = DecSingleT<false>;
using DecEmitSingle = DecSingleT<true>;
struct DecArray {
    const cf_dec_buffer *a;
    static constexpr bool kChecked = true;
    static constexpr bool kEmit = false;
    static constexpr bool kPublish = false, kWait = false;
    __device__ __forceinline__ DecPtrs get(int64_t i) const {
        const cf_dec_buffer *e = a + i;
        DecPtrs p;
        p.codes = ldg_ptr(&e->codes);
        p.scales = ldg_ptr(&e->scales);
        p.recon = ldg_ptr(&e->recon_r);
        p.out = nullptr;
        return p;
    }
};
struct DecEmitArray {
    const cf_dec_emit_buffer *a;
    static constexpr bool kChecked = true;
    static constexpr bool kEmit = true;
    static constexpr bool kPublish = false, kWait = false;
    __device__ __forceinline__ DecPtrs get(int64_t i) const {
        const cf_dec_emit_buffer *e = a + i;
        DecPtrs p;
        p.codes = ldg_ptr(&e->codes);
        p.scales = ldg_ptr(&e->scales);
        p.recon = ldg_ptr(&e->recon_r);
        p.out = ldg_ptr(&e->out);
        return p;
    }
};

// 8 fp32 values -> 8 bf16 (round to nearest even) packed in 16 bytes.
__device__ __forceinline__ uint4 pack_bf16x8(const float *v) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
        w[k] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Scales are per-token fp32 scalars: 4-byte alignment suffices for them.
__device__ __forceinline__ bool misaligned4(const void *p) {
    return (reinterpret_cast<uintptr_t>(p) & 3u) != 0;
}
template <bool DELTA, bool PUBLISH = false>
__device__ __forceinline__ int enc_ptr_status(const EncPtrs &p) {
    const void *state = DELTA ? static_cast<const void *>(p.xprev) : static_cast<const void *>(p.recon);
    if (PUBLISH) {  // codes and scales go to the destinations, at these offsets
        if (!p.x || !state || !p.err || p.codes_off < 0 || p.scales_off < 0) return CF_ERR_INVALID_ARG;
        if (misaligned16(p.x) || misaligned16(state) || misaligned16(p.err) || (p.codes_off & 15) ||
            (p.scales_off & 3))
            return CF_ERR_ALIGNMENT;
        return CF_OK;
    }
    if (!p.x || !state || !p.err || !p.codes || !p.scales) return CF_ERR_INVALID_ARG;
    if (misaligned16(p.x) || misaligned16(state) || misaligned16(p.err) ||
        misaligned16(p.codes) || misaligned4(p.scales))
        return CF_ERR_ALIGNMENT;
    return CF_OK;
}
template <bool EMIT, bool WAIT = false>
__device__ __forceinline__ int dec_ptr_status(const DecPtrs &p) {
    if (!p.codes || !p.scales || !p.recon || (EMIT && !p.out) || (WAIT && !p.ready))
        return CF_ERR_INVALID_ARG;
    if (misaligned16(p.codes) || misaligned4(p.scales) || misaligned16(p.recon) ||
        (EMIT && misaligned16(p.out)) || (WAIT && (reinterpret_cast<uintptr_t>(p.ready) & 7u)))
        return CF_ERR_ALIGNMENT;
    return CF_OK;
}

__device__ __forceinline__ void report(int32_t *status, int code) {
    if (status) atomicCAS(status, (int32_t)CF_OK, (int32_t)code);
}

// ---- exchange counters (publishing encode / waiting decode)

__device__ __forceinline__ uint64_t ld_acquire_sys(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Polls of a counter before a wait gives up; with the backoff below (up to
// about a microsecond between polls) that is on the order of a second.
constexpr uint32_t kCounterPolls = 1u << 20;

// Bounded wait until *p >= target (system-scope acquire); false on expiry.
__device__ __forceinline__ bool wait_counter(const uint64_t *p, uint64_t target,
                                             uint32_t polls = kCounterPolls) {
    uint32_t ns = 32;
    for (uint32_t i = 0; i < polls; ++i) {
        if (ld_acquire_sys(p) >= target) return true;
        __nanosleep(ns);
        if (ns < 1024) ns <<= 1;
    }
    return false;
}

// Publishing encode: buffers of cf_enc_publish_buffer, destinations of
// cf_publish_dst (the library's host code caps ndst at 8).
struct EncPublishArray {
    const cf_enc_publish_buffer *a;
    const cf_publish_dst *dst;
    int ndst;
    uint64_t ack_target;
    static constexpr bool kChecked = true;
    static constexpr bool kDelta = false;
    static constexpr bool kPublish = true, kWait = false;
    __device__ __forceinline__ EncPtrs get(int64_t i) const {
        const cf_enc_publish_buffer *e = a + i;
        EncPtrs p;
        p.x = ldg_ptr(&e->x);
        p.recon = ldg_ptr(&e->recon_s);
        p.err = ldg_ptr(&e->err);
        p.codes = nullptr;
        p.scales = nullptr;
        p.xprev = nullptr;
        p.codes_off = __ldg(reinterpret_cast<const long long *>(&e->codes_offset));
        p.scales_off = __ldg(reinterpret_cast<const long long *>(&e->scales_offset));
        return p;
    }
    // Destination pointers valid and aligned, then every ack counter at the
    // target (bounded).  On failure records the status and returns false.
    __device__ bool check_and_wait(int32_t *status) const {
        for (int d = 0; d < ndst; ++d) {
            const uint8_t *pl = ldg_ptr(&dst[d].payload);
            const uint64_t *rd = ldg_ptr(&dst[d].ready);
            const uint64_t *ak = ldg_ptr(&dst[d].ack);
            if (!pl || !rd) {
                report(status, CF_ERR_INVALID_ARG);
                return false;
            }
            if (misaligned16(pl) || (reinterpret_cast<uintptr_t>(rd) & 7u) ||
                (reinterpret_cast<uintptr_t>(ak) & 7u)) {
                report(status, CF_ERR_ALIGNMENT);
                return false;
            }
        }
        if (ack_target == 0) return true;
        for (int d = 0; d < ndst; ++d) {
            const uint64_t *ak = ldg_ptr(&dst[d].ack);
            if (ak && !wait_counter(ak, ack_target)) {
                report(status, CF_ERR_TIMEOUT);
                return false;
            }
        }
        return true;
    }
    // A warp's gathered code words of one unit block into every destination:
    // with 16-byte code rows (W % 4 == 0) lanes 0 .. nvec - 1 store q[0..3],
    // words w0 + 4 lane .. + 3; otherwise each word's first lane (own) stores
    // its word at index wi.  w0 is a multiple of 4, so a vector never
    // straddles the end of a row.
    __device__ __forceinline__ void store_words(const EncPtrs &p, int64_t t, int64_t W, int64_t w0, int lane,
                                                int nvec, const uint32_t *q, uint32_t word, bool own,
                                                int64_t wi) const {
        const bool vec = (W & 3) == 0;
        for (int d = 0; d < ndst; ++d) {
            uint32_t *crow = reinterpret_cast<uint32_t *>(ldg_ptr(&dst[d].payload) + p.codes_off) + t * W;
            if (vec) {
                if (lane < nvec && w0 + 4 * lane + 4 <= W)
                    *reinterpret_cast<uint4 *>(crow + w0 + 4 * lane) = make_uint4(q[0], q[1], q[2], q[3]);
            } else if (own && CF_IN(wi < W)) {
                crow[wi] = word;
            }
        }
    }
    __device__ __forceinline__ void store_scale(const EncPtrs &p, int64_t t, float scale) const {
        for (int d = 0; d < ndst; ++d)
            reinterpret_cast<float *>(ldg_ptr(&dst[d].payload) + p.scales_off)[t] = scale;
    }
    // Release of this CTA's rows: the fence orders every store the CTA made
    // (observed through the barrier before this call) before the adds.
    __device__ __forceinline__ void publish(uint64_t rows) const {
        __threadfence_system();
        for (int d = 0; d < ndst; ++d)
            atomicAdd_system(reinterpret_cast<unsigned long long *>(ldg_ptr(&dst[d].ready)),
                             (unsigned long long)rows);
    }
};

// Waiting decode: buffers of cf_dec_wait_buffer, all waited for up to the
// same ready target.
struct DecWaitArray {
    const cf_dec_wait_buffer *a;
    uint64_t target;
    static constexpr bool kChecked = true;
    static constexpr bool kEmit = false;
    static constexpr bool kPublish = false, kWait = true;
    __device__ __forceinline__ DecPtrs get(int64_t i) const {
        const cf_dec_wait_buffer *e = a + i;
        DecPtrs p;
        p.codes = ldg_ptr(&e->codes);
        p.scales = ldg_ptr(&e->scales);
        p.recon = ldg_ptr(&e->recon_r);
        p.out = nullptr;
        p.ready = ldg_ptr(&e->ready);
        return p;
    }
    __device__ __forceinline__ bool wait_ready(int64_t i) const {
        return wait_counter(ldg_ptr(&a[i].ready), target);
    }
};


// Code of one residual value.  1 bit: [v >= 0].  2 bits: number of the
// thresholds -A/2, 0, A/2 that v reaches (ties go to the upper bin).
template <int BITS>
__device__ __forceinline__ uint32_t quantize(float v, float half) {
    if (BITS == 1) return v >= 0.0f ? 1u : 0u;
    return (uint32_t)(v >= -half) + (uint32_t)(v >= 0.0f) + (uint32_t)(v >= half);
}

// Reconstruction level: 1 bit +-s; 2 bits (2k-3)/4 * A, i.e. the centres of
// the four equal bins of [-A, A].  (2k-3)/4 is exact; one rounded product.
template <int BITS>
__device__ __forceinline__ float dequantize(uint32_t code, float scale) {
    if (BITS == 1) return code ? scale : -scale;
    const float lvl = (float)((int)(2u * code) - 3) * 0.25f;
    return __fmul_rn(lvl, scale);
}

// Residual of 8 channels from their raw bf16 words.  Standard sender:
// v = (float)x - recon.  Delta-state sender: v = ((float)x - (float)x_prev)
// + err_old, two roundings in that order.  r holds recon or err_old.
template <bool DELTA>
__device__ __forceinline__ void residual8(const uint4 &xw, const uint4 &pw, const float *r, float *v) {
    const uint32_t w4[4] = {xw.x, xw.y, xw.z, xw.w};
    const uint32_t p4[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float xf = bf16_bits_to_f32((w4[e >> 1] >> ((e & 1) * 16)) & 0xffffu);
        if (DELTA) {
            const float pf = bf16_bits_to_f32((p4[e >> 1] >> ((e & 1) * 16)) & 0xffffu);
            v[e] = __fadd_rn(__fsub_rn(xf, pf), r[e]);
        } else {
            v[e] = __fsub_rn(xf, r[e]);
        }
    }
}

// The same for 4 channels (two bf16 words), used by the TMA pipeline.
template <bool DELTA>
__device__ __forceinline__ void residual4(const uint2 &xw, const uint2 &pw, const float *r, float *v) {
    const uint32_t w2[2] = {xw.x, xw.y};
    const uint32_t p2[2] = {pw.x, pw.y};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float xf = bf16_bits_to_f32((w2[e >> 1] >> ((e & 1) * 16)) & 0xffffu);
        if (DELTA) {
            const float pf = bf16_bits_to_f32((p2[e >> 1] >> ((e & 1) * 16)) & 0xffffu);
            v[e] = __fadd_rn(__fsub_rn(xf, pf), r[e]);
        } else {
            v[e] = __fsub_rn(xf, r[e]);
        }
    }
}

// 4 fp32 values -> 4 bf16 (round to nearest even) packed in 8 bytes.
__device__ __forceinline__ uint2 pack_bf16x4(const float *v) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    return make_uint2(*reinterpret_cast<const uint32_t *>(&a), *reinterpret_cast<const uint32_t *>(&b));
}

template <int BITS, int GPT, bool VEC, class Src>
__global__ void __launch_bounds__(512)
encode_rows_kernel(Src src, int64_t T, int64_t C, int64_t rows, int32_t *status) {
    constexpr int GPW = 4 / BITS;  // 8-channel groups per 32-bit code word
    const int tid = threadIdx.x;
    const int nt = blockDim.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int nw = nt >> 5;
    const int64_t G = (C + 7) >> 3;
    const int64_t W = (C * BITS + 31) >> 5;

    __shared__ double sh_sum[2][32];
    __shared__ float sh_max[2][32];

    // par alternates the scale slots between consecutive rows that reach
    // the row barrier.  A skipped row (bad buffer) reaches no barrier, so it
    // must not flip par: otherwise a fast warp could write the next row's
    // slot while a slow one still reads it for the previous row.
    int par = 0;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        const int64_t b = row / T;
        const int64_t t = row - b * T;
        const EncPtrs p = src.get(b);
        if (Src::kChecked) {
            const int st = enc_ptr_status<Src::kDelta>(p);
            if (st != CF_OK) {
                if (tid == 0) report(status, st);
                continue;  // uniform across the CTA
            }
        }
        const uint16_t *xr = p.x + t * C;
        // r: the reconstruction (standard sender) or the old error (delta)
        float *rr = (Src::kDelta ? p.err : p.recon) + t * C;
        const uint16_t *pr = Src::kDelta ? p.xprev + t * C : nullptr;
        float *er = p.err + t * C;
        uint32_t *cw = p.codes + t * W;

        // Phase 1: issue every load of this thread's groups.
        uint4 xraw[GPT], praw[GPT];
        float r[GPT][8];
#pragma unroll
        for (int j = 0; j < GPT; ++j) {
            const int64_t g = (int64_t)j * nt + tid;
            if (VEC) {
                if (g < G && CF_IN(8 * g + 8 <= C && t < T)) {
                    xraw[j] = ld_ro_v4(xr + 8 * g);
                    if (Src::kDelta) praw[j] = ld_ro_v4(pr + 8 * g);
                    const float4 a = ld_state_v4(rr + 8 * g);
                    const float4 c = ld_state_v4(rr + 8 * g + 4);
                    r[j][0] = a.x; r[j][1] = a.y; r[j][2] = a.z; r[j][3] = a.w;
                    r[j][4] = c.x; r[j][5] = c.y; r[j][6] = c.z; r[j][7] = c.w;
                } else {
                    xraw[j] = praw[j] = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int e = 0; e < 8; ++e) r[j][e] = 0.0f;
                }
            } else {
                uint32_t h[8], hp[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int64_t c = 8 * g + e;
                    const bool ok = (g < G) && (c < C);
                    h[e] = ok ? (uint32_t)xr[c] : 0u;
                    hp[e] = (Src::kDelta && ok) ? (uint32_t)pr[c] : 0u;
                    r[j][e] = ok ? rr[c] : 0.0f;
                }
                xraw[j] = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16),
                                     h[4] | (h[5] << 16), h[6] | (h[7] << 16));
                praw[j] = make_uint4(hp[0] | (hp[1] << 16), hp[2] | (hp[3] << 16),
                                     hp[4] | (hp[5] << 16), hp[6] | (hp[7] << 16));
            }
        }

        // Phase 2: residual (padding lanes hold zeros, so v = 0).
        float v[GPT][8];
#pragma unroll
        for (int j = 0; j < GPT; ++j)
            residual8<Src::kDelta>(xraw[j], praw[j], r[j], v[j]);

        // Phase 3: per-token scale.
        float scale;
        if (BITS == 1) {
            double acc = 0.0;
#pragma unroll
            for (int j = 0; j < GPT; ++j)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc += (double)fabsf(v[j][e]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFullMask, acc, o);
            if (lane == 0) sh_sum[par][warp] = acc;
            __syncthreads();
            double tot = 0.0;
            for (int w = 0; w < nw; ++w) tot += sh_sum[par][w];
            scale = __fdiv_rn(__double2float_rn(tot), (float)C);
        } else {
            float m = 0.0f;
#pragma unroll
            for (int j = 0; j < GPT; ++j)
#pragma unroll
                for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[j][e]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
            if (lane == 0) sh_max[par][warp] = m;
            __syncthreads();
            float tot = 0.0f;
            for (int w = 0; w < nw; ++w) tot = fmaxf(tot, sh_max[par][w]);
            scale = tot;
        }
        par ^= 1;
        const float half = __fmul_rn(0.5f, scale);

        // Phase 4: quantise, error feedback, mirror update, pack, store.
#pragma unroll
        for (int j = 0; j < GPT; ++j) {
            const int64_t g = (int64_t)j * nt + tid;
            uint32_t field = 0;
            float eo[8], ro[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const bool ok = VEC ? (g < G) : ((g < G) && (8 * g + e < C));
                uint32_t code = quantize<BITS>(v[j][e], half);
                code = ok ? code : 0u;
                field |= code << (e * BITS);
                const float d = dequantize<BITS>(code, scale);
                eo[e] = __fsub_rn(v[j][e], d);
                ro[e] = __fadd_rn(r[j][e], d);
            }
            uint32_t word = field << ((lane % GPW) * 8 * BITS);
#pragma unroll
            for (int o = 1; o < GPW; o <<= 1) word |= __shfl_xor_sync(kFullMask, word, o);
            if (g < G && CF_IN(8 * g + (VEC ? 8 : 1) <= C && t < T)) {
                if (VEC) {
                    st_stream_v4(er + 8 * g, make_float4(eo[0], eo[1], eo[2], eo[3]));
                    st_stream_v4(er + 8 * g + 4, make_float4(eo[4], eo[5], eo[6], eo[7]));
                    if (!Src::kDelta) {
                        st_state_v4(rr + 8 * g, make_float4(ro[0], ro[1], ro[2], ro[3]));
                        st_state_v4(rr + 8 * g + 4, make_float4(ro[4], ro[5], ro[6], ro[7]));
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int64_t c = 8 * g + e;
                        if (c < C) {
                            er[c] = eo[e];
                            if (!Src::kDelta) rr[c] = ro[e];
                        }
                    }
                }
                if ((lane % GPW) == 0 && CF_IN(g / GPW < W)) cw[g / GPW] = word;
            }
        }
        if (tid == 0 && CF_IN(t < T)) p.scales[t] = scale;
    }
}

template <int BITS, int GPT, bool VEC, class Src>
__global__ void __launch_bounds__(512)
decode_rows_kernel(Src src, int64_t T, int64_t C, int64_t rows, int32_t *status) {
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    const int tid = threadIdx.x;
    const int nt = blockDim.x;
    const int64_t G = (C + 7) >> 3;
    const int64_t W = (C * BITS + 31) >> 5;

    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        const int64_t b = row / T;
        const int64_t t = row - b * T;
        const DecPtrs p = src.get(b);
        if (Src::kChecked) {
            const int st = dec_ptr_status<Src::kEmit>(p);
            if (st != CF_OK) {
                if (tid == 0) report(status, st);
                continue;
            }
        }
        const float scale = __ldg(p.scales + t);
        const uint32_t *cw = p.codes + t * W;
        float *rr = p.recon + t * C;

        uint32_t field[GPT];
        float r[GPT][8];
#pragma unroll
        for (int j = 0; j < GPT; ++j) {
            const int64_t g = (int64_t)j * nt + tid;
            if (g < G && CF_IN((g + 1) * BITS <= 4 * W && t < T)) {
                // group g's 8*BITS bits: byte g (1 bit) or half-word g (2 bits)
                if (BITS == 1)
                    field[j] = __ldg(reinterpret_cast<const uint8_t *>(cw) + g);
                else
                    field[j] = __ldg(reinterpret_cast<const uint16_t *>(cw) + g);
            } else {
                field[j] = 0u;
            }
            if (VEC) {
                if (g < G && CF_IN(8 * g + 8 <= C)) {
                    const float4 a = ld_state_v4(rr + 8 * g);
                    const float4 c = ld_state_v4(rr + 8 * g + 4);
                    r[j][0] = a.x; r[j][1] = a.y; r[j][2] = a.z; r[j][3] = a.w;
                    r[j][4] = c.x; r[j][5] = c.y; r[j][6] = c.z; r[j][7] = c.w;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int64_t c = 8 * g + e;
                    r[j][e] = ((g < G) && (c < C)) ? rr[c] : 0.0f;
                }
            }
        }
#pragma unroll
        for (int j = 0; j < GPT; ++j) {
            const int64_t g = (int64_t)j * nt + tid;
            if (g >= G || !CF_IN(8 * g + (VEC ? 8 : 1) <= C)) continue;
            float ro[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t code = (field[j] >> (e * BITS)) & MASK;
                ro[e] = __fadd_rn(r[j][e], dequantize<BITS>(code, scale));
            }
            if (VEC) {
                st_state_v4(rr + 8 * g, make_float4(ro[0], ro[1], ro[2], ro[3]));
                st_state_v4(rr + 8 * g + 4, make_float4(ro[4], ro[5], ro[6], ro[7]));
                if (Src::kEmit)
                    *reinterpret_cast<uint4 *>(p.out + t * C + 8 * g) = pack_bf16x8(ro);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int64_t c = 8 * g + e;
                    if (c < C) {
                        rr[c] = ro[e];
                        if (Src::kEmit) {
                            const __nv_bfloat16 h = __float2bfloat16_rn(ro[e]);
                            p.out[t * C + c] = *reinterpret_cast<const uint16_t *>(&h);
                        }
                    }
                }
            }
        }
    }
}

// Warmup: recon = (float)x0, err = 0 (err may be null).  Flat over n
// elements; 8-element vector body, scalar tail.
__global__ void state_init_kernel(const uint16_t *x0, float *recon, float *err, int64_t n) {
    // recon or err may be null (not both; the host checks)
    const int64_t groups = n >> 3;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += stride) {
        if (!CF_IN(8 * g + 8 <= n)) continue;
        if (recon) {
            const uint4 xv = ld_ro_v4(x0 + 8 * g);
            const uint32_t w4[4] = {xv.x, xv.y, xv.z, xv.w};
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = bf16_bits_to_f32((w4[e >> 1] >> ((e & 1) * 16)) & 0xffffu);
            st_state_v4(recon + 8 * g, make_float4(f[0], f[1], f[2], f[3]));
            st_state_v4(recon + 8 * g + 4, make_float4(f[4], f[5], f[6], f[7]));
        }
        if (err) {
            st_stream_v4(err + 8 * g, make_float4(0.f, 0.f, 0.f, 0.f));
            st_stream_v4(err + 8 * g + 4, make_float4(0.f, 0.f, 0.f, 0.f));
        }
    }
    if (blockIdx.x == 0 && (int64_t)threadIdx.x < n - 8 * groups) {
        const int64_t i = 8 * groups + threadIdx.x;
        if (recon) recon[i] = bf16_bits_to_f32(x0[i]);
        if (err) err[i] = 0.0f;
    }
}

}  // namespace cf
