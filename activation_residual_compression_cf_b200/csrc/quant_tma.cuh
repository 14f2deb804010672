// quant_tma.cuh -- quantize-mode encode/decode with TMA row staging.
//
// Same per-row arithmetic as quant_kernels.cuh (identical device helpers,
// so the results are bit-identical), different memory pipeline:
//  * warp 0 (one lane) is a producer: for each row this CTA owns it issues
//    1-D bulk copies (cp.async.bulk global -> shared, no multicast) of the
//    row's x and recon (encode) or codes and recon (decode) into a ring of
//    `stages` shared-memory slots, completing on the slot's mbarrier;
//  * the remaining warps are consumers: they wait for the slot, read the
//    row from shared memory, reduce the scale over a named barrier that only
//    the consumers join, quantise, and write err, recon and codes straight
//    to global memory; then they release the slot.
// A consumer thread owns UPT units of K consecutive channels (K = 4 or 8),
// unit u of the row going to consumer thread u % (consumer threads).  With
// K = 4 one warp-wide 16-byte store of err or recon covers 512 contiguous
// bytes and the 16-byte shared-memory reads of a recon row are free of bank
// conflicts; with K = 8 a lane stores two 16-byte halves of a 32-byte
// sector and reads shared memory at a 32-byte stride, but packs twice the
// code bits per lane.  Which is faster depends on the shape and the bit
// width (the launch code picks it from measurements).
// Many rows are in flight per SM regardless of the register budget, which
// is what the register-resident kernel is short of.
// Every wait is bounded; on expiry CF_ERR_TIMEOUT goes to the status word
// (when given) and the CTA stops.
//
// Publishing encode / waiting decode (the exchange with the payload transfer
// fused in): with a publishing source the encode's warps gather their code
// words with shuffles and store them, 16 bytes per lane where the row
// allows, into every destination payload slot (which may be another GPU's
// memory), write the scale there too, and after its last row add
// the rows it walked to each destination's ready counter with a
// system-scope release.  With a waiting source the decode's producer reads
// a buffer's rows only after that buffer's ready counter has reached the
// target (a bounded acquire poll); every load of a TMA copy here reads this
// GPU's own memory.
#pragma once

#include "bounds.cuh"
#include "cf.h"
#include "cf_common.cuh"
#include "mbar.cuh"
#include "quant_kernels.cuh"

namespace cf {
namespace tma {

__device__ __forceinline__ uint32_t saddr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void bar_init(uint32_t b, uint32_t n) { mbar_init(b, n); }
__device__ __forceinline__ void bar_expect(uint32_t b, uint32_t bytes) { mbar_expect_tx(b, bytes); }
__device__ __forceinline__ void bar_arrive(uint32_t b) { mbar_arrive(b); }
__device__ __forceinline__ bool bar_wait(uint32_t b, uint32_t parity) { return mbar_wait(b, parity); }
// 1-D bulk copy global -> shared; both addresses 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
// 1-D bulk copy shared -> global (the copy engine writes the row), in the
// executing thread's bulk group; both addresses 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void bulk_s2g(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// this thread's bulk stores have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// this thread's bulk stores have completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void consumer_sync(int nthreads) {
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Residual of unit u of a staged row: x (bf16) at sx, x_prev (delta-state
// sender) at sp, recon or the old err (fp32) at sr.
template <int K, bool DELTA>
__device__ __forceinline__ void load_unit(const uint8_t *sx, const uint8_t *sp, const float *sr, int u,
                                          float *r, float *v) {
    if constexpr (K == 8) {
        const uint4 xw = *reinterpret_cast<const uint4 *>(sx + 16 * u);
        const uint4 pw = DELTA ? *reinterpret_cast<const uint4 *>(sp + 16 * u) : make_uint4(0, 0, 0, 0);
        const float4 a = *reinterpret_cast<const float4 *>(sr + 8 * u);
        const float4 c = *reinterpret_cast<const float4 *>(sr + 8 * u + 4);
        r[0] = a.x; r[1] = a.y; r[2] = a.z; r[3] = a.w;
        r[4] = c.x; r[5] = c.y; r[6] = c.z; r[7] = c.w;
        residual8<DELTA>(xw, pw, r, v);
    } else {
        const uint2 xw = *reinterpret_cast<const uint2 *>(sx + 8 * u);
        const uint2 pw = DELTA ? *reinterpret_cast<const uint2 *>(sp + 8 * u) : make_uint2(0, 0);
        const float4 a = *reinterpret_cast<const float4 *>(sr + 4 * u);
        r[0] = a.x; r[1] = a.y; r[2] = a.z; r[3] = a.w;
        residual4<DELTA>(xw, pw, r, v);
    }
}

// K fp32 values of unit u to a row in shared memory (an output row of the
// bulk-store path): one or two 16-byte stores.
template <int K>
__device__ __forceinline__ void store_unit_shared(float *row, int u, const float *o) {
    *reinterpret_cast<float4 *>(row + K * u) = make_float4(o[0], o[1], o[2], o[3]);
    if constexpr (K == 8) *reinterpret_cast<float4 *>(row + K * u + 4) = make_float4(o[4], o[5], o[6], o[7]);
}

// K fp32 values of unit u to a row: one or two 16-byte stores.
template <int K, bool STREAM>
__device__ __forceinline__ void store_unit(float *row, int u, const float *o) {
    if constexpr (STREAM) {
        st_stream_v4(row + K * u, make_float4(o[0], o[1], o[2], o[3]));
        if constexpr (K == 8) st_stream_v4(row + K * u + 4, make_float4(o[4], o[5], o[6], o[7]));
    } else {
        st_state_v4(row + K * u, make_float4(o[0], o[1], o[2], o[3]));
        if constexpr (K == 8) st_state_v4(row + K * u + 4, make_float4(o[4], o[5], o[6], o[7]));
    }
}

// Shared layout: [stages][slot bytes] then full[stages], empty[stages].
// Encode slot: x row (2C bytes) then recon row (4C bytes); delta-state
// encode: x row (2C), x_prev row (2C), err row (4C).
// Decode slot: codes row (4W bytes, padded to 16) then recon row (4C bytes).

// The two kernels below are the TMA pipeline with units of 8 channels and
// plain pointer sources, as the default launches use them: the same
// arithmetic, pipeline and results as the general kernels further down
// (encode_tma_unit_kernel, decode_tma_unit_kernel), written without their
// unit-width and exchange options.  Measured on B200 in the encode ->
// decode sequence, this form runs 3 % (2-bit decode at C = 1920) to 6 %
// (1-bit encode at C = 3072) faster than the general kernel instantiated
// for the same shape: same instruction count, but the general form's
// schedule stalls more and, for the 1-bit encode, spills a register.

// BULK (the standard sender): the consumers write each row's err and recon
// into one of two shared-memory output rows, and one thread has the copy
// engine store them (cp.async.bulk shared -> global) once every consumer has
// passed the next row's scale barrier, or the final barrier after the last
// row.  Before that barrier the same thread waits until the store issued
// at the previous barrier has read its output row, so the row written after
// the barrier is free.  Measured on B200, bulk stores move the encode's
// write-heavy byte mix (6 B read, 8 B written per element) near the copy
// rate, where per-thread 16-byte stores stay at ~0.87 of it.
template <int BITS, int GPT, class Src, bool BULK = false>
__global__ void __launch_bounds__(512)
encode_tma_kernel(Src src, int64_t T, int64_t C, int64_t rows, int32_t *status, int stages) {
    constexpr int GPW = 4 / BITS;
    static_assert(!(BULK && Src::kDelta), "bulk stores serve the standard sender");
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ double sh_sum[2][32];
    __shared__ float sh_max[2][32];
    __shared__ int abort_row[2];  // set before the row's barrier, read after it
    const int64_t G = C >> 3;  // C % 8 == 0 on this path
    const int64_t W = (C * BITS + 31) >> 5;
    const uint32_t slot = (uint32_t)((Src::kDelta ? 8 : 6) * C);
    const uint32_t base = saddr(smem);
    // BULK: two output rows of err (4C bytes) then recon (4C) after the ring
    const uint32_t obytes = BULK ? (uint32_t)(8 * C) : 0u;
    const uint32_t bars = base + (uint32_t)stages * slot + 2u * obytes;
    const int tid = threadIdx.x;
    const int nc = blockDim.x - 32;  // consumer threads
    if (tid == 0) {
        abort_row[0] = abort_row[1] = 0;
        for (int s = 0; s < stages; ++s) {
            bar_init(bars + 8u * s, 1);                    // full: producer arrival + tx
            bar_init(bars + 8u * (stages + s), (uint32_t)(nc / 32));  // empty: one per consumer warp
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (tid < 32) {
        if (tid != 0) return;
        int i = 0;
        for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
            const int64_t b = row / T, t = row - b * T;
            const EncPtrs p = src.get(b);
            if (Src::kChecked && enc_ptr_status<Src::kDelta>(p) != CF_OK) continue;
            const int s = i % stages;
            const uint32_t ph = (uint32_t)(i / stages) & 1u;
            if (!bar_wait(bars + 8u * (stages + s), ph ^ 1u)) {
                // consumers stopped releasing slots; they time out on their
                // own waits and leave together
                if (status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
                return;
            }
            const uint32_t dst = base + (uint32_t)s * slot;
            if (!CF_IN(t < T && b * T + t == row && s < stages)) continue;
            bar_expect(bars + 8u * s, slot);
            bulk_g2s(dst, p.x + t * C, (uint32_t)(2 * C), bars + 8u * s);
            if (Src::kDelta) {
                bulk_g2s(dst + (uint32_t)(2 * C), p.xprev + t * C, (uint32_t)(2 * C), bars + 8u * s);
                bulk_g2s(dst + (uint32_t)(4 * C), p.err + t * C, (uint32_t)(4 * C), bars + 8u * s);
            } else {
                bulk_g2s(dst + (uint32_t)(2 * C), p.recon + t * C, (uint32_t)(4 * C), bars + 8u * s);
            }
            ++i;
        }
        return;
    }

    const int ct = tid - 32;  // consumer thread index
    const int lane = ct & 31, warp = ct >> 5, nw = nc >> 5;
    int i = 0, par = 0;
    // BULK, thread ct 0: the row whose outputs wait in output row (pend_i & 1)
    float *pend_err = nullptr, *pend_rec = nullptr;
    int pend_i = 0, orow = 0;   // orow: rows whose outputs this CTA has written
    const uint32_t obase = base + (uint32_t)stages * slot;
    // issue the pending row's bulk stores (after a barrier that every
    // consumer passed once it had written its part of that row)
    auto flush_pending = [&]() {
        if (BULK && ct == 0 && pend_err) {
            const uint32_t ob = obase + (uint32_t)(pend_i & 1) * obytes;
            bulk_s2g(pend_err, ob, (uint32_t)(4 * C));
            bulk_s2g(pend_rec, ob + (uint32_t)(4 * C), (uint32_t)(4 * C));
            bulk_commit();
            pend_err = pend_rec = nullptr;
        }
    };
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        const int64_t b = row / T, t = row - b * T;
        const EncPtrs p = src.get(b);
        if (Src::kChecked) {
            const int st = enc_ptr_status<Src::kDelta>(p);
            if (st != CF_OK) {
                if (ct == 0) report(status, st);
                continue;
            }
        }
        const int s = i % stages;
        const uint32_t ph = (uint32_t)(i / stages) & 1u;
        bool ok = true;
        if (lane == 0) ok = bar_wait(bars + 8u * s, ph);
        ok = __shfl_sync(kFullMask, ok ? 1 : 0, 0) != 0;
        if (!ok && lane == 0) abort_row[par] = 1;  // acted on after the barrier
        const uint8_t *sx = smem + (size_t)s * slot;
        const uint8_t *sp = sx + 2 * C;   // x_prev row (delta-state sender)
        // recon (standard) or the old err (delta-state)
        const float *sr = reinterpret_cast<const float *>(sx + (Src::kDelta ? 4 : 2) * C);
        float *rr = Src::kDelta ? nullptr : p.recon + t * C;
        float *er = p.err + t * C;
        uint32_t *cw = p.codes + t * W;

        float r[GPT][8], v[GPT][8];
#pragma unroll
        for (int j = 0; j < GPT; ++j) {
            const int64_t g = (int64_t)j * nc + ct;
            if (ok && g < G && CF_IN(8 * g + 8 <= C)) {
                const uint4 xw = *reinterpret_cast<const uint4 *>(sx + 16 * g);
                const uint4 pw = Src::kDelta ? *reinterpret_cast<const uint4 *>(sp + 16 * g)
                                             : make_uint4(0, 0, 0, 0);
                const float4 a = *reinterpret_cast<const float4 *>(sr + 8 * g);
                const float4 c = *reinterpret_cast<const float4 *>(sr + 8 * g + 4);
                r[j][0] = a.x; r[j][1] = a.y; r[j][2] = a.z; r[j][3] = a.w;
                r[j][4] = c.x; r[j][5] = c.y; r[j][6] = c.z; r[j][7] = c.w;
                residual8<Src::kDelta>(xw, pw, r[j], v[j]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) r[j][e] = v[j][e] = 0.0f;
            }
        }
        // the slot is no longer read: release it to the producer.  The reads
        // above are generic-proxy accesses and the producer's next bulk copy
        // into this slot is an async-proxy write: the proxy fence orders them
        // (without it a late read can see the next row's bytes).
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) bar_arrive(bars + 8u * (stages + s));
        ++i;

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
            if (BULK && ct == 0) bulk_wait_read();   // output row i % 2 is free after the barrier
            consumer_sync(nc);
            if (*(volatile int *)&abort_row[par]) {
                if (ct == 0 && status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
                if (BULK && ct == 0) bulk_wait_all();
                return;  // every consumer warp sees the same flag here
            }
            flush_pending();
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
            if (BULK && ct == 0) bulk_wait_read();   // output row i % 2 is free after the barrier
            consumer_sync(nc);
            if (*(volatile int *)&abort_row[par]) {
                if (ct == 0 && status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
                if (BULK && ct == 0) bulk_wait_all();
                return;
            }
            flush_pending();
            float tot = 0.0f;
            for (int w = 0; w < nw; ++w) tot = fmaxf(tot, sh_max[par][w]);
            scale = tot;
        }
        par ^= 1;
        const float half = __fmul_rn(0.5f, scale);
#pragma unroll
        for (int j = 0; j < GPT; ++j) {
            const int64_t g = (int64_t)j * nc + ct;
            uint32_t field = 0;
            float eo[8], ro[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                uint32_t code = quantize<BITS>(v[j][e], half);
                code = (g < G) ? code : 0u;
                field |= code << (e * BITS);
                const float d = dequantize<BITS>(code, scale);
                eo[e] = __fsub_rn(v[j][e], d);
                ro[e] = __fadd_rn(r[j][e], d);
            }
            uint32_t word = field << ((lane % GPW) * 8 * BITS);
#pragma unroll
            for (int o = 1; o < GPW; o <<= 1) word |= __shfl_xor_sync(kFullMask, word, o);
            if (g < G && CF_IN(8 * g + 8 <= C && t < T && g / GPW < W)) {
                if constexpr (BULK) {
                    float *oe = reinterpret_cast<float *>(smem + (size_t)stages * slot + (size_t)(orow & 1) * obytes);
                    float *orr = oe + C;
                    *reinterpret_cast<float4 *>(oe + 8 * g) = make_float4(eo[0], eo[1], eo[2], eo[3]);
                    *reinterpret_cast<float4 *>(oe + 8 * g + 4) = make_float4(eo[4], eo[5], eo[6], eo[7]);
                    *reinterpret_cast<float4 *>(orr + 8 * g) = make_float4(ro[0], ro[1], ro[2], ro[3]);
                    *reinterpret_cast<float4 *>(orr + 8 * g + 4) = make_float4(ro[4], ro[5], ro[6], ro[7]);
                } else {
                    st_stream_v4(er + 8 * g, make_float4(eo[0], eo[1], eo[2], eo[3]));
                    st_stream_v4(er + 8 * g + 4, make_float4(eo[4], eo[5], eo[6], eo[7]));
                    if (!Src::kDelta) {
                        // streaming (evict-first) like err: measured 0.3-1.3 % faster
                        // than a plain store for the reconstruction too
                        st_stream_v4(rr + 8 * g, make_float4(ro[0], ro[1], ro[2], ro[3]));
                        st_stream_v4(rr + 8 * g + 4, make_float4(ro[4], ro[5], ro[6], ro[7]));
                    }
                }
                if ((lane % GPW) == 0) cw[g / GPW] = word;
            }
        }
        if (ct == 0 && CF_IN(t < T)) p.scales[t] = scale;
        if constexpr (BULK) {
            // this thread's output-row writes, visible to the copy engine
            // once every consumer has passed the next barrier
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            if (ct == 0) {
                pend_err = er;
                pend_rec = rr;
                pend_i = orow;
            }
            ++orow;
        }
    }
    if constexpr (BULK) {
        // the last row's outputs: every consumer has written its part
        consumer_sync(nc);
        flush_pending();
        if (ct == 0) bulk_wait_all();
    }
}

template <int BITS, int GPT, class Src>
__global__ void __launch_bounds__(512)
decode_tma_kernel(Src src, int64_t T, int64_t C, int64_t rows, int32_t *status, int stages) {
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    extern __shared__ __align__(16) uint8_t smem[];
    const int64_t G = C >> 3;
    const int64_t W = (C * BITS + 31) >> 5;
    const uint32_t cbytes = (uint32_t)(W * 4);
    const uint32_t slot = cbytes + (uint32_t)(4 * C);
    const uint32_t base = saddr(smem);
    const uint32_t bars = base + (uint32_t)stages * slot;
    const int tid = threadIdx.x;
    const int nc = blockDim.x - 32;
    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            bar_init(bars + 8u * s, 1);
            bar_init(bars + 8u * (stages + s), (uint32_t)(nc / 32));
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (tid < 32) {
        if (tid != 0) return;
        int i = 0;
        for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
            const int64_t b = row / T, t = row - b * T;
            const DecPtrs p = src.get(b);
            if (Src::kChecked && dec_ptr_status<Src::kEmit>(p) != CF_OK) continue;
            const int s = i % stages;
            const uint32_t ph = (uint32_t)(i / stages) & 1u;
            if (!bar_wait(bars + 8u * (stages + s), ph ^ 1u)) {
                if (status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
                return;
            }
            const uint32_t dst = base + (uint32_t)s * slot;
            if (!CF_IN(t < T && b * T + t == row && s < stages && (W & 3) == 0)) continue;
            // W % 4 == 0 on this path (host check): codes rows are 16-byte
            // aligned multiples of 16 bytes
            bar_expect(bars + 8u * s, cbytes + (uint32_t)(4 * C));
            bulk_g2s(dst, p.codes + t * W, cbytes, bars + 8u * s);
            bulk_g2s(dst + cbytes, p.recon + t * C, (uint32_t)(4 * C), bars + 8u * s);
            ++i;
        }
        return;
    }

    const int ct = tid - 32;
    const int lane = ct & 31;
    int i = 0;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        const int64_t b = row / T, t = row - b * T;
        const DecPtrs p = src.get(b);
        if (Src::kChecked) {
            const int st = dec_ptr_status<Src::kEmit>(p);
            if (st != CF_OK) {
                if (ct == 0) report(status, st);
                continue;
            }
        }
        const int s = i % stages;
        const uint32_t ph = (uint32_t)(i / stages) & 1u;
        bool ok = true;
        if (lane == 0) ok = bar_wait(bars + 8u * s, ph);
        ok = __shfl_sync(kFullMask, ok ? 1 : 0, 0) != 0;
        if (!ok) {  // decode warps are independent: each leaves on its own
            if (lane == 0 && status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
            return;
        }
        const uint8_t *sc = smem + (size_t)s * slot;
        const float *sr = reinterpret_cast<const float *>(sc + cbytes);
        const float scale = __ldg(p.scales + t);
        float *rr = p.recon + t * C;
        uint32_t field[GPT];
        float r[GPT][8];
#pragma unroll
        for (int j = 0; j < GPT; ++j) {
            const int64_t g = (int64_t)j * nc + ct;
            if (g < G && CF_IN(8 * g + 8 <= C && (g + 1) * BITS <= (int64_t)cbytes)) {
                const uint32_t off = (uint32_t)(g * BITS);  // byte offset of the group's field
                field[j] = BITS == 1 ? (uint32_t)sc[off]
                                     : (uint32_t)*reinterpret_cast<const uint16_t *>(sc + off);
                const float4 a = *reinterpret_cast<const float4 *>(sr + 8 * g);
                const float4 c = *reinterpret_cast<const float4 *>(sr + 8 * g + 4);
                r[j][0] = a.x; r[j][1] = a.y; r[j][2] = a.z; r[j][3] = a.w;
                r[j][4] = c.x; r[j][5] = c.y; r[j][6] = c.z; r[j][7] = c.w;
            } else {
                field[j] = 0u;
#pragma unroll
                for (int e = 0; e < 8; ++e) r[j][e] = 0.0f;
            }
        }
        // release the slot; proxy fence as in the encode kernel
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) bar_arrive(bars + 8u * (stages + s));
        ++i;
#pragma unroll
        for (int j = 0; j < GPT; ++j) {
            const int64_t g = (int64_t)j * nc + ct;
            if (g >= G || !CF_IN(8 * g + 8 <= C && t < T)) continue;
            float ro[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t code = (field[j] >> (e * BITS)) & MASK;
                ro[e] = __fadd_rn(r[j][e], dequantize<BITS>(code, scale));
            }
            st_state_v4(rr + 8 * g, make_float4(ro[0], ro[1], ro[2], ro[3]));
            st_state_v4(rr + 8 * g + 4, make_float4(ro[4], ro[5], ro[6], ro[7]));
            if (Src::kEmit) *reinterpret_cast<uint4 *>(p.out + t * C + 8 * g) = pack_bf16x8(ro);
        }
    }
}

// BULK: the standard encode's bulk-store path (two shared-memory output
// rows, stores issued after the next row's scale barrier), as in
// encode_tma_kernel.
template <int BITS, int K, int UPT, class Src, bool BULK = false>
__device__ __forceinline__ void encode_unit_body(const Src &src, int64_t T, int64_t C, int64_t rows,
                                                 int32_t *status, int stages) {
    static_assert(K == 4 || K == 8, "units of 4 or 8 channels");
    static_assert(!(BULK && Src::kDelta), "bulk stores serve the standard sender");
    constexpr int UPW = 32 / (K * BITS);  // units per 32-bit code word
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ double sh_sum[2][32];
    __shared__ float sh_max[2][32];
    __shared__ int abort_row[2];  // set before the row's barrier, read after it
    __shared__ int cta_abort;     // publishing: a destination check or an ack wait failed
    const int NU = (int)(C / K);  // units per row (C % 8 == 0 and C <= 16384 on this path)
    const int64_t W = (C * BITS + 31) >> 5;
    const uint32_t slot = (uint32_t)((Src::kDelta ? 8 : 6) * C);
    const uint32_t base = saddr(smem);
    const uint32_t obytes = BULK ? (uint32_t)(8 * C) : 0u;   // BULK output row: err, then recon
    const uint32_t obase = base + (uint32_t)stages * slot;
    const uint32_t bars = obase + 2u * obytes;
    const int tid = threadIdx.x;
    const int nc = blockDim.x - 32;  // consumer threads
    if (tid == 0) {
        abort_row[0] = abort_row[1] = 0;
        for (int s = 0; s < stages; ++s) {
            bar_init(bars + 8u * s, 1);                    // full: producer arrival + tx
            bar_init(bars + 8u * (stages + s), (uint32_t)(nc / 32));  // empty: one per consumer warp
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        cta_abort = 0;
        if constexpr (Src::kPublish) cta_abort = src.check_and_wait(status) ? 0 : 1;
    }
    __syncthreads();
    if constexpr (Src::kPublish) {
        if (cta_abort) return;  // uniform: nothing was issued yet
    }

    if (tid < 32) {
        if (tid != 0) return;
        int i = 0;
        for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
            const int64_t b = row / T, t = row - b * T;
            const EncPtrs p = src.get(b);
            if (Src::kChecked && enc_ptr_status<Src::kDelta, Src::kPublish>(p) != CF_OK) continue;
            const int s = i % stages;
            const uint32_t ph = (uint32_t)(i / stages) & 1u;
            if (!bar_wait(bars + 8u * (stages + s), ph ^ 1u)) {
                // consumers stopped releasing slots; they time out on their
                // own waits and leave together
                if (status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
                return;
            }
            const uint32_t dst = base + (uint32_t)s * slot;
            if (!CF_IN(t < T && b * T + t == row && s < stages)) continue;
            bar_expect(bars + 8u * s, slot);
            bulk_g2s(dst, p.x + t * C, (uint32_t)(2 * C), bars + 8u * s);
            if (Src::kDelta) {
                bulk_g2s(dst + (uint32_t)(2 * C), p.xprev + t * C, (uint32_t)(2 * C), bars + 8u * s);
                bulk_g2s(dst + (uint32_t)(4 * C), p.err + t * C, (uint32_t)(4 * C), bars + 8u * s);
            } else {
                bulk_g2s(dst + (uint32_t)(2 * C), p.recon + t * C, (uint32_t)(4 * C), bars + 8u * s);
            }
            ++i;
        }
        return;
    }

    const int ct = tid - 32;  // consumer thread index
    const int lane = ct & 31, warp = ct >> 5, nw = nc >> 5;
    int i = 0, par = 0;
    uint64_t walked = 0;  // rows this CTA walked, skipped ones included (publishing)
    float *pend_err = nullptr, *pend_rec = nullptr;   // BULK, thread ct 0: the row in output row pend_o
    int pend_o = 0, orow = 0;
    auto flush_pending = [&]() {
        if (BULK && ct == 0 && pend_err) {
            const uint32_t ob = obase + (uint32_t)(pend_o & 1) * obytes;
            bulk_s2g(pend_err, ob, (uint32_t)(4 * C));
            bulk_s2g(pend_rec, ob + (uint32_t)(4 * C), (uint32_t)(4 * C));
            bulk_commit();
            pend_err = pend_rec = nullptr;
        }
    };
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        const int64_t b = row / T, t = row - b * T;
        const EncPtrs p = src.get(b);
        ++walked;
        if (Src::kChecked) {
            const int st = enc_ptr_status<Src::kDelta, Src::kPublish>(p);
            if (st != CF_OK) {
                if (ct == 0) report(status, st);
                continue;
            }
        }
        const int s = i % stages;
        const uint32_t ph = (uint32_t)(i / stages) & 1u;
        bool ok = true;
        if (lane == 0) ok = bar_wait(bars + 8u * s, ph);
        ok = __shfl_sync(kFullMask, ok ? 1 : 0, 0) != 0;
        if (!ok && lane == 0) abort_row[par] = 1;  // acted on after the barrier
        const uint8_t *sx = smem + (size_t)s * slot;
        const uint8_t *sp = sx + 2 * C;   // x_prev row (delta-state sender)
        // recon (standard) or the old err (delta-state)
        const float *sr = reinterpret_cast<const float *>(sx + (Src::kDelta ? 4 : 2) * C);
        float *rr = Src::kDelta ? nullptr : p.recon + t * C;
        float *er = p.err + t * C;

        float r[UPT][K], v[UPT][K];
#pragma unroll
        for (int j = 0; j < UPT; ++j) {
            const int u = j * nc + ct;
            if (ok && u < NU && CF_IN(K * u + K <= C)) {
                load_unit<K, Src::kDelta>(sx, sp, sr, u, r[j], v[j]);
            } else {
#pragma unroll
                for (int e = 0; e < K; ++e) r[j][e] = v[j][e] = 0.0f;
            }
        }
        // the slot is no longer read: release it to the producer.  The reads
        // above are generic-proxy accesses and the producer's next bulk copy
        // into this slot is an async-proxy write: the proxy fence orders them
        // (without it a late read can see the next row's bytes).
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) bar_arrive(bars + 8u * (stages + s));
        ++i;

        float scale;
        if (BITS == 1) {
            double acc = 0.0;
#pragma unroll
            for (int j = 0; j < UPT; ++j)
#pragma unroll
                for (int e = 0; e < K; ++e) acc += (double)fabsf(v[j][e]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFullMask, acc, o);
            if (lane == 0) sh_sum[par][warp] = acc;
            if (BULK && ct == 0) bulk_wait_read();   // output row orow % 2 is free after the barrier
            consumer_sync(nc);
            if (*(volatile int *)&abort_row[par]) {
                if (ct == 0 && status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
                if (BULK && ct == 0) bulk_wait_all();
                return;  // every consumer warp sees the same flag here
            }
            flush_pending();
            double tot = 0.0;
            for (int w = 0; w < nw; ++w) tot += sh_sum[par][w];
            scale = __fdiv_rn(__double2float_rn(tot), (float)C);
        } else {
            float m = 0.0f;
#pragma unroll
            for (int j = 0; j < UPT; ++j)
#pragma unroll
                for (int e = 0; e < K; ++e) m = fmaxf(m, fabsf(v[j][e]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
            if (lane == 0) sh_max[par][warp] = m;
            if (BULK && ct == 0) bulk_wait_read();   // output row orow % 2 is free after the barrier
            consumer_sync(nc);
            if (*(volatile int *)&abort_row[par]) {
                if (ct == 0 && status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
                if (BULK && ct == 0) bulk_wait_all();
                return;
            }
            flush_pending();
            float tot = 0.0f;
            for (int w = 0; w < nw; ++w) tot = fmaxf(tot, sh_max[par][w]);
            scale = tot;
        }
        par ^= 1;
        const float half = __fmul_rn(0.5f, scale);
        uint32_t *cw = Src::kPublish ? nullptr : p.codes + t * W;
#pragma unroll
        for (int j = 0; j < UPT; ++j) {
            const int u = j * nc + ct;
            uint32_t field = 0;
            float eo[K], ro[K];
#pragma unroll
            for (int e = 0; e < K; ++e) {
                uint32_t code = quantize<BITS>(v[j][e], half);
                code = (u < NU) ? code : 0u;
                field |= code << (e * BITS);
                const float d = dequantize<BITS>(code, scale);
                eo[e] = __fsub_rn(v[j][e], d);
                ro[e] = __fadd_rn(r[j][e], d);
            }
            if (u < NU && CF_IN(K * u + K <= C && t < T)) {
                if constexpr (BULK) {
                    float *oe = reinterpret_cast<float *>(smem + (size_t)stages * slot + (size_t)(orow & 1) * obytes);
                    store_unit_shared<K>(oe, u, eo);
                    store_unit_shared<K>(oe + C, u, ro);
                } else {
                    store_unit<K, true>(er, u, eo);
                    if (!Src::kDelta) store_unit<K, false>(rr, u, ro);
                }
            }
            // nc is a multiple of 32, so u % UPW == lane % UPW: the UPW
            // lanes of one code word are adjacent and aligned
            uint32_t word = field << ((lane % UPW) * K * BITS);
#pragma unroll
            for (int o = 1; o < UPW; o <<= 1) word |= __shfl_xor_sync(kFullMask, word, o);
            if constexpr (Src::kPublish) {
                // This warp's code words of unit block j are contiguous: 32 / UPW
                // words from w0, the word of lane group g (every lane of which
                // holds it after the butterfly above) at w0 + g.  w0 is a
                // multiple of 4 (nc is a multiple of 32), so lanes
                // 0 .. 8 / UPW - 1 each gather four words and store them as one
                // 16-byte vector to every destination.
                const int64_t w0 = (int64_t)(j * nc + 32 * warp) / UPW;
                uint32_t q[4];
#pragma unroll
                for (int m = 0; m < 4; ++m) q[m] = __shfl_sync(kFullMask, word, ((4 * lane + m) * UPW) & 31);
                src.store_words(p, t, W, w0, lane, 8 / UPW, q, word, u < NU && (lane % UPW) == 0, u / UPW);
            } else if (u < NU && (lane % UPW) == 0 && CF_IN(u / UPW < W)) {
                cw[u / UPW] = word;
            }
        }
        if constexpr (Src::kPublish) {
            if (ct == 0 && CF_IN(t < T)) src.store_scale(p, t, scale);
        } else {
            if (ct == 0 && CF_IN(t < T)) p.scales[t] = scale;
        }
        if constexpr (BULK) {
            // this thread's output-row writes, visible to the copy engine
            // once every consumer has passed the next barrier
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            if (ct == 0) {
                pend_err = er;
                pend_rec = rr;
                pend_o = orow;
            }
            ++orow;
        }
    }
    if constexpr (Src::kPublish || BULK) {
        // every consumer's stores of this CTA precede the barrier; the
        // system-scope fence of the publishing thread is cumulative over
        // them; BULK: the last row's outputs are in shared memory
        consumer_sync(nc);
        flush_pending();
        if constexpr (Src::kPublish) {
            if (ct == 0) src.publish(walked);
        }
        if (BULK && ct == 0) bulk_wait_all();
    }
}

template <int BITS, int K, int UPT, class Src>
__global__ void __launch_bounds__(512)
encode_tma_unit_kernel(Src src, int64_t T, int64_t C, int64_t rows, int32_t *status, int stages) {
    encode_unit_body<BITS, K, UPT, Src>(src, T, C, rows, status, stages);
}

// The publishing form: at most 80 registers a thread, so that three CTAs of
// a C = 3072 launch (7 warps each) still fit on an SM as they do for the
// plain encode: the warps of an SM's CTAs spread over its four 16K-register
// sub-partitions, and the sub-partition that holds 6 of the 21 warps needs
// 6 x 32 x R <= 16384.  Without the cap the destination stores raise R past
// 110, and at 96 only two CTAs fit (measured: 296-CTA grid, 40 % slower).
template <int BITS, int K, int UPT, class Src, bool BULK = false>
__global__ void __maxnreg__(80)
encode_tma_publish_kernel(Src src, int64_t T, int64_t C, int64_t rows, int32_t *status, int stages) {
    encode_unit_body<BITS, K, UPT, Src, BULK>(src, T, C, rows, status, stages);
}

template <int BITS, int K, int UPT, class Src>
__global__ void __launch_bounds__(512)
decode_tma_unit_kernel(Src src, int64_t T, int64_t C, int64_t rows, int32_t *status, int stages) {
    static_assert(K == 4 || K == 8, "units of 4 or 8 channels");
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int dec_abort;  // waiting decode: the producer gave up on a ready counter
    const int NU = (int)(C / K);  // C <= 16384
    const int64_t W = (C * BITS + 31) >> 5;
    const uint32_t cbytes = (uint32_t)(W * 4);
    const uint32_t slot = cbytes + (uint32_t)(4 * C);
    const uint32_t base = saddr(smem);
    const uint32_t bars = base + (uint32_t)stages * slot;
    const int tid = threadIdx.x;
    const int nc = blockDim.x - 32;
    if (tid == 0) {
        dec_abort = 0;
        for (int s = 0; s < stages; ++s) {
            bar_init(bars + 8u * s, 1);
            bar_init(bars + 8u * (stages + s), (uint32_t)(nc / 32));
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (tid < 32) {
        if (tid != 0) return;
        int i = 0;
        int64_t ready_b = -1;  // waiting decode: the last buffer whose counter was seen ready
        for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
            const int64_t b = row / T, t = row - b * T;
            const DecPtrs p = src.get(b);
            if (Src::kChecked && dec_ptr_status<Src::kEmit, Src::kWait>(p) != CF_OK) continue;
            const int s = i % stages;
            const uint32_t ph = (uint32_t)(i / stages) & 1u;
            if (!bar_wait(bars + 8u * (stages + s), ph ^ 1u)) {
                if (status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
                return;
            }
            if constexpr (Src::kWait) {
                if (b != ready_b) {  // rows walk buffers in increasing order
                    if (!src.wait_ready(b)) {
                        // Give up: flag it and complete this slot's phase
                        // without data, so every consumer waiting on it wakes,
                        // sees the flag and stops.
                        report(status, CF_ERR_TIMEOUT);
                        *(volatile int *)&dec_abort = 1;
                        bar_arrive(bars + 8u * s);
                        return;
                    }
                    ready_b = b;
                    // the bulk copies below (async proxy) read what the
                    // acquire above made visible (generic proxy)
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                }
            }
            const uint32_t dst = base + (uint32_t)s * slot;
            if (!CF_IN(t < T && b * T + t == row && s < stages && (W & 3) == 0)) continue;
            // W % 4 == 0 on this path (host check): codes rows are 16-byte
            // aligned multiples of 16 bytes
            bar_expect(bars + 8u * s, cbytes + (uint32_t)(4 * C));
            bulk_g2s(dst, p.codes + t * W, cbytes, bars + 8u * s);
            bulk_g2s(dst + cbytes, p.recon + t * C, (uint32_t)(4 * C), bars + 8u * s);
            ++i;
        }
        return;
    }

    const int ct = tid - 32;
    const int lane = ct & 31;
    int i = 0;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        const int64_t b = row / T, t = row - b * T;
        const DecPtrs p = src.get(b);
        if (Src::kChecked) {
            const int st = dec_ptr_status<Src::kEmit, Src::kWait>(p);
            if (st != CF_OK) {
                if (ct == 0) report(status, st);
                continue;
            }
        }
        const int s = i % stages;
        const uint32_t ph = (uint32_t)(i / stages) & 1u;
        bool ok = true;
        if (lane == 0) ok = bar_wait(bars + 8u * s, ph);
        ok = __shfl_sync(kFullMask, ok ? 1 : 0, 0) != 0;
        if (!ok) {  // decode warps are independent: each leaves on its own
            if (lane == 0 && status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
            return;
        }
        if constexpr (Src::kWait) {
            if (*(volatile int *)&dec_abort) return;  // status already recorded
        }
        const uint8_t *sc = smem + (size_t)s * slot;
        const float *sr = reinterpret_cast<const float *>(sc + cbytes);
        // a waiting decode reads a scale another GPU may have just written:
        // through L2 (the coherence point), not the non-coherent path
        const float scale = Src::kWait ? __ldcg(p.scales + t) : __ldg(p.scales + t);
        float *rr = p.recon + t * C;
        uint32_t field[UPT];
        float r[UPT][K];
#pragma unroll
        for (int j = 0; j < UPT; ++j) {
            const int u = j * nc + ct;
            if (u < NU && CF_IN(K * u + K <= C && (K * BITS * (u + 1) + 7) / 8 <= (int)cbytes)) {
                // unit u's K*BITS code bits
                if constexpr (K * BITS == 4)
                    field[j] = (uint32_t)sc[u >> 1] >> ((u & 1) * 4);
                else if constexpr (K * BITS == 8)
                    field[j] = (uint32_t)sc[u];
                else
                    field[j] = (uint32_t)reinterpret_cast<const uint16_t *>(sc)[u];
                const float4 a = *reinterpret_cast<const float4 *>(sr + K * u);
                r[j][0] = a.x; r[j][1] = a.y; r[j][2] = a.z; r[j][3] = a.w;
                if constexpr (K == 8) {
                    const float4 c = *reinterpret_cast<const float4 *>(sr + K * u + 4);
                    r[j][4] = c.x; r[j][5] = c.y; r[j][6] = c.z; r[j][7] = c.w;
                }
            } else {
                field[j] = 0u;
#pragma unroll
                for (int e = 0; e < K; ++e) r[j][e] = 0.0f;
            }
        }
        // release the slot; proxy fence as in the encode kernel
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) bar_arrive(bars + 8u * (stages + s));
        ++i;
#pragma unroll
        for (int j = 0; j < UPT; ++j) {
            const int u = j * nc + ct;
            if (u >= NU || !CF_IN(K * u + K <= C && t < T)) continue;
            float ro[K];
#pragma unroll
            for (int e = 0; e < K; ++e) {
                const uint32_t code = (field[j] >> (e * BITS)) & MASK;
                ro[e] = __fadd_rn(r[j][e], dequantize<BITS>(code, scale));
            }
            store_unit<K, false>(rr, u, ro);
            if constexpr (Src::kEmit) {
                if constexpr (K == 8)
                    *reinterpret_cast<uint4 *>(p.out + t * C + 8 * u) = pack_bf16x8(ro);
                else
                    *reinterpret_cast<uint2 *>(p.out + t * C + 4 * u) = pack_bf16x4(ro);
            }
        }
    }
}

// After a waiting decode: one release add per sender's ack counter (stream
// order puts it after every read of the decode).
__global__ void exchange_ack_kernel(uint64_t *const *acks, int n) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= n) return;
    uint64_t *a = ldg_ptr(acks + k);
    __threadfence_system();
    atomicAdd_system(reinterpret_cast<unsigned long long *>(a), 1ull);
}

}  // namespace tma
}  // namespace cf
