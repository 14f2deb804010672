// lowrank_apply_tc.cuh -- D = (qP sP)(qQ sQ)^T on the tensor cores, fused with
// the error-feedback update (sender) or the accumulate (receiver).
//
// One CTA per tile of 128 channels x 128 tokens.  The product is formed
// transposed, D^T[c][t] = sum_k qQ[c][k] * (qP[t][k] sP[k] sQ[k]):
//   A = the INT4 codes of Q as fp32 integers (exact in tf32),   M = 128 ch
//   B = b[t][k] = qP[t][k] * (sP[k] sQ[k]) split as b = hi + lo, both
//       tf32-exact parts (hi keeps the top 10 mantissa bits), N = 128 tok
//   D^T = A hi^T + A lo^T, tcgen05.mma kind::tf32, fp32 accumulation in
//       TMEM: TMEM lane = channel, column = token.
// The split keeps ~21 significant bits of every product, so D matches the
// exact product of the payload to ~1e-6 relative.  Sender and receiver run
// this same kernel on the same payload, so their D is bit-identical.
// Epilogue: x and recon arrive in shared memory through bulk copies issued
// by a producer warp (below); warp w reads TMEM lanes 32 (w % 4) .. +31
// (channels) and, of every 16-token stage, the token columns of half w / 4;
// for each token its 32 lanes write 32 consecutive channels, one 128-byte
// transaction per warp per array.
#pragma once

#include <cuda_bf16.h>

#include "bounds.cuh"
#include "cf.h"
#include "cf_common.cuh"
#include "lowrank_kernels.cuh"
#include "lowrank_umma.cuh"

namespace cf {
namespace umma {

constexpr int kApplyTile = 128;

__device__ __forceinline__ int int4_code_at(const uint8_t *row, int k) {
    const uint32_t byte = row[k >> 1];
    const int q = (int)((byte >> ((k & 1) * 4)) & 0xFu);
    return q >= 8 ? q - 16 : q;
}

// kind::tf32 instruction descriptor: D f32, A/B tf32, both K-major, M = 128.
__host__ __device__ constexpr uint32_t idesc_tf32(int n) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(128 >> 4) << 24);
}

// Byte offset of fp32 element (row, k) in a K-major 128-byte-swizzled tile
// of 128 rows: atom blocks of 32 k (128 B per row) and 128 rows (16 KB).
__device__ __forceinline__ uint32_t sw128_f32_offset(int row, int k) {
    const int atom = k >> 5, kin = k & 31;
    const int chunk = (kin >> 2) ^ (row & 7);
    return (uint32_t)(atom * 16384 + row * 128 + chunk * 16 + (kin & 3) * 4);
}

// 32 TMEM lanes x 8 columns of fp32 into 8 registers of this thread.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float *v) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    // the wait takes the destination registers as operands, so no use of
    // them can be scheduled above it
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7])
                 :
                 : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// Staging of x and recon: a tile's 128 tokens are stages of STOK token rows;
// a stage holds the rows' recon (STOK x 128 fp32) and, for the sender, x
// (STOK x 128 bf16).  Each consumer warp takes STOK / 2 tokens of a stage.
// Ring depth per kernel, sized so that rank <= 32 keeps two CTAs per SM
// (measured on B200 with per-warp cp.async staging: 16-token stages 4 deep
// for both directions; the receiver at 32-token stages 3 deep, or 16 x 6,
// was slower).
template <bool SENDER>
__host__ __device__ constexpr int apply_stage_tok() {
    return 16;
}
constexpr int kApplyConsumers = 256;            // 8 warps: 4 channel quarters x 2 token halves
constexpr int kApplyMmaWarp = kApplyConsumers / 32;        // warps 8, 9: B operands;
constexpr int kApplyBuilders = 64;                          // warp 8 also issues the MMAs
constexpr int kApplyThreads = kApplyConsumers + kApplyBuilders;
// Token tiles per CTA at most: the receiver's tiles carry half the bytes of
// the sender's, so it takes twice as many to amortise a CTA's set-up
// (measured on B200: 16 tiles gave the receiver 0.92 of HBM against 0.89).
template <bool SENDER>
__host__ __device__ constexpr int apply_max_tiles_per_cta() {
    return SENDER ? 8 : 16;
}

template <bool SENDER>
__host__ __device__ constexpr int apply_stage_bytes() {
    return apply_stage_tok<SENDER>() * kApplyTile * (SENDER ? 6 : 4);
}
template <bool SENDER, int KP>
__host__ __device__ constexpr int apply_ring() {
    return KP <= 32 ? 4 : 8;
}
template <bool SENDER, int KP>
__host__ __device__ constexpr int apply_tc_smem() {
    return 1024 + 3 * (KP / 32) * 16384 + apply_ring<SENDER, KP>() * apply_stage_bytes<SENDER>() + 512;
}

// 16-byte asynchronous copy global -> shared (src-size 0: 16 zero bytes)
__device__ __forceinline__ void apply_cp16(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void apply_cp_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void apply_cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// consumers + the builder warps, once, after the first operands are built
__device__ __forceinline__ void operand_sync() {
    asm volatile("bar.sync 1, %0;" ::"r"(kApplyConsumers + kApplyBuilders) : "memory");
}
// the two builder warps, once per token tile
__device__ __forceinline__ void builder_sync() {
    asm volatile("bar.sync 2, %0;" ::"r"(kApplyBuilders) : "memory");
}

// B operand of one token tile: b[t][k] = qP[t][k] * s[k] (s[k] = sP[k] sQ[k],
// precomputed in shared memory) split into the tf32-exact hi part and the
// remainder; 16-byte chunks of 4 consecutive k, threads [tid0, tid0 + nthr).
template <int KP>
__device__ __forceinline__ void apply_build_b(uint8_t *gbh, uint8_t *gbl, const uint8_t *pc,
                                              const float *sk, int64_t t0, int64_t T, int r,
                                              int nb, int tid, int nthr) {
    for (int idx = tid; idx < kApplyTile * (KP / 4); idx += nthr) {
        const int row = idx / (KP / 4), k0 = (idx - row * (KP / 4)) * 4;
        const int64_t t = t0 + row;
        float h[4], l[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int k = k0 + u;
            float b = 0.0f;
            if (t < T && k < r) b = __fmul_rn((float)int4_code_at(pc + t * nb, k), sk[k]);
            h[u] = __uint_as_float(__float_as_uint(b) & 0xFFFFE000u);
            l[u] = __fsub_rn(b, h[u]);
        }
        const uint32_t off = sw128_f32_offset(row, k0);
        *reinterpret_cast<float4 *>(gbh + off) = make_float4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<float4 *>(gbl + off) = make_float4(l[0], l[1], l[2], l[3]);
    }
}

// The same B operand built by one warp: lane l owns token rows l, l + 32,
// l + 64, l + 96.  The packed codes of all four rows are loaded before any
// is used -- as 32-bit words when the rows are 4-byte aligned (nb % 4 == 0
// and an aligned code array: the usual case), else byte by byte one row at
// a time -- then each row's KP values are written as hi and lo 16-byte chunks.
template <int KP>
__device__ __forceinline__ void apply_b_row(uint8_t *gbh, uint8_t *gbl, const uint32_t *w,
                                            const float *sk, int row, int r) {
#pragma unroll
    for (int k0 = 0; k0 < KP; k0 += 4) {
        float h[4], l[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int k = k0 + u;
            const int q = (int)((w[k >> 3] >> ((k & 7) * 4)) & 0xFu);
            const float b = k < r ? __fmul_rn((float)(q >= 8 ? q - 16 : q), sk[k]) : 0.0f;
            h[u] = __uint_as_float(__float_as_uint(b) & 0xFFFFE000u);
            l[u] = __fsub_rn(b, h[u]);
        }
        const uint32_t off = sw128_f32_offset(row, k0);
        *reinterpret_cast<float4 *>(gbh + off) = make_float4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<float4 *>(gbl + off) = make_float4(l[0], l[1], l[2], l[3]);
    }
}

template <int KP>
__device__ __forceinline__ void apply_build_b_warp(uint8_t *gbh, uint8_t *gbl, const uint8_t *pc,
                                                   const float *sk, int64_t t0, int64_t T, int r,
                                                   int nb, int lane, int part) {
    constexpr int NW = KP / 8;                 // 32-bit words of codes per row (at most)
    constexpr int NP = kApplyBuilders / 32;    // builder warps
    constexpr int RPL = kApplyTile / 32 / NP;  // rows per lane: lane + 32 (NP rr + part)
    const bool words = (nb & 3) == 0 && (reinterpret_cast<uintptr_t>(pc) & 3u) == 0;
    if (words) {
        const int nw = nb >> 2;
        uint32_t w[RPL][NW];
#pragma unroll
        for (int rr = 0; rr < RPL; ++rr) {
            const int64_t t = t0 + lane + 32 * (NP * rr + part);
            const uint32_t *src = reinterpret_cast<const uint32_t *>(pc + t * nb);
#pragma unroll
            for (int j = 0; j < NW; ++j) w[rr][j] = (t < T && j < nw) ? __ldg(src + j) : 0u;
        }
#pragma unroll
        for (int rr = 0; rr < RPL; ++rr) apply_b_row<KP>(gbh, gbl, w[rr], sk, lane + 32 * (NP * rr + part), r);
    } else {
#pragma unroll 1
        for (int rr = 0; rr < RPL; ++rr) {
            const int64_t t = t0 + lane + 32 * (NP * rr + part);
            const uint8_t *src = pc + t * nb;
            uint32_t w[NW];
#pragma unroll
            for (int j = 0; j < NW; ++j) w[j] = 0u;
#pragma unroll
            for (int j = 0; j < 4 * NW; ++j)
                if (t < T && j < nb) w[j >> 2] |= (uint32_t)__ldg(src + j) << (8 * (j & 3));
            apply_b_row<KP>(gbh, gbl, w, sk, lane + 32 * (NP * rr + part), r);
        }
    }
}

// Persistent over a run of token tiles: CTA (x, y, z) owns channel block x of
// buffer z and token tiles [y * tpc, (y + 1) * tpc).  Warp roles (320
// threads):
//   warps 0-7 : with warps 8-9, build the A operand (Q codes of the channel
//               block) and tile 0's B operand; then each warp combines one
//               channel quarter (w % 4, its TMEM lanes) x one half (w / 4) of
//               every stage of every tile, reading x and recon from shared
//               memory and D from TMEM, and writes err and recon.  A warp
//               stages exactly the rows and channels it combines itself:
//               16-byte asynchronous copies (cp.async) into a ring of S
//               stages, issued S stages ahead from the kernel's first
//               instructions on, so its loads never wait on its arithmetic
//               and no other warp has to hand it the data;
//   warps 8-9 : for tile i, once tile i-1's product is done (its commit
//               barrier) write tile i's B operand (single buffer, half the
//               rows each), and once the consumers have released accumulator
//               i % 2 (tile i-2 combined) warp 8 issues the MMAs of tile i
//               into it.
// So the consumers never wait on operand building: the product of the next
// tile is formed while the current one is combined.
// Every wait is bounded; on expiry CF_ERR_TIMEOUT goes to the buffer's status
// word and the waiting warp stops (the others then run out of their own
// waits), every warp drains its copies still in flight, and TMEM is freed.
template <bool SENDER, int KP>
__global__ void __launch_bounds__(kApplyThreads, (KP <= 32 ? 2 : 1))
lr_apply_tc_kernel(const cf_lowrank::LrBatch B, const cf_lowrank::Layout L, int tpc) {
    const int bz = blockIdx.z;
    if (lr_skipped(B, L, bz)) return;
    const cf_lowrank::LrPtrs pp = B.get(bz);
    if (!SENDER && B.dec && !lr_dec_ptrs_ok(B, pp)) return;
    const uint16_t *x = pp.x;
    float *recon = pp.recon, *err = pp.err;
    const uint8_t *pc = pp.pc, *qc = pp.qc;
    const float *ps = pp.ps, *qs = pp.qs;
    const int64_t T = L.T, C = L.C;
    const int r = L.r;
    int32_t *status = B.ws ? B.at<int32_t>(bz, L.off_status) + cf_lowrank::kStatusWord
                           : (SENDER ? nullptr : B.dec_status);
    constexpr int NA = KP / 32;       // 128-byte K atoms per operand
    constexpr int OPB = NA * 16384;   // bytes per operand tile
    constexpr int S = apply_ring<SENDER, KP>();
    constexpr int SB = apply_stage_bytes<SENDER>();
    constexpr int STOK = apply_stage_tok<SENDER>();
    constexpr int TPW = STOK / 2;                        // tokens per warp per stage
    constexpr int RB = STOK * kApplyTile * 4;            // recon part of a stage
    extern __shared__ uint8_t dsm[];
    const uint32_t base = (smem_u32(dsm) + 1023u) & ~1023u;
    uint8_t *gb = dsm + (base - smem_u32(dsm));
    const uint32_t sA = base, sBh = base + OPB, sBl = base + 2 * OPB;
    const uint32_t ring = base + 3 * OPB;
    uint8_t *gring = gb + 3 * OPB;
    // barriers: mma[2], acc_free[2]
    const uint32_t bars = ring + S * SB;
    const uint32_t mma0 = bars, accf0 = bars + 16u;
    float *sk = reinterpret_cast<float *>(gring + S * SB + 8 * 4);   // [KP]
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sk + KP);
    int *abort_flag = reinterpret_cast<int *>(tslot + 1);   // builder warps give up together

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t c0 = (int64_t)blockIdx.x * kApplyTile;
    const int64_t ntt = (T + kApplyTile - 1) / kApplyTile;
    const int64_t ty0 = (int64_t)blockIdx.y * tpc;
    if (ty0 >= ntt) return;
    const int nt = (int)((ntt - ty0 < tpc) ? ntt - ty0 : tpc);        // tiles of this CTA
    const int64_t tbeg = ty0 * kApplyTile;
    const int64_t tend = (tbeg + (int64_t)nt * kApplyTile < T) ? tbeg + (int64_t)nt * kApplyTile : T;
    const int nb = (r + 1) / 2;
    const int64_t cw = (C - c0 < kApplyTile) ? C - c0 : kApplyTile;   // channels in the block

    if (tid == 0) {
        for (int j = 0; j < 2; ++j) {
            mbar_init(mma0 + 8u * j, 1);                         // tcgen05.commit
            mbar_init(accf0 + 8u * j, kApplyConsumers / 32);     // one per consumer warp
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (tid < KP) sk[tid] = tid < r ? __fmul_rn(__ldg(ps + tid), __ldg(qs + tid)) : 0.0f;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tslot)),
                     "r"(256u)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tslot;

    {
        // Consumer warps: their first S stages' copies go out before the
        // operand build, so the loads overlap it.
        const int q = warp & 3, half = warp >> 2;
        const int cl = 32 * q + lane;              // channel within the block
        const int64_t c = c0 + cl;
        const bool col_ok = cl < cw;
        const uint32_t tlane = (uint32_t)(32 * q) << 16;
        // Global stage g covers tokens [tbeg + g STOK, +STOK) (tiles are
        // full except possibly the CTA's last).  issue(g) stages this
        // warp's TPW rows x 32 channels of it: recon in 16-byte chunks of
        // 4 channels, x in chunks of 8; one commit group per stage.
        const int64_t gstages = (tend - tbeg + STOK - 1) / STOK;
        auto issue = [&](int64_t gg) {
            if (gg < gstages) {
                const uint32_t sr0 = ring + (uint32_t)((gg % S) * SB);
                const int64_t tb = tbeg + gg * STOK + TPW * half;
#pragma unroll
                for (int id = lane; id < TPW * 8; id += 32) {
                    const int row = id >> 3, ch = 32 * q + 4 * (id & 7);
                    const int64_t t = tb + row;
                    const bool ok = t < tend && ch < cw && CF_IN(t < T && c0 + ch + 4 <= C);
                    apply_cp16(sr0 + (uint32_t)((TPW * half + row) * (kApplyTile * 4) + ch * 4),
                               ok ? (const void *)(recon + t * C + c0 + ch) : (const void *)recon, ok);
                }
                if (SENDER) {
#pragma unroll
                    for (int id = lane; id < TPW * 4; id += 32) {
                        const int row = id >> 2, ch = 32 * q + 8 * (id & 3);
                        const int64_t t = tb + row;
                        const bool ok = t < tend && ch < cw && CF_IN(t < T && c0 + ch + 8 <= C);
                        apply_cp16(sr0 + (uint32_t)(RB + (TPW * half + row) * (kApplyTile * 2) + ch * 2),
                                   ok ? (const void *)(x + t * C + c0 + ch) : (const void *)x, ok);
                    }
                }
            }
            apply_cp_commit();
        };
        if (warp < kApplyMmaWarp)
            for (int gg = 0; gg < S; ++gg) issue(gg);
        // A = the INT4 codes of Q for this channel block, and tile 0's B:
        // built once by the consumers and the MMA warp together.
        const int ot = warp >= kApplyMmaWarp ? kApplyConsumers + 32 * (warp - kApplyMmaWarp) + lane : tid;
        constexpr int kOpThreads = kApplyConsumers + kApplyBuilders;
        for (int idx = ot; idx < kApplyTile * (KP / 4); idx += kOpThreads) {
            const int row = idx / (KP / 4), k0 = (idx - row * (KP / 4)) * 4;
            const int64_t c = c0 + row;
            float a[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int k = k0 + u;
                a[u] = (c < C && k < r) ? (float)int4_code_at(qc + c * nb, k) : 0.0f;
            }
            *reinterpret_cast<float4 *>(gb + sw128_f32_offset(row, k0)) = make_float4(a[0], a[1], a[2], a[3]);
        }
        apply_build_b<KP>(gb + OPB, gb + 2 * OPB, pc, sk, tbeg, T, r, nb, ot, kOpThreads);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        fence_before_sync();
        operand_sync();
        fence_after_sync();

        if (warp >= kApplyMmaWarp) {
            // ---------------- B operands and MMAs ----------------
            // Both builder warps reach builder_sync exactly once per tile and
            // leave together on a shared flag, so a bounded wait that gives
            // up in one of them cannot strand the other at the barrier.
            const int part = warp - kApplyMmaWarp;
            const int ksteps = (r + 7) / 8;
            constexpr uint32_t idesc = idesc_tf32(kApplyTile);
            for (int i = 0; i < nt; ++i) {
                bool ok = true;
                if (i > 0) {
                    // tile i-1's product has read the B buffer
                    ok = __all_sync(kFullMask, mbar_wait(mma0 + 8u * ((i - 1) & 1), (uint32_t)(((i - 1) >> 1) & 1)));
                    if (ok)
                        apply_build_b_warp<KP>(gb + OPB, gb + 2 * OPB, pc, sk, tbeg + (int64_t)i * kApplyTile,
                                               T, r, nb, lane, part);
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                // accumulator i % 2 is free once tile i-2 has been combined
                if (ok && i >= 2)
                    ok = __all_sync(kFullMask, mbar_wait(accf0 + 8u * (i & 1), (uint32_t)(((i - 2) >> 1) & 1)));
                if (!ok && lane == 0) {
                    *(volatile int *)abort_flag = 1;
                    if (status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
                }
                builder_sync();
                if (*(volatile int *)abort_flag) break;
                fence_after_sync();
                if (part == 0 && lane == 0) {
                    const uint32_t acc = tmem + (uint32_t)(128 * (i & 1));
                    for (int kk = 0; kk < ksteps; ++kk) {
                        const uint32_t off = (uint32_t)((kk >> 2) * 16384 + (kk & 3) * 32);
                        const uint64_t da = sw128_desc(sA + off, 16, 1024);
                        mma_tf32(acc, da, sw128_desc(sBh + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
                        mma_tf32(acc, da, sw128_desc(sBl + off, 16, 1024), idesc, 1u);
                    }
                    mma_commit(mma0 + 8u * (i & 1));
                }
                __syncwarp();
            }
        } else {
            // ---------------- combine ----------------
            int64_t g = 0;                             // stages consumed so far
            for (int i = 0; i < nt; ++i) {
                if (!__all_sync(kFullMask, mbar_wait(mma0 + 8u * (i & 1), (uint32_t)((i >> 1) & 1)))) {
                    if (lane == 0 && status) atomicCAS(status, (int32_t)CF_OK, (int32_t)CF_ERR_TIMEOUT);
                    break;
                }
                fence_after_sync();
                const int64_t t0 = tbeg + (int64_t)i * kApplyTile;
                const uint32_t acc = tmem + tlane + (uint32_t)(128 * (i & 1));
                const int64_t tw = (T - t0 < kApplyTile) ? T - t0 : kApplyTile;
                const int ns = (int)((tw + STOK - 1) / STOK);
                for (int st = 0; st < ns; ++st, ++g) {
                    const int slot = (int)(g % S);
                    // this warp's copies of stage g have landed (one group
                    // per stage, S in flight)
                    apply_cp_wait<S - 1>();
                    __syncwarp();
                    const int tl = st * STOK + TPW * half;   // first token column of this warp
                    float dv[TPW];
                    if (TPW == 16)
                        tmem_ld16(acc + (uint32_t)tl, dv);
                    else
                        tmem_ld8(acc + (uint32_t)tl, dv);
                    const float *sr = reinterpret_cast<const float *>(gring + slot * SB) + TPW * half * kApplyTile;
                    const uint16_t *sx = reinterpret_cast<const uint16_t *>(gring + slot * SB + RB) + TPW * half * kApplyTile;
                    if (col_ok) {
#pragma unroll
                        for (int j = 0; j < TPW; ++j) {
                            if (tl + j >= tw) break;
                            if (!CF_IN(t0 + tl + j < T && c < C)) break;
                            const float rv = sr[j * kApplyTile + cl];
                            const int64_t o = (t0 + tl + j) * C + c;
                            if (SENDER) {
                                const float v = __fsub_rn(bf16_bits_to_f32(sx[j * kApplyTile + cl]), rv);
                                __stcs(err + o, __fsub_rn(v, dv[j]));
                            }
                            __stcs(recon + o, __fadd_rn(rv, dv[j]));
                        }
                    }
                    // every lane has read its rows of the slot: refill it
                    __syncwarp();
                    issue(g + S);
                }
                // this warp's reads of accumulator i % 2 are complete
                fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(accf0 + 8u * (i & 1));
            }
            // no copy may land after this CTA's shared memory is released
            asm volatile("cp.async.wait_all;" ::: "memory");
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256u)
                     : "memory");
    }
}

}  // namespace umma
}  // namespace cf
