// lowrank_api.cuh -- internal interface of the low-rank implementation:
// limits, tile constants and the workspace layout.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "cf.h"

namespace cf_lowrank {

constexpr int kMaxRank = 64;
constexpr int kMaxIters = 16;

constexpr int64_t kChunkA = 512;   // channels per split of Y = V Q (CUDA-core engine)
constexpr int64_t kChunkB = 512;   // tokens per split of Q = V^T P (CUDA-core engine)
constexpr int kGramTok = 32;       // tokens per Gram CTA
constexpr int kGramGroup = 16;     // Gram partial blocks summed per first-level group
constexpr int kApplyTok = 32;      // D tile: tokens
constexpr int kApplyCh = 256;      // D tile: channels
constexpr int kApplyThreads = 256;
constexpr int64_t kTileRows = 128;  // output rows per tcgen05 projection tile

// Workspace layout (byte offsets, each region 256-byte aligned).  rp is
// the rank padded to a multiple of 16 (MMA N granularity); Tp the token
// count padded to a multiple of 8 (16-byte rows of the bf16 P^T copy).
struct Layout {
    int64_t T, C;
    int r, rp;
    int64_t Tp;
    int splitsA, splitsB, nGram, nGroups;
    int nTileT, nTileC;  // 128-row tiles of the two projections
    size_t off_status, off_gt, off_gp, off_gg, off_rmat, off_amax, off_vb, off_qt, off_yp, off_y,
        off_p, off_pt, off_zp, off_q, total;
};

// Descriptor checks shared by cf_payload_bytes and the low-rank entry points.
cf_status check_desc(const cf_desc *d);
Layout make_layout(int64_t T, int64_t C, int r);

// Per-buffer status region (off_status): [0] status word, [1] final Gram
// ticket, [2] skip flag (set when the buffer's pointers failed validation),
// all cleared at the start of every encode; [4] and [5] the warm-start tag,
// kept across encodes: kWarmMagic | r and C once an encode has left a
// usable Q (its bf16 copy Qt) in the workspace.
constexpr int kStatusWord = 0, kTicketWord = 1, kSkipWord = 2, kWarmTag = 4, kWarmC = 5;
constexpr uint32_t kWarmMagic = 0x51570000u;

// One buffer's caller pointers (sender fields; the receiver uses the payload
// and recon).
struct LrPtrs {
    const uint16_t *x;
    float *recon;
    float *err;
    const float *omega;
    const uint8_t *pc;
    const float *ps;
    const uint8_t *qc;
    const float *qs;
    uint8_t *pc_out;
    float *ps_out;
    uint8_t *qc_out;
    float *qs_out;
};

// What every low-rank kernel receives by value: where each buffer's caller
// pointers and workspace slice are.  Exactly one of enc / dec / single use
// is active: `enc` (batched encode), `dec` (batched decode), else `one`.
struct LrBatch {
    const cf_lowrank_buffer *enc;
    const cf_lowrank_dec_buffer *dec;
    LrPtrs one;
    uint8_t *ws;
    int64_t ws_stride;
    int32_t *dec_status;  // batched decode: optional caller status word

#ifdef __CUDACC__
    template <class P>
    __device__ __forceinline__ static P ld(P const *field) {
        return reinterpret_cast<P>(__ldg(reinterpret_cast<const unsigned long long *>(field)));
    }
    __device__ __forceinline__ LrPtrs get(int b) const {
        if (enc) {
            const cf_lowrank_buffer *e = enc + b;
            LrPtrs p;
            p.x = ld(&e->x);
            p.recon = ld(&e->recon_s);
            p.err = ld(&e->err);
            p.omega = ld(&e->omega);
            p.pc_out = ld(&e->p_codes);
            p.ps_out = ld(&e->p_scales);
            p.qc_out = ld(&e->q_codes);
            p.qs_out = ld(&e->q_scales);
            p.pc = p.pc_out;
            p.ps = p.ps_out;
            p.qc = p.qc_out;
            p.qs = p.qs_out;
            return p;
        }
        if (dec) {
            const cf_lowrank_dec_buffer *e = dec + b;
            LrPtrs p = {};
            p.pc = ld(&e->p_codes);
            p.ps = ld(&e->p_scales);
            p.qc = ld(&e->q_codes);
            p.qs = ld(&e->q_scales);
            p.recon = ld(&e->recon_r);
            return p;
        }
        return one;
    }
    template <class T>
    __device__ __forceinline__ T *at(int b, size_t off) const {
        return reinterpret_cast<T *>(ws + (int64_t)b * ws_stride + off);
    }
#endif
};

}  // namespace cf_lowrank
