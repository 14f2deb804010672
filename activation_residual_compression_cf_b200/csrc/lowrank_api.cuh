// lowrank_api.cuh -- internal interface of the low-rank implementation:
// limits, tile constants and the workspace layout.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "cf.h"

namespace cf_lowrank {

constexpr int kMaxRank = 64;
constexpr int kMaxIters = 16;

constexpr int64_t kChunkA = 512;   // channels per split of the Y = V Q pass
constexpr int64_t kChunkB = 512;   // tokens per split of the Q = V^T P pass
constexpr int kGramTok = 32;       // tokens per Gram CTA
constexpr int kGramGroup = 16;     // Gram partial blocks summed per first-level group
constexpr int kApplyTok = 32;      // D tile: tokens
constexpr int kApplyCh = 256;      // D tile: channels
constexpr int kApplyThreads = 256;

// Workspace layout (byte offsets, each region 256-byte aligned).  rp is
// the rank padded to a multiple of 16 (MMA N granularity); Tp the token
// count padded to a multiple of 8 (16-byte rows of the bf16 P^T copy).
struct Layout {
    int64_t T, C;
    int r, rp;
    int64_t Tp;
    int splitsA, splitsB, nGram, nGroups;
    size_t off_status, off_gt, off_gp, off_gg, off_rmat, off_amax, off_vb, off_qt, off_yp, off_y, off_p, off_pt,
        off_zp, off_q, total;
};

// Descriptor checks shared by cf_payload_bytes and the low-rank entry points.
cf_status check_desc(const cf_desc *d);
Layout make_layout(int64_t T, int64_t C, int r);

}  // namespace cf_lowrank
