// lowrank_api.cuh -- internal interface between the C-ABI translation unit
// and the low-rank implementation (lowrank.cu).
#pragma once

#include "cf.h"

namespace cf_lowrank {

constexpr int kMaxRank = 64;
constexpr int kMaxIters = 16;

// Descriptor checks shared by cf_payload_bytes and the low-rank entry points.
cf_status check_desc(const cf_desc *d);

}  // namespace cf_lowrank
