// lowrank.cu -- low-rank mode (subspace iteration + INT4 factors).
#include <cuda_runtime.h>

#include "cf.h"
#include "lowrank_api.cuh"

namespace cf_lowrank {

cf_status check_desc(const cf_desc *d) {
    if (!d) return CF_ERR_INVALID_ARG;
    if (d->tokens < 0 || d->channels < 1) return CF_ERR_INVALID_ARG;
    if (d->bits != 0 || d->scale_kind != 0) return CF_ERR_INVALID_ARG;
    if (d->rank < 1 || d->rank > kMaxRank) return CF_ERR_UNSUPPORTED;
    if (d->iters < 1 || d->iters > kMaxIters) return CF_ERR_UNSUPPORTED;
    if (d->rank > d->channels || (d->tokens > 0 && d->rank > d->tokens)) return CF_ERR_INVALID_ARG;
    return CF_OK;
}

}  // namespace cf_lowrank

extern "C" {

int64_t cf_lowrank_workspace_bytes(const cf_desc *d) {
    if (cf_lowrank::check_desc(d) != CF_OK) return 0;
    return 0;
}

int64_t cf_lowrank_factor_bytes(int64_t rows, int32_t rank) {
    if (rows < 0 || rank < 1) return 0;
    return rows * ((rank + 1) / 2);
}

cf_status cf_lowrank_encode(const cf_desc *, const uint16_t *, float *, float *, const float *,
                            uint8_t *, float *, uint8_t *, float *, void *, size_t, void *) {
    return CF_ERR_UNSUPPORTED;
}

cf_status cf_lowrank_decode(const cf_desc *, const uint8_t *, const float *, const uint8_t *,
                            const float *, float *, void *) {
    return CF_ERR_UNSUPPORTED;
}

cf_status cf_lowrank_status(void *, void *) { return CF_ERR_UNSUPPORTED; }

}  // extern "C"
