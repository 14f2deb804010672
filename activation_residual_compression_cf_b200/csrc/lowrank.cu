// lowrank.cu -- low-rank mode: subspace iteration + INT4 factors + error
// feedback ("Accelerating Parallel Diffusion Model Serving with Residual
// Compression": "Approach" -- low-rank compression with INT4 factors;
// "Key results" -- rank 32 INT4 gives about 100x; "Builds on" -- PowerSGD
// style subspace iteration; "Measured effects" -- 2 vs 10 iterations).
//
// Per buffer and step, with V = (float)x - recon_s:
//   Vb  = bf16(V)                       formed by the first projection from
//                                       x and recon (tensor cores), or by a
//                                       residual pass (CUDA cores)
//   Qt  = bf16(Omega)^T                 [rp][C], K-major B operand (or the
//                                       previous encode's, warm start)
//   repeat iters:
//     Y    = Vb Q          128-token tiles over all channels; tile Grams
//     G    = Y^T Y         (fp64, summed in tile order), R = chol(G)
//     P    = Y R^-1        (fp32 [T][rp], bf16 copy Pt [rp][Tp])
//     Q    = Vb^T P        128-channel blocks over all tokens
//   INT4 per column of P and Q, packed
//   D = (qP sP)(qQ sQ)^T ; err = V - D ; recon_s += D     (exact fp32 V)
// The receiver adds the same D, formed by the same device routine.  The
// CUDA-core engine (cross-checks) splits the two products over K and sums
// the partials in fixed order instead.
//
// The workspace is caller-allocated (cf_lowrank_workspace_bytes); its
// layout is computed here from (T, C, r).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>

#include "cf.h"
#include "cf_diag.h"
#include "cf_trace.h"
#include "cf_common.cuh"
#include "lowrank_api.cuh"
#include "lowrank_kernels.cuh"
#include "lowrank_umma.cuh"
#include "lowrank_apply_tc.cuh"

namespace cf_lowrank {

cf_status check_desc(const cf_desc *d) {
    if (!d) return CF_ERR_INVALID_ARG;
    if (d->tokens < 0 || d->channels < 1) return CF_ERR_INVALID_ARG;
    if (d->bits != 0 || d->scale_kind != 0) return CF_ERR_INVALID_ARG;
    if (d->rank < 1 || d->rank > kMaxRank) return CF_ERR_UNSUPPORTED;
    if (d->iters < 1 || d->iters > kMaxIters) return CF_ERR_UNSUPPORTED;
    if (d->rank > d->channels || (d->tokens > 0 && d->rank > d->tokens)) return CF_ERR_INVALID_ARG;
    if (d->channels % 8 != 0) return CF_ERR_UNSUPPORTED;
    if (d->tokens > (int64_t(1) << 40) / d->channels) return CF_ERR_INVALID_ARG;
    return CF_OK;
}

Layout make_layout(int64_t T, int64_t C, int r) {
    Layout L;
    L.T = T;
    L.C = C;
    L.r = r;
    L.rp = (r + 15) / 16 * 16;
    L.Tp = (T + 7) / 8 * 8;
    L.splitsA = (int)((C + kChunkA - 1) / kChunkA);
    L.splitsB = (int)((T + kChunkB - 1) / kChunkB);
    L.nGram = (int)((T + kGramTok - 1) / kGramTok);
    L.nGroups = (L.nGram + kGramGroup - 1) / kGramGroup;
    L.nTileT = (int)((T + kTileRows - 1) / kTileRows);
    L.nTileC = (int)((C + kTileRows - 1) / kTileRows);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += (bytes + 255) / 256 * 256;
        return o;
    };
    L.off_status = take(16);                          // status word, final ticket
    L.off_gt = take((size_t)L.nGroups * 4);           // group tickets
    // partial Grams: per 32-token block (CUDA-core engine) or per 128-token
    // tile (tensor-core engine); the former count is the larger
    L.off_gp = take((size_t)L.nGram * L.rp * L.rp * 8);
    L.off_gg = take((size_t)L.nGroups * L.rp * L.rp * 8);
    L.off_rmat = take((size_t)L.rp * L.rp * 4 + (size_t)L.rp * 4);
    L.off_amax = take((size_t)2 * L.rp * 4);
    L.off_vb = take((size_t)T * C * 2);
    L.off_qt = take((size_t)L.rp * C * 2);
    L.off_yp = take((size_t)L.splitsA * T * L.rp * 4);
    L.off_y = take((size_t)T * L.rp * 4);
    L.off_p = take((size_t)T * L.rp * 4);
    L.off_pt = take((size_t)L.rp * L.Tp * 2);
    L.off_zp = take((size_t)L.splitsB * C * L.rp * 4);
    L.off_q = take((size_t)C * L.rp * 4);
    L.total = off;
    return L;
}

}  // namespace cf_lowrank

namespace {

using namespace cf_lowrank;

cf_status check_ptr(const void *p, uintptr_t align = 16) {
    if (!p) return CF_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(p) & (align - 1)) != 0) return CF_ERR_ALIGNMENT;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return CF_ERR_INVALID_ARG;
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return CF_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return CF_ERR_CUDA;
    if (a.type == cudaMemoryTypeDevice && a.device != dev) return CF_ERR_INVALID_ARG;
    return CF_OK;
}

#define LR_TRY(expr)                \
    do {                            \
        cf_status _s = (expr);      \
        if (_s != CF_OK) return _s; \
    } while (0)

#define LR_LAUNCHED()                                              \
    do {                                                           \
        if (cudaGetLastError() != cudaSuccess) return CF_ERR_CUDA; \
    } while (0)

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

std::atomic<int> g_engine{0};  // 0 = tensor cores (tcgen05), 1 = CUDA cores
std::atomic<int> g_group{0};   // batched encode: buffers per pass of every stage (0 = all)

// Events recorded around the apply launch (measurement hook), per direction.
std::atomic<void *> g_apply_ev[2][2] = {};

cf_status record_apply_event(bool sender, int which, cudaStream_t st) {
    void *ev = g_apply_ev[sender ? 0 : 1][which].load();
    if (!ev) return CF_OK;
    return cudaEventRecord(static_cast<cudaEvent_t>(ev), st) == cudaSuccess ? CF_OK : CF_ERR_CUDA;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::atomic<bool> tried{false};
    if (!fn && !tried.exchange(true)) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            (void)cudaGetLastError();
    }
    return fn;
}

// 3-D bf16 tensor map over n buffers of a row-major [rows][cols] array each
// (row pitch `pitch` elements, buffer stride `bstride` bytes), box {64
// columns, box_rows rows, 1 buffer}, 128-byte swizzle, zero fill outside.
bool make_map(CUtensorMap *m, const void *base, int64_t cols, int64_t rows, int64_t pitch,
              int64_t n, int64_t bstride, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)n};
    const cuuint64_t strides[2] = {(cuuint64_t)pitch * 2, (cuuint64_t)bstride};
    const cuuint32_t box[3] = {64, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
cf_status launch_project(const LrBatch &B, const Layout &L, int n, cudaStream_t st) {
    CUtensorMap mv, mq;
    if (!make_map(&mv, B.ws + L.off_vb, L.C, L.T, L.C, n, B.ws_stride, 128) ||
        !make_map(&mq, B.ws + L.off_qt, L.C, L.rp, L.C, n, B.ws_stride, BN))
        return CF_ERR_CUDA;
    auto k = cf::umma::project_kernel<BN>;
    const int smem = cf::umma::StageGeom<BN>::kSmem;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return CF_ERR_CUDA;
    dim3 grid((unsigned)L.nTileT, 1, (unsigned)n);
    k<<<grid, 128, smem, st>>>(mv, mq, B, L);
    return cudaGetLastError() == cudaSuccess ? CF_OK : CF_ERR_CUDA;
}

template <int BN>
cf_status launch_project_residual(const LrBatch &B, const Layout &L, int n, cudaStream_t st) {
    CUtensorMap mq;
    if (!make_map(&mq, B.ws + L.off_qt, L.C, L.rp, L.C, n, B.ws_stride, BN)) return CF_ERR_CUDA;
    auto k = cf::umma::project_residual_kernel<BN>;
    const int smem = cf::umma::FusedGeom<BN>::kSmem;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return CF_ERR_CUDA;
    dim3 grid((unsigned)L.nTileT, 1, (unsigned)n);
    k<<<grid, cf::umma::kFusedThreads, smem, st>>>(mq, B, L);
    return cudaGetLastError() == cudaSuccess ? CF_OK : CF_ERR_CUDA;
}

// First projection of a tensor-core encode, fused with the residual.
cf_status project_residual(const LrBatch &B, const Layout &L, int n, cudaStream_t st) {
    switch (L.rp) {
        case 16: return launch_project_residual<16>(B, L, n, st);
        case 32: return launch_project_residual<32>(B, L, n, st);
        case 48: return launch_project_residual<48>(B, L, n, st);
        case 64: return launch_project_residual<64>(B, L, n, st);
    }
    return CF_ERR_UNSUPPORTED;
}

template <int BN>
cf_status launch_backproject(const LrBatch &B, const Layout &L, int n, bool last, cudaStream_t st) {
    CUtensorMap mv, mp;
    if (!make_map(&mv, B.ws + L.off_vb, L.C, L.T, L.C, n, B.ws_stride, 64) ||
        !make_map(&mp, B.ws + L.off_pt, L.Tp, L.rp, L.Tp, n, B.ws_stride, BN))
        return CF_ERR_CUDA;
    auto k = cf::umma::backproject_kernel<BN>;
    const int smem = cf::umma::StageGeom<BN>::kSmem;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return CF_ERR_CUDA;
    dim3 grid((unsigned)L.nTileC, 1, (unsigned)n);
    k<<<grid, 128, smem, st>>>(mv, mp, B, L, last ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? CF_OK : CF_ERR_CUDA;
}

cf_status project(const LrBatch &B, const Layout &L, int n, cudaStream_t st) {
    if (g_engine.load() == 0) {
        switch (L.rp) {
            case 16: return launch_project<16>(B, L, n, st);
            case 32: return launch_project<32>(B, L, n, st);
            case 48: return launch_project<48>(B, L, n, st);
            case 64: return launch_project<64>(B, L, n, st);
        }
    }
    cf::lr_project_simt<<<dim3((unsigned)((L.T + 63) / 64), (unsigned)L.splitsA, (unsigned)n), 256, 0,
                          st>>>(B, L);
    return cudaGetLastError() == cudaSuccess ? CF_OK : CF_ERR_CUDA;
}

cf_status backproject(const LrBatch &B, const Layout &L, int n, bool last, cudaStream_t st) {
    if (g_engine.load() == 0) {
        switch (L.rp) {
            case 16: return launch_backproject<16>(B, L, n, last, st);
            case 32: return launch_backproject<32>(B, L, n, last, st);
            case 48: return launch_backproject<48>(B, L, n, last, st);
            case 64: return launch_backproject<64>(B, L, n, last, st);
        }
    }
    cf::lr_backproject_simt<<<dim3((unsigned)((L.C + 63) / 64), (unsigned)L.splitsB, (unsigned)n), 256,
                              0, st>>>(B, L);
    return cudaGetLastError() == cudaSuccess ? CF_OK : CF_ERR_CUDA;
}

cf_status orth(const LrBatch &B, const Layout &L, int n, bool last, cudaStream_t st) {
#define CF_ORTH(RP)                                                                                   \
    cf::lr_orth_kernel<RP><<<dim3((unsigned)((L.Tp + cf::orth_threads<RP>() - 1) / cf::orth_threads<RP>()), \
                                  1, (unsigned)n),                                                        \
                             cf::orth_threads<RP>(), 0, st>>>(B, L, last ? 1 : 0)
    switch (L.rp) {
        case 16: CF_ORTH(16); break;
        case 32: CF_ORTH(32); break;
        case 48: CF_ORTH(48); break;
        case 64: CF_ORTH(64); break;
        default: return CF_ERR_UNSUPPORTED;
    }
#undef CF_ORTH
    return cudaGetLastError() == cudaSuccess ? CF_OK : CF_ERR_CUDA;
}

cf_status reduce_q(const LrBatch &B, const Layout &L, int n, bool last, cudaStream_t st) {
    const dim3 grid((unsigned)((L.C + 31) / 32), 1, (unsigned)n);
#define CF_RQ(RP) cf::lr_reduce_q_kernel<RP><<<grid, 32, 0, st>>>(B, L, last ? 1 : 0)
    switch (L.rp) {
        case 16: CF_RQ(16); break;
        case 32: CF_RQ(32); break;
        case 48: CF_RQ(48); break;
        case 64: CF_RQ(64); break;
        default: return CF_ERR_UNSUPPORTED;
    }
#undef CF_RQ
    return cudaGetLastError() == cudaSuccess ? CF_OK : CF_ERR_CUDA;
}

template <bool SENDER, int KP>
cf_status launch_apply_tc(const LrBatch &B, const Layout &L, int n, cudaStream_t st) {
    auto k = cf::umma::lr_apply_tc_kernel<SENDER, KP>;
    constexpr int smem = cf::umma::apply_tc_smem<SENDER, KP>();
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return CF_ERR_CUDA;
    // Token tiles per CTA: enough CTAs for two waves of resident CTAs, and
    // up to apply_max_tiles_per_cta tiles each so the per-CTA set-up (TMEM,
    // A operand, first product) is amortised.
    const int64_t ncb = (L.C + 127) / 128, ntt = (L.T + 127) / 128;
    const int64_t tiles = ncb * ntt * n;
    const int64_t slots = (int64_t)sm_count() * (KP <= 32 ? 2 : 1);
    int64_t tpc = tiles / (2 * slots);
    if (tpc < 1) tpc = 1;
    constexpr int max_tpc = cf::umma::apply_max_tiles_per_cta<SENDER>();
    if (tpc > max_tpc) tpc = max_tpc;
    dim3 grid((unsigned)ncb, (unsigned)((ntt + tpc - 1) / tpc), (unsigned)n);
    k<<<grid, cf::umma::kApplyThreads, smem, st>>>(B, L, (int)tpc);
    return cudaGetLastError() == cudaSuccess ? CF_OK : CF_ERR_CUDA;
}

// D = P^ Q^T applied to the state.  Engine 0: tensor cores (tcgen05 tf32,
// hi/lo split); engine 1: CUDA-core FMA chain.  A buffer's sender and
// receiver must use the same engine to stay bit-identical.
cf_status apply_launch(bool sender, const LrBatch &B, const Layout &L, int n, cudaStream_t st) {
    if (g_engine.load() == 0) {
        if (L.rp <= 32)
            return sender ? launch_apply_tc<true, 32>(B, L, n, st) : launch_apply_tc<false, 32>(B, L, n, st);
        return sender ? launch_apply_tc<true, 64>(B, L, n, st) : launch_apply_tc<false, 64>(B, L, n, st);
    }
    const int64_t gx = (L.C + kApplyCh - 1) / kApplyCh;
    const int64_t ntiles = (L.T + kApplyTok - 1) / kApplyTok;
    int64_t gy = (2 * (int64_t)sm_count() + gx - 1) / gx;
    if (gy > ntiles) gy = ntiles;
    if (gy < 1) gy = 1;
    dim3 grid((unsigned)gx, (unsigned)gy, (unsigned)n);
    const size_t smem = (size_t)L.r * (kApplyTok + kApplyCh) * sizeof(float);
    if (sender) {
        auto k = cf::lr_apply_kernel<true>;
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return CF_ERR_CUDA;
        k<<<grid, kApplyThreads, smem, st>>>(B, L);
    } else {
        auto k = cf::lr_apply_kernel<false>;
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return CF_ERR_CUDA;
        k<<<grid, kApplyThreads, smem, st>>>(B, L);
    }
    LR_LAUNCHED();
    return CF_OK;
}

cf_status apply(bool sender, const LrBatch &B, const Layout &L, int n, cudaStream_t st) {
    const cf_status e0 = record_apply_event(sender, 0, st);
    const cf_status k = apply_launch(sender, B, L, n, st);
    const cf_status e1 = record_apply_event(sender, 1, st);
    if (k != CF_OK) return k;
    return e0 != CF_OK ? e0 : e1;
}

cf_status encode_group(const cf_desc *d, const Layout &L, int n, const LrBatch &B, cudaStream_t st);

// The whole sender for n buffers (n = 1 for the single-buffer call): every
// stage launched once for all n, or, with a group size g set, for g buffers
// at a time (the buffers of a group then share the L2 between the passes).
cf_status encode_impl(const cf_desc *d, const Layout &L, int n, const LrBatch &B, cudaStream_t st) {
    const int g = g_group.load();
    if (g <= 0 || g >= n || !B.enc) return encode_group(d, L, n, B, st);
    for (int b0 = 0; b0 < n; b0 += g) {
        LrBatch Bg = B;
        Bg.enc = B.enc + b0;
        Bg.ws = B.ws + (int64_t)b0 * B.ws_stride;
        const cf_status s = encode_group(d, L, n - b0 < g ? n - b0 : g, Bg, st);
        if (s != CF_OK) return s;
    }
    return CF_OK;
}

cf_status encode_group(const cf_desc *d, const Layout &L, int n, const LrBatch &B, cudaStream_t st) {
    const bool fused = g_engine.load() == 0;
    cf::lr_prep_kernel<<<(unsigned)n, 128, 0, st>>>(B, L);
    LR_LAUNCHED();
    {
        // tensor-core engine: the first projection forms Vb itself
        if (!fused) {
            const int64_t groups = L.T * L.C / 8;
            int64_t blocks = (groups + 255) / 256;
            const int64_t cap = (int64_t)sm_count() * 8 / n + 1;
            if (blocks > cap) blocks = cap;
            cf::lr_residual_kernel<<<dim3((unsigned)blocks, 1, (unsigned)n), 256, 0, st>>>(B, L);
            LR_LAUNCHED();
        }
        const int64_t ctiles = (L.C + 31) / 32;
        cf::lr_omega_kernel<<<dim3((unsigned)((ctiles + cf::kOmegaTilesPerBlock - 1) / cf::kOmegaTilesPerBlock),
                                   (unsigned)((L.rp + 31) / 32), (unsigned)n),
                              dim3(32, 8), 0, st>>>(B, L);
        LR_LAUNCHED();
    }
    // Tensor-core engine: each projection CTA accumulates its whole K range,
    // so the projection also forms G and factors it (last tile of the
    // buffer) and the back-projection writes Q's transpose and maxima: an
    // iteration is three launches, and the first projection also forms the
    // bf16 residual (no separate residual pass).  CUDA-core engine: the
    // residual kernel, split-K partials with separate Gram / Cholesky and
    // Q-reduction kernels.
    for (int it = 0; it < d->iters; ++it) {
        const bool last = (it == d->iters - 1);
        LR_TRY(it == 0 && fused ? project_residual(B, L, n, st) : project(B, L, n, st));
        if (!fused) {
            cf::lr_gram_chol_kernel<<<dim3((unsigned)L.nGram, 1, (unsigned)n), 256, 0, st>>>(B, L);
            LR_LAUNCHED();
        }
        LR_TRY(orth(B, L, n, last, st));
        LR_TRY(backproject(B, L, n, last, st));
        if (!fused) LR_TRY(reduce_q(B, L, n, last, st));
    }
    // INT4 factors: quantise and pack against the column maxima.
    {
        const int64_t rows = L.T > L.C ? L.T : L.C;
        const dim3 grid((unsigned)((rows + cf::kPackThreads - 1) / cf::kPackThreads), 2, (unsigned)n);
        switch (L.rp) {
            case 16: cf::lr_int4_pack_kernel<16><<<grid, cf::kPackThreads, 0, st>>>(B, L); break;
            case 32: cf::lr_int4_pack_kernel<32><<<grid, cf::kPackThreads, 0, st>>>(B, L); break;
            case 48: cf::lr_int4_pack_kernel<48><<<grid, cf::kPackThreads, 0, st>>>(B, L); break;
            case 64: cf::lr_int4_pack_kernel<64><<<grid, cf::kPackThreads, 0, st>>>(B, L); break;
            default: return CF_ERR_UNSUPPORTED;
        }
        LR_LAUNCHED();
    }
    return apply(true, B, L, n, st);
}

}  // namespace

// Bounds-checked debug build: this translation unit's first failed index
// check, read and cleared (synchronises the device).
#ifdef CF_DEBUG_BOUNDS
int32_t cf_bounds_take_lowrank() {
    int32_t v = 0;
    const int32_t z = 0;
    if (cudaMemcpyFromSymbol(&v, cf::g_bounds_hit, sizeof v) != cudaSuccess ||
        cudaMemcpyToSymbol(cf::g_bounds_hit, &z, sizeof z) != cudaSuccess) {
        (void)cudaGetLastError();
        return -1;
    }
    return v;
}
#endif

extern "C" {

int64_t cf_lowrank_workspace_bytes(const cf_desc *d) {
    if (check_desc(d) != CF_OK) return 0;
    return (int64_t)make_layout(d->tokens, d->channels, d->rank).total;
}

int64_t cf_lowrank_factor_bytes(int64_t rows, int32_t rank) {
    if (rows < 0 || rank < 1) return 0;
    return rows * ((rank + 1) / 2);
}

cf_status cf_lowrank_encode(const cf_desc *d, const uint16_t *x, float *recon_s, float *err,
                            const float *omega, uint8_t *p_codes, float *p_scales,
                            uint8_t *q_codes, float *q_scales, void *workspace,
                            size_t workspace_bytes, void *stream) {
    cf::TraceRange trace_("cf_lowrank_encode");
    LR_TRY(check_desc(d));
    if (d->tokens == 0) return CF_OK;
    const Layout L = make_layout(d->tokens, d->channels, d->rank);
    if (workspace_bytes < L.total) return CF_ERR_WORKSPACE;
    LR_TRY(check_ptr(x));
    LR_TRY(check_ptr(recon_s));
    LR_TRY(check_ptr(err));
    if (omega) LR_TRY(check_ptr(omega, 4));   // NULL: warm start
    LR_TRY(check_ptr(p_codes, 1));
    LR_TRY(check_ptr(p_scales, 4));
    LR_TRY(check_ptr(q_codes, 1));
    LR_TRY(check_ptr(q_scales, 4));
    LR_TRY(check_ptr(workspace));
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return CF_ERR_ALIGNMENT;
    LrBatch B = {};
    B.one.x = x;
    B.one.recon = recon_s;
    B.one.err = err;
    B.one.omega = omega;
    B.one.pc = B.one.pc_out = p_codes;
    B.one.ps = B.one.ps_out = p_scales;
    B.one.qc = B.one.qc_out = q_codes;
    B.one.qs = B.one.qs_out = q_scales;
    B.ws = static_cast<uint8_t *>(workspace);
    B.ws_stride = (int64_t)L.total;
    return encode_impl(d, L, 1, B, (cudaStream_t)stream);
}

cf_status cf_lowrank_encode_batched(const cf_desc *d, int32_t n, const cf_lowrank_buffer *bufs_dev,
                                    void *workspace, size_t workspace_bytes, void *stream) {
    cf::TraceRange trace_("cf_lowrank_encode_batched");
    LR_TRY(check_desc(d));
    if (n < 0) return CF_ERR_INVALID_ARG;
    if (n == 0 || d->tokens == 0) return CF_OK;
    if (n > 65535) return CF_ERR_UNSUPPORTED;
    const Layout L = make_layout(d->tokens, d->channels, d->rank);
    if (workspace_bytes / (size_t)n < L.total) return CF_ERR_WORKSPACE;
    LR_TRY(check_ptr(bufs_dev));
    LR_TRY(check_ptr(workspace));
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return CF_ERR_ALIGNMENT;
    LrBatch B = {};
    B.enc = bufs_dev;
    B.ws = static_cast<uint8_t *>(workspace);
    B.ws_stride = (int64_t)L.total;
    return encode_impl(d, L, n, B, (cudaStream_t)stream);
}

cf_status cf_lowrank_decode(const cf_desc *d, const uint8_t *p_codes, const float *p_scales,
                            const uint8_t *q_codes, const float *q_scales, float *recon_r,
                            void *stream) {
    cf::TraceRange trace_("cf_lowrank_decode");
    LR_TRY(check_desc(d));
    if (d->tokens == 0) return CF_OK;
    LR_TRY(check_ptr(p_codes, 1));
    LR_TRY(check_ptr(p_scales, 4));
    LR_TRY(check_ptr(q_codes, 1));
    LR_TRY(check_ptr(q_scales, 4));
    LR_TRY(check_ptr(recon_r));
    const Layout L = make_layout(d->tokens, d->channels, d->rank);
    LrBatch B = {};
    B.one.pc = p_codes;
    B.one.ps = p_scales;
    B.one.qc = q_codes;
    B.one.qs = q_scales;
    B.one.recon = recon_r;
    return apply(false, B, L, 1, (cudaStream_t)stream);
}

cf_status cf_lowrank_decode_batched(const cf_desc *d, int32_t n, const cf_lowrank_dec_buffer *bufs_dev,
                                    int32_t *status_dev, void *stream) {
    cf::TraceRange trace_("cf_lowrank_decode_batched");
    LR_TRY(check_desc(d));
    if (n < 0) return CF_ERR_INVALID_ARG;
    if (n == 0 || d->tokens == 0) return CF_OK;
    if (n > 65535) return CF_ERR_UNSUPPORTED;
    LR_TRY(check_ptr(bufs_dev));
    if (status_dev) LR_TRY(check_ptr(status_dev, 4));
    const Layout L = make_layout(d->tokens, d->channels, d->rank);
    LrBatch B = {};
    B.dec = bufs_dev;
    B.dec_status = status_dev;
    return apply(false, B, L, n, (cudaStream_t)stream);
}

cf_status cf_set_lowrank_group(int32_t buffers) {
    if (buffers < 0 || buffers > 65535) return CF_ERR_INVALID_ARG;
    g_group.store(buffers);
    return CF_OK;
}

cf_status cf_set_lowrank_engine(int32_t engine) {
    if (engine < 0 || engine > 1) return CF_ERR_INVALID_ARG;
    g_engine.store(engine);
    return CF_OK;
}

cf_status cf_lowrank_set_apply_events(void *enc_start, void *enc_stop, void *dec_start,
                                      void *dec_stop) {
    if ((enc_start == nullptr) != (enc_stop == nullptr) ||
        (dec_start == nullptr) != (dec_stop == nullptr))
        return CF_ERR_INVALID_ARG;
    g_apply_ev[0][0].store(enc_start);
    g_apply_ev[0][1].store(enc_stop);
    g_apply_ev[1][0].store(dec_start);
    g_apply_ev[1][1].store(dec_stop);
    return CF_OK;
}

cf_status cf_lowrank_status(void *workspace, void *stream) {
    if (!workspace) return CF_ERR_INVALID_ARG;
    int32_t h = 0;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&h, workspace, sizeof h, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return CF_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return CF_ERR_CUDA;
    const int32_t zero = 0;
    if (cudaMemcpyAsync(workspace, &zero, sizeof zero, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return CF_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return CF_ERR_CUDA;
    return (cf_status)h;
}

cf_status cf_lowrank_status_async(const void *workspace, int64_t slice_bytes, int32_t n,
                                  int32_t *host_status, void *stream) {
    if (n < 0) return CF_ERR_INVALID_ARG;
    if (n == 0) return CF_OK;
    if (!workspace || !host_status || slice_bytes <= 0) return CF_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || slice_bytes % 256 != 0 ||
        (reinterpret_cast<uintptr_t>(host_status) & 3u) != 0)
        return CF_ERR_ALIGNMENT;
    LR_TRY(check_ptr(workspace, 256));
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, host_status) != cudaSuccess) {
        (void)cudaGetLastError();
        return CF_ERR_INVALID_ARG;
    }
    if (a.type != cudaMemoryTypeHost) return CF_ERR_INVALID_ARG;   // pageable or device memory
    // one strided copy: row b is the first int32 of slice b
    if (cudaMemcpy2DAsync(host_status, sizeof(int32_t), workspace, (size_t)slice_bytes,
                          sizeof(int32_t), (size_t)n, cudaMemcpyDeviceToHost,
                          (cudaStream_t)stream) != cudaSuccess) {
        (void)cudaGetLastError();
        return CF_ERR_CUDA;
    }
    return CF_OK;
}

}  // extern "C"
