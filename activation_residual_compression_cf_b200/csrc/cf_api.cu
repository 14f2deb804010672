// cf_api.cu -- host side of libcf.so: argument validation, launch-shape
// choice and kernel launches behind the C ABI declared in cf.h.
//
// Nothing here allocates device memory or synchronises a stream (except
// cf_lowrank_status, documented as synchronising).
#include <cuda_runtime.h>

#include <mutex>

#include "cf.h"
#include "cf_diag.h"
#include "cf_trace.h"
#include "lowrank_api.cuh"
#include "quant_kernels.cuh"
#include "quant_tma.cuh"

namespace {

// ---------------------------------------------------------------- helpers

constexpr int kMaxGroupsPerThread = 4;
constexpr int64_t kMaxDynSmem = 227 * 1024;   // dynamic shared memory a CTA may opt into
constexpr int64_t kSmemPerSM = 228 * 1024;    // shared memory of an SM (1 KB of it reserved per CTA)
constexpr int kMaxThreads = 512;
constexpr int64_t kMaxChannels = 8LL * kMaxGroupsPerThread * kMaxThreads;  // 16384

struct Override {
    int gpt = 0, threads = 0, blocks_per_sm = 0;
};
Override g_override[2];
int g_pipeline[2] = {1, 1};  // 0 = register-resident rows, 1 = TMA row staging (default)
int g_stages[2] = {0, 0};    // TMA ring depth (0 = built-in choice)
int g_unit[2] = {0, 0};      // TMA channels per thread unit, 4 or 8 (0 = built-in choice)
std::mutex g_mu;

int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    static int cache[64] = {0};
    if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64) cache[dev] = n;
    return n;
}

cf_status check_dev_ptr(const void *p, uintptr_t align = 16) {
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

#define CF_TRY(expr)                         \
    do {                                     \
        cf_status _s = (expr);               \
        if (_s != CF_OK) return _s;          \
    } while (0)

cf_status check_quant_desc(const cf_desc *d) {
    if (!d) return CF_ERR_INVALID_ARG;
    if (d->tokens < 0 || d->channels < 1) return CF_ERR_INVALID_ARG;
    if (d->scale_kind != 0) return CF_ERR_UNSUPPORTED;
    if (d->bits != 1 && d->bits != 2) return CF_ERR_UNSUPPORTED;
    if (d->rank != 0 || d->iters != 0) return CF_ERR_INVALID_ARG;
    if (d->channels > kMaxChannels) return CF_ERR_UNSUPPORTED;
    if (d->tokens > (int64_t(1) << 40) / d->channels) return CF_ERR_INVALID_ARG;
    return CF_OK;
}

struct Shape {
    int gpt;
    int threads;
    int blocks_per_sm;
    int pipeline = 0;
    int unit = 8;    // TMA pipeline: channels per thread unit (4 or 8)
};

// Channels per thread unit of the TMA kernels, measured on B200 in the
// encode -> decode sequence (two alternating repeats of 300 steps each):
// 4-channel units make every warp store 512 contiguous bytes and remove the
// shared-memory bank conflicts of the recon reads, which helped the 2-bit
// encode at C = 3072 (+3.5 %), but cost the 1-bit encode at C = 3072 4 %
// and the 2-bit decode at C = 1920 4 %; elsewhere the two tie.
int choose_unit(int kernel, int bits, int64_t C, bool delta) {
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (g_unit[kernel]) return g_unit[kernel];
    }
    if (kernel == 0 && !delta && bits == 2 && C >= 2048) return 4;
    return 8;
}

// Launch shape per row: threads (a multiple of 32) x groups of 8 channels
// per thread.  Chosen from sweeps on B200 timed in the encode -> decode
// sequence (C = 1920 and 3072): TMA encode 2 groups per thread under the
// sustained power cap (delta-state encode: 2 at 1 bit, 4 at 2 bits), TMA
// decode 3; the register pipeline 2.
Shape choose_shape(int kernel, int64_t C, int pipeline, int bits, bool delta = false) {
    const int64_t G = (C + 7) / 8;
    Shape s;
    int gpt;
    if (pipeline == 1) {
        if (kernel == 0)
            gpt = delta ? (bits == 1 ? 2 : 4) : 2;
        else
            gpt = 3;
    } else {
        gpt = (int)((G + 191) / 192);
        if (gpt < 2) gpt = 2;
    }
    if (gpt > kMaxGroupsPerThread) gpt = kMaxGroupsPerThread;
    while (gpt > 1 && (G + gpt - 1) / gpt < 32 && (G + gpt - 2) / (gpt - 1) <= 32) --gpt;
    int64_t thr = (G + gpt - 1) / gpt;
    thr = (thr + 31) / 32 * 32;
    while (thr > kMaxThreads && gpt < kMaxGroupsPerThread) {
        ++gpt;
        thr = ((G + gpt - 1) / gpt + 31) / 32 * 32;
    }
    s.gpt = gpt;
    s.threads = (int)thr;
    s.blocks_per_sm = 0;
    std::lock_guard<std::mutex> lk(g_mu);
    const Override &o = g_override[kernel];
    if (o.gpt > 0 && o.threads > 0 && (int64_t)o.gpt * o.threads >= G) {
        s.gpt = o.gpt;
        s.threads = o.threads;
    }
    if (o.blocks_per_sm > 0) s.blocks_per_sm = o.blocks_per_sm;
    return s;
}

template <class K>
int grid_for(K kernel, int threads, int blocks_per_sm_cap, int64_t rows) {
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, 0) != cudaSuccess ||
        occ < 1) {
        (void)cudaGetLastError();
        occ = 1;
    }
    if (blocks_per_sm_cap > 0 && blocks_per_sm_cap < occ) occ = blocks_per_sm_cap;
    int64_t g = (int64_t)device_sm_count() * occ;
    if (g < 1) g = 1;
    if (rows < g) g = rows;
    return (int)g;
}

cf_status launch_result() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? CF_OK : CF_ERR_CUDA;
}

template <int BITS, int GPT, bool VEC, class Src>
cf_status launch_encode_t(const Src &src, int64_t T, int64_t C, int64_t rows, int32_t *status,
                          const Shape &s, cudaStream_t st) {
    auto k = cf::encode_rows_kernel<BITS, GPT, VEC, Src>;
    const int grid = grid_for(k, s.threads, s.blocks_per_sm, rows);
    k<<<grid, s.threads, 0, st>>>(src, T, C, rows, status);
    return launch_result();
}

template <int BITS, int GPT, bool VEC, class Src>
cf_status launch_decode_t(const Src &src, int64_t T, int64_t C, int64_t rows, int32_t *status,
                          const Shape &s, cudaStream_t st) {
    auto k = cf::decode_rows_kernel<BITS, GPT, VEC, Src>;
    const int grid = grid_for(k, s.threads, s.blocks_per_sm, rows);
    k<<<grid, s.threads, 0, st>>>(src, T, C, rows, status);
    return launch_result();
}

// TMA-staged variants: C % 8 == 0 (16-byte rows) and, for decode, 16-byte
// code rows (W % 4 == 0); at most 480 consumer threads.
constexpr int kDecodeConsumerWarpsPerSM = 12;

// The standard sender's encode (not the delta-state one): the sources whose
// dedicated TMA kernel stores err and recon with bulk copies.
template <bool ENC, class Src>
constexpr bool standard_encode() {
    if constexpr (ENC)
        return !Src::kDelta;
    else
        return false;
}

template <bool ENC, int BITS, int GPT, int K, class Src>
cf_status launch_tma(const Src &src, int64_t T, int64_t C, int64_t rows, int32_t *status,
                     const Shape &s, int stages_req, cudaStream_t st) {
    const int64_t W = (C * BITS + 31) / 32;
    int64_t slot = 4 * W + 4 * C;
    if constexpr (ENC) slot = (Src::kDelta ? 8 : 6) * C;
    // Ring depth, measured on B200 (C = 1920 and 3072) in runs long enough
    // for the power cap to hold the SM clock down, as in sustained use:
    // encode with per-thread stores 4 slots (with 2 groups per thread that
    // keeps 3-4 CTAs and 16-18 consumer warps per SM, 6-8 % above 5 slots at
    // 2 CTAs); the bulk-store encode 2 (below); decode 5.  The delta-state
    // encode's slots are a third larger (8C bytes): at C = 3072, 3 slots,
    // which keep three CTAs per SM, beat 4 (two CTAs) by ~10 %; at C <= 2048
    // it takes 2 (below).
    // a thread's GPT groups of 8 channels as 8 / K * GPT units of K; the
    // plain 8-channel launches take the dedicated kernels (faster schedule),
    // and the standard sender's dedicated encode stores err and recon with
    // bulk copies from two shared-memory output rows (8C bytes each)
    constexpr bool kPlain = K == 8 && !Src::kPublish && !Src::kWait;
    bool delta = false;
    if constexpr (ENC) delta = Src::kDelta;
    constexpr bool kBulk = kPlain && standard_encode<ENC, Src>();
    const int threads = 32 + s.threads;
    void (*k)(Src, int64_t, int64_t, int64_t, int32_t *, int);
    // Bulk-store encode: measured on B200 in the encode -> decode sequence,
    // it beats the per-thread stores when a 2-slot ring plus the two output
    // rows still lets four CTAs share an SM (C = 1920: encode +4 %), and
    // loses where fewer fit (C = 3072, two CTAs: -15 %; C = 1920 with 3 or 4
    // slots: -4 to -22 %).  So it runs with 2 slots, and only where the
    // occupancy query gives four CTAs.
    // The publishing encode (8-channel units) takes the same bulk-store path
    // for its local err and recon rows under the same condition; its codes
    // and scales still go straight to the receivers' slots.
    constexpr bool kBulkPub = ENC && Src::kPublish && K == 8;
    bool bulk = false;
    if constexpr (kBulk || kBulkPub) {
        const size_t smem2 = 2 * (size_t)slot + 16 * (size_t)C + 32;
        void (*kb)(Src, int64_t, int64_t, int64_t, int32_t *, int);
        if constexpr (kBulk)
            kb = cf::tma::encode_tma_kernel<BITS, GPT, Src, true>;
        else
            kb = cf::tma::encode_tma_publish_kernel<BITS, K, 8 / K * GPT, Src, true>;
        int occ_b = 0;
        if (smem2 <= (size_t)kMaxDynSmem &&
            cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2) == cudaSuccess &&
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_b, kb, threads, smem2) == cudaSuccess)
            bulk = occ_b >= 4;
        (void)cudaGetLastError();
    }
    const int64_t out_rows = bulk ? 16 * C : 0;
    int stages = stages_req;
    if (stages <= 0) {
        // delta-state encode: 2 slots where a slot (8C bytes) is at most
        // 16 KB, measured on B200 at C = 1920 (4 groups per thread):
        // 6042-6060 GB/s against 5052 with 4 slots, as more CTAs share an
        // SM; at C = 3072, 3 slots (75 KB) stay best (2: -4 to -6 %)
        if (bulk)
            stages = 2;
        else if (delta)
            stages = slot <= 16384 ? 2 : (int)(75000 / slot);
        else
            stages = (int)(120000 / slot);
        const int cap = (ENC && !delta) ? 4 : 5;
        if (stages > cap) stages = cap;
    }
    if (stages > 8) stages = 8;
    if (stages < 2) stages = 2;
    size_t smem = (size_t)stages * slot + (size_t)out_rows + 16 * (size_t)stages;
    while (smem > (size_t)kMaxDynSmem && stages > 2)
        smem = (size_t)--stages * slot + (size_t)out_rows + 16 * (size_t)stages;
    if (smem > (size_t)kMaxDynSmem) return CF_ERR_UNSUPPORTED;
    if constexpr (ENC) {
        if constexpr (kPlain)
            k = bulk ? cf::tma::encode_tma_kernel<BITS, GPT, Src, kBulk>
                     : cf::tma::encode_tma_kernel<BITS, GPT, Src, false>;
        else if constexpr (Src::kPublish)
            k = bulk ? cf::tma::encode_tma_publish_kernel<BITS, K, 8 / K * GPT, Src, kBulkPub>
                     : cf::tma::encode_tma_publish_kernel<BITS, K, 8 / K * GPT, Src, false>;
        else
            k = cf::tma::encode_tma_unit_kernel<BITS, K, 8 / K * GPT, Src>;
    } else {
        if constexpr (kPlain)
            k = cf::tma::decode_tma_kernel<BITS, GPT, Src>;
        else
            k = cf::tma::decode_tma_unit_kernel<BITS, K, 8 / K * GPT, Src>;
    }
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return CF_ERR_CUDA;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, threads, smem) != cudaSuccess || occ < 1) {
        (void)cudaGetLastError();
        occ = 1;
    }
    if (s.blocks_per_sm > 0) {
        if (s.blocks_per_sm < occ) occ = s.blocks_per_sm;
    } else if constexpr (!ENC) {
        // Decode: measured on B200 (C = 1920 and 3072, ring depths 3-7), the
        // rate depends on the consumer warps per SM and peaks at 12 (6.4-6.6
        // TB/s); 15 or 9 lose 10-14 %.  Cap the CTAs per SM accordingly.
        const int cap = kDecodeConsumerWarpsPerSM / (s.threads / 32);
        if (cap >= 1 && cap < occ) occ = cap;
    }
    int64_t grid = (int64_t)device_sm_count() * occ;
    if (grid > rows) grid = rows;
    if (grid < 1) grid = 1;
    k<<<(unsigned)grid, threads, smem, st>>>(src, T, C, rows, status, stages);
    return launch_result();
}

template <bool ENC, int BITS, int GPT, bool VEC, class Src>
cf_status launch_one(const Src &src, int64_t T, int64_t C, int64_t rows, int32_t *status,
                     const Shape &s, cudaStream_t st) {
    constexpr bool kFused = Src::kPublish || Src::kWait;   // TMA pipeline only
    if constexpr (VEC) {
        if (s.pipeline == 1) {
            int stages;
            {
                std::lock_guard<std::mutex> lk(g_mu);
                stages = g_stages[ENC ? 0 : 1];
            }
            if (s.unit == 4) return launch_tma<ENC, BITS, GPT, 4>(src, T, C, rows, status, s, stages, st);
            return launch_tma<ENC, BITS, GPT, 8>(src, T, C, rows, status, s, stages, st);
        }
    }
    if constexpr (kFused) {
        return CF_ERR_UNSUPPORTED;
    } else if constexpr (ENC) {
        return launch_encode_t<BITS, GPT, VEC>(src, T, C, rows, status, s, st);
    } else {
        return launch_decode_t<BITS, GPT, VEC>(src, T, C, rows, status, s, st);
    }
}

// Runtime (bits, gpt, vec) -> template instance.
// The TMA pipeline applies when rows are 16-byte multiples (C % 8 == 0),
// decode code rows too (ceil(C*bits/32) % 4 == 0), and a 2-slot ring fits.
bool tma_applies(bool enc, int bits, int64_t C, bool delta = false) {
    if (C % 8 != 0) return false;
    if (!enc && ((C * bits + 31) / 32) % 4 != 0) return false;
    return 2 * (enc ? (delta ? 8 : 6) * C : 4 * C + C * bits / 8) <= 200000;
}

template <bool ENC, class Src>
cf_status dispatch(const Src &src, int bits, int64_t T, int64_t C, int64_t rows,
                   int32_t *status, cudaStream_t st) {
    int pipe;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        pipe = g_pipeline[ENC ? 0 : 1];
    }
    bool delta = false;
    if constexpr (ENC) delta = Src::kDelta;
    constexpr bool kFused = Src::kPublish || Src::kWait;
    if (kFused) pipe = 1;     // the publishing and waiting kernels are TMA-staged
    if (pipe == 1 && !tma_applies(ENC, bits, C, delta)) pipe = 0;
    Shape s = choose_shape(ENC ? 0 : 1, C, pipe, bits, delta);
    if (pipe == 1 && s.threads > 480) s = choose_shape(ENC ? 0 : 1, C, pipe = 0, bits, delta);
    if (kFused && pipe != 1) return CF_ERR_UNSUPPORTED;
    s.pipeline = pipe;
    s.unit = choose_unit(ENC ? 0 : 1, bits, C, delta);
    if constexpr (Src::kPublish) {
        // the publishing encode at 4-channel units needs more registers than
        // the 80 that keep three CTAs per SM (it spills): 8-channel units
        // unless a sweep overrides it
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_unit[0]) s.unit = 8;
    }
    if constexpr (!ENC) {
        if constexpr (Src::kEmit) {
            // The emitting decode writes recon (fp32) and the bf16 copy; with
            // 8-channel units each recon store instruction fills 32 half
            // sectors.  4-channel units write whole sectors: measured on B200
            // in the encode -> decode sequence, 6713 against 5594 GB/s at
            // C = 1920 (+20 %) and +1.6 % at C = 3072.
            std::lock_guard<std::mutex> lk(g_mu);
            if (!g_unit[1]) s.unit = 4;
        }
    }
    if constexpr (ENC && !kFused) {
        // The standard encode with bulk stores (TMA pipeline, 8-channel
        // units): measured on B200 at C = 1920 in the encode -> decode
        // sequence, 4 groups of 8 channels per thread (two consumer warps
        // per CTA) and four CTAs per SM ran the encode 5-14 % above the
        // per-thread stores at their best shape (2 groups, 4 warps); the
        // same 4-group shape with per-thread stores was 6 % slower, and
        // with bulk stores at fewer CTAs 15 % slower.  It applies where a
        // 2-slot ring and the two output rows leave room for four CTAs.
        bool overridden;
        {
            std::lock_guard<std::mutex> lk(g_mu);
            overridden = g_override[0].gpt > 0;
        }
        // The 4-channel-unit encode (2-bit, C >= 2048) also runs best at 4
        // groups per thread: measured on two B200 boxes at C = 3072, encode
        // +2.9 % and +3.1 % over 2 groups (4 slots, three CTAs per SM).
        const bool bulk_shape = s.unit == 8 && 4 * (28 * C + 32 + 1024) <= kSmemPerSM;
        if (!delta && pipe == 1 && !overridden && (bulk_shape || s.unit == 4)) {
            const int64_t G = (C + 7) / 8;
            int gpt = kMaxGroupsPerThread;
            while (gpt > 1 && (G + gpt - 1) / gpt < 32 && (G + gpt - 2) / (gpt - 1) <= 32) --gpt;
            s.gpt = gpt;
            s.threads = (int)(((G + gpt - 1) / gpt + 31) / 32 * 32);
        }
    }
    const bool vec = (C % 8) == 0;
#define CF_CASE(B, G, V)                                     \
    if (bits == B && s.gpt == G && vec == V)                 \
        return launch_one<ENC, B, G, V>(src, T, C, rows, status, s, st);
#define CF_CASES_G(B, V) CF_CASE(B, 1, V) CF_CASE(B, 2, V) CF_CASE(B, 3, V) CF_CASE(B, 4, V)
    CF_CASES_G(1, true)
    CF_CASES_G(1, false)
    CF_CASES_G(2, true)
    CF_CASES_G(2, false)
#undef CF_CASES_G
#undef CF_CASE
    return CF_ERR_UNSUPPORTED;
}

}  // namespace

// Bounds-checked debug build: this translation unit's first failed index
// check, read and cleared (synchronises the device).
#ifdef CF_DEBUG_BOUNDS
int32_t cf_bounds_take_api() {
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

#ifdef CF_DEBUG_BOUNDS
int32_t cf_bounds_take_lowrank();
int32_t cf_bounds_take_diag();
#endif

// ------------------------------------------------------------------ C ABI

extern "C" {

const char *cf_status_string(cf_status s) {
    switch (s) {
        case CF_OK: return "CF_OK";
        case CF_ERR_INVALID_ARG: return "CF_ERR_INVALID_ARG: null, host or out-of-range argument";
        case CF_ERR_ALIGNMENT: return "CF_ERR_ALIGNMENT: device pointer not 16-byte aligned";
        case CF_ERR_UNSUPPORTED: return "CF_ERR_UNSUPPORTED: bits/rank/scale_kind/shape not supported";
        case CF_ERR_WORKSPACE: return "CF_ERR_WORKSPACE: low-rank workspace too small";
        case CF_ERR_CUDA: return "CF_ERR_CUDA: CUDA runtime call or kernel launch failed";
        case CF_ERR_NUMERIC: return "CF_ERR_NUMERIC: Gram matrix not positive definite";
        case CF_ERR_TIMEOUT: return "CF_ERR_TIMEOUT: bounded device wait gave up";
    }
    return "unknown cf_status";
}

int32_t cf_abi_version(void) { return CF_ABI_VERSION; }

int64_t cf_codes_words_per_row(const cf_desc *d) {
    if (check_quant_desc(d) != CF_OK) return 0;
    return (d->channels * d->bits + 31) / 32;
}

int64_t cf_payload_bytes(const cf_desc *d) {
    if (!d) return 0;
    if (d->bits == 0 && d->rank > 0) {
        if (cf_lowrank::check_desc(d) != CF_OK) return 0;
        const int64_t nb = (d->rank + 1) / 2;
        return d->tokens * nb + d->channels * nb + 8LL * d->rank;
    }
    if (check_quant_desc(d) != CF_OK) return 0;
    return d->tokens * cf_codes_words_per_row(d) * 4 + d->tokens * 4;
}

cf_status cf_state_init(const cf_desc *d, const uint16_t *x0, float *recon, float *err,
                        void *stream) {
    cf::TraceRange trace_("cf_state_init");
    if (!d || d->tokens < 0 || d->channels < 1) return CF_ERR_INVALID_ARG;
    if (d->tokens > (int64_t(1) << 40) / d->channels) return CF_ERR_INVALID_ARG;
    const int64_t n = d->tokens * d->channels;
    if (n == 0) return CF_OK;
    CF_TRY(check_dev_ptr(x0));
    if (!recon && !err) return CF_ERR_INVALID_ARG;
    if (recon) CF_TRY(check_dev_ptr(recon));
    if (err) CF_TRY(check_dev_ptr(err));
    const int threads = 256;
    int64_t blocks = (n / 8 + threads - 1) / threads;
    const int64_t cap = (int64_t)device_sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    cf::state_init_kernel<<<(int)blocks, threads, 0, (cudaStream_t)stream>>>(x0, recon, err, n);
    return launch_result();
}

cf_status cf_encode(const cf_desc *d, const uint16_t *x, float *recon_s, float *err,
                    uint32_t *codes, float *scales, void *stream) {
    cf::TraceRange trace_("cf_encode");
    CF_TRY(check_quant_desc(d));
    if (d->tokens == 0) return CF_OK;
    CF_TRY(check_dev_ptr(x));
    CF_TRY(check_dev_ptr(recon_s));
    CF_TRY(check_dev_ptr(err));
    CF_TRY(check_dev_ptr(codes));
    CF_TRY(check_dev_ptr(scales, 4));
    cf::EncSingle src{{x, recon_s, err, codes, scales}};
    return dispatch<true>(src, d->bits, d->tokens, d->channels, d->tokens, nullptr,
                          (cudaStream_t)stream);
}

cf_status cf_encode_delta(const cf_desc *d, const uint16_t *x, const uint16_t *x_prev, float *err,
                          uint32_t *codes, float *scales, void *stream) {
    cf::TraceRange trace_("cf_encode_delta");
    CF_TRY(check_quant_desc(d));
    if (d->tokens == 0) return CF_OK;
    CF_TRY(check_dev_ptr(x));
    CF_TRY(check_dev_ptr(x_prev));
    CF_TRY(check_dev_ptr(err));
    CF_TRY(check_dev_ptr(codes));
    CF_TRY(check_dev_ptr(scales, 4));
    cf::EncDeltaSingle src{{x, nullptr, err, codes, scales, x_prev}};
    return dispatch<true>(src, d->bits, d->tokens, d->channels, d->tokens, nullptr,
                          (cudaStream_t)stream);
}

cf_status cf_decode(const cf_desc *d, const uint32_t *codes, const float *scales, float *recon_r,
                    void *stream) {
    cf::TraceRange trace_("cf_decode");
    CF_TRY(check_quant_desc(d));
    if (d->tokens == 0) return CF_OK;
    CF_TRY(check_dev_ptr(codes));
    CF_TRY(check_dev_ptr(scales, 4));
    CF_TRY(check_dev_ptr(recon_r));
    cf::DecSingle src{{codes, scales, recon_r}};
    return dispatch<false>(src, d->bits, d->tokens, d->channels, d->tokens, nullptr,
                           (cudaStream_t)stream);
}

cf_status cf_decode_emit(const cf_desc *d, const uint32_t *codes, const float *scales,
                         float *recon_r, uint16_t *out, void *stream) {
    cf::TraceRange trace_("cf_decode_emit");
    CF_TRY(check_quant_desc(d));
    if (d->tokens == 0) return CF_OK;
    CF_TRY(check_dev_ptr(codes));
    CF_TRY(check_dev_ptr(scales, 4));
    CF_TRY(check_dev_ptr(recon_r));
    CF_TRY(check_dev_ptr(out));
    cf::DecEmitSingle src{{codes, scales, recon_r, out}};
    return dispatch<false>(src, d->bits, d->tokens, d->channels, d->tokens, nullptr,
                           (cudaStream_t)stream);
}

cf_status cf_decode_emit_batched(const cf_desc *d, int32_t n, const cf_dec_emit_buffer *bufs_dev,
                                 int32_t *status_dev, void *stream) {
    cf::TraceRange trace_("cf_decode_emit_batched");
    CF_TRY(check_quant_desc(d));
    if (n < 0) return CF_ERR_INVALID_ARG;
    if (n == 0 || d->tokens == 0) return CF_OK;
    CF_TRY(check_dev_ptr(bufs_dev));
    if (status_dev) CF_TRY(check_dev_ptr(status_dev));
    cf::DecEmitArray src{bufs_dev};
    return dispatch<false>(src, d->bits, d->tokens, d->channels, d->tokens * (int64_t)n,
                           status_dev, (cudaStream_t)stream);
}

cf_status cf_encode_batched(const cf_desc *d, int32_t n, const cf_enc_buffer *bufs_dev,
                            int32_t *status_dev, void *stream) {
    cf::TraceRange trace_("cf_encode_batched");
    CF_TRY(check_quant_desc(d));
    if (n < 0) return CF_ERR_INVALID_ARG;
    if (n == 0 || d->tokens == 0) return CF_OK;
    CF_TRY(check_dev_ptr(bufs_dev));
    if (status_dev) CF_TRY(check_dev_ptr(status_dev));
    cf::EncArray src{bufs_dev};
    return dispatch<true>(src, d->bits, d->tokens, d->channels, d->tokens * (int64_t)n,
                          status_dev, (cudaStream_t)stream);
}

cf_status cf_encode_delta_batched(const cf_desc *d, int32_t n, const cf_enc_delta_buffer *bufs_dev,
                                  int32_t *status_dev, void *stream) {
    cf::TraceRange trace_("cf_encode_delta_batched");
    CF_TRY(check_quant_desc(d));
    if (n < 0) return CF_ERR_INVALID_ARG;
    if (n == 0 || d->tokens == 0) return CF_OK;
    CF_TRY(check_dev_ptr(bufs_dev));
    if (status_dev) CF_TRY(check_dev_ptr(status_dev));
    cf::EncDeltaArray src{bufs_dev};
    return dispatch<true>(src, d->bits, d->tokens, d->channels, d->tokens * (int64_t)n,
                          status_dev, (cudaStream_t)stream);
}

cf_status cf_decode_batched(const cf_desc *d, int32_t n, const cf_dec_buffer *bufs_dev,
                            int32_t *status_dev, void *stream) {
    cf::TraceRange trace_("cf_decode_batched");
    CF_TRY(check_quant_desc(d));
    if (n < 0) return CF_ERR_INVALID_ARG;
    if (n == 0 || d->tokens == 0) return CF_OK;
    CF_TRY(check_dev_ptr(bufs_dev));
    if (status_dev) CF_TRY(check_dev_ptr(status_dev));
    cf::DecArray src{bufs_dev};
    return dispatch<false>(src, d->bits, d->tokens, d->channels, d->tokens * (int64_t)n,
                           status_dev, (cudaStream_t)stream);
}

cf_status cf_encode_publish_batched(const cf_desc *d, int32_t n, const cf_enc_publish_buffer *bufs_dev,
                                    int32_t ndst, const cf_publish_dst *dsts_dev, uint64_t ack_target,
                                    int32_t *status_dev, void *stream) {
    cf::TraceRange trace_("cf_encode_publish_batched");
    CF_TRY(check_quant_desc(d));
    if (n < 0 || ndst < 1 || ndst > 8) return CF_ERR_INVALID_ARG;
    if (n == 0 || d->tokens == 0) return CF_OK;
    if (!tma_applies(true, d->bits, d->channels)) return CF_ERR_UNSUPPORTED;
    CF_TRY(check_dev_ptr(bufs_dev));
    CF_TRY(check_dev_ptr(dsts_dev));
    if (status_dev) CF_TRY(check_dev_ptr(status_dev, 4));
    cf::EncPublishArray src{bufs_dev, dsts_dev, ndst, ack_target};
    return dispatch<true>(src, d->bits, d->tokens, d->channels, d->tokens * (int64_t)n,
                          status_dev, (cudaStream_t)stream);
}

cf_status cf_decode_wait_batched(const cf_desc *d, int32_t n, const cf_dec_wait_buffer *bufs_dev,
                                 uint64_t ready_target, int32_t nack, uint64_t *const *acks_dev,
                                 int32_t *status_dev, void *stream) {
    cf::TraceRange trace_("cf_decode_wait_batched");
    CF_TRY(check_quant_desc(d));
    if (n < 0 || nack < 0 || nack > 64) return CF_ERR_INVALID_ARG;
    if (nack > 0) CF_TRY(check_dev_ptr(acks_dev, 8));
    if (status_dev) CF_TRY(check_dev_ptr(status_dev, 4));
    cudaStream_t st = (cudaStream_t)stream;
    if (n > 0 && d->tokens > 0) {
        if (!tma_applies(false, d->bits, d->channels)) return CF_ERR_UNSUPPORTED;
        CF_TRY(check_dev_ptr(bufs_dev));
        cf::DecWaitArray src{bufs_dev, ready_target};
        CF_TRY(dispatch<false>(src, d->bits, d->tokens, d->channels, d->tokens * (int64_t)n,
                               status_dev, st));
    }
    if (nack > 0) {
        cf::tma::exchange_ack_kernel<<<1, 64, 0, st>>>(acks_dev, nack);
        return launch_result();
    }
    return CF_OK;
}

int32_t cf_debug_bounds_checked(void) { return cf::kBoundsChecked ? 1 : 0; }

int32_t cf_debug_bounds_take(void) {
#ifdef CF_DEBUG_BOUNDS
    int32_t first = 0;
    for (int32_t v : {cf_bounds_take_api(), cf_bounds_take_lowrank(), cf_bounds_take_diag()})
        if (first == 0 && v != 0) first = v;
    return first;
#else
    return 0;
#endif
}

cf_status cf_set_quant_unit(int32_t kernel, int32_t channels) {
    if (kernel < 0 || kernel > 1) return CF_ERR_INVALID_ARG;
    if (channels != 0 && channels != 4 && channels != 8) return CF_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    g_unit[kernel] = channels;
    return CF_OK;
}

cf_status cf_set_quant_pipeline(int32_t kernel, int32_t pipeline, int32_t stages) {
    if (kernel < 0 || kernel > 1) return CF_ERR_INVALID_ARG;
    if (pipeline < 0 || pipeline > 1) return CF_ERR_INVALID_ARG;
    if (stages < 0 || stages == 1 || stages > 8) return CF_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    g_pipeline[kernel] = pipeline;
    g_stages[kernel] = stages;
    return CF_OK;
}

cf_status cf_set_launch_override(int32_t kernel, int32_t groups_per_thread, int32_t threads,
                                 int32_t blocks_per_sm) {
    if (kernel < 0 || kernel > 1) return CF_ERR_INVALID_ARG;
    if (groups_per_thread < 0 || groups_per_thread > kMaxGroupsPerThread) return CF_ERR_INVALID_ARG;
    if (threads < 0 || threads > kMaxThreads || threads % 32 != 0) return CF_ERR_INVALID_ARG;
    if (blocks_per_sm < 0 || blocks_per_sm > 64) return CF_ERR_INVALID_ARG;
    if ((groups_per_thread == 0) != (threads == 0)) return CF_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    g_override[kernel].gpt = groups_per_thread;
    g_override[kernel].threads = threads;
    g_override[kernel].blocks_per_sm = blocks_per_sm;
    return CF_OK;
}

}  // extern "C"
