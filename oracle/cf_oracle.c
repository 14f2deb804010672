/*
 * cf_oracle.c -- plain, slow, single-threaded CPU oracle for the quantize
 * mode of CompactFusion-style residual compression.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link or call
 * this file: only the tests, __graft_entry__.smoke() and bench.py's CPU
 * baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA library; the two meet only through the arrays a test hands both.
 *
 * Source of the method: the page "Accelerating Parallel Diffusion Model
 * Serving with Residual Compression" (atlas.scime.ai summary of the
 * CompactFusion paper).  Its "Approach" section fixes the method: send the
 * step-wise residual against the previously *reconstructed* activation,
 * keep a sender-side error-feedback buffer so compression error does not
 * accumulate, and compress with 1/2-bit quantisation or INT4 low-rank
 * factors.  Its "Measured effects" table names the 1-bit and 2-bit
 * variants and the 1-step warmup.  The page gives no equations; every
 * formula below is the plainest reading of those facts, listed with the
 * reason for each reading in the design notes:
 *
 *   init   (warmup step, sent uncompressed):
 *          recon = (float)x0 ; err = 0
 *   encode (every later step, per token row t, channels c = 0..C-1):
 *     1. v_c   = (float)x_t[c] - recon_s[c]              fp32, one rounding
 *        (this residual already carries the previous step's dropped part,
 *        because recon_s + err == x after every step; see the EF identity)
 *     2. scale b=1: s = (float)(sum_c |v_c| summed in fp64) / C   (mean-abs)
 *              b=2: A = max_c |v_c|                               (absmax)
 *     3. code  b=1: bit = [v_c >= 0]           deq = bit ? s : -s
 *              b=2: k = [v>=-A/2] + [v>=0] + [v>=A/2]  in 0..3
 *                   deq = lvl[k] * A, lvl = {-3/4, -1/4, 1/4, 3/4}
 *     4. err_c     = v_c - deq_c                          fp32
 *     5. recon_s_c = recon_s_c + deq_c                    fp32
 *     6. pack: element c of a row goes to word (c*b)/32, bits
 *        [(c*b)%32, +b), least significant first; unused tail bits are 0.
 *   decode: recon_r_c = recon_r_c + deq(code_c, scale)  -- the same
 *           expression as step 3/5, so recon_r tracks recon_s exactly.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math (no FMA contraction, SSE
 * float arithmetic, IEEE round-to-nearest-even).  See oracle/build.py.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
static float bf16_bits_to_float(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Number of uint32 code words per token row: ceil(C*b/32). */
int64_t orc_words_per_row(int64_t C, int32_t bits) {
    return (C * (int64_t)bits + 31) / 32;
}

/* Reconstruction level of a code.  b=1: +-s.  b=2: the centre of one of
 * four equal bins that split [-A, A]. */
static float dequant(int32_t bits, uint32_t code, float scale) {
    if (bits == 1) {
        return code ? scale : -scale;
    } else {
        static const float lvl[4] = {-0.75f, -0.25f, 0.25f, 0.75f};
        float d = lvl[code] * scale; /* one fp32 rounding */
        return d;
    }
}

/* Warmup step: the first step is sent uncompressed, so both ends start
 * from the exact activation and an empty error buffer. */
void orc_state_init(int64_t T, int64_t C, const uint16_t *x0, float *recon,
                    float *err) {
    for (int64_t i = 0; i < T * C; ++i) {
        recon[i] = bf16_bits_to_float(x0[i]);
        if (err) err[i] = 0.0f;
    }
}

/* Steps 2-6 for one token row: scale, codes, error feedback, mirror update
 * (when rr is not NULL) and packing, from the row's residual v. */
static void quantize_row(int64_t C, int32_t bits, const float *v, float *er, float *rr,
                         uint32_t *cw, int64_t W, float *scale_out) {
    /* 2. per-token scale */
    float scale;
    if (bits == 1) {
        double acc = 0.0;
        for (int64_t c = 0; c < C; ++c) acc += fabs((double)v[c]);
        float sum32 = (float)acc;
        scale = (C > 0) ? sum32 / (float)C : 0.0f;
    } else {
        float a = 0.0f;
        for (int64_t c = 0; c < C; ++c) {
            float m = fabsf(v[c]);
            if (m > a) a = m;
        }
        scale = a;
    }
    *scale_out = scale;

    /* 3-6. quantise, error feedback, mirror update, pack */
    for (int64_t w = 0; w < W; ++w) cw[w] = 0u;
    const float half = 0.5f * scale;
    for (int64_t c = 0; c < C; ++c) {
        uint32_t code;
        if (bits == 1) {
            code = (v[c] >= 0.0f) ? 1u : 0u;
        } else {
            code = (uint32_t)(v[c] >= -half) + (uint32_t)(v[c] >= 0.0f) +
                   (uint32_t)(v[c] >= half);
        }
        float d = dequant(bits, code, scale);
        er[c] = v[c] - d;
        if (rr) rr[c] = rr[c] + d;
        int64_t bitpos = c * (int64_t)bits;
        cw[bitpos / 32] |= code << (bitpos % 32);
    }
}

/* One compressed step of the sender for T token rows.  Returns 0, or -1 for
 * an unsupported bit width.  v_scratch must hold C floats. */
int orc_encode(int64_t T, int64_t C, int32_t bits, const uint16_t *x,
               float *recon_s, float *err, uint32_t *codes, float *scales,
               float *v_scratch) {
    if (bits != 1 && bits != 2) return -1;
    const int64_t W = orc_words_per_row(C, bits);
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t *xr = x + t * C;
        float *rr = recon_s + t * C;
        float *v = v_scratch;
        /* 1. residual against the sender's copy of the receiver state */
        for (int64_t c = 0; c < C; ++c) v[c] = bf16_bits_to_float(xr[c]) - rr[c];
        quantize_row(C, bits, v, err + t * C, rr, codes + t * W, W, scales + t);
    }
    return 0;
}

/* The same sender with its state kept as the previous activation x_prev
 * and the error buffer err (read, then overwritten) instead of a
 * reconstruction copy:
 *   1'. v_c = ((float)x_t[c] - (float)x_prev[c]) + err[c]    two roundings
 * then steps 2-6 as above, without the mirror update.  In exact arithmetic
 * v equals step 1's residual, because recon_s + err == x after every step
 * (the "Approach" section's error feedback, kept in another form). */
int orc_encode_delta(int64_t T, int64_t C, int32_t bits, const uint16_t *x,
                     const uint16_t *x_prev, float *err, uint32_t *codes, float *scales,
                     float *v_scratch) {
    if (bits != 1 && bits != 2) return -1;
    const int64_t W = orc_words_per_row(C, bits);
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t *xr = x + t * C;
        const uint16_t *pr = x_prev + t * C;
        float *er = err + t * C;
        float *v = v_scratch;
        for (int64_t c = 0; c < C; ++c) {
            float d = bf16_bits_to_float(xr[c]) - bf16_bits_to_float(pr[c]);
            v[c] = d + er[c];
        }
        quantize_row(C, bits, v, er, NULL, codes + t * W, W, scales + t);
    }
    return 0;
}

/* fp32 -> bf16 bit pattern, round to nearest, ties to even; NaN stays a
 * (quiet) NaN.  The attention layer that consumes the reconstruction reads
 * bf16, so a receiver that also emits bf16 writes this rounding of recon_r. */
uint16_t orc_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x0040u);
    const uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7fffu + lsb) >> 16);
}

/* Receiver that also emits the bf16 reconstruction: recon_r as orc_decode,
 * then out[i] = bf16_rne(recon_r[i]). */
int orc_decode_emit(int64_t T, int64_t C, int32_t bits, const uint32_t *codes,
                    const float *scales, float *recon_r, uint16_t *out);

/* Receiver: unpack, dequantise and accumulate into recon_r. */
int orc_decode(int64_t T, int64_t C, int32_t bits, const uint32_t *codes,
               const float *scales, float *recon_r) {
    if (bits != 1 && bits != 2) return -1;
    const int64_t W = orc_words_per_row(C, bits);
    const uint32_t mask = (1u << bits) - 1u;
    for (int64_t t = 0; t < T; ++t) {
        const uint32_t *cw = codes + t * W;
        float *rr = recon_r + t * C;
        for (int64_t c = 0; c < C; ++c) {
            int64_t bitpos = c * (int64_t)bits;
            uint32_t code = (cw[bitpos / 32] >> (bitpos % 32)) & mask;
            rr[c] = rr[c] + dequant(bits, code, scales[t]);
        }
    }
    return 0;
}

int orc_decode_emit(int64_t T, int64_t C, int32_t bits, const uint32_t *codes,
                    const float *scales, float *recon_r, uint16_t *out) {
    int rc = orc_decode(T, C, bits, codes, scales, recon_r);
    if (rc != 0) return rc;
    for (int64_t i = 0; i < T * C; ++i) out[i] = orc_f32_to_bf16(recon_r[i]);
    return 0;
}
