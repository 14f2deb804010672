/*
 * cf.h -- C ABI of libcf.so: B200 (sm_100a) CompactFusion-style residual
 * compression of exchanged activations.
 *
 * Method: "Accelerating Parallel Diffusion Model Serving with Residual
 * Compression" (atlas.scime.ai summary of the CompactFusion paper).  Per
 * the page's "Approach": the sender transmits the step-wise residual against
 * the previously reconstructed activation instead of the activation, keeps
 * a sender-side error-feedback buffer so compression error does not build
 * up, and compresses either to 1/2-bit codes or to low-rank factors
 * quantised to INT4.  The receiver decodes and accumulates into its own
 * reconstruction.  The "Measured effects" table names the 1-bit and 2-bit
 * variants, the 1-step warmup and subspace iteration; "Key results" gives
 * about 100x compression at rank 32 with INT4 factors.
 *
 * Conventions for every entry point
 *  - Ownership: the caller allocates and owns every buffer.  The library
 *    allocates nothing, frees nothing and never synchronises the stream
 *    (except cf_lowrank_status, which says so).
 *  - All device work is enqueued asynchronously on `stream`, a
 *    cudaStream_t passed as void* (NULL = the legacy default stream).
 *  - Pointers named *_dev or documented as device pointers must be device
 *    (or managed) memory of the current device.  Single-buffer calls check
 *    this with cudaPointerGetAttributes and return CF_ERR_INVALID_ARG for
 *    host memory instead of launching.
 *  - Every device pointer must be 16-byte aligned (CF_ERR_ALIGNMENT), except
 *    the scale arrays (per-token in the quantize mode, so [n][T] packed
 *    scales of any T are valid; per-column in the low-rank mode) and the
 *    low-rank start block omega, which need 4 bytes, and the low-rank INT4
 *    code arrays, which need 1 byte.
 *  - Argument errors are reported synchronously and launch nothing.  A
 *    failed launch returns CF_ERR_CUDA.  Numeric trouble found on the
 *    device (low-rank mode) is written to a status word in the workspace.
 *  - Layouts are row-major and dense: an activation is [tokens][channels].
 *  - bf16 values are passed as their 16-bit patterns (the upper half of an
 *    IEEE binary32).
 *  - Inputs must be finite; NaN/Inf give unspecified codes.
 *
 * Quantize-mode arithmetic (fp32 IEEE round-to-nearest-even, no fused
 * multiply-add anywhere on the state path), per token row:
 *   v      = (float)x - recon_s
 *   1 bit: s = (float)(sum |v| accumulated in fp64) / C ;  code = [v >= 0] ;
 *          deq = code ? s : -s
 *   2 bit: A = max |v| ; code = [v >= -A/2] + [v >= 0] + [v >= A/2] ;
 *          deq = lvl[code] * A with lvl = {-3/4, -1/4, 1/4, 3/4}
 *   err    = v - deq ;  recon_s = recon_s + deq
 *   decode: recon_r = recon_r + deq (same expression, so recon_r == recon_s
 *           bit for bit when both started from the same cf_state_init)
 * Code layout: row t of the codes is ceil(C*bits/32) uint32 words; element
 * c sits in word (c*bits)/32 at bit (c*bits)%32, least significant first;
 * unused tail bits are zero.  One fp32 scale per token (s or A).
 */
#ifndef CF_H
#define CF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CF_ABI_VERSION 1

typedef enum cf_status {
    CF_OK = 0,
    CF_ERR_INVALID_ARG = 1,  /* null/host pointer, negative size, bad field */
    CF_ERR_ALIGNMENT = 2,    /* a device pointer is not aligned as required  */
    CF_ERR_UNSUPPORTED = 3,  /* bits/rank/scale_kind outside what is built  */
    CF_ERR_WORKSPACE = 4,    /* low-rank workspace too small                 */
    CF_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed         */
    CF_ERR_NUMERIC = 6,      /* low-rank: Gram matrix not positive definite */
    CF_ERR_TIMEOUT = 7       /* a bounded device wait (mbarrier of a TMA or
                                tensor-core pipeline) gave up; recorded in
                                the status word (batched status_dev or the
                                low-rank workspace), never returned by a
                                call                                         */
} cf_status;

/* Problem description, as the pages state the problem: one exchanged
 * activation buffer of `tokens` x `channels`, compressed at `bits` (quantize
 * mode) or at `rank` with `iters` subspace iterations (low-rank mode). */
typedef struct cf_desc {
    int64_t tokens;      /* T >= 0 (T == 0 is a no-op)                     */
    int64_t channels;    /* C >= 1; quantize mode C <= 16384                */
    int32_t bits;        /* quantize mode: 1 or 2; low-rank mode: 0         */
    int32_t rank;        /* low-rank mode: 1..64, <= min(T, C); else 0      */
    int32_t iters;       /* low-rank mode: 1..16; else 0                    */
    int32_t scale_kind;  /* 0 = 1-bit mean-abs / 2-bit absmax (only value)  */
} cf_desc;

/* One sender buffer set for the batched encode (all device pointers). */
typedef struct cf_enc_buffer {
    const uint16_t *x;   /* bf16 [T][C], this step's activation             */
    float *recon_s;      /* fp32 [T][C], sender copy of the reconstruction  */
    float *err;          /* fp32 [T][C], error-feedback buffer (written)    */
    uint32_t *codes;     /* uint32 [T][ceil(C*bits/32)] (written)           */
    float *scales;       /* fp32 [T] (written)                              */
} cf_enc_buffer;

/* One receiver buffer set for the batched decode (all device pointers). */
typedef struct cf_dec_buffer {
    const uint32_t *codes;
    const float *scales;
    float *recon_r;      /* fp32 [T][C], receiver reconstruction (updated)  */
} cf_dec_buffer;

/* One receiver buffer set for the batched emitting decode. */
typedef struct cf_dec_emit_buffer {
    const uint32_t *codes;
    const float *scales;
    float *recon_r;      /* fp32 [T][C], receiver reconstruction (updated)  */
    uint16_t *out;       /* bf16 [T][C], written: bf16_rne(new recon_r)     */
} cf_dec_emit_buffer;

/* Streams and graphs: every call except cf_lowrank_status only enqueues
 * work on the given stream (no allocation, no synchronisation, no host read
 * of device memory), so a step of batched calls can be captured into a CUDA
 * graph and replayed; the host-side argument checks run at capture time.
 * cf_lowrank_encode_noalloc's first call on a device must precede capture. */

/* Tuning knobs, measurement hooks and the bounded-wait self-test are
 * declared apart, in cf_diag.h: product callers need none of them. */

/* Human-readable name of a status code (static string, never NULL). */
const char *cf_status_string(cf_status s);

/* CF_ABI_VERSION of the loaded library. */
int32_t cf_abi_version(void);

/* uint32 code words per token row: ceil(channels * bits / 32); 0 for an
 * invalid descriptor.  Cite: the 1- and 2-bit variants of the "Measured
 * effects" table (b bits per element); the word layout is this library's
 * (least significant bit first, see above). */
int64_t cf_codes_words_per_row(const cf_desc *d);

/* Bytes on the wire for one buffer: codes + scales (quantize mode) or INT4
 * factors + scales (low-rank mode); 0 for an invalid descriptor.  Cite:
 * "Key results" (rank 32 with INT4 factors compresses about 100x: at
 * 1024 x 3072 this size gives 95.6x) and the 1/2-bit rows of "Measured
 * effects" (16/b x before the per-token scales). */
int64_t cf_payload_bytes(const cf_desc *d);

/* Warmup step ("Measured effects": the first step is sent uncompressed).
 * recon[i] = (float)x0[i] when recon != NULL; err[i] = 0 when err != NULL
 * (at least one of them).  Call it for the sender (with err) and for the
 * receiver (err = NULL) on the same x0; the delta-state sender below keeps
 * no reconstruction and calls it with recon = NULL.
 * x0: bf16 [T][C] device; recon, err: fp32 [T][C] device. */
cf_status cf_state_init(const cf_desc *d, const uint16_t *x0, float *recon,
                        float *err, void *stream);

/* Sender, quantize mode, one buffer: residual with error feedback, per-token
 * scale, quantise, pack, error update and mirror update in one pass.
 * Cite: "Approach" (transmit the residual against the previous
 * reconstruction; keep a sender-side error-feedback buffer) and the
 * Compact-1bit / Compact-2bit rows of the "Measured effects" table.
 * x: bf16 [T][C]; recon_s: fp32 [T][C] read and updated in place;
 * err: fp32 [T][C] written; codes: uint32 [T][words_per_row] written;
 * scales: fp32 [T] written.  All device pointers, non-overlapping.
 * Errors: CF_ERR_INVALID_ARG (null or host pointer, T < 0, C < 1, rank or
 * iters set), CF_ERR_UNSUPPORTED (bits not 1 or 2, C > 16384, scale_kind
 * not 0), CF_ERR_ALIGNMENT, CF_ERR_CUDA; nothing is launched on an error. */
cf_status cf_encode(const cf_desc *d, const uint16_t *x, float *recon_s,
                    float *err, uint32_t *codes, float *scales, void *stream);

/* Receiver, quantize mode, one buffer: unpack, dequantise, accumulate.
 * Cite: "Approach" (the receiver adds the decoded residual to its own
 * reconstruction of the previous step).
 * codes, scales as written by cf_encode; recon_r: fp32 [T][C] updated.
 * Never reads sender state.  Errors as cf_encode. */
cf_status cf_decode(const cf_desc *d, const uint32_t *codes,
                    const float *scales, float *recon_r, void *stream);

/* Receiver that also emits the reconstruction in bf16, the dtype the
 * attention layer consumes (the decoded K/V go straight to attention), in
 * the same pass: recon_r is updated exactly as by cf_decode and
 * out[t][c] = bf16 round-to-nearest-even of the new recon_r[t][c].
 * out: bf16 [T][C] device, written. */
cf_status cf_decode_emit(const cf_desc *d, const uint32_t *codes, const float *scales,
                         float *recon_r, uint16_t *out, void *stream);

/* Batched forms: `n` buffers of the same shape in ONE launch, with the same
 * per-buffer semantics as cf_encode / cf_decode (cite: as those; a diffusion
 * transformer exchanges the K and V buffers of every layer at every step,
 * "Approach" and the sequence-parallel setting of "Key results").  n < 0 is
 * CF_ERR_INVALID_ARG; n == 0 launches nothing.  `bufs_dev` is a DEVICE
 * array of n descriptors (it must stay valid until the work completes).
 * Pointers inside it are checked on the device: a buffer with a null or
 * misaligned pointer is skipped and, when `status_dev` (device int32) is
 * not NULL, the first such error code is stored there with atomicCAS over
 * an initial CF_OK (the caller zeroes it).  Pointers inside must be device
 * memory: the host cannot check them. */
cf_status cf_encode_batched(const cf_desc *d, int32_t n,
                            const cf_enc_buffer *bufs_dev, int32_t *status_dev,
                            void *stream);
cf_status cf_decode_batched(const cf_desc *d, int32_t n,
                            const cf_dec_buffer *bufs_dev, int32_t *status_dev,
                            void *stream);
cf_status cf_decode_emit_batched(const cf_desc *d, int32_t n,
                                 const cf_dec_emit_buffer *bufs_dev,
                                 int32_t *status_dev, void *stream);

/* ------------------------------------------------------------------------
 * Publishing encode and waiting decode: the sequence-parallel exchange with
 * the payload transfer fused into the codec kernels.  Cite: "Approach"
 * (senders transmit the compressed residual; every receiver keeps its own
 * reconstruction), the 6.7x communication-bound speed-up of "Key results"
 * (the transfer is what the compression shortens) and the ring-attention row
 * of "Measured effects" (each rank's K/V reach every other rank).
 *
 * The encode writes each row's codes and scale straight into the payload
 * slot that every receiver keeps for this sender -- plain stores, 16 bytes
 * wide where the code row allows it, to memory that may be another GPU's
 * (peer access) or this GPU's own -- instead of into a local payload that a
 * collective then copies.  Synchronisation is by monotonic 64-bit counters
 * in the receivers' memory:
 *  - ready: rows published.  After its last row every CTA of the encode
 *    adds the rows it walked to each destination's ready counter with a
 *    system-scope release (fence, then atomic add).  For step e (1, 2, ...)
 *    of a sender publishing R = n * T rows per step, the counter reaches
 *    e * R when step e is complete, since a sender's steps are ordered.
 *  - ack: steps decoded.  After its decode the receiver adds 1 to an ack
 *    counter per sender (in that sender's memory).  With two payload slots
 *    per (receiver, sender) used alternately (step e writes slot e % 2), the
 *    sender at step e waits, before its first store to a destination, until
 *    that destination's ack is >= e - 2 (ack_target), i.e. until the slot's
 *    previous contents were decoded.
 * Every wait is bounded (about a second): on expiry the CTA records
 * CF_ERR_TIMEOUT in status_dev and stops, and nothing hangs.  A sender that
 * stopped publishes nothing, so its receivers time out in turn.
 * Requirements: C % 8 == 0; the decode also ceil(C*bits/32) % 4 == 0 (the
 * TMA row pipeline); otherwise CF_ERR_UNSUPPORTED.  No TMA load ever reads
 * another GPU's memory: the sender's loads are local, the receiver's bulk
 * copies read its own memory.  Both calls only enqueue work, so they can be
 * stream-captured; the counter targets are arguments of the captured
 * launches, so a captured step waits for the same counts on every replay
 * (capture per step, or call them eagerly). */

/* One destination of a publishing encode (all device pointers; the first
 * two may be another GPU's memory mapped for peer access). */
typedef struct cf_publish_dst {
    uint8_t *payload;        /* this sender's payload slot at the receiver, 16-byte aligned */
    uint64_t *ready;         /* the receiver's ready counter for this sender, 8-byte aligned */
    const uint64_t *ack;     /* this sender's ack counter for that receiver, or NULL: no wait */
} cf_publish_dst;

/* One buffer of a publishing encode: the sender state as in cf_enc_buffer,
 * and where the buffer's codes ([T][ceil(C*bits/32)] uint32) and scales
 * ([T] fp32) sit in every destination's payload slot. */
typedef struct cf_enc_publish_buffer {
    const uint16_t *x;       /* bf16 [T][C], this step's activation             */
    float *recon_s;          /* fp32 [T][C], updated                            */
    float *err;              /* fp32 [T][C], written                            */
    int64_t codes_offset;    /* bytes from a slot's base, multiple of 16        */
    int64_t scales_offset;   /* bytes from a slot's base, multiple of 4         */
} cf_enc_publish_buffer;

/* Sender: cf_encode_batched's arithmetic for n buffers, with codes and
 * scales stored into each of the ndst (1..8) destinations instead of local
 * arrays, the ack wait before the stores and the ready publication after
 * them.  bufs_dev: DEVICE array of n cf_enc_publish_buffer; dsts_dev: DEVICE
 * array of ndst cf_publish_dst; both valid until the work completes.
 * ack_target: see above (0 = no wait).  Buffer pointers are checked on the
 * device as in cf_encode_batched (a bad buffer is skipped, its rows still
 * count as published); a destination with a null or misaligned pointer
 * stops every CTA before any store with CF_ERR_INVALID_ARG / ALIGNMENT in
 * status_dev (device int32, zeroed by the caller; may be NULL). */
cf_status cf_encode_publish_batched(const cf_desc *d, int32_t n,
                                    const cf_enc_publish_buffer *bufs_dev, int32_t ndst,
                                    const cf_publish_dst *dsts_dev, uint64_t ack_target,
                                    int32_t *status_dev, void *stream);

/* One buffer of a waiting decode: cf_dec_buffer plus the ready counter of
 * the sender whose payload holds this buffer's codes and scales. */
typedef struct cf_dec_wait_buffer {
    const uint32_t *codes;
    const float *scales;
    float *recon_r;          /* fp32 [T][C], updated                            */
    const uint64_t *ready;   /* 8-byte aligned, in this receiver's memory       */
} cf_dec_wait_buffer;

/* Receiver: cf_decode_batched for n buffers, where a CTA reads a buffer's
 * codes only after that buffer's ready counter is >= ready_target (the
 * sender's step e: e * rows published per step).  Then adds 1 to each of the
 * nack (0..64) counters in acks_dev (DEVICE array of uint64_t*, each 8-byte
 * aligned, possibly another GPU's memory), with a system-scope release after
 * the decode.  A wait that expires records CF_ERR_TIMEOUT in status_dev,
 * the CTA stops, and the acks are still sent (so that a sender does not
 * block on a receiver that gave up). */
cf_status cf_decode_wait_batched(const cf_desc *d, int32_t n,
                                 const cf_dec_wait_buffer *bufs_dev, uint64_t ready_target,
                                 int32_t nack, uint64_t *const *acks_dev,
                                 int32_t *status_dev, void *stream);

/* ------------------------------------------------------------------------
 * Delta-state sender: the same residual-with-error-feedback ("Approach") kept
 * as the previous activation and the error buffer instead of a sender copy
 * of the reconstruction.  With x_prev the previous step's activation (bf16,
 * kept by the caller: x_0 after the warmup step) and err the error buffer:
 *   v = ((float)x - (float)x_prev) + err       two fp32 roundings
 * then the per-token scale, codes, packing and err = v - deq exactly as in
 * cf_encode; the receiver is unchanged (cf_decode).  In exact arithmetic v
 * equals cf_encode's x - recon_s (recon_s + err == x after every step), so
 * the two senders agree up to fp32 rounding, and at the first compressed
 * step after the warmup they are bit-identical.  It moves 12 bytes per
 * element instead of 14 (recon_s is neither read nor written).  Warmup:
 * cf_state_init(d, x0, NULL, err, stream), x_prev = x0.  Alignment as
 * cf_encode (x_prev 16 bytes). */
cf_status cf_encode_delta(const cf_desc *d, const uint16_t *x, const uint16_t *x_prev,
                          float *err, uint32_t *codes, float *scales, void *stream);

/* One sender buffer set of the batched delta-state encode. */
typedef struct cf_enc_delta_buffer {
    const uint16_t *x;       /* bf16 [T][C], this step's activation             */
    const uint16_t *x_prev;  /* bf16 [T][C], the previous step's activation     */
    float *err;              /* fp32 [T][C], error-feedback buffer (updated)    */
    uint32_t *codes;         /* uint32 [T][ceil(C*bits/32)] (written)           */
    float *scales;           /* fp32 [T] (written)                              */
} cf_enc_delta_buffer;

/* Batched delta-state encode: rules as cf_encode_batched. */
cf_status cf_encode_delta_batched(const cf_desc *d, int32_t n,
                                  const cf_enc_delta_buffer *bufs_dev,
                                  int32_t *status_dev, void *stream);

/* ------------------------------------------------------------------------
 * Low-rank mode ("Approach", "Key results", "Builds on": PowerSGD-style
 * subspace iteration, INT4 factors).  With V = (float)x - recon_s:
 *   Q = omega ; repeat iters: Y = V Q ; P = orth(Y) ; Q = V^T P
 *   INT4 per column of P [T][r] and Q [C][r]: s_j = max|col_j| / 7,
 *   q = clamp(rint(col / s_j), -7, 7)
 *   D = (q_P s_P)(q_Q s_Q)^T ; err = V - D ; recon_s = recon_s + D
 * orth() is CholeskyQR with an fp64 Gram matrix: P = Y R^-1 with R the
 * Cholesky factor of Y^T Y, i.e. the unique thin QR with diag(R) > 0.
 * Factor layout: row-major [rows][ceil(r/2)] bytes, two's-complement
 * nibbles, even column in the low nibble.  Scales: fp32 [r] per factor.
 * ---------------------------------------------------------------------- */

/* Device workspace bytes cf_lowrank_encode needs for this descriptor (the
 * subspace-iteration intermediates of "Approach" / "Builds on": the bf16
 * residual copy, Y, P, Q, the Gram partials); 0 for an invalid descriptor. */
int64_t cf_lowrank_workspace_bytes(const cf_desc *d);

/* Bytes of one packed INT4 factor with `rows` rows at rank `rank`:
 * rows * ceil(rank / 2) ("Key results": INT4 factors); 0 if rows < 0 or
 * rank < 1. */
int64_t cf_lowrank_factor_bytes(int64_t rows, int32_t rank);

/* Sender, low-rank mode.  Alignment: x, recon_s, err 16 bytes; omega and the
 * scales 4 bytes; the code arrays 1 byte.
 * x: bf16 [T][C]; recon_s: fp32 [T][C] updated;
 * err: fp32 [T][C] written; omega: fp32 [C][r] Gaussian start block chosen
 * by the caller, or NULL for a warm start ("Builds on": PowerSGD reuses the
 * previous step's factor as the next start block): the iteration then starts
 * from the Q that the previous encode left in this workspace, rounded to
 * bf16 as every Q operand is.  A warm start needs an earlier encode of the
 * same shape and rank on the same workspace (slice); without one the buffer
 * is skipped and CF_ERR_INVALID_ARG is recorded in its status word.
 * p_codes: [T][ceil(r/2)] bytes, p_scales: fp32 [r];
 * q_codes: [C][ceil(r/2)] bytes, q_scales: fp32 [r] (all written);
 * workspace: device, >= cf_lowrank_workspace_bytes(d) bytes, 256-byte
 * aligned, contents need not be initialised.  If the fp64 Gram matrix of an
 * iteration is not positive definite (Y rank deficient, e.g. a zero
 * residual) the affected columns of P are set to zero, which still yields a
 * valid (lower-rank) D, and CF_ERR_NUMERIC is recorded in the workspace
 * status word (see cf_lowrank_status). */
cf_status cf_lowrank_encode(const cf_desc *d, const uint16_t *x, float *recon_s,
                            float *err, const float *omega, uint8_t *p_codes,
                            float *p_scales, uint8_t *q_codes, float *q_scales,
                            void *workspace, size_t workspace_bytes,
                            void *stream);

/* One buffer of a batched low-rank encode (device pointers; rules as for
 * cf_lowrank_encode). */
typedef struct cf_lowrank_buffer {
    const uint16_t *x;       /* bf16 [T][C]                                  */
    float *recon_s;          /* fp32 [T][C], updated                         */
    float *err;              /* fp32 [T][C], written                         */
    const float *omega;      /* fp32 [C][r] start block, or NULL: warm start */
    uint8_t *p_codes;        /* [T][ceil(r/2)], written                      */
    float *p_scales;         /* fp32 [r], written                            */
    uint8_t *q_codes;        /* [C][ceil(r/2)], written                      */
    float *q_scales;         /* fp32 [r], written                            */
} cf_lowrank_buffer;

/* One buffer of a batched low-rank decode. */
typedef struct cf_lowrank_dec_buffer {
    const uint8_t *p_codes;
    const float *p_scales;
    const uint8_t *q_codes;
    const float *q_scales;
    float *recon_r;          /* fp32 [T][C], updated                         */
} cf_lowrank_dec_buffer;

/* Batched low-rank sender: `n` buffers of the same shape, every stage of the
 * method launched once for all of them (the latency-bound small steps of
 * different buffers then overlap).  bufs_dev: DEVICE array of n
 * cf_lowrank_buffer, valid until the work completes.  workspace: device,
 * 256-byte aligned, >= n * cf_lowrank_workspace_bytes(d) bytes; buffer b
 * uses the slice at b * cf_lowrank_workspace_bytes(d), and its status word
 * is read with cf_lowrank_status(workspace + that offset, stream).  Pointers
 * inside bufs_dev are checked on the device: a buffer with a null pointer or
 * a misaligned x/recon_s/err (16 B) or omega/scales (4 B) is skipped and
 * its status word gets CF_ERR_INVALID_ARG / CF_ERR_ALIGNMENT. */
cf_status cf_lowrank_encode_batched(const cf_desc *d, int32_t n,
                                    const cf_lowrank_buffer *bufs_dev, void *workspace,
                                    size_t workspace_bytes, void *stream);

/* Batched low-rank receiver: recon_r += D for `n` buffers in one launch.
 * bufs_dev: DEVICE array of n cf_lowrank_dec_buffer.  A buffer with a null
 * pointer or misaligned recon_r (16 B) / scales (4 B) is skipped and, when
 * status_dev (device int32, zeroed by the caller) is given, the first such
 * error is stored there. */
cf_status cf_lowrank_decode_batched(const cf_desc *d, int32_t n,
                                    const cf_lowrank_dec_buffer *bufs_dev,
                                    int32_t *status_dev, void *stream);

/* Receiver, low-rank mode: recon_r += D, with D formed from the payload by
 * the same device routine the sender uses (so recon_r == recon_s bit for
 * bit).  recon_r: fp32 [T][C] device, updated. */
cf_status cf_lowrank_decode(const cf_desc *d, const uint8_t *p_codes,
                            const float *p_scales, const uint8_t *q_codes,
                            const float *q_scales, float *recon_r,
                            void *stream);

/* Size of the device scratch array behind cf_lowrank_encode_noalloc: 40 MiB,
 * enough for 4096 tokens x 3072 channels at rank 32 (about 33.5 MB). */
#define CF_LOWRANK_NOALLOC_SCRATCH_BYTES (40ull << 20)

/* Low-rank sender for callers that cannot allocate device memory.  The
 * paper has no counterpart to this call; it exists for callers such as a
 * plug-in running inside a framework that owns all device memory and gives
 * it no allocator, or a serving loop that must not call cudaMalloc mid-step
 * (the call can synchronise the device).  Same arguments and results as
 * cf_lowrank_encode without the workspace pair: the scratch lives in one
 * file-scope device array of CF_LOWRANK_NOALLOC_SCRATCH_BYTES bytes that
 * every GPU using the library holds until the process exits.  The call
 * allocates nothing and calls no allocating routine; inputs and outputs are
 * still the caller's.
 *  - Problems whose cf_lowrank_workspace_bytes exceeds the array return
 *    CF_ERR_WORKSPACE without launching anything.
 *  - The first call on a device looks up the array's device address on the
 *    current device (cudaGetSymbolAddress) and caches it; make that first
 *    call before any stream capture on that device.  The cached address
 *    belongs to the device's primary context: after cudaDeviceReset (or any
 *    reset of the primary context) it is stale and this library does not
 *    notice, so do not call this entry point again in a process that has
 *    reset the device.
 *  - Every call on a device shares the one array, which keeps the previous
 *    call's contents (the implementation clears what must start at zero).
 *    Calls whose work overlaps on the GPU -- different streams without
 *    ordering between them -- race on the array and corrupt each other.
 *  - The status word is in the array as well: cf_lowrank_status cannot
 *    reach it; CF_ERR_NUMERIC cases still yield a valid, lower-rank D.
 *  - omega must not be NULL (a warm start would read whichever buffer the
 *    shared array saw last): CF_ERR_INVALID_ARG. */
cf_status cf_lowrank_encode_noalloc(const cf_desc *d, const uint16_t *x, float *recon_s,
                                    float *err, const float *omega, uint8_t *p_codes,
                                    float *p_scales, uint8_t *q_codes, float *q_scales,
                                    void *stream);

/* Synchronises `stream`, then returns the status word the last
 * cf_lowrank_encode on `workspace` recorded (CF_OK or CF_ERR_NUMERIC) and
 * clears it.  Returns CF_ERR_CUDA if the copy or the sync fails. */
cf_status cf_lowrank_status(void *workspace, void *stream);

/* Non-blocking form for a batch: enqueues on `stream` one strided
 * device-to-host copy of the status words of n workspace slices -- slice b
 * at workspace + b * slice_bytes, slice_bytes normally
 * cf_lowrank_workspace_bytes(d) -- into host_status[0..n-1] (int32), and
 * returns without waiting.  The words are valid once the stream has passed
 * this point (record an event after the call and wait on it, or read them
 * after a later synchronisation), and they hold what the encodes enqueued
 * before this call recorded.  Nothing is cleared: every encode resets its
 * slice's word when it starts.  host_status must be page-locked host memory
 * (cudaHostAlloc / cudaHostRegister), so that the copy is asynchronous;
 * pageable memory is CF_ERR_INVALID_ARG.  workspace: device, 256-byte
 * aligned; slice_bytes a positive multiple of 256 (CF_ERR_ALIGNMENT
 * otherwise); n >= 0 (0 enqueues nothing).  Returns CF_ERR_CUDA if the copy
 * cannot be enqueued.  Usable inside stream capture: the copy becomes a
 * graph node. */
cf_status cf_lowrank_status_async(const void *workspace, int64_t slice_bytes, int32_t n,
                                  int32_t *host_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* CF_H */
