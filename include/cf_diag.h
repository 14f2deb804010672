/*
 * cf_diag.h -- tuning knobs, measurement hooks and a device self-test of
 * libcf.so, declared apart from the product API in cf.h.
 *
 * None of these has a counterpart in the paper ("Accelerating Parallel
 * Diffusion Model Serving with Residual Compression").  They exist for
 * launch-shape sweeps, cross-checks of the two low-rank engines, timing of
 * one kernel inside a whole call, and a check that the bounded device waits
 * end.  The setters change PROCESS-WIDE state without synchronisation
 * against calls in flight on other host threads: a setting made by one
 * caller changes the kernels every other caller in the process launches
 * next.  A product caller should not call them; the defaults are the
 * measured choices.  Same conventions as cf.h (caller-owned buffers,
 * asynchronous on `stream`, argument errors returned synchronously).
 */
#ifndef CF_DIAG_H
#define CF_DIAG_H

#include "cf.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Checks on the device that the bounded wait every TMA and tensor-core
 * pipeline uses ends.  One CTA waits, with at most `polls` polls (1 ..
 * 65536), on an mbarrier it has signalled itself and on one that nothing
 * signals, and writes out_dev[0..1] (device int32[2], 4-byte aligned):
 * [0] = 1 if the signalled wait completed; [1] = CF_ERR_TIMEOUT if the
 * unsignalled wait gave up (CF_OK otherwise).  The GPU never hangs or
 * faults: the unsignalled wait stops after `polls`. */
cf_status cf_diag_bounded_wait(int32_t polls, int32_t *out_dev, void *stream);

/* Engine of the low-rank dense products in this process: 0 (the default) =
 * tcgen05 tensor cores (the two subspace-iteration products with bf16
 * operands, and D = P^ Q^T in tf32 with a hi/lo split of the scaled P
 * factor, fp32 accumulation in TMEM), 1 = CUDA cores (same operands, fp32
 * FMA).  For cross-checks and diagnosis; both satisfy the same parity bar.
 * The sender and the receiver of a buffer must use the same engine: D is
 * bit-identical only within one engine.  Returns CF_ERR_INVALID_ARG for any
 * other value. */
cf_status cf_set_lowrank_engine(int32_t engine);

/* Buffers per pass of a batched low-rank encode in this process: 0 (the
 * default) launches every stage once for all buffers of the call; g > 0
 * runs the whole sender for g buffers at a time, so a group's bf16 residual
 * copies can stay in L2 between the four projection passes.  Results are
 * bit-identical either way.  Returns CF_ERR_INVALID_ARG outside 0..65535. */
cf_status cf_set_lowrank_group(int32_t buffers);

/* Measurement hook (no counterpart in the paper): CUDA events (cudaEvent_t,
 * passed as void*) that the low-rank calls record around their apply kernel
 * -- the kernel that forms D and updates the state -- so a caller can time
 * that one kernel inside a whole call.  When enc_start/enc_stop are non-null,
 * every later cf_lowrank_encode(_batched) records enc_start on its stream
 * immediately before the apply launch and enc_stop immediately after it;
 * dec_start/dec_stop likewise for cf_lowrank_decode(_batched).  Null pairs
 * (the default) record nothing.  Process-wide; the events stay the caller's
 * (create them before, destroy them after the calls that record them).  An
 * event that fails to record makes the call return CF_ERR_CUDA after its
 * launches.  Returns CF_ERR_INVALID_ARG if exactly one of a pair is null. */
cf_status cf_lowrank_set_apply_events(void *enc_start, void *enc_stop, void *dec_start,
                                      void *dec_stop);

/* Memory pipeline of the quantize-mode kernels in this process: kernel 0 =
 * encode, 1 = decode; pipeline 0 = register-resident rows (each thread
 * loads its channel groups straight into registers), 1 = TMA row staging
 * (a producer warp streams whole rows into a ring of `stages` shared-memory
 * slots with 1-D bulk copies; consumer warps compute from shared memory;
 * the default).  stages 0 = built-in choice, else 2..8.  Both give bit-identical results;
 * the TMA pipeline applies when C % 8 == 0 (decode also needs
 * ceil(C*bits/32) % 4 == 0) and otherwise the call uses pipeline 0.
 * Returns CF_ERR_INVALID_ARG for out-of-range values. */
cf_status cf_set_quant_pipeline(int32_t kernel, int32_t pipeline, int32_t stages);

/* A reference for the encode's byte mix (no counterpart in the paper): one
 * streaming pass over n elements (n % 8 == 0) that reads x (bf16 [n]) and r
 * (fp32 [n]) and writes a = (float)x - r and r = (float)x + r (fp32 [n]
 * each), i.e. the 6 bytes read and 8 written per element of the quantize
 * encode with none of its per-row work.  Timed next to the encode, it shows
 * what HBM gives a plain streaming kernel with that read/write mix, which
 * is less than it gives a copy's even split.  Device pointers, 16-byte aligned,
 * non-overlapping; overwrites r and a.  n < 0 or n % 8 != 0:
 * CF_ERR_INVALID_ARG. */
cf_status cf_diag_stream_mix(const uint16_t *x, float *r, float *a, int64_t n, void *stream);

/* The same byte mix moved by the quantize encode's own memory pipeline (no
 * counterpart in the paper): rows x rows of C channels, x bf16 [rows][C] and
 * r fp32 [rows][C] read, a = (float)x - r and r = (float)x + r written
 * (fp32 [rows][C] each).  A producer lane bulk-copies each row's x and r into
 * a ring of shared-memory slots; consumer warps compute from shared memory
 * and write a and r with the encode's store path: bulk = 0, per-thread
 * streaming stores (the encode's launch shape for long rows); bulk = 1,
 * two shared-memory output rows stored by the copy engine after each row's
 * barrier, 4 groups of 8 channels per thread and 2 slots (the standard
 * encode's shape where four CTAs fit on an SM).  It does none of the
 * encode's per-row work (scale reduction, quantisation, codes), so the
 * encode's time over this kernel's time is what that work costs.  Device
 * pointers, 16-byte aligned, non-overlapping; overwrites r and a.
 * status_dev: optional device int32 (4-byte aligned) that receives
 * CF_ERR_TIMEOUT if a bounded pipeline wait expires.  rows < 0, C < 8,
 * C % 8 != 0, C > 16384 or bulk not 0 or 1: CF_ERR_INVALID_ARG; rows needing
 * more than 480 consumer threads (C > 15360) or more shared memory than a
 * CTA may have (bulk: C > 8300): CF_ERR_UNSUPPORTED. */
cf_status cf_diag_stream_mix_tma(const uint16_t *x, float *r, float *a, int64_t rows, int64_t C, int32_t bulk,
                                 int32_t *status_dev, void *stream);

/* Bounds-checked debug build.  The library built with CF_DEBUG_BOUNDS
 * (libcf_debug.so) checks, at the global and shared-memory accesses of its
 * kernels, that the index arithmetic stays inside the array; a failed check
 * skips the access and records the first failure, and nothing traps.
 * cf_debug_bounds_checked: 1 in that build, 0 in the release build.
 * cf_debug_bounds_take: the first failure since the last call as
 * (tag << 16) | line, the tag a 15-bit FNV-1a hash of the source file's
 * base name, or 0 if none; clears it; synchronises the device.  Always 0 in
 * the release build.  -1 if reading the record failed. */
int32_t cf_debug_bounds_checked(void);
int32_t cf_debug_bounds_take(void);

/* Positive control of those checks (debug build only): writes
 * out_dev[i] = i for i < n (device int32[n], 4-byte aligned, 2 <= n <=
 * 2^20) through a check that declares an extent of n / 2, so the upper
 * half is skipped and a failure in diag.cu is recorded.  Every write stays
 * inside out_dev.  Release build: CF_ERR_UNSUPPORTED, nothing launched. */
cf_status cf_diag_bounds_selftest(int32_t *out_dev, int32_t n, void *stream);

/* Channels per thread unit of the TMA-staged quantize kernels in this
 * process: kernel 0 = encode, 1 = decode; channels 4 or 8, or 0 for the
 * built-in choice (measured per bit width and row length).  Both give
 * bit-identical results.  Returns CF_ERR_INVALID_ARG for other values. */
cf_status cf_set_quant_unit(int32_t kernel, int32_t channels);

/* Launch-shape override for tuning sweeps: kernel 0 = encode, 1 = decode;
 * groups_per_thread in 1..4 (8 channels per group), threads a multiple of
 * 32 in 32..512, or 0 to restore the built-in choice; blocks_per_sm caps
 * the persistent grid (0 = occupancy limit).  Affects later launches in
 * this process only.  Returns CF_ERR_INVALID_ARG for out-of-range values. */
cf_status cf_set_launch_override(int32_t kernel, int32_t groups_per_thread,
                                 int32_t threads, int32_t blocks_per_sm);

#ifdef __cplusplus
}
#endif

#endif /* CF_DIAG_H */
