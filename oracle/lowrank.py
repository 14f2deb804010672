"""Plain fp64 CPU oracle for the low-rank mode (subspace iteration + INT4).

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and bench.py's CPU-baseline leg, never by the product package.  It shares no
code with the CUDA library.

Source: the page "Accelerating Parallel Diffusion Model Serving with Residual
Compression" (atlas.scime.ai summary of CompactFusion).
  * "Approach": the residual against the previous reconstruction, with
    sender-side error feedback, may be compressed by a low-rank
    factorisation whose factors are quantised to INT4.
  * "Key results": rank 32 with INT4 factors gives about 100x compression.
  * "Measured effects" table: the factorisation is subspace iteration;
    going from 2 to 10 iterations at rank 8 changed FID only slightly.
  * "Builds on": subspace iteration in the style of PowerSGD gradient
    compression.

Steps, in the order the pages give them (readings, not printed formulas):
  V = (float)x_t - recon_s                 fp32 residual, one rounding
  Q = Omega                                caller-supplied Gaussian [C, r]
  repeat iters times:  Y = V Q ;  P = orth(Y) ;  Q = V^T P
      (fp64 products; orth = Householder thin QR with diag(R) > 0)
  INT4 per column j of P and of Q:
      s_j = fp32(max_i |col_j| / 7);  q = clamp(rint(col / s_j), -7, 7)
      (rint rounds half to even; s_j == 0 gives q == 0)
  D = (q_P s_P)(q_Q s_Q)^T                 fp64 product, rounded once to fp32
  err = V - D ; recon_s = recon_s + D      fp32
  receiver: recon_r = recon_r + D          the same D from the payload
Packing: INT4 two's complement, two per byte, the even column in the low
nibble, one row of ceil(r/2) bytes per factor row.

Parity pins live in tests/test_oracle_lowrank.py (Eckart-Young optimum from
LAPACK SVD, exact recovery at rank <= r, orthonormality, INT4 bounds, the
compression-ratio closed form; reconstruct: hand-worked payloads in
tests/golden/lowrank_reconstruct_cases.json and the elementwise INT4
rounding bound on |D - P Q^T|).
"""
from __future__ import annotations

import numpy as np

INT4_MAX = 7


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def residual(x_bits: np.ndarray, recon_s: np.ndarray) -> np.ndarray:
    """V = (float)x - recon_s, in fp32 (one IEEE rounding per element)."""
    return bf16_bits_to_f32(x_bits) - recon_s.astype(np.float32)


def orth(y: np.ndarray) -> np.ndarray:
    """Orthonormal basis of the columns of ``y`` by Householder QR (LAPACK
    geqrf through numpy), column signs fixed so that diag(R) > 0.  With a
    positive diagonal the thin QR factorisation is unique, so any other
    correct QR of the same Y (CholeskyQR, Gram-Schmidt) gives the same P."""
    q, r = np.linalg.qr(y, mode="reduced")
    d = np.sign(np.diag(r))
    d[d == 0] = 1.0
    return q * d[None, :]


def subspace_iteration(v: np.ndarray, omega: np.ndarray, iters: int):
    """Rank-r factors of ``v`` by subspace iteration from ``omega``.

    Returns (P, Q) in fp64 with P orthonormal [T, r] and Q = V^T P [C, r],
    so that V ~ P Q^T.  ``iters`` >= 1 rounds of Y = V Q, P = orth(Y),
    Q = V^T P, starting from Q = omega."""
    v64 = np.asarray(v, dtype=np.float64)
    q = np.asarray(omega, dtype=np.float64)
    p = None
    for _ in range(iters):
        y = v64 @ q
        p = orth(y)
        q = v64.T @ p
    return p, q


def int4_quantize_columns(f: np.ndarray):
    """Per-column symmetric INT4: s_j = fp32(max|f_j| / 7), codes in [-7, 7].

    Returns (codes int8 [rows, r], scales float32 [r])."""
    f = np.asarray(f, dtype=np.float64)
    amax = np.max(np.abs(f), axis=0) if f.shape[0] else np.zeros(f.shape[1])
    s = (amax / INT4_MAX).astype(np.float32)
    s64 = s.astype(np.float64)
    safe = np.where(s64 > 0, s64, 1.0)
    q = np.rint(f / safe[None, :])
    q = np.clip(q, -INT4_MAX, INT4_MAX)
    q[:, s64 == 0] = 0
    return q.astype(np.int8), s


def int4_pack(codes: np.ndarray) -> np.ndarray:
    """Two's-complement nibbles, two per byte, even column in the low nibble.
    A row of r codes becomes ceil(r/2) bytes; an odd tail nibble is 0."""
    rows, r = codes.shape
    nb = (r + 1) // 2
    nib = np.zeros((rows, 2 * nb), dtype=np.uint8)
    nib[:, :r] = codes.astype(np.int16).astype(np.uint8) & 0xF
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def int4_unpack(packed: np.ndarray, r: int) -> np.ndarray:
    """Inverse of int4_pack: bytes [rows, ceil(r/2)] -> int8 codes [rows, r]."""
    lo = (packed & 0xF).astype(np.int16)
    hi = (packed >> 4).astype(np.int16)
    nib = np.empty((packed.shape[0], 2 * packed.shape[1]), dtype=np.int16)
    nib[:, 0::2] = lo
    nib[:, 1::2] = hi
    nib = np.where(nib >= 8, nib - 16, nib)
    return nib[:, :r].astype(np.int8)


def reconstruct(p_packed, p_scales, q_packed, q_scales, r: int) -> np.ndarray:
    """D = (q_P s_P)(q_Q s_Q)^T from the payload: fp64 product, one fp32
    rounding.  Sender and receiver both call this, so they add the same D."""
    qp = int4_unpack(p_packed, r).astype(np.float64) * np.asarray(p_scales, np.float64)[None, :]
    qq = int4_unpack(q_packed, r).astype(np.float64) * np.asarray(q_scales, np.float64)[None, :]
    return (qp @ qq.T).astype(np.float32)


def lowrank_encode(x_bits, recon_s, omega, iters: int):
    """One compressed low-rank step of the sender.

    Inputs: x_bits uint16 [T, C] (bf16 patterns), recon_s float32 [T, C]
    (updated in place), omega float32 [C, r].  Returns a dict with the
    payload (p_codes, p_scales, q_codes, q_scales), the fp32 error-feedback
    buffer ``err``, the unquantised fp64 factors P, Q, and D."""
    v = residual(x_bits, recon_s)
    p, q = subspace_iteration(v, omega, iters)
    r = omega.shape[1]
    pc, ps = int4_quantize_columns(p)
    qc, qs = int4_quantize_columns(q)
    p_packed, q_packed = int4_pack(pc), int4_pack(qc)
    d = reconstruct(p_packed, ps, q_packed, qs, r)
    err = v - d
    recon_s[...] = recon_s + d
    return dict(p_codes=p_packed, p_scales=ps, q_codes=q_packed, q_scales=qs,
                err=err, P=p, Q=q, D=d, V=v)


def lowrank_decode(p_packed, p_scales, q_packed, q_scales, recon_r, r: int):
    """Receiver: recon_r += D (in place)."""
    d = reconstruct(p_packed, p_scales, q_packed, q_scales, r)
    recon_r[...] = recon_r + d
    return d


def payload_bytes(tokens: int, channels: int, rank: int) -> int:
    """Bytes on the wire per buffer in low-rank mode: both INT4 factors plus
    one fp32 scale per factor column."""
    nb = (rank + 1) // 2
    return tokens * nb + channels * nb + 2 * 4 * rank
