"""CPU oracle for the weight-only-quantised linear layer.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module:
only the tests, the smoke check and the benchmark's CPU-baseline leg call it.
It shares no code with the CUDA library (``dequant_gemv_packed_b200/csrc``)
and it never imports that package.

What it computes, in the plainest form that the pages support
(``Y = rht(X) . dequant(Wq)^T``):

* ``pack`` / ``unpack``  -- integer codes <-> a per-row little-endian bit
  stream along the reduction dimension K ("24B0978-Week01-Track2_20-Submission01",
  section "How these techniques accelerate inference on CUDA", paragraph
  "Group-wise affine integer quantisation": codes plus one scale and zero point
  per group of 128 along K).  Mixed widths per 64-row block follow
  "25M2111-Week02-Track2-40-Submission01", section "Method, selection, and
  reproduction" (dense mixed-width codes with byte selectors).
* ``dequant64`` -- w = s * (q - z) evaluated in float64 (same paragraph).
* ``dequant16`` -- the fp16 weight that the library exposes: t = fp32(q) - fp32(z)
  and p = fp32(s) * t, each rounded once to fp32, then rounded once to fp16.
* ``hadamard`` -- the explicit Sylvester matrix H[i, j] = (-1)^popcount(i & j).
* ``rht64`` -- random Hadamard transform of the activations: per block of 128
  along K, flip signs then multiply by the orthonormal H / sqrt(128)
  ("24B0978-Week01-Track2_20-Submission01", paragraph "Random Hadamard
  transform"; "24B0978-Week02-Track2-40-Submission01", section "Recipe").
  Dense 128x128 products, not a butterfly.
* ``linear64`` -- the fp64 matmul of the rotated activations with the fp64
  dequantised weight.
* ``hessian64`` / ``hessian_inverse_factor`` / ``gptq_columns32`` / ``gptq32`` /
  ``quantize_gptq`` -- GPTQ error compensation ("24B0978-Week02-Track2-40-
  Submission01", section "Recipe": RHT + GPTQ 6-bit g128 from a calibration
  Hessian of 128 sequences, the compensation run in the rotated basis;
  "24B0908-Week03-Track1-40-Submission01": GPTQ int3 g128 on the MLP; the
  Hessian is H = 2 X^T X over the calibration inputs, as the SparseGPT page
  "24B0908-Week02-Track1-40-Submission01" writes it).  The pages name the
  method, not its steps; these follow the published column-by-column form:
  columns in order, each group's grid taken by round-to-nearest from the
  weights as they stand when the group starts, each column's quantisation
  error divided by the diagonal of the upper Cholesky factor U of the damped
  inverse Hessian and subtracted, times U's row, from the later columns.
* ``rotate_weight32`` / ``rtn32`` / ``quantize_rtn`` -- the offline weight side:
  each weight row rotated with the activations' signs and H / sqrt(128) (the
  weight side of the rotation is folded in offline, "24B0978-Week01-Track2_20-
  Submission01", paragraph "Random Hadamard transform"), rounded once to fp32,
  then asymmetric round-to-nearest per group of 128 ("24B0978-Week02-Track2-40-
  Submission01", recipe op "quant_rtn": bits, group 128) in fp32 arithmetic:
  s = fp16((max - min) / (2^b - 1)) (1 if not > 0), z = fp16(-min / s),
  q = clip(rint(w / s + z), 0, 2^b - 1).

Readings where the pages leave a step open (the library documents the same readings):

* FWHT normalisation is 1/sqrt(128) (orthonormal): the pages call the transform
  orthogonal and function preserving.
* One independent sign per K index; sign bit set means -1; signs are applied
  before H.
* The rotated activation is rounded once to fp16 (``rht16``).
* Code bits above the width are ignored by ``pack``.
* Round-to-nearest quantisation works per group in fp32 with the min/max
  affine form above; a zero minimum counts as +0 (so z is -0).
* GPTQ: damping 1 % of the mean Hessian diagonal; natural column order; the
  working weights, the factor U and every update in fp32, each product and
  difference rounded on its own (no fused multiply-add), updates applied to
  each later column one source column at a time in column order.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, brute force, exact rational arithmetic or a library
routine; none is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

GROUP = 128          # codes per scale/zero group along K
BLOCK_ROWS = 64      # rows per width block in the mixed-width format
HADAMARD_BLOCK = 128  # block size of the activation rotation
WIDTHS = (3, 4, 6, 8)


# --------------------------------------------------------------------------
# Packed code layout
# --------------------------------------------------------------------------

def row_widths(N: int, bits: int | None = None, block_bits=None) -> np.ndarray:
    """Code width of every row: uniform ``bits``, or ``block_bits[n // 64]``."""
    if block_bits is None:
        if bits not in WIDTHS:
            raise ValueError(f"unsupported width {bits}")
        return np.full(N, bits, dtype=np.int64)
    block_bits = np.asarray(block_bits, dtype=np.int64)
    if N % BLOCK_ROWS or block_bits.shape != (N // BLOCK_ROWS,):
        raise ValueError("mixed widths need N % 64 == 0 and one width per 64-row block")
    if not np.isin(block_bits, WIDTHS).all():
        raise ValueError("unsupported block width")
    return np.repeat(block_bits, BLOCK_ROWS)


def row_byte_offsets(N: int, K: int, bits: int | None = None, block_bits=None) -> np.ndarray:
    """Byte offset of each row's bit stream, plus the total, as int64 [N + 1].

    Row n holds K codes of b_n bits each, i.e. K * b_n / 8 bytes; rows follow
    one another with no padding.
    """
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    w = row_widths(N, bits, block_bits)
    off = np.zeros(N + 1, dtype=np.int64)
    off[1:] = np.cumsum(w * K // 8)
    return off


def pack(codes: np.ndarray, bits: int | None = None, block_bits=None) -> np.ndarray:
    """Pack integer codes [N, K] into the per-row little-endian bit stream.

    Code k of a row occupies stream bits [b*k, b*k + b), least significant bit
    first; stream bit j is bit (j mod 8) of byte j // 8 of the row (so, read as
    little-endian 32-bit words, bit j mod 32 of word j // 32).  Returns uint8.
    """
    codes = np.asarray(codes)
    N, K = codes.shape
    w = row_widths(N, bits, block_bits)
    off = row_byte_offsets(N, K, bits, block_bits)
    out = np.zeros(int(off[-1]), dtype=np.uint8)
    q = codes.astype(np.uint8)
    for b in np.unique(w):
        rows = np.nonzero(w == b)[0]
        # bit i of code k, i < b  ->  stream bit b*k + i
        bitplanes = np.unpackbits(q[rows][..., None], axis=-1, bitorder="little")[..., :b]
        stream = bitplanes.reshape(len(rows), K * int(b))
        rowbytes = np.packbits(stream, axis=-1, bitorder="little")
        for r, n in enumerate(rows):
            out[off[n]:off[n + 1]] = rowbytes[r]
    return out


def unpack(packed: np.ndarray, N: int, K: int, bits: int | None = None, block_bits=None,
           rows=None) -> np.ndarray:
    """Inverse of ``pack``: read codes [len(rows), K] (uint8) from the bit stream."""
    packed = np.asarray(packed, dtype=np.uint8)
    w = row_widths(N, bits, block_bits)
    off = row_byte_offsets(N, K, bits, block_bits)
    rows = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((len(rows), K), dtype=np.uint8)
    for i, n in enumerate(rows):
        b = int(w[n])
        stream = np.unpackbits(packed[off[n]:off[n + 1]], bitorder="little")
        bitplanes = stream.reshape(K, b).astype(np.uint16)
        out[i] = (bitplanes << np.arange(b, dtype=np.uint16)).sum(axis=1).astype(np.uint8)
    return out


# --------------------------------------------------------------------------
# Dequantisation
# --------------------------------------------------------------------------

def _per_k(a: np.ndarray, K: int) -> np.ndarray:
    """Broadcast a per-group array [N, K/128] to per-code [N, K]."""
    return np.repeat(np.asarray(a), GROUP, axis=1)[:, :K]


def dequant64(codes: np.ndarray, scales: np.ndarray, zeros: np.ndarray) -> np.ndarray:
    """w[n, k] = s[n, k//128] * (q[n, k] - z[n, k//128]) in float64."""
    K = codes.shape[1]
    s = _per_k(scales, K).astype(np.float64)
    z = _per_k(zeros, K).astype(np.float64)
    return s * (codes.astype(np.float64) - z)


def dequant16(codes: np.ndarray, scales: np.ndarray, zeros: np.ndarray) -> np.ndarray:
    """The fp16 weight: fp32 subtract, fp32 multiply, one rounding to fp16.

    numpy float32 arithmetic is IEEE single precision with round-to-nearest-even
    and no fused multiply-add, and ``astype(float16)`` rounds to nearest even.
    """
    K = codes.shape[1]
    s = _per_k(scales, K).astype(np.float32)
    z = _per_k(zeros, K).astype(np.float32)
    t = codes.astype(np.float32) - z
    p = s * t
    return p.astype(np.float16)


# --------------------------------------------------------------------------
# Random Hadamard transform of the activations
# --------------------------------------------------------------------------

def hadamard(n: int = HADAMARD_BLOCK) -> np.ndarray:
    """Sylvester Hadamard matrix of order n (a power of two), int64 entries +-1."""
    if n <= 0 or n & (n - 1):
        raise ValueError("order must be a power of two")
    i = np.arange(n, dtype=np.int64)
    a = i[:, None] & i[None, :]
    parity = np.zeros_like(a)
    while a.any():
        parity ^= a & 1
        a >>= 1
    return 1 - 2 * parity


def signs_from_bits(sign_bits: np.ndarray, K: int) -> np.ndarray:
    """+-1 float64 [K]: bit (k mod 32) of word k // 32 set means d_k = -1."""
    words = np.asarray(sign_bits, dtype=np.uint32)
    if words.shape != (K // 32,):
        raise ValueError("sign_bits must hold K/32 words")
    k = np.arange(K)
    bit = (words[k // 32] >> (k % 32).astype(np.uint32)) & 1
    return 1.0 - 2.0 * bit.astype(np.float64)


def rht64(x: np.ndarray, sign_bits: np.ndarray) -> np.ndarray:
    """x~ = (1/sqrt(128)) H diag(d) x, block by block of 128 along K, in float64."""
    x = np.asarray(x, dtype=np.float64)
    M, K = x.shape
    if K % HADAMARD_BLOCK:
        raise ValueError("K must be a multiple of 128")
    d = signs_from_bits(sign_bits, K)
    H = hadamard(HADAMARD_BLOCK).astype(np.float64)
    inv_sqrt = 1.0 / math.sqrt(HADAMARD_BLOCK)
    out = np.empty_like(x)
    for b0 in range(0, K, HADAMARD_BLOCK):
        xb = x[:, b0:b0 + HADAMARD_BLOCK] * d[b0:b0 + HADAMARD_BLOCK]
        out[:, b0:b0 + HADAMARD_BLOCK] = (xb @ H.T) * inv_sqrt
    return out


def rht16(x: np.ndarray, sign_bits: np.ndarray) -> np.ndarray:
    """The rotated activation rounded once to fp16."""
    return rht64(x, sign_bits).astype(np.float16)


# --------------------------------------------------------------------------
# Offline weight side: rotation and round-to-nearest quantisation
# --------------------------------------------------------------------------

def rotate_weight32(w: np.ndarray, sign_bits: np.ndarray) -> np.ndarray:
    """Each fp16 weight row rotated like the activations (``rht64``: signs, then
    H / sqrt(128) per block of 128), rounded once to fp32.  For fp16 input the
    fp64 sums are exact (multiples of 2^-24 below 2^23), so this is the fp32
    rounding of one fp64 product of the exact sum with 1/sqrt(128)."""
    return rht64(np.asarray(w, np.float16).astype(np.float64), sign_bits).astype(np.float32)


def rtn32(wr: np.ndarray, bits: int | None = None, block_bits=None):
    """Asymmetric round-to-nearest per group of 128 of fp32 rows ``wr`` [N, K],
    every step an fp32 operation rounded to nearest:
    s = fp16((max - min) / (2^b - 1)), replaced by 1 unless > 0;
    z = fp16(-min / s) with a zero minimum taken as +0;
    q = clip(rint(w / s + z), 0, 2^b - 1).
    Returns (codes uint8 [N, K], scales fp16 [N, K/128], zeros fp16 [N, K/128])."""
    wr = np.asarray(wr, np.float32)
    N, K = wr.shape
    g = wr.reshape(N, K // GROUP, GROUP)
    qmax = (np.float32(2.0) ** row_widths(N, bits, block_bits).astype(np.float32) - np.float32(1.0))[:, None]
    mn = g.min(axis=-1) + np.float32(0.0)
    mx = g.max(axis=-1)
    s16 = ((mx - mn) / qmax).astype(np.float16)
    s16 = np.where(s16.astype(np.float32) > np.float32(0.0), s16, np.float16(1.0))
    s32 = s16.astype(np.float32)
    z16 = (-mn / s32).astype(np.float16)
    z32 = z16.astype(np.float32)
    q = np.clip(np.rint(g / s32[..., None] + z32[..., None]), np.float32(0.0), qmax[..., None])
    return q.astype(np.uint8).reshape(N, K), s16, z16


def quantize_rtn(w: np.ndarray, sign_bits: np.ndarray, bits: int | None = None, block_bits=None):
    """The offline weight side: ``rtn32(rotate_weight32(w))``."""
    return rtn32(rotate_weight32(w, sign_bits), bits, block_bits)


# --------------------------------------------------------------------------
# GPTQ: error-compensated quantisation against a calibration Hessian
# --------------------------------------------------------------------------

def hessian64(x: np.ndarray) -> np.ndarray:
    """H = 2 X^T X / n for calibration inputs x [n, K] (rows are the inputs the
    layer sees), in float64."""
    x = np.asarray(x, dtype=np.float64)
    return (2.0 / x.shape[0]) * (x.T @ x)


def hessian_inverse_factor(H: np.ndarray, damp: float = 0.01) -> np.ndarray:
    """Upper-triangular U (float64) with U^T U = (H + damp * mean(diag H) * I)^-1:
    the lower Cholesky factor of the damped inverse, transposed."""
    H = np.asarray(H, dtype=np.float64)
    Hd = H + damp * float(np.mean(np.diag(H))) * np.eye(H.shape[0])
    return np.ascontiguousarray(np.linalg.cholesky(np.linalg.inv(Hd)).T)


def gptq_columns32(w: np.ndarray, U: np.ndarray, qmax: np.ndarray, group: int = GROUP):
    """The GPTQ column loop on fp32 rows w [N, K] with the fp32 factor U [K, K]
    and the largest code of each row, qmax [N]:

        for each column i in order:
            at the first column of a group: its grid (s, z) by round-to-nearest
                from the group's weights as they are now (the ``rtn32`` formulas);
            q_i   = clip(rint(w_i / s + z), 0, qmax)
            e_i   = (w_i - s (q_i - z)) / U[i, i]
            w_j  -= e_i U[i, j]            for every later column j

    every operation an fp32 operation rounded to nearest.  Returns (codes uint8
    [N, K], scales fp16 [N, K/group], zeros fp16 [N, K/group], e fp32 [N, K])."""
    W = np.array(w, dtype=np.float32, copy=True)
    U = np.asarray(U, dtype=np.float32)
    N, K = W.shape
    if K % group or U.shape != (K, K):
        raise ValueError("K must be a multiple of the group and U must be K x K")
    qmax = np.asarray(qmax, dtype=np.float32).reshape(N)
    codes = np.zeros((N, K), dtype=np.uint8)
    s16 = np.zeros((N, K // group), dtype=np.float16)
    z16 = np.zeros((N, K // group), dtype=np.float16)
    err = np.zeros((N, K), dtype=np.float32)
    s32 = z32 = None
    for i in range(K):
        g, j = divmod(i, group)
        if j == 0:
            blk = W[:, i:i + group]
            mn = blk.min(axis=1) + np.float32(0.0)
            mx = blk.max(axis=1)
            sg = ((mx - mn) / qmax).astype(np.float16)
            sg = np.where(sg.astype(np.float32) > np.float32(0.0), sg, np.float16(1.0))
            s32 = sg.astype(np.float32)
            zg = (-mn / s32).astype(np.float16)
            z32 = zg.astype(np.float32)
            s16[:, g], z16[:, g] = sg, zg
        q = np.clip(np.rint(W[:, i] / s32 + z32), np.float32(0.0), qmax)
        wq = s32 * (q - z32)
        e = (W[:, i] - wq) / U[i, i]
        W[:, i + 1:] -= np.outer(e, U[i, i + 1:])
        codes[:, i] = q.astype(np.uint8)
        err[:, i] = e
    return codes, s16, z16, err


def gptq32(w: np.ndarray, U: np.ndarray, bits: int | None = None, block_bits=None):
    """GPTQ of fp32 rows w [N, K] in groups of 128 with each row's width (uniform
    ``bits`` or per 64-row block); returns (codes, scales, zeros) like ``rtn32``."""
    w = np.asarray(w, dtype=np.float32)
    qmax = np.float32(2.0) ** row_widths(w.shape[0], bits, block_bits).astype(np.float32) - np.float32(1.0)
    codes, s16, z16, _ = gptq_columns32(w, U, qmax, GROUP)
    return codes, s16, z16


def quantize_gptq(w: np.ndarray, sign_bits: np.ndarray, U: np.ndarray, bits: int | None = None, block_bits=None):
    """The offline weight side with error compensation: ``gptq32`` of the rotated
    rows ``rotate_weight32(w)``; U is the factor of the Hessian of the rotated
    activations (the compensation runs in the rotated basis)."""
    return gptq32(rotate_weight32(w, sign_bits), U, bits, block_bits)


# --------------------------------------------------------------------------
# The quantised linear layer
# --------------------------------------------------------------------------

def linear64(x: np.ndarray, codes: np.ndarray, scales: np.ndarray, zeros: np.ndarray,
             sign_bits: np.ndarray) -> np.ndarray:
    """Y[m, n] = sum_k rht64(x)[m, k] * dequant64(w)[n, k], in float64.

    ``codes``/``scales``/``zeros`` may hold any subset of the weight rows; the
    result then holds the matching output columns.
    """
    xr = rht64(x, sign_bits)
    w = dequant64(codes, scales, zeros)
    return xr @ w.T


def algorithmic_bytes(N: int, K: int, bits: int | None = None, block_bits=None) -> int:
    """Bytes a kernel must read from memory for one pass over the weight:
    packed codes plus the fp16 scale and zero of every group (plus one selector
    byte per 64-row block in the mixed format)."""
    code_bytes = int(row_byte_offsets(N, K, bits, block_bits)[-1])
    sz_bytes = 2 * 2 * N * (K // GROUP)
    sel = 0 if block_bits is None else N // BLOCK_ROWS
    return code_bytes + sz_bytes + sel


def parity_errors(y: np.ndarray, y_ref: np.ndarray) -> tuple[float, float]:
    """(max|y - y_ref| / max|y_ref|, ||y - y_ref||_F / ||y_ref||_F)."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    diff = y - y_ref
    den_max = float(np.abs(y_ref).max()) if y_ref.size else 0.0
    den_fro = float(np.linalg.norm(y_ref)) if y_ref.size else 0.0
    rel_max = float(np.abs(diff).max()) / den_max if den_max > 0 else float(np.abs(diff).max(initial=0.0))
    rel_fro = float(np.linalg.norm(diff)) / den_fro if den_fro > 0 else float(np.linalg.norm(diff))
    return rel_max, rel_fro
