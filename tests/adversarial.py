"""Adversarial inputs of the layer, for the parity tests.

The workload generator draws round-to-nearest weights (positive scales, zero
points inside the code range) and N(0, 1) activations.  These inputs stress the
two places where the kernels evaluate the layer differently from the plain
formula:

* the scale and zero applied to each group's partial sum,
  sum_k s (q_k - z) x_k = s (sum_k q_k x_k - z sum_k x_k): stressed by trained-
  like zero points (non-integer, both signs, up to four times the code range;
  training moves the zeros, "24B0978-Week01-Track2_20-Submission01", paragraph
  "End-to-end training changes nothing at inference") and by scales of both
  signs spanning 2^16;
* the 16-bit integer form of the rotated activations inside the M = 1 kernel
  (one power-of-two scale per run of 64 values, or 32 for 8-bit codes):
  stressed by runs whose values span 2^10 and by runs of fp16 subnormals.

An activation block of kind "wide" or "subnormal" is built from an integer
vector a as x = D H a 2^-e (D the block's signs, H the Sylvester matrix), which
is exact in fp16, so that its rotation is known in closed form:
rht(x) = H D x / sqrt(128) = sqrt(128) a 2^-e.
Test infrastructure: builds inputs with the oracle's Hadamard matrix and sign
expansion, never with the library.
"""
from __future__ import annotations

import numpy as np
import torch

from dequant_gemv_packed_b200 import workloads as W
from oracle import qlin_oracle as O

BLOCK = 128
KINDS = ("wide", "subnormal", "plain")
WIDE_EXP, SUBNORMAL_EXP = 13, 24
BIG = 1023


def _widths(N, bits, block_bits):
    return np.full(N, bits) if bits else np.repeat(np.asarray(block_bits, dtype=np.int64), 64)


def _pack_weight(N, K, bits, block_bits, codes, s, z) -> W.QuantWeight:
    bb = None if bits else torch.as_tensor(np.asarray(block_bits), dtype=torch.uint8)
    return W.QuantWeight(N, K, bits, bb, torch.from_numpy(codes), torch.from_numpy(s), torch.from_numpy(z))


def weight(N: int, K: int, bits: int, seed: int, block_bits=None, zero_span: float = 4.0,
           scale_exp=(-14.0, 2.0)) -> W.QuantWeight:
    """Codes uniform over each row's width; zero points uniform in
    (-zero_span, zero_span) * 2^b, rounded to fp16 (non-integer, both signs);
    scales of random sign with |s| = 2^u / (5 * 2^b), u uniform in scale_exp,
    independently per group, rounded to fp16 (down to fp16 subnormals).
    Every dequantised weight then satisfies |w| <= 2^max(scale_exp)."""
    rng = np.random.default_rng(seed)
    G = K // BLOCK
    widths = _widths(N, bits, block_bits)
    qmax = np.exp2(widths.astype(np.float64))[:, None]
    codes = (rng.integers(0, 256, (N, K)) & ((1 << widths) - 1)[:, None]).astype(np.uint8)
    z = (rng.uniform(-zero_span, zero_span, (N, G)) * qmax).astype(np.float16)
    sign = np.where(rng.random((N, G)) < 0.5, -1.0, 1.0)
    s = (sign * np.exp2(rng.uniform(*scale_exp, (N, G))) / (5.0 * qmax)).astype(np.float16)
    return _pack_weight(N, K, bits, block_bits, codes, s, z)


def block_weight(N: int, K: int, bits: int, seed: int, kinds, block_bits=None) -> W.QuantWeight:
    """Codes uniform, zero points uniform in [0, 2^b - 1] (non-integer), and the
    scale of each group sized to its activation block's kind, so that every
    group adds a comparable amount to the output: the tiny rotated values of a
    subnormal block meet large weights (|w| up to ~2^14), the plain and wide
    blocks ordinary ones."""
    rng = np.random.default_rng(seed)
    G = K // BLOCK
    widths = _widths(N, bits, block_bits)
    qmax = np.exp2(widths.astype(np.float64))[:, None]
    codes = (rng.integers(0, 256, (N, K)) & ((1 << widths) - 1)[:, None]).astype(np.uint8)
    z = (rng.uniform(0.0, 1.0, (N, G)) * (qmax - 1.0)).astype(np.float16)
    target = np.array([{"plain": 0.02, "wide": 0.15, "subnormal": 1.4e4}[k] for k in kinds])[None, :]
    sign = np.where(rng.random((N, G)) < 0.5, -1.0, 1.0)
    s = (sign * target * rng.uniform(0.5, 1.0, (N, G)) / qmax).astype(np.float16)
    return _pack_weight(N, K, bits, block_bits, codes, s, z)


def activation(M: int, K: int, seed: int, kinds=None):
    """Activations [M, K] fp16 and sign bits, block by block of 128 along K:

    * "wide": a = +-1 except one entry +-1023, x = D H a 2^-13; its rotation
      sqrt(128) a 2^-13 holds one value of ~1.41 among values of ~1.4e-3, so
      the 64-value run holding it spans 2^10;
    * "subnormal": a in {+-1, +-2, +-3}, x = D H a 2^-24; x and its rotation
      (~6.7e-7 .. 2.0e-6) are fp16 subnormals;
    * "plain": x ~ N(0, 1).

    The kind of each block is the same for all M rows (`kinds`, drawn if None);
    a is drawn per row.  Returns (workloads.Activation on the CPU, kinds)."""
    rng = np.random.default_rng(seed)
    nb = K // BLOCK
    sb = rng.integers(0, 2 ** 32, K // 32, dtype=np.uint64).astype(np.uint32)
    d = O.signs_from_bits(sb, K)
    H = O.hadamard(BLOCK).astype(np.float64)
    if kinds is None:
        kinds = list(rng.choice(KINDS, nb))
    x = np.empty((M, K), np.float64)
    for m in range(M):
        for j, kind in enumerate(kinds):
            sl = slice(BLOCK * j, BLOCK * (j + 1))
            if kind == "plain":
                x[m, sl] = rng.standard_normal(BLOCK)
                continue
            if kind == "wide":
                a = rng.choice([-1.0, 1.0], BLOCK)
                a[rng.integers(BLOCK)] *= BIG
                e = WIDE_EXP
            else:
                a = rng.choice([-3.0, -2.0, -1.0, 1.0, 2.0, 3.0], BLOCK)
                e = SUBNORMAL_EXP
            x[m, sl] = d[sl] * (H @ a) * 2.0 ** -e
    x16 = x.astype(np.float16)
    exact = np.array([k != "plain" for k in kinds]).repeat(BLOCK)
    assert np.array_equal(x16.astype(np.float64)[:, exact], x[:, exact]), "construction must be exact in fp16"
    return W.Activation(torch.from_numpy(x16), torch.from_numpy(sb.view(np.int32))), list(kinds)


def reference_r16(w: W.QuantWeight, a: W.Activation) -> np.ndarray:
    """The layer with the rotated activations rounded once to fp16, as the
    kernels use them, and everything else exact: fp64 rht16(x) times the fp64
    dequantised weight.  For subnormal rotated values that rounding is a
    relative error of several per cent, far above the output tolerance, so
    those inputs are compared with this reference rather than with the exact
    rotation."""
    xr = O.rht16(a.x.cpu().numpy(), a.sign_bits.cpu().numpy().view(np.uint32)).astype(np.float64)
    wd = O.dequant64(w.codes.cpu().numpy(), w.scales.cpu().numpy(), w.zeros.cpu().numpy())
    return xr @ wd.T
