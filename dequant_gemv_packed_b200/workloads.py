"""Seeded synthetic workloads for the quantised linear layer.

This module only *draws* inputs: Gaussian weights with a fixed share of
outliers, their round-to-nearest group quantisation (the stand-in for the
pages' offline quantisers), Gaussian activations and random sign bits.  It
contains none of the layer's runtime arithmetic (no unpacking, dequantisation,
Hadamard transform or matmul), so the CUDA path and the CPU oracle can both
consume its outputs without sharing any of that arithmetic.

Everything is produced with ``torch`` random generators, on the device given
(CPU for small cases, CUDA for full-size ones).  A CPU draw and a CUDA draw of
the same workload differ (the two generator engines differ); each is fully
determined by its seed.

Workloads (sizes as in the decode and prefill shapes of a 4B-class decoder):

* ``tiny``     K=256,  N=512,  M=1, int4, weights N(0, 0.02), no outliers.
* ``gateup``   K=2560, N=9728, M=1, int4, weights N(0, 0.02) with 0.1 % x20 outliers.
* ``down``     K=9728, N=2560, M in {1, 4, 16}, int3, same weight distribution.
* ``stack``    36 layers x {q 2560->4096, k/v 2560->1024, o 4096->2560,
               gate/up 2560->9728, down 9728->2560} int6, plus an int8 tied
               lm_head 2560->151936, M=1; every linear has its own x and signs.
* ``prefill``  M in {256, 1024, 2048}, K=2560, N=9728, 64-row blocks of int6/int8
               (17 % of blocks int8, seeded), same weight distribution.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterator, Optional

import torch

GROUP = 128
BLOCK_ROWS = 64
WEIGHT_STD = 0.02
OUTLIER_SHARE = 0.001
OUTLIER_FACTOR = 20.0
INT8_BLOCK_SHARE = 0.17

# independent random streams of one workload
_STREAM_WEIGHTS, _STREAM_OUTLIERS, _STREAM_ACT, _STREAM_SIGNS, _STREAM_WIDTHS = range(5)


def _gen(device, seed: int, stream: int, index: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + stream * 7_919 + index * 104_729) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


@dataclasses.dataclass
class QuantWeight:
    """One quantised weight: codes [N, K] uint8, scales/zeros [N, K/128] fp16."""
    N: int
    K: int
    bits: int                       # 3, 4, 6, 8, or 0 for mixed widths
    block_bits: Optional[torch.Tensor]  # uint8 [N/64] (host) when bits == 0
    codes: torch.Tensor
    scales: torch.Tensor
    zeros: torch.Tensor

    def to(self, device) -> "QuantWeight":
        return dataclasses.replace(self, codes=self.codes.to(device), scales=self.scales.to(device),
                                   zeros=self.zeros.to(device))


@dataclasses.dataclass
class Activation:
    """Activations x [M, K] fp16 and the Hadamard sign bits [K/32] (int32 bit patterns)."""
    x: torch.Tensor
    sign_bits: torch.Tensor

    def to(self, device) -> "Activation":
        return Activation(self.x.to(device), self.sign_bits.to(device))


def rtn_quantise(w: torch.Tensor, bits: int) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Round-to-nearest asymmetric quantisation per group of 128 along K (fp32).

    scale = fp16((max - min) / (2^b - 1)) (1 if the group is constant),
    zero = fp16(-min / scale), q = clamp(round_half_even(w / scale + zero), 0, 2^b - 1).
    """
    N, K = w.shape
    qmax = float(2 ** bits - 1)
    wg = w.float().reshape(N, K // GROUP, GROUP)
    mn = wg.amin(dim=-1)
    mx = wg.amax(dim=-1)
    s = (mx - mn) / qmax
    s = torch.where(mx > mn, s, torch.ones_like(s))
    s16 = s.half()
    s16 = torch.where(s16 > 0, s16, torch.ones_like(s16))
    s32 = s16.float()
    z16 = (-mn / s32).half()
    z32 = z16.float()
    q = torch.round(wg / s32[..., None] + z32[..., None]).clamp_(0.0, qmax)
    return q.to(torch.uint8).reshape(N, K), s16, z16


def _draw_w32(N: int, K: int, seed: int, index: int, outliers: bool, device) -> torch.Tensor:
    """W ~ N(0, 0.02) [N, K] (fp32) with exactly round(0.1 % * N * K) entries,
    chosen without replacement, scaled by 20."""
    gw = _gen(device, seed, _STREAM_WEIGHTS, index)
    w = torch.randn(N, K, generator=gw, device=device, dtype=torch.float32) * WEIGHT_STD
    if outliers:
        n_out = int(math.floor(OUTLIER_SHARE * N * K + 0.5))
        go = _gen(device, seed, _STREAM_OUTLIERS, index)
        pos = torch.randperm(N * K, generator=go, device=device)[:n_out]
        w.view(-1)[pos] *= OUTLIER_FACTOR
        del pos
    return w


def draw_fp16_weight(N: int, K: int, *, seed: int = 0, index: int = 0, outliers: bool = True,
                     device="cpu") -> torch.Tensor:
    """The unquantised weight of `draw_weight` (same draw), rounded to fp16: the
    input of the offline rotation and quantisation."""
    return _draw_w32(N, K, seed, index, outliers, device).half()


def draw_weight(N: int, K: int, bits: int, *, seed: int = 0, index: int = 0, outliers: bool = True,
                block_bits: Optional[torch.Tensor] = None, device="cpu") -> QuantWeight:
    """Draw W ~ N(0, 0.02) [N, K] (fp32), scale exactly round(0.1 % * N * K) entries,
    chosen without replacement, by 20, and RTN-quantise each row with its width."""
    w = _draw_w32(N, K, seed, index, outliers, device)
    if bits:
        codes, s, z = rtn_quantise(w, bits)
        return QuantWeight(N, K, bits, None, codes, s, z)
    assert block_bits is not None and N % BLOCK_ROWS == 0
    codes = torch.empty(N, K, dtype=torch.uint8, device=device)
    s = torch.empty(N, K // GROUP, dtype=torch.float16, device=device)
    z = torch.empty_like(s)
    row_bits = torch.repeat_interleave(block_bits.to(device).long(), BLOCK_ROWS)
    for b in (3, 4, 6, 8):
        rows = torch.nonzero(row_bits == b).flatten()
        if rows.numel():
            c, ss, zz = rtn_quantise(w[rows], b)
            codes[rows], s[rows], z[rows] = c, ss, zz
    return QuantWeight(N, K, 0, block_bits.cpu().to(torch.uint8), codes, s, z)


def draw_block_bits(N: int, *, seed: int = 0, index: int = 0, share8: float = INT8_BLOCK_SHARE) -> torch.Tensor:
    """Widths of the 64-row blocks: exactly round(share8 * N/64) blocks of 8 bits,
    picked by a seeded permutation, the rest 6 bits (uint8 [N/64], host)."""
    nb = N // BLOCK_ROWS
    n8 = int(math.floor(share8 * nb + 0.5))
    perm = torch.randperm(nb, generator=_gen("cpu", seed, _STREAM_WIDTHS, index))
    bb = torch.full((nb,), 6, dtype=torch.uint8)
    bb[perm[:n8]] = 8
    return bb


def draw_activation(M: int, K: int, *, seed: int = 0, index: int = 0, device="cpu") -> Activation:
    """x ~ N(0, 1) rounded to fp16 [M, K]; one random sign bit per K index."""
    ga = _gen(device, seed, _STREAM_ACT, index)
    x = torch.randn(M, K, generator=ga, device=device, dtype=torch.float32).half()
    gs = _gen(device, seed, _STREAM_SIGNS, index)
    sb = torch.randint(-(2 ** 31), 2 ** 31, (K // 32,), generator=gs, device=device, dtype=torch.int64)
    return Activation(x, sb.to(torch.int32))


CALIB_SEQUENCES = 128
CALIB_TOKENS = 16
CALIB_HEAVY_SHARE = 0.01
CALIB_HEAVY_FACTOR = 8.0
CALIB_RANK = 8


def draw_calibration(K: int, *, seed: int = 0, index: int = 0, n: int = CALIB_SEQUENCES * CALIB_TOKENS,
                     device="cpu") -> torch.Tensor:
    """Synthetic calibration inputs of a layer, x [n, K] fp32 (the stand-in for
    128 calibration sequences): N(0, 1) plus a shared rank-8 component (so the
    channels correlate), with exactly round(1 % * K) channels, chosen without
    replacement, scaled by 8 (activation outlier channels)."""
    g = _gen(device, seed, _STREAM_ACT, 1000 + index)
    x = torch.randn(n, K, generator=g, device=device, dtype=torch.float32)
    basis = torch.randn(CALIB_RANK, K, generator=g, device=device, dtype=torch.float32)
    coef = torch.randn(n, CALIB_RANK, generator=g, device=device, dtype=torch.float32)
    x += coef @ basis
    heavy = torch.randperm(K, generator=_gen("cpu", seed, _STREAM_OUTLIERS, 1000 + index))[
        :int(math.floor(CALIB_HEAVY_SHARE * K + 0.5))]
    x[:, heavy.to(device)] *= CALIB_HEAVY_FACTOR
    return x


# ---------------------------------------------------------------------------
# Named workloads
# ---------------------------------------------------------------------------

STACK_LAYERS = 36
HIDDEN = 2560
STACK_SHAPES = (  # (name, K, N): in -> out
    ("q_proj", 2560, 4096),
    ("k_proj", 2560, 1024),
    ("v_proj", 2560, 1024),
    ("o_proj", 4096, 2560),
    ("gate_proj", 2560, 9728),
    ("up_proj", 2560, 9728),
    ("down_proj", 9728, 2560),
)
LM_HEAD = ("lm_head", 2560, 151936)
STACK_BITS = 6
LM_HEAD_BITS = 8


def tiny(device="cpu", seed: int = 0):
    w = draw_weight(512, 256, 4, seed=seed, outliers=False, device=device)
    a = draw_activation(1, 256, seed=seed, device=device)
    return w, a


def gateup(device="cpu", seed: int = 0, M: int = 1):
    w = draw_weight(9728, 2560, 4, seed=seed, device=device)
    a = draw_activation(M, 2560, seed=seed, device=device)
    return w, a


def down(M: int = 1, device="cpu", seed: int = 0):
    w = draw_weight(2560, 9728, 3, seed=seed, device=device)
    a = draw_activation(M, 9728, seed=seed, device=device)
    return w, a


def prefill(M: int = 256, device="cpu", seed: int = 0, N: int = 9728, K: int = 2560):
    bb = draw_block_bits(N, seed=seed)
    w = draw_weight(N, K, 0, seed=seed, block_bits=bb, device=device)
    a = draw_activation(M, K, seed=seed, device=device)
    return w, a


def stack_linears() -> list[tuple[str, int, int, int]]:
    """(name, K, N, bits) of every linear of the 36-layer stack, lm_head last."""
    out = []
    for layer in range(STACK_LAYERS):
        for name, K, N in STACK_SHAPES:
            out.append((f"layers.{layer}.{name}", K, N, STACK_BITS))
    out.append((LM_HEAD[0], LM_HEAD[1], LM_HEAD[2], LM_HEAD_BITS))
    return out


def stack(device="cpu", seed: int = 0) -> Iterator[tuple[str, QuantWeight, Activation]]:
    """Yield (name, weight, activation) for every linear of the stack, in order."""
    for i, (name, K, N, bits) in enumerate(stack_linears()):
        w = draw_weight(N, K, bits, seed=seed, index=i + 1, device=device)
        a = draw_activation(1, K, seed=seed, index=i + 1, device=device)
        yield name, w, a


def concat_rows(ws: list[QuantWeight]) -> QuantWeight:
    """One weight whose output rows are those of `ws` in order (same K, same
    uniform width): the fused projection of linears that read the same x."""
    K, bits = ws[0].K, ws[0].bits
    assert bits and all(w.K == K and w.bits == bits for w in ws), "fusion needs one K and one uniform width"
    return QuantWeight(sum(w.N for w in ws), K, bits, None, torch.cat([w.codes for w in ws]),
                       torch.cat([w.scales for w in ws]), torch.cat([w.zeros for w in ws]))


# Projections of one layer that read the same x, fused into one weight each.
STACK_FUSED = (("qkv_proj", ("q_proj", "k_proj", "v_proj")), ("o_proj", ("o_proj",)),
               ("gate_up_proj", ("gate_proj", "up_proj")), ("down_proj", ("down_proj",)))


def stack_fused(device="cpu", seed: int = 0) -> Iterator[tuple[str, QuantWeight, Activation]]:
    """The stack's weights (the same draws as `stack`) with q/k/v and gate/up
    each fused into one weight of N = 6144 and 19456 rows; a fused projection
    reads the x of its first member.  Yields (name, weight, activation) for
    the 36 x 4 fused linears and the lm_head."""
    lin = stack_linears()
    index = {name: i for i, (name, _, _, _) in enumerate(lin)}
    for layer in range(STACK_LAYERS):
        for fused, members in STACK_FUSED:
            ids = [index[f"layers.{layer}.{m}"] for m in members]
            ws = [draw_weight(lin[i][2], lin[i][1], lin[i][3], seed=seed, index=i + 1, device=device) for i in ids]
            a = draw_activation(1, lin[ids[0]][1], seed=seed, index=ids[0] + 1, device=device)
            yield f"layers.{layer}.{fused}", (ws[0] if len(ws) == 1 else concat_rows(ws)), a
    i = len(lin) - 1
    name, K, N, bits = lin[i]
    yield name, draw_weight(N, K, bits, seed=seed, index=i + 1, device=device), \
        draw_activation(1, K, seed=seed, index=i + 1, device=device)
