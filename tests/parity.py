"""Shared helpers of the GPU parity tests: move workloads between devices,
run the oracle on (a sample of) the output, and apply the tolerances.

Tolerances of the layer output (fp16 in, fp32 accumulate, fp16 out):
    max|y - y_ref| <= 2e-3 * max|y_ref|   and   ||y - y_ref||_F <= 1e-3 ||y_ref||_F
where y_ref is the oracle's float64 result.  Codes, packed bytes and fp16
dequantised weights must match bit for bit.
"""
import numpy as np
import torch

from dequant_gemv_packed_b200 import qlin as Q
from oracle import qlin_oracle as O

MAX_REL = 2e-3
FRO_REL = 1e-3


def np_u32(sign_bits: torch.Tensor) -> np.ndarray:
    return sign_bits.cpu().numpy().view(np.uint32)


def host(w, a):
    """numpy copies of a weight and activation: codes, scales, zeros, x, sign bits."""
    return (w.codes.cpu().numpy(), w.scales.cpu().numpy(), w.zeros.cpu().numpy(), a.x.cpu().numpy(),
            np_u32(a.sign_bits))


def oracle_rows(w, a, rows=None):
    """Oracle output [M, len(rows)] for the given weight rows (all rows if None)."""
    rows = np.arange(w.N) if rows is None else np.asarray(rows)
    t = torch.as_tensor(rows, device=w.codes.device)
    codes = w.codes[t].cpu().numpy()
    s = w.scales[t].cpu().numpy()
    z = w.zeros[t].cpu().numpy()
    return O.linear64(a.x.cpu().numpy(), codes, s, z, np_u32(a.sign_bits))


def assert_close(y, y_ref, what=""):
    y = y.float().cpu().numpy() if isinstance(y, torch.Tensor) else np.asarray(y, np.float64)
    assert np.isfinite(y).all(), f"{what}: non-finite output"
    rel_max, rel_fro = O.parity_errors(y, y_ref)
    assert rel_max <= MAX_REL and rel_fro <= FRO_REL, f"{what}: max rel {rel_max:.3e}, fro rel {rel_fro:.3e}"
    return rel_max, rel_fro


def assert_dot_bound(y, w, a, rows=None, what=""):
    """Extra per-element check beside the output tolerance: every output is a
    dot product of K terms, and its error is held to 2e-3 of the sum of the
    terms' magnitudes, |y - y_ref| <= 2e-3 * sum_k |x~_k w_k| (fp64 oracle
    terms).  Unlike the max-relative bound it does not depend on the other
    outputs, so it also bounds outputs that cancel to far below their terms."""
    rows = np.arange(w.N) if rows is None else np.asarray(rows)
    t = torch.as_tensor(rows, device=w.codes.device)
    xr = O.rht64(a.x.cpu().numpy(), np_u32(a.sign_bits))
    wd = O.dequant64(w.codes[t].cpu().numpy(), w.scales[t].cpu().numpy(), w.zeros[t].cpu().numpy())
    ref = xr @ wd.T
    bound = MAX_REL * (np.abs(xr) @ np.abs(wd).T)
    y = y.float().cpu().numpy() if isinstance(y, torch.Tensor) else np.asarray(y, np.float64)
    err = np.abs(y - ref)
    assert (err <= bound).all(), f"{what}: worst error/bound {float((err / bound).max()):.3f}"


def packed_on_device(w):
    """Desc and packed buffer (packed on the GPU by qlin_pack)."""
    d = Q.Desc.of(w)
    return d, Q.qlin_pack(d, w.codes)


def sample_rows(N: int, count: int, seed: int = 0) -> np.ndarray:
    """Sorted sample of rows that always includes the first and last row."""
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(N, size=min(count, N), replace=False).tolist())
    rows.update({0, N - 1})
    return np.array(sorted(rows))
