"""GPU parity on adversarial inputs, and on every output column of full-size
layers.

* Trained-like zero points (non-integer, both signs, |z| up to 4 * 2^b) and
  scales of both signs over 2^16 (down to fp16 subnormals): they stress the
  per-group scale and zero applied to each group's partial sum.
* Activations whose 64-value runs span 2^10 ("wide" blocks) and runs of fp16
  subnormals: they stress the 16-bit integer form of the rotated activations
  in the M = 1 kernel (4- and 8-bit codes) and the fp16 operands of the
  tensor-core paths.
Each case runs on the M = 1 kernel (3, 4, 6 and 8 bits), the tensor-core GEMV
(M = 4 and 16) and the GEMM (M = 256), against the fp64 oracle with the output
tolerance: max|y - y_ref| <= 2e-3 max|y_ref| and relative Frobenius error
<= 1e-3.
"""
import numpy as np
import pytest
import torch

from dequant_gemv_packed_b200 import qlin as Q
from dequant_gemv_packed_b200 import workloads as W
from oracle import qlin_oracle as O

import adversarial as A
from parity import assert_close, assert_dot_bound, np_u32, oracle_rows, packed_on_device

pytestmark = pytest.mark.gpu
DEV = "cuda"
K = 2560
N = 448


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dequant_gemv_packed_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    Q.lib()


def _run(w, a, M):
    d, packed = packed_on_device(w)
    fn = Q.qlin_gemv if M <= 16 else Q.qlin_gemm
    y = fn(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    return y


PATHS = [(1, 3), (1, 4), (1, 6), (1, 8), (2, 6), (4, 3), (4, 8), (9, 3), (16, 4), (16, 6), (32, 0), (64, 8),
         (256, 6), (256, 0)]


def _bb(bits, n):
    return None if bits else ([6, 8, 3, 4, 8, 6, 8] * 8)[:n // 64]


@pytest.mark.parametrize("M,bits", PATHS)
def test_trained_zeros_and_signed_scales(M, bits):
    w = A.weight(N, K, bits, seed=10 * M + bits, block_bits=_bb(bits, N)).to(DEV)
    a = W.draw_activation(M, K, seed=M + 3).to(DEV)
    y = _run(w, a, M)
    ref = oracle_rows(w, a)
    assert_close(y, ref, f"adversarial s/z M{M} b{bits}")
    assert_dot_bound(y, w, a, what=f"adversarial s/z M{M} b{bits}")


@pytest.mark.parametrize("M,bits", PATHS)
def test_wide_activation_runs(M, bits):
    """Rotated runs that span 2^10 (and plain blocks), against the exact oracle."""
    kinds = ["wide", "plain"] * (K // 256)
    a, kinds = A.activation(M, K, seed=20 + M + bits, kinds=kinds)
    w = A.block_weight(N, K, bits, seed=30 + M + bits, kinds=kinds, block_bits=_bb(bits, N)).to(DEV)
    a = a.to(DEV)
    y = _run(w, a, M)
    assert_close(y, oracle_rows(w, a), f"wide runs M{M} b{bits}")


@pytest.mark.parametrize("M,bits", PATHS)
def test_subnormal_and_wide_runs(M, bits):
    """Subnormal, wide and plain blocks in every row, each group adding a
    comparable share of the output.  The fp16 rounding of a subnormal rotated
    value is a relative error of several per cent, so the reference is the
    exact layer on the fp16-rounded rotation (the reading that the rotated
    activations are rounded once to fp16)."""
    kinds = (["subnormal", "wide", "plain", "subnormal"] * K)[:K // 128]
    a, kinds = A.activation(M, K, seed=40 + M + bits, kinds=kinds)
    w = A.block_weight(N, K, bits, seed=50 + M + bits, kinds=kinds, block_bits=_bb(bits, N)).to(DEV)
    a = a.to(DEV)
    y = _run(w, a, M)
    ref = A.reference_r16(w, a)
    assert_close(y, ref, f"subnormal runs M{M} b{bits}")
    # the subnormal groups matter: without them the output would be far off
    keep = np.repeat(np.array([k != "subnormal" for k in kinds]), 128)
    xr = O.rht16(a.x.cpu().numpy(), np_u32(a.sign_bits)).astype(np.float64)
    wd = O.dequant64(w.codes.cpu().numpy(), w.scales.cpu().numpy(), w.zeros.cpu().numpy())
    partial = xr[:, keep] @ wd[:, keep].T
    assert O.parity_errors(partial, ref)[1] > 0.1


# ------------------------------------------------------------ all columns ----

def test_gemm_prefill256_all_columns():
    """The mixed int6/int8 prefill GEMM at M = 256: every one of the 9728 output
    columns against the oracle."""
    w, a = W.prefill(M=256, device=DEV)
    d, packed = packed_on_device(w)
    y = Q.qlin_gemm(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
    torch.cuda.synchronize()
    assert_close(y, oracle_rows(w, a), "prefill M=256, all columns")
    assert Q.qlin_device_error() == 0


def _oracle_chunked(w, a, chunk=8192):
    out = []
    for r0 in range(0, w.N, chunk):
        out.append(oracle_rows(w, a, np.arange(r0, min(w.N, r0 + chunk))))
    return np.concatenate(out, axis=1)


@pytest.mark.parametrize("which", list(range(7)) + [-1])
def test_stack_layer_all_rows(which):
    """One full linear of each shape of the 36-layer stack (layer 0: q, k, v, o,
    gate, up, down; int6) and the whole int8 lm_head, every output row against
    the oracle."""
    lin = W.stack_linears()
    i = which if which >= 0 else len(lin) - 1
    name, Kl, Nl, bits = lin[i]
    w = W.draw_weight(Nl, Kl, bits, seed=0, index=i + 1, device=DEV)
    a = W.draw_activation(1, Kl, seed=0, index=i + 1, device=DEV)
    d, packed = packed_on_device(w)
    y = Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
    torch.cuda.synchronize()
    assert_close(y, _oracle_chunked(w, a), f"{name}, all rows")
    assert Q.qlin_device_error() == 0
