"""The allocation-free GEMM entry point, qlin_gemm_noalloc.

Callers that cannot allocate device memory where they run the layer (a plugin
whose host runtime owns every allocation, or a serving loop that forbids
allocation once running) use qlin_gemm_noalloc, which keeps the rotated
activations in an array inside the library instead of a caller workspace.
This test calls it through the C ABI twice in a row, with different shapes so
that stale contents of the shared array would show, and compares each result
with qlin_gemm's on the same inputs and with the CPU oracle, within the parity
tolerances.  qlin_gemm_noalloc has no workspace for split tiles, so it runs the
one-CTA-per-tile schedule (each output tile summed by one CTA over all of K);
the oracle comparison is what checks that schedule.  It lives in a file of its
own that pytest collects last.
"""
import ctypes

import numpy as np
import pytest
import torch

from dequant_gemv_packed_b200 import qlin as Q
from dequant_gemv_packed_b200 import workloads as W
from oracle import qlin_oracle as O

pytestmark = pytest.mark.gpu

MAX_REL, FRO_REL = 2e-3, 1e-3
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dequant_gemv_packed_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    Q.lib()


def _noalloc(desc, packed, s, z, sb, x, y):
    L = Q.lib()
    stream = torch.cuda.current_stream().cuda_stream
    return L.qlin_gemm_noalloc(desc.ref(), packed.data_ptr(), s.data_ptr(), z.data_ptr(), sb.data_ptr(),
                               x.data_ptr(), y.data_ptr(), x.shape[0], ctypes.c_void_p(stream))


def _case(M, N, K, block_bits, seed):
    w = W.draw_weight(N, K, 0, seed=seed, block_bits=torch.as_tensor(block_bits, dtype=torch.uint8)).to(DEV)
    a = W.draw_activation(M, K, seed=seed).to(DEV)
    d = Q.Desc.of(w)
    packed = Q.qlin_pack(d, w.codes)
    return w, a, d, packed


def test_noalloc_matches_gemm_on_two_calls():
    cases = [(300, 256, 2560, [6, 8, 6, 6], 11), (96, 320, 1280, [8, 6, 6, 8, 6], 12)]
    for M, N, K, bb, seed in cases:
        w, a, d, packed = _case(M, N, K, bb, seed)
        ref = Q.qlin_gemm(d, packed, w.scales, w.zeros, a.sign_bits, a.x).float().cpu().numpy()
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device=DEV)
        assert _noalloc(d, packed, w.scales, w.zeros, a.sign_bits, a.x, y) == 0
        torch.cuda.synchronize()
        got = y.float().cpu().numpy()
        assert np.isfinite(got).all()
        rel_max, rel_fro = O.parity_errors(got, ref)
        assert rel_max <= MAX_REL and rel_fro <= FRO_REL, (M, N, K, rel_max, rel_fro)
        oracle = O.linear64(a.x.cpu().numpy(), w.codes.cpu().numpy(), w.scales.cpu().numpy(),
                            w.zeros.cpu().numpy(), a.sign_bits.cpu().numpy().view(np.uint32))
        rel_max, rel_fro = O.parity_errors(got, oracle)
        assert rel_max <= MAX_REL and rel_fro <= FRO_REL, ("oracle", M, N, K, rel_max, rel_fro)
    assert Q.qlin_device_error() == 0


def test_noalloc_rejects_oversize():
    w, a, d, packed = _case(64, 64, 128, [6], 13)
    big_m = (8 << 20) // 128 + 1
    x = torch.zeros(big_m, 128, dtype=torch.float16, device=DEV)
    y = torch.empty(big_m, 64, dtype=torch.float16, device=DEV)
    assert _noalloc(d, packed, w.scales, w.zeros, a.sign_bits, x, y) == -3  # QLIN_ERR_SHAPE
