"""GPU parity of the split-K tensor-core GEMV (qlin_gemv at M = 2..16 with one
code width) in the cases its launch plan makes special: every M from 2 to 16
(one or two n8 tiles of x rows, unused columns), rectangles streamed through
two shared-memory buffers in rounds, K slices of unequal length, a workspace
that holds garbage on entry, and one workspace shared by calls of different
shapes.  Every output is compared with the oracle (sampled rows where the
layer is large), at the tolerances of the output definition.
"""
import numpy as np
import pytest
import torch

from dequant_gemv_packed_b200 import qlin as Q
from dequant_gemv_packed_b200 import workloads as W

from parity import assert_close, assert_dot_bound, oracle_rows, packed_on_device, sample_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dequant_gemv_packed_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    Q.lib()


def _case(N, K, bits, M, seed, rows=None, workspace=None):
    w = W.draw_weight(N, K, bits, seed=seed).to(DEV)
    a = W.draw_activation(M, K, seed=seed + 1).to(DEV)
    d, packed = packed_on_device(w)
    assert Q.qlin_gemv_plan(d, M)["kernel"] == 4
    y = Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, a.x, workspace=workspace)
    torch.cuda.synchronize()
    got = y if rows is None else y[:, torch.as_tensor(rows, device=DEV)]
    assert_close(got, oracle_rows(w, a, rows), f"b{bits} N{N} K{K} M{M}")
    return w, a, d, packed, y


@pytest.mark.parametrize("bits", [3, 4, 6, 8])
def test_every_m(bits):
    """M = 2..16 on a ragged layer (N not a multiple of 32, several slices)."""
    for M in range(2, 17):
        w, a, d, packed, y = _case(333, 1280, bits, M, seed=40 + M)
        assert_dot_bound(y, w, a, what=f"b{bits} M{M}")


@pytest.mark.parametrize("bits,M,N", [(8, 16, 20000), (3, 4, 40000), (6, 9, 20000), (4, 2, 40000)])
def test_rounds_sampled(bits, M, N):
    """A layer whose CTA rectangles do not fit shared memory at once: the codes
    go through two buffers in rounds (plan stages == 2)."""
    K = 2560
    d = Q.Desc(N, K, bits)
    p = Q.qlin_gemv_plan(d, M)
    assert p["stages"] == 2, p
    rows = sample_rows(N, 64, seed=bits)
    _case(N, K, bits, M, seed=bits, rows=rows)


def test_garbage_workspace_and_repeat():
    """The workspace may hold anything on entry; two calls give the same bits."""
    N, K, bits, M = 2560, 9728, 3, 16
    d = Q.Desc(N, K, bits)
    ws = torch.full((Q.qlin_gemv_workspace_bytes(d, M),), 0xFF, dtype=torch.uint8, device=DEV)
    assert ws.numel() > 0
    w, a, d, packed, y1 = _case(N, K, bits, M, seed=7, rows=sample_rows(N, 96, seed=7), workspace=ws)
    ws.fill_(0xA5)
    y2 = Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, a.x, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_shared_workspace_across_shapes():
    """One workspace for layers of different shapes, called in turn on one
    stream (a decoder stack's pattern): each result equals the same call with a
    workspace of its own, bit for bit."""
    shapes = [(2560, 9728, 3, 4), (9728, 2560, 4, 16), (1024, 2560, 6, 8), (2560, 4096, 6, 2), (300, 1280, 8, 5)]
    cases = []
    need = 0
    for i, (N, K, bits, M) in enumerate(shapes):
        w = W.draw_weight(N, K, bits, seed=60 + i).to(DEV)
        a = W.draw_activation(M, K, seed=70 + i).to(DEV)
        d, packed = packed_on_device(w)
        need = max(need, Q.qlin_gemv_workspace_bytes(d, M))
        own = Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
        cases.append((w, a, d, packed, own))
    shared = torch.empty(need, dtype=torch.uint8, device=DEV)
    for rep in range(2):
        for i, (w, a, d, packed, own) in enumerate(cases):
            y = Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, a.x, workspace=shared)
            torch.cuda.synchronize()
            assert torch.equal(y.view(torch.int16), own.view(torch.int16)), (rep, shapes[i])
    for i, (w, a, d, packed, own) in enumerate(cases):
        rows = sample_rows(w.N, 48, seed=i)
        assert_close(own[:, torch.as_tensor(rows, device=DEV)], oracle_rows(w, a, rows), f"shape {shapes[i]}")


@pytest.mark.parametrize("bits", [3, 4, 6, 8])
@pytest.mark.parametrize("N,K,M", [(1, 128, 16), (31, 128, 2), (33, 9728, 2), (2560, 128, 9), (4097, 256, 8),
                                   (9728, 2560, 16), (1024, 9728, 3)])
def test_edge_shapes(bits, N, K, M):
    """One group (K = 128, a single slice), one row, a row count just past a
    tile, very long K with few rows, many rows with short K, and the gate/up
    shape at M = 16 (sampled rows where the layer is large)."""
    rows = None if N * K <= (1 << 22) else sample_rows(N, 96, seed=N + K)
    w, a, d, packed, y = _case(N, K, bits, M, seed=N + K + M, rows=rows)
    if rows is None:
        assert_dot_bound(y, w, a, what=f"b{bits} N{N} K{K} M{M}")


def test_no_tc_errors():
    assert Q.qlin_device_error() == 0
