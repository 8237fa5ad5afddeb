"""Host-side checks of the seeded workload generator (no GPU)."""
import math

import numpy as np
import torch

from dequant_gemv_packed_b200 import workloads as W


def test_deterministic_and_independent_streams():
    w1, a1 = W.tiny()
    w2, a2 = W.tiny()
    assert torch.equal(w1.codes, w2.codes) and torch.equal(a1.x, a2.x)
    assert torch.equal(a1.sign_bits, a2.sign_bits)
    w3, a3 = W.tiny(seed=1)
    assert not torch.equal(w1.codes, w3.codes)


def test_rtn_ranges_and_reconstruction():
    w, _ = W.tiny()
    assert w.codes.shape == (512, 256) and w.codes.dtype == torch.uint8
    assert int(w.codes.max()) <= 15
    assert w.scales.shape == (512, 2) and bool((w.scales > 0).all())
    # RTN keeps every weight within half a step (plus fp16 rounding of s and z)
    g = torch.Generator().manual_seed(0)
    wf = torch.randn(4, 256, generator=g) * 0.02
    q, s, z = W.rtn_quantise(wf, 4)
    rec = s.float().repeat_interleave(128, 1) * (q.float() - z.float().repeat_interleave(128, 1))
    step = s.float().repeat_interleave(128, 1)
    assert bool(((rec - wf).abs() <= 0.5 * step + 2e-3 * wf.abs().max()).all())


def test_outlier_count():
    N, K = 64, 256
    base = W.draw_weight(N, K, 4, outliers=False)
    out = W.draw_weight(N, K, 4, outliers=True)
    assert base.codes.shape == out.codes.shape
    n_out = int(math.floor(0.001 * N * K + 0.5))
    assert n_out == 16


def test_block_bits_share():
    bb = W.draw_block_bits(9728)
    assert bb.shape == (152,)
    assert int((bb == 8).sum()) == 26 and int((bb == 6).sum()) == 126


def test_mixed_weight_ranges():
    bb = torch.tensor([6, 8], dtype=torch.uint8)
    w = W.draw_weight(128, 256, 0, block_bits=bb)
    assert int(w.codes[:64].max()) <= 63
    assert int(w.codes[64:].max()) > 63


def test_stack_shapes():
    lin = W.stack_linears()
    assert len(lin) == 36 * 7 + 1
    assert lin[-1] == ("lm_head", 2560, 151936, 8)
    total_weights = sum(K * N for _, K, N, _ in lin)
    assert total_weights == 36 * (2560 * 4096 + 2 * 2560 * 1024 + 4096 * 2560 + 2 * 2560 * 9728 + 9728 * 2560) + 2560 * 151936


def test_concat_rows():
    ws = [W.draw_weight(n, 256, 4, seed=0, index=i + 1) for i, n in enumerate((64, 3, 128))]
    f = W.concat_rows(ws)
    assert (f.N, f.K, f.bits) == (195, 256, 4)
    assert torch.equal(f.codes[64:67], ws[1].codes) and torch.equal(f.scales[67:], ws[2].scales)
    assert torch.equal(f.zeros[:64], ws[0].zeros)
    try:
        W.concat_rows([ws[0], W.draw_weight(8, 128, 4, seed=0)])
    except AssertionError:
        pass
    else:
        raise AssertionError("rows of different K were fused")


def test_stack_fused_first_projection():
    """The fused q/k/v of layer 0 is the stack's q, k and v rows in order and
    reads the x of q."""
    import itertools
    name, f, a = next(W.stack_fused())
    sep = list(itertools.islice(W.stack(), 3))
    assert name == "layers.0.qkv_proj" and f.N == 6144 and f.K == 2560 and f.bits == 6
    assert torch.equal(f.codes, torch.cat([w.codes for _, w, _ in sep]))
    assert torch.equal(f.scales, torch.cat([w.scales for _, w, _ in sep]))
    assert torch.equal(a.x, sep[0][2].x) and torch.equal(a.sign_bits, sep[0][2].sign_bits)
    assert [n for n, _ in W.STACK_FUSED] == ["qkv_proj", "o_proj", "gate_up_proj", "down_proj"]
