"""GPU parity of the error-compensated offline quantiser (qlin_quantize_gptq)
against the oracle's quantize_gptq: codes, scales and zeros bit for bit, on
the same fp16 weights, signs and fp32 inverse-Hessian factor.  The factor is
computed once on the CPU from synthetic calibration inputs (rotated, since the
compensation runs in the rotated basis) and handed to both sides as an input.
"""
import numpy as np
import pytest
import torch

from dequant_gemv_packed_b200 import qlin as Q
from dequant_gemv_packed_b200 import workloads as W
from oracle import qlin_oracle as O

from parity import assert_close, np_u32, packed_on_device

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dequant_gemv_packed_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    Q.lib()


def _inputs(N, K, seed):
    w = W.draw_fp16_weight(N, K, seed=seed, index=N + K)
    a = W.draw_activation(1, K, seed=seed, index=N + K)
    sb = np_u32(a.sign_bits)
    xcal = W.draw_calibration(K, seed=seed, index=K)
    U = O.hessian_inverse_factor(O.hessian64(O.rht64(xcal.numpy(), sb))).astype(np.float32)
    return w, a, sb, U


def _gpu(N, K, bits, block_bits, w, a, U):
    d = Q.Desc(N, K, bits, block_bits)
    c, s, z = Q.qlin_quantize_gptq(d, w.to(DEV), a.sign_bits.to(DEV), torch.from_numpy(U).to(DEV))
    torch.cuda.synchronize()
    return d, c, s, z


def _same(got, ref, what):
    c, s, z = got
    rc, rs, rz = ref
    assert np.array_equal(c.cpu().numpy(), rc), f"{what}: codes differ ({int((c.cpu().numpy() != rc).sum())})"
    assert np.array_equal(s.cpu().numpy().view(np.uint16), rs.view(np.uint16)), f"{what}: scales differ"
    assert np.array_equal(z.cpu().numpy().view(np.uint16), rz.view(np.uint16)), f"{what}: zeros differ"


@pytest.mark.parametrize("N,K,bits", [(64, 256, 4), (77, 384, 3), (130, 512, 6), (33, 1280, 8), (1, 128, 4),
                                      (200, 2560, 3)])
def test_gptq_bit_exact(N, K, bits):
    """Ragged row counts (tiles of the trailing update cut by N), one group, many groups."""
    w, a, sb, U = _inputs(N, K, seed=bits)
    d, c, s, z = _gpu(N, K, bits, None, w, a, U)
    _same((c, s, z), O.quantize_gptq(w.numpy(), sb, U, bits), f"b{bits} N{N} K{K}")


def test_gptq_mixed_widths_bit_exact():
    bb = [6, 8, 3, 4, 6]
    N, K = 64 * len(bb), 768
    w, a, sb, U = _inputs(N, K, seed=11)
    d, c, s, z = _gpu(N, K, 0, bb, w, a, U)
    _same((c, s, z), O.quantize_gptq(w.numpy(), sb, U, None, bb), "mixed")


def test_gptq_gateup_shape_sampled_rows():
    """The gate/up shape (9728 x 2560, int4): GPTQ treats rows independently, so
    the oracle on sampled rows (with the same factor) fixes those rows."""
    N, K = 9728, 2560
    w = W.draw_fp16_weight(N, K, seed=0)
    a = W.draw_activation(1, K, seed=0)
    sb = np_u32(a.sign_bits)
    xcal = W.draw_calibration(K, seed=0)
    U = O.hessian_inverse_factor(O.hessian64(O.rht64(xcal.numpy(), sb))).astype(np.float32)
    d, c, s, z = _gpu(N, K, 4, None, w, a, U)
    rows = np.array([0, 1, 31, 32, 4095, 4864, 9000, N - 1])
    t = torch.as_tensor(rows, device=DEV)
    _same((c[t], s[t], z[t]), O.quantize_gptq(w.numpy()[rows], sb, U, 4), "gate/up rows")


def test_gptq_layer_and_objective():
    """The GPTQ weight packed and run through qlin_gemv matches the oracle layer,
    and its Hessian-weighted error is below round-to-nearest's on the same rows."""
    N, K = 256, 1024
    w, a, sb, U = _inputs(N, K, seed=5)
    d, c, s, z = _gpu(N, K, 4, None, w, a, U)
    packed = Q.qlin_pack(d, c)
    x = a.x.to(DEV)
    y = Q.qlin_gemv(d, packed, s, z, a.sign_bits.to(DEV), x)
    torch.cuda.synchronize()
    ref = O.linear64(a.x.numpy(), c.cpu().numpy(), s.cpu().numpy(), z.cpu().numpy(), sb)
    assert_close(y, ref, "gptq layer")
    rc, rs, rz = Q.qlin_quantize_rtn(d, w.to(DEV), a.sign_bits.to(DEV))
    wr = O.rotate_weight32(w.numpy(), sb).astype(np.float64)
    Hd = np.linalg.inv(U.astype(np.float64).T @ U.astype(np.float64))
    def objective(cc, ss, zz):
        E = wr - O.dequant64(cc.cpu().numpy(), ss.cpu().numpy(), zz.cpu().numpy())
        return float(np.einsum("rk,kl,rl->", E, Hd, E))
    assert objective(c, s, z) < 0.8 * objective(rc, rs, rz)


def test_gptq_identity_factor_is_rtn():
    """A diagonal factor: the GPU GPTQ equals the GPU round-to-nearest tool."""
    N, K = 96, 512
    w = W.draw_fp16_weight(N, K, seed=6)
    a = W.draw_activation(1, K, seed=6)
    U = O.hessian_inverse_factor(np.eye(K)).astype(np.float32)
    d, c, s, z = _gpu(N, K, 6, None, w, a, U)
    rc, rs, rz = Q.qlin_quantize_rtn(d, w.to(DEV), a.sign_bits.to(DEV))
    assert torch.equal(c, rc) and torch.equal(s.view(torch.int16), rs.view(torch.int16))
    assert torch.equal(z.view(torch.int16), rz.view(torch.int16))


def test_gptq_rejects_small_workspace():
    N, K = 64, 256
    d = Q.Desc(N, K, 4)
    w = torch.zeros(N, K, dtype=torch.float16, device=DEV)
    sb = torch.zeros(K // 32, dtype=torch.int32, device=DEV)
    U = torch.eye(K, dtype=torch.float32, device=DEV)
    small = torch.empty(Q.qlin_gptq_workspace_bytes(d) - 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(Q.QlinError) as e:
        Q.qlin_quantize_gptq(d, w, sb, U, workspace=small)
    assert e.value.status == -6
