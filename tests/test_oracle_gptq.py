"""Pins of the oracle's GPTQ (error-compensated quantisation) against what the
mathematics fixes: a case worked by hand in exact binary fractions, the
reduction to round-to-nearest when the Hessian is a multiple of I, the exact
identity between the Hessian-weighted error and the column errors, the
optimal-brain-surgeon update computed from the inverse Hessian directly, the
advantage over round-to-nearest on a correlated Hessian, and the composition
with the weight rotation.  CPU only."""
import numpy as np
import pytest
import torch

from dequant_gemv_packed_b200 import workloads as W
from oracle import qlin_oracle as O


def test_hand_worked_case():
    """K = 4, one group of 4, 2-bit codes; every step exact in binary:
    grid from [0.5625, 0.25, 1, 0.625]: s = (1 - 0.25) / 3 = 0.25, z = -1;
    col 0: 0.5625/0.25 - 1 = 1.25 -> q 1, w^ 0.5, e = 0.0625 / 1;
           col 1 -= 0.0625 * 0.5 -> 0.21875, col 2 -= 0.0625 * 0.25 -> 0.984375;
    col 1: 0.875 - 1 = -0.125 -> q 0, w^ 0.25, e = -0.03125;
           col 2 -> 1.0, col 3 -> 0.625 + 0.03125 * 0.5 = 0.640625;
    col 2: 4 - 1 = 3 -> q 3, e = 0;  col 3: 2.5625 - 1 = 1.5625 -> q 2, e = -0.109375."""
    U = np.array([[1, .5, .25, 0], [0, 1, .5, .5], [0, 0, 1, .25], [0, 0, 0, 1]], np.float32)
    c, s, z, e = O.gptq_columns32(np.array([[0.5625, 0.25, 1.0, 0.625]]), U, np.array([3.0]), group=4)
    assert c.tolist() == [[1, 0, 3, 2]]
    assert s.tolist() == [[0.25]] and z.tolist() == [[-1.0]]
    assert e.tolist() == [[0.0625, -0.03125, 0.0, -0.109375]]


@pytest.mark.parametrize("bits,block_bits", [(3, None), (4, None), (6, None), (8, None), (None, [6, 8, 3])])
def test_identity_hessian_is_round_to_nearest(bits, block_bits):
    """H = I: the damped inverse factor is diagonal, nothing propagates, and
    GPTQ is round-to-nearest with the same grids, bit for bit."""
    rng = np.random.default_rng(bits or 0)
    N = 192 if block_bits else 50
    w = (rng.standard_normal((N, 256)) * 0.02).astype(np.float32)
    w[3, :128] = 0.0
    U = O.hessian_inverse_factor(np.eye(256)).astype(np.float32)
    assert np.count_nonzero(U - np.diag(np.diag(U))) == 0
    got = O.gptq32(w, U, bits, block_bits)
    ref = O.rtn32(w, bits, block_bits)
    for a, b in zip(got, ref):
        assert a.dtype == b.dtype and np.array_equal(a.view(np.uint8), b.view(np.uint8))


def _hessian(K, seed):
    x = W.draw_calibration(K, seed=seed).numpy()
    return O.hessian64(x)


def test_weighted_error_equals_column_errors():
    """With U^T U = H^-1, the final error E = w - w^ equals e U, so
    E H E^T = |e|^2 for every row (exact arithmetic; fp32 rounding here)."""
    rng = np.random.default_rng(1)
    K = 256
    H = _hessian(K, 1)
    Hd = H + 0.01 * np.mean(np.diag(H)) * np.eye(K)
    U = O.hessian_inverse_factor(H).astype(np.float32)
    w = (rng.standard_normal((32, K)) * 0.02).astype(np.float32)
    c, s, z, e = O.gptq_columns32(w, U, np.full(32, 15.0), 128)
    E = w.astype(np.float64) - O.dequant64(c, s, z)
    lhs = np.einsum("rk,kl,rl->r", E, Hd, E)
    rhs = (e.astype(np.float64) ** 2).sum(axis=1)
    assert np.allclose(lhs, rhs, rtol=2e-3), np.abs(lhs / rhs - 1).max()
    assert np.allclose(E, e.astype(np.float64) @ U.astype(np.float64), atol=1e-6)


def test_first_update_is_the_obs_step():
    """After column 0, column j holds w_j - (w_0 - w^_0) [H^-1]_0j / [H^-1]_00
    (the optimal-brain-surgeon update), with H^-1 from a plain inverse."""
    rng = np.random.default_rng(2)
    K = 128
    H = _hessian(K, 2)
    Hinv = np.linalg.inv(H + 0.01 * np.mean(np.diag(H)) * np.eye(K))
    U = O.hessian_inverse_factor(H).astype(np.float32)
    w = (rng.standard_normal((16, K)) * 0.02).astype(np.float32)
    c, s, z, e = O.gptq_columns32(w, U, np.full(16, 7.0), 128)
    w0hat = O.dequant64(c, s, z)[:, 0]
    # column 1 as quantised: e_1 U_11 + w^_1 (its error definition), before any later update
    w1_used = e[:, 1].astype(np.float64) * float(U[1, 1]) + O.dequant64(c, s, z)[:, 1]
    obs = w[:, 1] - (w[:, 0] - w0hat) * Hinv[0, 1] / Hinv[0, 0]
    assert np.allclose(w1_used, obs, atol=1e-6), np.abs(w1_used - obs).max()


def test_beats_round_to_nearest_on_correlated_hessian():
    """The Hessian-weighted error tr(E H E^T) of GPTQ is well below that of
    round-to-nearest on the same weights."""
    rng = np.random.default_rng(3)
    K = 512
    H = _hessian(K, 3)
    U = O.hessian_inverse_factor(H).astype(np.float32)
    w = (rng.standard_normal((64, K)) * 0.02).astype(np.float32)
    for bits in (3, 4):
        g = O.gptq32(w, U, bits)
        r = O.rtn32(w, bits)
        Eg = w - O.dequant64(*g)
        Er = w - O.dequant64(*r)
        lg = np.einsum("rk,kl,rl->", Eg, H, Eg)
        lr = np.einsum("rk,kl,rl->", Er, H, Er)
        assert lg < 0.8 * lr, (bits, lg / lr)


def test_composes_with_the_rotation():
    """quantize_gptq rotates first: with H = I it is quantize_rtn, bit for bit;
    and its codes are GPTQ of the rotated rows."""
    w = W.draw_fp16_weight(64, 256, seed=4).numpy()
    sb = W.draw_activation(1, 256, seed=4).sign_bits.numpy().view(np.uint32)
    I = O.hessian_inverse_factor(np.eye(256)).astype(np.float32)
    for a, b in zip(O.quantize_gptq(w, sb, I, 4), O.quantize_rtn(w, sb, 4)):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))
    H = _hessian(256, 4)
    U = O.hessian_inverse_factor(H).astype(np.float32)
    for a, b in zip(O.quantize_gptq(w, sb, U, 6), O.gptq32(O.rotate_weight32(w, sb), U, 6)):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


def test_factor_is_the_upper_cholesky_factor_of_the_damped_inverse():
    H = _hessian(128, 5)
    U = O.hessian_inverse_factor(H, damp=0.05)
    assert np.allclose(np.tril(U, -1), 0.0)
    Hd = H + 0.05 * np.mean(np.diag(H)) * np.eye(128)
    assert np.allclose(U.T @ U @ Hd, np.eye(128), atol=1e-8)
    assert (np.diag(U) > 0).all()


def test_calibration_draw():
    x = W.draw_calibration(1024, seed=0)
    assert x.shape == (2048, 1024) and x.dtype == torch.float32
    std = x.std(dim=0)
    assert int((std > 10).sum()) == 10  # round(1% of 1024) heavy channels, x8
    assert torch.equal(x, W.draw_calibration(1024, seed=0))
