"""CPU checks of the adversarial parity inputs (tests/adversarial.py): the
activation blocks rotate to the closed forms they are built for, and the
weights have the zero points and scales they are meant to stress."""
import numpy as np

from oracle import qlin_oracle as O

import adversarial as A

K = 1024


def _rot(a):
    return O.rht64(a.x.numpy(), a.sign_bits.numpy().view(np.uint32))


def test_wide_blocks_rotate_to_sqrt128_times_integers():
    kinds = ["wide", "plain"] * (K // 256)
    a, kinds = A.activation(3, K, seed=1, kinds=kinds)
    xr = _rot(a)
    unit = np.sqrt(128.0) * 2.0 ** -A.WIDE_EXP
    for j, kind in enumerate(kinds):
        if kind != "wide":
            continue
        v = xr[:, 128 * j:128 * (j + 1)] / unit
        assert np.allclose(v, np.rint(v), atol=1e-9)
        mag = np.sort(np.abs(np.rint(v)), axis=1)
        assert (mag[:, -1] == A.BIG).all() and (mag[:, :-1] == 1).all()
        # the 64-value run holding the large value spans a factor 1023
        runs = np.abs(v).reshape(3, 2, 64)
        spans = runs.max(axis=2) / runs.min(axis=2)
        assert np.isclose(spans.max(axis=1), A.BIG).all()


def test_subnormal_blocks_are_subnormal_before_and_after_rotation():
    kinds = ["subnormal"] * (K // 128)
    a, _ = A.activation(2, K, seed=2, kinds=kinds)
    x = a.x.numpy().astype(np.float64)
    tiny = 2.0 ** -14
    assert (np.abs(x) < tiny).all()
    xr = _rot(a)
    v = xr / (np.sqrt(128.0) * 2.0 ** -A.SUBNORMAL_EXP)
    assert np.allclose(v, np.rint(v), atol=1e-9) and set(np.abs(np.rint(v)).ravel()) <= {1.0, 2.0, 3.0}
    r16 = O.rht16(a.x.numpy(), a.sign_bits.numpy().view(np.uint32)).astype(np.float64)
    assert (r16 != 0).all() and (np.abs(r16) < tiny).all()
    # fp16 rounding of these values is a relative error of several per cent
    assert np.abs(r16 / xr - 1).max() > 0.02


def test_subnormal_groups_carry_a_share_of_the_output():
    kinds = (["subnormal", "wide", "plain", "subnormal"] * K)[:K // 128]
    a, kinds = A.activation(2, K, seed=3, kinds=kinds)
    w = A.block_weight(128, K, 6, seed=4, kinds=kinds)
    ref = A.reference_r16(w, a)
    keep = np.repeat(np.array([k != "subnormal" for k in kinds]), 128)
    xr = O.rht16(a.x.numpy(), a.sign_bits.numpy().view(np.uint32)).astype(np.float64)
    wd = O.dequant64(w.codes.numpy(), w.scales.numpy(), w.zeros.numpy())
    assert O.parity_errors(xr[:, keep] @ wd[:, keep].T, ref)[1] > 0.1
    assert np.abs(wd).max() < 65504  # the fp16 weights stay finite


def test_adversarial_weights():
    for bits in (3, 4, 6, 8):
        w = A.weight(256, K, bits, seed=bits)
        z = w.zeros.numpy().astype(np.float64)
        s = w.scales.numpy().astype(np.float64)
        q = 2.0 ** bits
        assert (z < 0).any() and (z > 0).any() and (np.abs(z) > q).any() and (np.abs(z) <= 4 * q).all()
        assert (z != np.rint(z)).any()
        assert (s < 0).any() and (s > 0).any()
        assert np.abs(s).max() / np.abs(s[s != 0]).min() > 2.0 ** 12
        wd = O.dequant64(w.codes.numpy(), w.scales.numpy(), w.zeros.numpy())
        assert np.abs(wd).max() <= 4.0 * 1.001
