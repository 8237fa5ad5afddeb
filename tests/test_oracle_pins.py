"""Pins for the CPU oracle, independent of the oracle's own code.

Each test checks one oracle function against something that is not a retyped
copy of it: a hand-derived layout example, a big-integer formulation of the
bit stream, scipy's Hadamard matrix, an independent butterfly transform, exact
rational arithmetic, brute-force loops, closed forms, or figures the pages
print (``tests/golden/page_figures.json``).  A dropped term, a wrong sign or
index, or a transposed operand in the oracle fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import qlin_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


def _bigint_stream(codes_row, b):
    """Row bit stream as one Python integer: sum_k q_k << (b*k)."""
    v = 0
    for k, q in enumerate(codes_row):
        v |= (int(q) & ((1 << b) - 1)) << (b * k)
    return v.to_bytes(len(codes_row) * b // 8, "little")


# ---------------------------------------------------------------- layout ----

def test_int4_word_example():
    # codes 0..7 in the first eight positions -> little-endian word 0x76543210
    codes = np.zeros((1, 128), dtype=np.uint8)
    codes[0, :8] = np.arange(8)
    p = O.pack(codes, bits=4)
    assert p[:4].view("<u4")[0] == 0x76543210
    assert len(p) == 64


def test_int8_word_example():
    codes = np.zeros((1, 128), dtype=np.uint8)
    codes[0, :4] = [0x11, 0x22, 0x33, 0x44]
    p = O.pack(codes, bits=8)
    assert p[:4].view("<u4")[0] == 0x44332211


def test_int3_straddling_code():
    # code 10 occupies stream bits 30..32: its two low bits end word 0, its top
    # bit starts word 1.  q10 = 0b101 -> word0 bit30 = 1, bit31 = 0, word1 bit0 = 1.
    codes = np.zeros((1, 128), dtype=np.uint8)
    codes[0, 10] = 5
    w = O.pack(codes, bits=3)[:8].view("<u4")
    assert w[0] == (1 << 30)
    assert w[1] == 1
    # one group of 128 int3 codes is exactly 12 words
    assert len(O.pack(codes, bits=3)) == 48


def test_int6_straddling_code():
    # code 5 occupies stream bits 30..35: q5 = 0b110101 -> word0 bits 30,31 = 1,0;
    # word1 bits 0..3 = q5 >> 2 = 0b1101.
    codes = np.zeros((1, 128), dtype=np.uint8)
    codes[0, 5] = 0b110101
    w = O.pack(codes, bits=6)[:8].view("<u4")
    assert w[0] == (1 << 30)
    assert w[1] == 0b1101


@pytest.mark.parametrize("b", [3, 4, 6, 8])
def test_pack_matches_bigint_stream(b):
    rng = np.random.default_rng(b)
    codes = rng.integers(0, 1 << b, size=(3, 256), dtype=np.uint8)
    p = O.pack(codes, bits=b)
    row = 256 * b // 8
    for n in range(3):
        assert p[n * row:(n + 1) * row].tobytes() == _bigint_stream(codes[n], b)


def test_pack_ignores_high_bits():
    codes = np.full((1, 128), 0xFF, dtype=np.uint8)
    for b in (3, 4, 6):
        assert np.array_equal(O.unpack(O.pack(codes, bits=b), 1, 128, bits=b),
                              np.full((1, 128), (1 << b) - 1, dtype=np.uint8))


@pytest.mark.parametrize("b", [3, 4, 6, 8])
def test_roundtrip_uniform(b):
    rng = np.random.default_rng(10 + b)
    N, K = 7, 384
    for codes in (rng.integers(0, 1 << b, size=(N, K), dtype=np.uint8),
                  np.zeros((N, K), dtype=np.uint8),
                  np.full((N, K), (1 << b) - 1, dtype=np.uint8)):
        p = O.pack(codes, bits=b)
        assert len(p) == N * K * b // 8
        assert np.array_equal(O.unpack(p, N, K, bits=b), codes)


def test_roundtrip_mixed_and_offsets():
    rng = np.random.default_rng(3)
    N, K = 256, 256
    bb = np.array([6, 8, 8, 6], dtype=np.uint8)
    row_b = np.repeat(bb, 64).astype(np.int64)
    codes = (rng.integers(0, 256, size=(N, K)) % (1 << row_b[:, None])).astype(np.uint8)
    p = O.pack(codes, block_bits=bb)
    off = O.row_byte_offsets(N, K, block_bits=bb)
    # block j spans 64 rows of K codes of its width, blocks back to back
    expect = np.concatenate([[0], np.cumsum(np.repeat(bb.astype(np.int64) * K // 8, 64))])
    assert np.array_equal(off, expect)
    assert len(p) == off[-1]
    assert np.array_equal(O.unpack(p, N, K, block_bits=bb), codes)
    # rows of the second block are the 8-bit bytes themselves
    assert np.array_equal(p[off[64]:off[65]], codes[64])
    # sampled-row unpack agrees with full unpack
    rows = [0, 63, 64, 200, 255]
    assert np.array_equal(O.unpack(p, N, K, block_bits=bb, rows=rows), codes[rows])


def test_mixed_width_page_figures():
    """212 blocks of 64 rows upgraded 6 -> 8 bits hold 36,012,032 weights; with a
    64-row block spanning all of K this is 199 blocks at K=2560 plus 13 at K=4096.
    The oracle's byte accounting must charge exactly 2 extra bits per weight."""
    fig = json.load(open(GOLDEN))["mixed_width_upgrade"]
    rows = fig["block_rows"]
    sols = [(a, fig["blocks_upgraded"] - a) for a in range(fig["blocks_upgraded"] + 1)
            if a * rows * 2560 + (fig["blocks_upgraded"] - a) * rows * 4096 == fig["weights_upgraded"]]
    assert sols == [(199, 13)]
    extra = 0
    for nblocks, K in ((199, 2560), (13, 4096)):
        N = nblocks * rows
        lo = O.row_byte_offsets(N, K, block_bits=np.full(nblocks, fig["from_bits"]))[-1]
        hi = O.row_byte_offsets(N, K, block_bits=np.full(nblocks, fig["to_bits"]))[-1]
        extra += hi - lo
    assert extra * 8 == fig["weights_upgraded"] * (fig["to_bits"] - fig["from_bits"])


def test_traffic_cut_page_figure():
    """Reading 3-4-bit codes instead of 16-bit weights cuts weight bytes by about 4-5x."""
    fig = json.load(open(GOLDEN))["weight_traffic_cut"]
    N, K = 64, 2560
    for b in fig["code_bits"]:
        cut = (N * K * fig["dense_bits"] / 8) / O.row_byte_offsets(N, K, bits=b)[-1]
        assert fig["cut_low"] <= cut <= fig["cut_high"]
        assert cut == pytest.approx(16 / b)
    # scales and zeros add 32 bits per 128 codes
    assert O.algorithmic_bytes(N, K, bits=4) * 8 == N * K * (4 + 32 / 128)


# ----------------------------------------------------------------- dequant --

def test_dequant64_exact_rational():
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 16, size=(2, 256), dtype=np.uint8)
    s = rng.uniform(1e-3, 0.1, size=(2, 2)).astype(np.float16)
    z = rng.uniform(0, 15, size=(2, 2)).astype(np.float16)
    w = O.dequant64(codes, s, z)
    for n in range(2):
        for k in range(0, 256, 37):
            exact = Fraction(float(s[n, k // 128])) * (int(codes[n, k]) - Fraction(float(z[n, k // 128])))
            assert w[n, k] == float(exact)  # product of an 11-bit and a <=19-bit value: exact in fp64


def _fp32(v: float) -> float:
    return float(np.float32(v))


def test_dequant16_independent_rounding():
    """fp16(fp32(fp32(s) * fp32(q - z))) computed with exact float64 steps and an
    explicit rounding to fp32 after each: q - z and s * t are exact in float64."""
    rng = np.random.default_rng(6)
    codes = rng.integers(0, 256, size=(4, 128), dtype=np.uint8)
    s = rng.uniform(1e-4, 0.5, size=(4, 1)).astype(np.float16)
    z = rng.uniform(-3, 260, size=(4, 1)).astype(np.float16)
    w16 = O.dequant16(codes, s, z)
    for n in range(4):
        for k in range(128):
            t = _fp32(float(codes[n, k]) - float(z[n, 0]))
            p = _fp32(float(s[n, 0]) * t)
            assert w16[n, k].tobytes() == np.float16(np.float32(p)).tobytes()


def test_dequant16_hand_cases():
    # s = 0.25, z = 1.5, q = 3 -> 0.375 exactly
    assert O.dequant16(np.array([[3] + [0] * 127], np.uint8), np.array([[0.25]], np.float16),
                       np.array([[1.5]], np.float16))[0, 0] == np.float16(0.375)
    # q == z gives +0; q < z gives a negative weight
    w = O.dequant16(np.array([[2, 1] + [0] * 126], np.uint8), np.array([[1.0]], np.float16),
                    np.array([[2.0]], np.float16))
    assert w[0, 0] == 0 and w[0, 1] == np.float16(-1.0)


# ---------------------------------------------------------------- hadamard --

def test_hadamard_orthogonal_and_scipy():
    H = O.hadamard(128)
    assert np.array_equal(H @ H.T, 128 * np.eye(128, dtype=np.int64))
    scipy_linalg = pytest.importorskip("scipy.linalg")
    assert np.array_equal(H, scipy_linalg.hadamard(128))


def test_hadamard_sylvester_recursion():
    H = np.array([[1]], dtype=np.int64)
    while H.shape[0] < 128:
        H = np.block([[H, H], [H, -H]])
    assert np.array_equal(O.hadamard(128), H)


def _butterfly(v):
    """Independent in-place FWHT: log2(n) stages of (u, v) -> (u + v, u - v)."""
    v = np.array(v, dtype=np.float64)
    n = v.shape[-1]
    h = 1
    stages = 0
    while h < n:
        for i in range(0, n, 2 * h):
            a = v[..., i:i + h].copy()
            b = v[..., i + h:i + 2 * h].copy()
            v[..., i:i + h] = a + b
            v[..., i + h:i + 2 * h] = a - b
        h *= 2
        stages += 1
    return v, stages


def test_rht_matches_butterfly():
    fig = json.load(open(GOLDEN))["hadamard"]
    rng = np.random.default_rng(7)
    M, K = 3, 384
    x = rng.standard_normal((M, K))
    sb = rng.integers(0, 2 ** 32, size=K // 32, dtype=np.uint64).astype(np.uint32)
    d = np.array([-1.0 if (int(sb[k // 32]) >> (k % 32)) & 1 else 1.0 for k in range(K)])
    ref = np.empty_like(x)
    for b0 in range(0, K, 128):
        out, stages = _butterfly(x[:, b0:b0 + 128] * d[b0:b0 + 128])
        assert stages == fig["add_sub_stages"]
        ref[:, b0:b0 + 128] = out / math.sqrt(fig["block"])
    assert np.allclose(O.rht64(x, sb), ref, rtol=0, atol=1e-12)


def test_rht_preserves_norm_per_block():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((4, 512))
    sb = rng.integers(0, 2 ** 32, size=16, dtype=np.uint64).astype(np.uint32)
    xr = O.rht64(x, sb)
    for b0 in range(0, 512, 128):
        assert np.allclose(np.linalg.norm(xr[:, b0:b0 + 128], axis=1),
                           np.linalg.norm(x[:, b0:b0 + 128], axis=1), rtol=1e-13)


def test_rht_unit_vector_closed_form():
    H = O.hadamard(128)
    K = 256
    zeros = np.zeros(K // 32, dtype=np.uint32)
    for j in (0, 1, 77, 128 + 5):
        e = np.zeros((1, K))
        e[0, j] = 1.0
        out = O.rht64(e, zeros)[0]
        blk = (j // 128) * 128
        expect = np.zeros(K)
        expect[blk:blk + 128] = H[:, j - blk] / math.sqrt(128)
        assert np.allclose(out, expect, atol=1e-15)
        # flipping the sign bit of index j negates the result
        sb = zeros.copy()
        sb[j // 32] = np.uint32(1 << (j % 32))
        assert np.allclose(O.rht64(e, sb)[0], -expect, atol=1e-15)


def test_rht_blocks_independent():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((1, 256))
    sb = rng.integers(0, 2 ** 32, size=8, dtype=np.uint64).astype(np.uint32)
    y0 = O.rht64(x, sb)
    x2 = x.copy()
    x2[0, 200] += 3.0
    y1 = O.rht64(x2, sb)
    assert np.array_equal(y0[0, :128], y1[0, :128])
    assert not np.allclose(y0[0, 128:], y1[0, 128:])


def test_rotation_invariance():
    """Rotating both activation and weight rows leaves every product unchanged."""
    rng = np.random.default_rng(11)
    K = 384
    x = rng.standard_normal((2, K))
    w = rng.standard_normal((5, K))
    sb = rng.integers(0, 2 ** 32, size=K // 32, dtype=np.uint64).astype(np.uint32)
    assert np.allclose(O.rht64(x, sb) @ O.rht64(w, sb).T, x @ w.T, rtol=1e-12, atol=1e-12)


def test_rht16_is_one_rounding():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((2, 128)).astype(np.float16)
    sb = np.zeros(4, dtype=np.uint32)
    assert np.array_equal(O.rht16(x, sb), O.rht64(x, sb).astype(np.float16))


# ------------------------------------------------------------------ matmul --

def test_linear_bruteforce_tiny():
    rng = np.random.default_rng(13)
    M, N, K = 2, 3, 256
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    s = rng.uniform(0.01, 0.1, size=(N, K // 128)).astype(np.float16)
    z = rng.uniform(0, 15, size=(N, K // 128)).astype(np.float16)
    x = rng.standard_normal((M, K)).astype(np.float16)
    sb = rng.integers(0, 2 ** 32, size=K // 32, dtype=np.uint64).astype(np.uint32)
    H = O.hadamard(128)
    y = O.linear64(x, codes, s, z, sb)
    for m in range(M):
        # rotated activation by explicit loops
        xr = [0.0] * K
        for k in range(K):
            sign = -1.0 if (int(sb[k // 32]) >> (k % 32)) & 1 else 1.0
            blk, i = divmod(k, 128)
            for j in range(128):
                sj = -1.0 if (int(sb[(blk * 128 + j) // 32]) >> ((blk * 128 + j) % 32)) & 1 else 1.0
                xr[k] += H[i, j] * sj * float(x[m, blk * 128 + j])
            xr[k] /= math.sqrt(128)
            del sign
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += xr[k] * float(s[n, k // 128]) * (int(codes[n, k]) - float(z[n, k // 128]))
            assert y[m, n] == pytest.approx(acc, rel=1e-12, abs=1e-12)


def test_linear_torch_library_fp64():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(14)
    M, N, K = 4, 16, 512
    codes = rng.integers(0, 8, size=(N, K), dtype=np.uint8)
    s = rng.uniform(0.01, 0.1, size=(N, K // 128)).astype(np.float16)
    z = rng.uniform(0, 7, size=(N, K // 128)).astype(np.float16)
    x = rng.standard_normal((M, K)).astype(np.float16)
    sb = rng.integers(0, 2 ** 32, size=K // 32, dtype=np.uint64).astype(np.uint32)
    xr = torch.from_numpy(O.rht64(x, sb))
    w = torch.from_numpy(O.dequant64(codes, s, z))
    ref = torch.nn.functional.linear(xr, w).numpy()
    assert np.allclose(O.linear64(x, codes, s, z, sb), ref, rtol=1e-12, atol=1e-12)


def test_linear_integer_special_case():
    """s = 1, z = 0, all signs +1 and x = row j of H: rht(x) = sqrt(128) e_j, so
    Y[:, n] = sqrt(128) * q[n, j] (this fails if the weight is transposed)."""
    rng = np.random.default_rng(15)
    N, K = 6, 256
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    s = np.ones((N, K // 128), np.float16)
    z = np.zeros((N, K // 128), np.float16)
    H = O.hadamard(128)
    for j in (3, 128 + 100):
        x = np.zeros((1, K))
        blk = (j // 128) * 128
        x[0, blk:blk + 128] = H[j - blk, :]
        y = O.linear64(x, codes, s, z, np.zeros(K // 32, np.uint32))
        assert np.allclose(y[0], math.sqrt(128) * codes[:, j].astype(np.float64), rtol=1e-13, atol=1e-12)


def test_parity_errors():
    r = np.array([[1.0, -2.0, 4.0]])
    assert O.parity_errors(r, r) == (0.0, 0.0)
    a, f = O.parity_errors(r + np.array([[0.0, 0.0, 0.04]]), r)
    assert a == pytest.approx(0.01) and f == pytest.approx(0.04 / math.sqrt(21))


# ------------------------------------------------- offline weight side ----

def _sylvester(n):
    """H_n by the recursion H_2n = [[H, H], [H, -H]] (integers)."""
    h = np.array([[1]], dtype=np.int64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def _sign_of(sign_bits, k):
    return -1 if (int(sign_bits[k // 32]) >> (k % 32)) & 1 else 1


def test_rotate_weight32_exact_integer_sums():
    """fp16 rows are integer multiples of 2^-24: the rotation as exact integer
    sums, scaled once in fp64 by 1/sqrt(128) and rounded to fp32, equals the
    oracle's (including subnormal and near-maximal fp16 values in one block)."""
    rng = np.random.default_rng(11)
    w = (rng.standard_normal((3, 256)) * 0.02).astype(np.float16)
    w[0, :4] = [np.float16(6.0e-8), np.float16(-65504.0), np.float16(3.0e-5), np.float16(0.0)]
    w[1, 130] = np.float16(-1.0e4)
    sb = rng.integers(0, 2 ** 32, size=256 // 32, dtype=np.uint64).astype(np.uint32)
    H = _sylvester(128)
    inv = 1.0 / math.sqrt(128.0)
    got = O.rotate_weight32(w, sb)
    for n in range(w.shape[0]):
        units = [int(Fraction(float(v)) * (1 << 24)) for v in w[n].astype(np.float64)]
        for b0 in range(0, 256, 128):
            dv = [_sign_of(sb, b0 + j) * units[b0 + j] for j in range(128)]
            for i in range(128):
                exact = sum(int(H[i, j]) * dv[j] for j in range(128))
                want = np.float32(float(exact) * 2.0 ** -24 * inv)
                assert got[n, b0 + i].view(np.uint32) == want.view(np.uint32), (n, b0, i)


def test_rtn32_hand_cases():
    ramp = np.tile(np.arange(16, dtype=np.float32), 8)[None, :]          # 0..15: s = 1, z = -0
    c, s, z = O.rtn32(ramp, bits=4)
    assert np.array_equal(c[0], ramp[0].astype(np.uint8))
    assert s[0, 0] == np.float16(1.0) and z.view(np.uint16)[0, 0] == 0x8000
    const = np.full((1, 128), 0.5, np.float32)                            # constant group: s = 1, z = -0.5, q = 0
    c, s, z = O.rtn32(const, bits=6)
    assert s[0, 0] == np.float16(1.0) and z[0, 0] == np.float16(-0.5) and not c.any()
    zero = np.zeros((1, 128), np.float32)
    zero[0, ::3] = -0.0                                                   # mixed zeros: still z = -0, q = 0
    c, s, z = O.rtn32(zero, bits=3)
    assert s[0, 0] == np.float16(1.0) and z.view(np.uint16)[0, 0] == 0x8000 and not c.any()
    shifted = ramp + np.float32(32.0)                                     # 32..47: s = 1, z = -32
    c, s, z = O.rtn32(shifted, bits=4)
    assert np.array_equal(c[0], ramp[0].astype(np.uint8)) and z[0, 0] == np.float16(-32.0)


def _ulp16(v):
    v = abs(float(v))
    e = max(math.floor(math.log2(v)) if v > 0 else -14, -14)
    return Fraction(2) ** (e - 10)


@pytest.mark.parametrize("b", [3, 4, 6, 8])
def test_rtn32_extremes_rounding_and_error_bound(b):
    """Against exact rationals: s is within an fp16 rounding (plus the fp32
    quotient's) of (max - min) / (2^b - 1), z within one of -min / s; the
    group minimum maps to 0 and maximum to 2^b - 1; every code is the nearest
    integer to w / s + z up to the fp32 evaluation, so s (q - z) is within s/2
    (plus that rounding) of w."""
    rng = np.random.default_rng(b)
    wr = (rng.standard_normal((4, 384)) * rng.uniform(0.01, 3.0, size=(4, 1))).astype(np.float32)
    c, s, z = O.rtn32(wr, bits=b)
    qmax = (1 << b) - 1
    assert c.max() <= qmax
    for n in range(4):
        for g in range(3):
            grp = wr[n, 128 * g:128 * (g + 1)]
            cg = c[n, 128 * g:128 * (g + 1)]
            mn, mx = Fraction(float(grp.min())), Fraction(float(grp.max()))
            S, Z = Fraction(float(s[n, g])), Fraction(float(z[n, g]))
            assert abs(S - (mx - mn) / qmax) <= _ulp16(s[n, g]) / 2 + (mx - mn) / qmax * Fraction(1, 1 << 23)
            assert abs(Z - (-mn / S)) <= _ulp16(z[n, g]) / 2 + abs(mn / S) * Fraction(1, 1 << 23)
            assert cg[np.argmin(grp)] == 0 and cg[np.argmax(grp)] == qmax
            for v, q in zip(grp, cg):
                t = Fraction(float(v)) / S + Z
                assert abs(Fraction(int(q)) - t) <= Fraction(1, 2) + abs(t) * Fraction(1, 1 << 21), (v, q, t)


def test_rtn32_mixed_widths():
    rng = np.random.default_rng(5)
    wr = rng.standard_normal((128, 256)).astype(np.float32)
    c, _, _ = O.rtn32(wr, block_bits=[8, 3])
    assert c[:64].max() == 255 and c[64:].max() == 7


def test_quantize_rtn_folds_the_rotation():
    """The weight side uses the activations' signs and H: with x rotated by
    rht64 and W by quantize_rtn, the layer reproduces x W^T (int8: to the
    quantisation noise)."""
    rng = np.random.default_rng(9)
    N, K = 40, 512
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    x = rng.standard_normal((3, K)).astype(np.float16)
    sb = rng.integers(0, 2 ** 32, size=K // 32, dtype=np.uint64).astype(np.uint32)
    c, s, z = O.quantize_rtn(w, sb, bits=8)
    y = O.linear64(x, c, s, z, sb)
    y0 = x.astype(np.float64) @ w.astype(np.float64).T
    rel = np.linalg.norm(y - y0) / np.linalg.norm(y0)
    assert rel < 0.02, rel
    bad = O.linear64(x, c, s, z, sb ^ np.uint32(1))  # one activation sign flipped: no longer the same function
    assert np.linalg.norm(bad - y0) / np.linalg.norm(y0) > 5 * rel
