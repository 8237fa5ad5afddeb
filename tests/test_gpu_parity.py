"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact: packed bytes, unpacked codes, fp16 dequantised weights.
RHT: within one fp16 ulp of the rounded fp64 transform.
Layer outputs: max|y - y_ref| <= 2e-3 max|y_ref| and relative Frobenius error
<= 1e-3 against the fp64 oracle, for every workload shape (tiny int4, gate/up
int4, down-proj int3 at M = 1/4/16, the 36-layer int6 stack with the int8
lm_head, the mixed int6/int8 prefill GEMM at M = 256/1024/2048) plus ragged
and degenerate shapes.
"""
import dataclasses

import numpy as np
import pytest
import torch

from dequant_gemv_packed_b200 import qlin as Q
from dequant_gemv_packed_b200 import workloads as W
from oracle import qlin_oracle as O

from parity import assert_close, assert_dot_bound, host, np_u32, oracle_rows, packed_on_device, sample_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dequant_gemv_packed_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    Q.lib()


def _rand_weight(N, K, bits, seed, block_bits=None):
    w = W.draw_weight(N, K, bits, seed=seed, block_bits=None if bits else torch.as_tensor(block_bits, dtype=torch.uint8))
    return w.to(DEV)


# ------------------------------------------------------------- bit-exact ------

@pytest.mark.parametrize("bits", [3, 4, 6, 8])
@pytest.mark.parametrize("N,K", [(77, 384), (1, 128), (130, 2560)])
def test_pack_unpack_bit_exact(bits, N, K):
    rng = np.random.default_rng(bits * 1000 + N)
    codes = rng.integers(0, 256, size=(N, K), dtype=np.uint8)  # high bits must be ignored
    d = Q.Desc(N, K, bits)
    packed = Q.qlin_pack(d, torch.from_numpy(codes).to(DEV))
    ref = O.pack(codes, bits=bits)
    got = packed.cpu().numpy()
    assert got[:len(ref)].tobytes() == ref.tobytes()
    back = Q.qlin_unpack(d, packed).cpu().numpy()
    assert np.array_equal(back, codes & ((1 << bits) - 1))


def test_pack_unpack_mixed_bit_exact():
    bb = np.array([6, 8, 3, 4, 8, 6], dtype=np.uint8)
    N, K = 64 * len(bb), 640
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    d = Q.Desc(N, K, 0, bb)
    packed = Q.qlin_pack(d, torch.from_numpy(codes).to(DEV)).cpu().numpy()
    ref = O.pack(codes, block_bits=bb)
    assert packed[:len(ref)].tobytes() == ref.tobytes()
    # block table: starts (16-byte units) and widths
    t0 = (len(ref) + 15) // 16 * 16
    starts = packed[t0:t0 + 4 * (len(bb) + 1)].view(np.uint32)
    off = O.row_byte_offsets(N, K, block_bits=bb)
    assert np.array_equal(starts.astype(np.int64) * 16, off[::64])
    assert np.array_equal(packed[t0 + 4 * (len(bb) + 1):t0 + 4 * (len(bb) + 1) + len(bb)], bb)
    back = Q.qlin_unpack(d, torch.from_numpy(packed).to(DEV)).cpu().numpy()
    mask = (1 << np.repeat(bb.astype(np.int64), 64)) - 1
    assert np.array_equal(back, codes & mask[:, None])


@pytest.mark.parametrize("bits", [3, 4, 6, 8, 0])
def test_dequant_bit_exact(bits):
    bb = [6, 8, 8, 4] if bits == 0 else None
    N, K = (256 if bits == 0 else 200), 384
    w = _rand_weight(N, K, bits, seed=bits + 7, block_bits=bb)
    d, packed = packed_on_device(w)
    got = Q.qlin_dequant(d, packed, w.scales, w.zeros).cpu().numpy()
    ref = O.dequant16(w.codes.cpu().numpy(), w.scales.cpu().numpy(), w.zeros.cpu().numpy())
    assert got.view(np.uint16).tobytes() == ref.view(np.uint16).tobytes()


def test_dequant_bit_exact_adversarial_scales():
    """Arbitrary fp16 scales and zeros (negative, tiny, large, non-integer)."""
    rng = np.random.default_rng(3)
    N, K = 64, 256
    codes = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    s = (rng.standard_normal((N, 2)) * np.exp(rng.uniform(-9, 4, (N, 2)))).astype(np.float16)
    z = (rng.standard_normal((N, 2)) * 100).astype(np.float16)
    d = Q.Desc(N, K, 8)
    packed = Q.qlin_pack(d, torch.from_numpy(codes).to(DEV))
    got = Q.qlin_dequant(d, packed, torch.from_numpy(s).to(DEV), torch.from_numpy(z).to(DEV)).cpu().numpy()
    ref = O.dequant16(codes, s, z)
    assert got.view(np.uint16).tobytes() == ref.view(np.uint16).tobytes()


def _wide_zero_points(rng, shape):
    """fp16 zero points of every magnitude, subnormals included, either sign."""
    z = np.exp(rng.uniform(-17.5, 6.0, shape)) * rng.choice([-1.0, 1.0], shape)
    return z.astype(np.float16)


@pytest.mark.parametrize("bits", [3, 4, 6, 8])
def test_dequant_bit_exact_tiny_zero_points(bits):
    """Zero points down to the fp16 subnormals: fp32(q) - z is then often not
    exact, so the two fp32 roundings (subtract, multiply) both show."""
    rng = np.random.default_rng(11 + bits)
    N, K = 96, 512
    codes = rng.integers(0, 1 << bits, size=(N, K), dtype=np.uint8)
    s = (np.exp(rng.uniform(-14, 3, (N, K // 128))) * rng.choice([-1.0, 1.0], (N, K // 128))).astype(np.float16)
    z = _wide_zero_points(rng, (N, K // 128))
    zk = np.repeat(z.astype(np.float64), 128, axis=1)
    inexact = (codes.astype(np.float32) - zk.astype(np.float32)).astype(np.float64) != codes - zk
    assert inexact.mean() > 0.05
    d = Q.Desc(N, K, bits)
    packed = Q.qlin_pack(d, torch.from_numpy(codes).to(DEV))
    got = Q.qlin_dequant(d, packed, torch.from_numpy(s).to(DEV), torch.from_numpy(z).to(DEV)).cpu().numpy()
    ref = O.dequant16(codes, s, z)
    assert got.view(np.uint16).tobytes() == ref.view(np.uint16).tobytes()


@pytest.mark.parametrize("bits", [3, 4, 6, 8])
def test_gemm_wide_zero_points(bits):
    """The GEMM dequantises in tensor memory with its own code extraction:
    arbitrary zero points (tiny, subnormal, negative, large) and scales of
    either sign, against the oracle."""
    rng = np.random.default_rng(21 + bits)
    N, K, M = 320, 1280, 96
    w = _rand_weight(N, K, bits, seed=5 + bits)
    G = K // 128
    s = (np.exp(rng.uniform(-12, -6, (N, G))) * rng.choice([-1.0, 1.0], (N, G))).astype(np.float16)
    z = _wide_zero_points(rng, (N, G))
    w = dataclasses.replace(w, scales=torch.from_numpy(s).to(DEV), zeros=torch.from_numpy(z).to(DEV))
    a = W.draw_activation(M, K, seed=bits).to(DEV)
    d, packed = packed_on_device(w)
    y = Q.qlin_gemm(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
    torch.cuda.synchronize()
    assert_close(y, oracle_rows(w, a), f"gemm wide zeros b{bits}")
    assert_dot_bound(y, w, a, what=f"gemm wide zeros b{bits}")


# ------------------------------------------------------------------- rht ------

def _ulp16(v):
    v = np.abs(v).astype(np.float16)
    return (np.nextafter(v, np.float16(np.inf)) - v).astype(np.float64)


@pytest.mark.parametrize("M,K", [(1, 128), (3, 384), (16, 9728), (257, 2560)])
def test_rht_within_one_ulp(M, K):
    a = W.draw_activation(M, K, seed=M)
    ref = O.rht64(a.x.numpy(), np_u32(a.sign_bits))
    got = Q.qlin_rht(a.x.to(DEV), a.sign_bits.to(DEV)).float().cpu().numpy()
    err = np.abs(got - ref)
    # one fp16 ulp of the exact value; values far below the block's scale may
    # additionally carry the fp32 rounding of the butterfly sums
    tol = _ulp16(ref) + 1e-6 * np.abs(a.x.float().numpy()).max()
    assert (err <= tol).all(), float((err - tol).max())


# --------------------------------------------------------------- gemv ---------

def _gemv_case(w, a, rows=None, what=""):
    d, packed = packed_on_device(w)
    y = Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
    torch.cuda.synchronize()
    ref = oracle_rows(w, a, rows)
    got = y if rows is None else y[:, torch.as_tensor(rows, device=y.device)]
    if rows is None and w.N * w.K <= (1 << 22):
        assert_dot_bound(got, w, a, rows, what)
    return assert_close(got, ref, what)


def test_gemv_tiny_int4():
    w, a = W.tiny(device=DEV)
    _gemv_case(w, a, what="tiny")


def test_gemv_gateup_int4_full():
    w, a = W.gateup(device=DEV)
    _gemv_case(w, a, what="gateup")


@pytest.mark.parametrize("M", [1, 4, 16])
def test_gemv_down_int3_full(M):
    w, a = W.down(M=M, device=DEV)
    _gemv_case(w, a, what=f"down M={M}")


def test_gemv_stack_int6_int8_sampled():
    """Every linear of the 36-layer stack (int6) and the int8 lm_head, sampled rows."""
    worst = (0.0, 0.0)
    for i, (name, w, a) in enumerate(W.stack(device=DEV)):
        rows = sample_rows(w.N, 24, seed=i)
        r = _gemv_case(w, a, rows, what=name)
        worst = tuple(max(p, q) for p, q in zip(worst, r))
        del w, a
    print("stack worst rel errors", worst)


def test_gemv_fused_projections():
    """Fused q/k/v (N = 6144) and gate/up (N = 19456) of one layer: one weight of
    the members' rows and one x.  Sampled rows of every member against the
    oracle; all rows consistent with the members' separate calls."""
    lin = W.stack_linears()
    index = {name: i for i, (name, _, _, _) in enumerate(lin)}
    for members in (("q_proj", "k_proj", "v_proj"), ("gate_proj", "up_proj")):
        ids = [index[f"layers.0.{m}"] for m in members]
        ws = [W.draw_weight(lin[i][2], lin[i][1], lin[i][3], seed=0, index=i + 1, device=DEV) for i in ids]
        a = W.draw_activation(1, lin[ids[0]][1], seed=0, index=ids[0] + 1, device=DEV)
        f = W.concat_rows(ws)
        rows, r0 = [], 0
        for k, w in enumerate(ws):  # both ends of every member's row range
            rows.extend((r0 + sample_rows(w.N, 16, seed=k)).tolist())
            r0 += w.N
        _gemv_case(f, a, rows, what="+".join(members))
        d, packed = packed_on_device(f)
        y = Q.qlin_gemv(d, packed, f.scales, f.zeros, a.sign_bits, a.x)
        parts = []
        for w in ws:
            dw, pw = packed_on_device(w)
            parts.append(Q.qlin_gemv(dw, pw, w.scales, w.zeros, a.sign_bits, a.x))
        separate = torch.cat(parts, dim=1).double().cpu().numpy()
        assert_close(y, separate, what="+".join(members) + " fused vs separate calls")


@pytest.mark.parametrize("bits", [3, 4, 6, 8])
@pytest.mark.parametrize("N,K,M", [(77, 384, 5), (333, 1280, 16), (64, 9728, 2)])
def test_gemv_ragged(bits, N, K, M):
    w = _rand_weight(N, K, bits, seed=N + bits)
    a = W.draw_activation(M, K, seed=N).to(DEV)
    _gemv_case(w, a, what=f"b{bits} N{N} K{K} M{M}")


@pytest.mark.parametrize("bits", [3, 4, 6, 8])
@pytest.mark.parametrize("M", [1, 3])
def test_gemv_single_row(bits, M):
    """The smallest layer, N = 1 and K = 128 (one group, one rotation block),
    called 16 times with independent draws; the 16 outputs together meet the
    output tolerance (max-relative over the set), and each one the dot-product
    bound."""
    ys, refs = [], []
    for i in range(16):
        w = _rand_weight(1, 128, bits, seed=100 * bits + i)
        a = W.draw_activation(M, 128, seed=200 + i).to(DEV)
        d, packed = packed_on_device(w)
        y = Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
        torch.cuda.synchronize()
        assert_dot_bound(y, w, a, what=f"b{bits} N1 K128 M{M} draw {i}")
        ys.append(y.float().cpu().numpy())
        refs.append(oracle_rows(w, a))
    assert_close(np.concatenate(ys, axis=1), np.concatenate(refs, axis=1), f"b{bits} N1 K128 M{M} x16")


@pytest.mark.parametrize("bits", [3, 4, 6, 8])
@pytest.mark.parametrize("N,K", [(77, 384), (149, 128), (333, 1280), (64, 9728), (1337, 2560), (4440, 4096)])
def test_gemv_m1_shapes(bits, N, K):
    """M = 1 across row counts that leave ragged chunks and idle lanes, shares
    that fit shared memory whole and ones that cycle the stage ring."""
    w = _rand_weight(N, K, bits, seed=3 * N + bits)
    a = W.draw_activation(1, K, seed=N + 1).to(DEV)
    _gemv_case(w, a, what=f"b{bits} N{N} K{K} M1")


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", [(2368, 1280), (2516, 1408), (2900, 2560), (2960, 1408), (3108, 1280), (9728, 1280),
                                 (2368, 3072), (4736, 2816), (4736, 2304)])
def test_gemv_m1_integer_last_tile(bits, N, K):
    """The integer M = 1 kernel with a CTA's last 16-row tile full (2368 rows: 16 a CTA) or holding 1,
    3, 4 or 5 rows (the rows past the CTA's share read its last row and store nothing), including an
    odd number of groups (K = 1408: the last group pair has one group), and 17 to 24 groups (K = 2304,
    2560, 2816, 3072: the groups past the sixteenth take a second rotation round), against the oracle on
    every row."""
    w = _rand_weight(N, K, bits, seed=7 * N + bits)
    a = W.draw_activation(1, K, seed=N + 3).to(DEV)
    d, packed = packed_on_device(w)
    assert Q.qlin_gemv_plan(d, 1)["kernel"] == 3
    y = Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
    torch.cuda.synchronize()
    assert_close(y, oracle_rows(w, a), f"b{bits} N{N} K{K} M1")
    assert_dot_bound(y, w, a, what=f"b{bits} N{N} K{K} M1")


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", [(147, 2560), (1337, 2560), (2368, 5120), (1184, 8192), (296, 9728)])
def test_gemv_m1_integer_rotation_rounds(bits, N, K):
    """The integer M = 1 kernel when its 16 warps rotate x in several rounds:
    20 groups (four warps take a second block; on 148 CTAs and on an odd grid
    of 147), 40, 64 and 76 groups (three to five rounds), against the oracle on
    every row."""
    w = _rand_weight(N, K, bits, seed=11 * N + bits)
    a = W.draw_activation(1, K, seed=N + 5).to(DEV)
    d, packed = packed_on_device(w)
    assert Q.qlin_gemv_plan(d, 1)["kernel"] == 3
    y = Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
    torch.cuda.synchronize()
    assert_close(y, oracle_rows(w, a), f"b{bits} N{N} K{K} M1")
    assert_dot_bound(y, w, a, what=f"b{bits} N{N} K{K} M1")


@pytest.mark.parametrize("bits", [3, 4, 6, 8])
@pytest.mark.parametrize("N,K", [(4737, 1280), (5000, 1024), (6000, 1536), (4800, 4096), (5000, 128), (9728, 384)])
def test_gemv_m1_tall_shapes(bits, N, K):
    """M = 1 with 32 or more rows a CTA: several consumer iterations a chunk,
    ragged last chunks, 1 to 10 consumer warps."""
    w = _rand_weight(N, K, bits, seed=5 * N + bits)
    a = W.draw_activation(1, K, seed=N + 2).to(DEV)
    _gemv_case(w, a, what=f"b{bits} N{N} K{K} M1")


def _quantize_case(N, K, bits, block_bits=None, seed=0):
    w = W.draw_fp16_weight(N, K, seed=seed, index=N + K)
    w[0, :128] = 0.0                        # a zero group (rotated: zeros of both signs)
    w[-1, -128:] = 0.25                     # a constant group
    if N > 2:
        w[1, :128] = 0.0                    # a one-hot group (rotated: +-c only)
        w[1, 5] = 0.5
    a = W.draw_activation(1, K, seed=seed, index=N + K)
    d = Q.Desc(N, K, bits, block_bits)
    c, s, z = Q.qlin_quantize_rtn(d, w.to(DEV), a.sign_bits.to(DEV))
    rc, rs, rz = O.quantize_rtn(w.numpy(), np_u32(a.sign_bits), bits or None, block_bits)
    assert np.array_equal(c.cpu().numpy(), rc), "codes differ"
    assert np.array_equal(s.cpu().numpy().view(np.uint16), rs.view(np.uint16)), "scales differ"
    assert np.array_equal(z.cpu().numpy().view(np.uint16), rz.view(np.uint16)), "zeros differ"
    return w, a, d, c, s, z


@pytest.mark.parametrize("N,K,bits", [(77, 384, 3), (130, 256, 4), (64, 1280, 6), (200, 2560, 8), (1, 128, 4),
                                      (9728, 2560, 4)])
def test_quantize_rtn_bit_exact(N, K, bits):
    """Offline rotation + round-to-nearest on the GPU: codes, scales and zeros
    bit-exact against the oracle (zero, constant and signed-zero groups,
    outliers, a single row, the gate/up shape)."""
    _quantize_case(N, K, bits)


def test_quantize_rtn_mixed_widths_and_layer():
    """Mixed 64-row widths (one launch per run of equal widths) bit-exact; then
    the packed result through qlin_gemv matches the oracle layer and, the
    rotation being folded, approximates x W^T of the unrotated weight."""
    bb = [6, 8, 8, 4, 3, 8]
    w, a, d, c, s, z = _quantize_case(64 * len(bb), 512, 0, bb, seed=3)
    packed = Q.qlin_pack(d, c)
    x = a.x.to(DEV)
    y = Q.qlin_gemv(d, packed, s, z, a.sign_bits.to(DEV), x)
    torch.cuda.synchronize()
    ref = O.linear64(a.x.numpy(), c.cpu().numpy(), s.cpu().numpy(), z.cpu().numpy(), np_u32(a.sign_bits))
    assert_close(y, ref, what="quantised layer")
    y0 = a.x.double().numpy() @ w.double().numpy().T
    rel = np.linalg.norm(y.double().cpu().numpy() - y0) / np.linalg.norm(y0)
    assert rel < 0.1, rel  # RTN noise of these inputs: 0.077 (oracle), 3- and 4-bit rows dominating


def test_gemv_mixed():
    bb = [6, 8, 4, 3, 8]
    w = _rand_weight(64 * len(bb), 1280, 0, seed=5, block_bits=bb)
    for M in (1, 3, 16):
        a = W.draw_activation(M, 1280, seed=M).to(DEV)
        _gemv_case(w, a, what=f"mixed M{M}")


def test_gemv_integer_special_case():
    """s = 1, z = 0, signs +1, x = row j of H: y[:, n] = sqrt(128) * q[n, j]."""
    N, K = 96, 256
    rng = np.random.default_rng(0)
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    H = O.hadamard(128)
    j = 37
    x = np.zeros((1, K), np.float16)
    x[0, :128] = H[j]
    d = Q.Desc(N, K, 4)
    packed = Q.qlin_pack(d, torch.from_numpy(codes).to(DEV))
    ones = torch.ones(N, 2, dtype=torch.float16, device=DEV)
    zeros = torch.zeros(N, 2, dtype=torch.float16, device=DEV)
    sb = torch.zeros(K // 32, dtype=torch.int32, device=DEV)
    y = Q.qlin_gemv(d, packed, ones, zeros, sb, torch.from_numpy(x).to(DEV)).float().cpu().numpy()[0]
    expect = (np.sqrt(128) * codes[:, j]).astype(np.float16).astype(np.float64)
    assert np.abs(y - expect).max() <= 2e-3 * np.abs(expect).max()


def test_gemv_deterministic_and_stream():
    w, a = W.gateup(device=DEV)
    d, packed = packed_on_device(w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y1 = Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
        y2 = Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
    s.synchronize()
    assert torch.equal(y1, y2)


def test_gemv_rejects_misaligned_and_small_workspace():
    w, a = W.tiny(device=DEV)
    d, packed = packed_on_device(w)
    buf = torch.empty(256 * 2 + 8, dtype=torch.float16, device=DEV)
    xm = buf[1:1 + 256].view(1, 256)  # 2-byte offset
    with pytest.raises(Q.QlinError) as e:
        Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, xm)
    assert e.value.status == -4
    x4 = W.draw_activation(4, 256).x.to(DEV)
    need = Q.qlin_gemv_workspace_bytes(d, 4)
    assert need > 0
    small = torch.empty(need - 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(Q.QlinError) as e:
        Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, x4, workspace=small)
    assert e.value.status == -6


# --------------------------------------------------------------- gemm ---------

@pytest.mark.parametrize("M", [32, 256, 1024, 2048])
def test_gemm_prefill_mixed_sampled(M):
    w, a = W.prefill(M=M, device=DEV)
    d, packed = packed_on_device(w)
    y = Q.qlin_gemm(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
    torch.cuda.synchronize()
    rows = sample_rows(w.N, 384, seed=M)
    ref = oracle_rows(w, a, rows)
    assert_close(y[:, torch.as_tensor(rows, device=DEV)], ref, f"prefill M={M}")
    assert torch.isfinite(y.float()).all()


@pytest.mark.parametrize("bits", [3, 4, 6, 8, 0])
@pytest.mark.parametrize("N,K,M", [(77, 384, 1), (64, 256, 65), (200, 1280, 17), (448, 2560, 300), (256, 640, 600)])
def test_gemm_ragged(bits, N, K, M):
    if bits == 0:
        N = (N + 63) // 64 * 64
        bb = ([6, 8] * 8)[:N // 64]
    else:
        bb = None
    w = _rand_weight(N, K, bits, seed=N + M, block_bits=bb)
    a = W.draw_activation(M, K, seed=M).to(DEV)
    d, packed = packed_on_device(w)
    y = Q.qlin_gemm(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
    torch.cuda.synchronize()
    assert_close(y, oracle_rows(w, a), f"gemm b{bits} N{N} K{K} M{M}")
    assert Q.qlin_device_error() == 0


@pytest.mark.parametrize("N,K,M", [(9728, 2560, 256), (77, 384, 1), (1000, 1280, 600)])
def test_gemm_deterministic_split_tiles(N, K, M):
    """Tiles split between CTAs are summed in a fixed order: repeated calls are
    bit-identical (and match the oracle)."""
    w = _rand_weight(N, K, 6, seed=N + 7)
    a = W.draw_activation(M, K, seed=3).to(DEV)
    d, packed = packed_on_device(w)
    y1 = Q.qlin_gemm(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
    y2 = Q.qlin_gemm(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    rows = sample_rows(N, 64, seed=1) if N > 2000 else None
    got = y1 if rows is None else y1[:, torch.as_tensor(rows, device=y1.device)]
    assert_close(got, oracle_rows(w, a, rows), f"gemm split N{N} K{K} M{M}")
    assert Q.qlin_device_error() == 0


def test_gemm_matches_gemv_at_m16():
    w, a = W.down(M=16, device=DEV)
    d, packed = packed_on_device(w)
    y1 = Q.qlin_gemv(d, packed, w.scales, w.zeros, a.sign_bits, a.x).float()
    y2 = Q.qlin_gemm(d, packed, w.scales, w.zeros, a.sign_bits, a.x).float()
    ref = oracle_rows(w, a)
    assert_close(y1, ref, "gemv")
    assert_close(y2, ref, "gemm")


@pytest.mark.parametrize("M,bits", [(1, 4), (1, 3), (4, 6), (32, 0)])
def test_linear_host_matches_device_call(M, bits):
    """qlin_linear_host (x from pinned host memory, y back to it, one call) gives
    the bits the device call gives, and both match the oracle."""
    N, K = 512, 1280
    w = _rand_weight(N, K, bits, seed=90 + M + bits, block_bits=[6, 8, 4, 3, 8, 6, 8, 4] if bits == 0 else None)
    a = W.draw_activation(M, K, seed=91 + M).to(DEV)
    d, packed = packed_on_device(w)
    fn = Q.qlin_gemv if M <= 16 else Q.qlin_gemm
    y_dev = fn(d, packed, w.scales, w.zeros, a.sign_bits, a.x)
    xh = a.x.cpu().pin_memory()
    yh = torch.full((M, N), float("nan"), dtype=torch.float16).pin_memory()
    xd = torch.empty_like(a.x)
    yd = torch.empty(M, N, dtype=torch.float16, device=DEV)
    Q.qlin_linear_host(d, packed, w.scales, w.zeros, a.sign_bits, xh, yh, xd, yd)
    torch.cuda.synchronize()
    assert torch.equal(yh.view(torch.int16), y_dev.cpu().view(torch.int16))
    assert_close(yh, oracle_rows(w, a), f"linear_host M{M} b{bits}")


def test_zz_no_device_errors():
    """No bounded wait in any kernel gave up during the tests above."""
    torch.cuda.synchronize()
    assert Q.qlin_device_error() == 0


def test_gemv_overlap_chain_matches_serial():
    """With qlin_set_overlap(1), each call may start before the previous one ends;
    a chain y_i = layer_i(y_{i-1}) must give the same bits as without overlap."""
    K = 2560
    layers = []
    for i in range(6):
        w = W.draw_weight(K, K, 4 if i % 2 == 0 else 8, seed=50 + i, device=DEV)
        sb = W.draw_activation(1, K, seed=60 + i, device=DEV).sign_bits
        d, packed = packed_on_device(w)
        layers.append((d, packed, w.scales, w.zeros, sb))
    x0 = W.draw_activation(1, K, seed=70, device=DEV).x

    def chain(overlap):
        prev = Q.qlin_set_overlap(overlap)
        try:
            x = x0
            outs = []
            for d, packed, s, z, sb in layers:
                y = torch.empty(1, K, dtype=torch.float16, device=DEV)
                Q.qlin_gemv(d, packed, s, z, sb, x, y)
                # keep magnitudes bounded through the chain
                x = y
                outs.append(y)
            torch.cuda.synchronize()
            return [o.clone() for o in outs]
        finally:
            Q.qlin_set_overlap(prev)

    serial, overlapped = chain(False), chain(True)
    for a, b in zip(serial, overlapped):
        assert torch.equal(a, b)
    assert torch.isfinite(serial[-1].float()).all()
