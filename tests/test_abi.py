"""CPU checks of the C ABI: the library builds and loads, exports every function
``include/qlin.h`` declares, and rejects bad arguments before touching a GPU.
No compute call is made here."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from dequant_gemv_packed_b200 import build as B
from dequant_gemv_packed_b200 import qlin as Q
from oracle import qlin_oracle as O

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "qlin.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return Q.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlin_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_expected():
    assert set(declared_functions()) == set(Q.EXPORTED)


def test_every_symbol_exported(lib):
    nm = subprocess.run(["nm", "-D", "--defined-only", Q.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (qlin_\w+)", nm))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_status_strings(lib):
    for code, name in Q.STATUS_NAMES.items():
        assert Q.status_string(code).startswith(name)


@pytest.mark.parametrize("bits", [3, 4, 6, 8])
def test_packed_bytes_matches_oracle(lib, bits):
    for N, K in ((1, 128), (77, 384), (9728, 2560), (2560, 9728), (151936, 2560)):
        d = Q.Desc(N, K, bits)
        code = int(O.row_byte_offsets(N, K, bits=bits)[-1])
        assert Q.qlin_code_bytes(d) == code
        assert Q.qlin_packed_bytes(d) == (code + 15) // 16 * 16


def test_packed_bytes_mixed(lib):
    bb = np.array([6, 8, 8, 6, 3, 4], dtype=np.uint8)
    N, K = 64 * len(bb), 2560
    d = Q.Desc(N, K, 0, bb)
    code = int(O.row_byte_offsets(N, K, block_bits=bb)[-1])
    assert Q.qlin_code_bytes(d) == code
    nb = len(bb)
    table = (code + 15) // 16 * 16 + 4 * (nb + 1) + nb
    assert Q.qlin_packed_bytes(d) == (table + 15) // 16 * 16


def test_invalid_descriptors(lib):
    for args in ((0, 128, 4), (8, 100, 4), (8, 128, 5), (8, 128, 2), (65, 128, 0)):
        bb = [6] * (args[0] // 64 + 1) if args[2] == 0 else None
        assert Q.qlin_packed_bytes(Q.Desc(*args, block_bits=bb)) == 0
    assert Q.qlin_packed_bytes(Q.Desc(64, 128, 0, [5])) == 0


def _call_gemv(lib, desc, M, ptr=16, ws=0, wsbytes=0):
    p = ctypes.c_void_p(ptr) if ptr else None
    return lib.qlin_gemv(desc.ref(), p, p, p, p, p, p, M, ctypes.c_void_p(ws) if ws else None, wsbytes, None)


def test_validation_returns_before_launch(lib):
    d = Q.Desc(512, 256, 4)
    assert _call_gemv(lib, d, 1, ptr=0) == -1          # null buffers
    assert _call_gemv(lib, d, 1, ptr=18) == -4         # misaligned
    assert _call_gemv(lib, d, 0) == -3                 # M out of range
    assert _call_gemv(lib, d, 17) == -3
    assert _call_gemv(lib, Q.Desc(512, 200, 4), 1) == -3
    assert _call_gemv(lib, Q.Desc(512, 256, 5), 1) == -2
    assert Q.qlin_gemv_workspace_bytes(d, 1) == 0  # fused rotation, no workspace
    need = Q.qlin_gemv_workspace_bytes(d, 4)
    if need:
        assert _call_gemv(lib, d, 4, ws=0) == -6
        assert _call_gemv(lib, d, 4, ws=4096, wsbytes=need - 1) == -6
    p = ctypes.c_void_p(16)
    assert lib.qlin_gemm(d.ref(), p, p, p, p, p, p, 64, None, 0, None) == -6
    assert lib.qlin_gemm(d.ref(), p, p, p, p, p, p, 0, p, 1 << 30, None) == -3
    assert lib.qlin_rht(p, p, p, 1, 256, None) == -1  # in-place not allowed
    assert lib.qlin_rht(p, ctypes.c_void_p(32), p, 1, 100, None) == -3
    assert lib.qlin_pack(Q.Desc(64, 128, 0, [7]).ref(), p, p, None) == -2


def test_library_refuses_without_build(tmp_path, monkeypatch):
    monkeypatch.setattr(Q, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(Q, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        Q.lib()


def test_quantize_validation_returns_before_launch(lib):
    """qlin_quantize_rtn rejects null, misaligned and bad-shape arguments
    before any CUDA call (the pointers here are never dereferenced)."""
    p = ctypes.c_void_p(16)
    d = Q.Desc(64, 128, 4)
    assert lib.qlin_quantize_rtn(None, p, p, p, p, p, None) == -1
    assert lib.qlin_quantize_rtn(d.ref(), None, p, p, p, p, None) == -1
    assert lib.qlin_quantize_rtn(d.ref(), p, p, p, p, None, None) == -1
    assert lib.qlin_quantize_rtn(d.ref(), ctypes.c_void_p(18), p, p, p, p, None) == -4
    assert lib.qlin_quantize_rtn(d.ref(), p, p, ctypes.c_void_p(24), p, p, None) == -4
    assert lib.qlin_quantize_rtn(Q.Desc(64, 100, 4).ref(), p, p, p, p, p, None) == -3
    assert lib.qlin_quantize_rtn(Q.Desc(64, 128, 5).ref(), p, p, p, p, p, None) == -2
    assert lib.qlin_quantize_rtn(Q.Desc(65, 128, 0, [6, 6]).ref(), p, p, p, p, p, None) == -3


def test_binding_rejects_host_tensors(lib):
    """Every entry point of the binding takes CUDA tensors only and raises for
    host tensors before calling the library: there is no CPU path."""
    import torch
    d = Q.Desc(64, 128, 4)
    h16 = torch.zeros(64, 128, dtype=torch.float16)
    s = torch.zeros(64, 1, dtype=torch.float16)
    sb = torch.zeros(4, dtype=torch.int32)
    x = torch.zeros(1, 128, dtype=torch.float16)
    packed = torch.zeros(Q.qlin_packed_bytes(d), dtype=torch.uint8)
    calls = [
        lambda: Q.qlin_pack(d, torch.zeros(64, 128, dtype=torch.uint8), packed),
        lambda: Q.qlin_unpack(d, packed, torch.zeros(64, 128, dtype=torch.uint8)),
        lambda: Q.qlin_dequant(d, packed, s, s, h16),
        lambda: Q.qlin_rht(x, sb, torch.zeros_like(x)),
        lambda: Q.qlin_quantize_rtn(d, h16, sb, torch.zeros(64, 128, dtype=torch.uint8), s.clone(), s.clone()),
        lambda: Q.qlin_gemv(d, packed, s, s, sb, x, torch.zeros(1, 64, dtype=torch.float16),
                            torch.zeros(256, dtype=torch.uint8)),
        lambda: Q.qlin_gemm(d, packed, s, s, sb, x, torch.zeros(1, 64, dtype=torch.float16),
                            torch.zeros(1 << 16, dtype=torch.uint8)),
    ]
    for call in calls:
        with pytest.raises(TypeError, match="CUDA tensor"):
            call()


def test_gemv_plan_invariants(lib):
    """Launch plans of qlin_gemv over a sweep of widths, K and N (host only):
    the invariants the kernels' index bounds rely on."""
    Ns = (1, 2, 63, 64, 147, 148, 149, 1000, 2560, 4096, 4737, 9728, 19456, 151936, 262144)
    smem_floor, smem_limit = 80 * 1024, 113 * 1024
    for bits in (3, 4, 6, 8):
        unit = 32 if bits == 8 else 64
        rows_per_pass = 4 if bits == 4 else 2
        for K in list(range(128, 4097, 128)) + [5120, 9728, 12288, 16384, 20480, 24576, 32768]:
            for N in Ns:
                d = Q.Desc(N, K, bits)
                p = Q.qlin_gemv_plan(d, 1)
                assert p["workspace_bytes"] == Q.qlin_gemv_workspace_bytes(d, 1)
                if p["kernel"] == 2:  # very long K: the tensor-core kernel with a workspace
                    assert K // unit > 320 and p["workspace_bytes"] > 0
                    continue
                if p["kernel"] == 3:  # integer tensor-core kernel: 4/8-bit, a CTA's rows all resident
                    assert bits in (4, 8) and p["workspace_bytes"] == 0
                    assert p["threads"] == 32 * (p["consumer_warps"] + 1)
                    assert p["grid"] == min(148, N) and p["rows_per_cta"] == -(-N // p["grid"])
                    assert p["rows_per_chunk"] == 16 and p["stages"] == -(-p["rows_per_cta"] // 16) <= 64
                    assert smem_floor <= p["smem_bytes"] <= smem_limit, (bits, K, N, p)
                    assert p["rows_per_cta"] * K * bits // 8 < p["smem_bytes"], (bits, K, N, p)
                    continue
                U, NW, UW = K // unit, p["consumer_warps"], p["units_per_warp"]
                assert 1 <= NW <= 10 and UW in (1, 2, 4, 8, 16, 32) and (NW - 1) * UW < U <= NW * UW
                assert p["threads"] == 32 * (NW + 1)
                assert smem_floor <= p["smem_bytes"] <= smem_limit, (bits, K, N, p)
                assert p["grid"] == min(148, N) and p["rows_per_cta"] == -(-N // p["grid"])
                assert p["rows_per_chunk"] % (rows_per_pass * 32 // UW) == 0
                nchunks = -(-p["rows_per_cta"] // p["rows_per_chunk"])
                assert 1 <= p["stages"] <= min(16, nchunks) and 1 <= p["chunks_in_flight"] <= p["stages"]
                row_bytes = K * bits // 8
                resident = p["rows_per_cta"] if p["stages"] == nchunks else p["stages"] * p["rows_per_chunk"]
                assert resident * row_bytes < p["smem_bytes"], (bits, K, N, p)
    for M in (2, 16):
        p = Q.qlin_gemv_plan(Q.Desc(2560, 9728, 3), M)
        assert p["kernel"] == 4 and p["workspace_bytes"] == Q.qlin_gemv_workspace_bytes(Q.Desc(2560, 9728, 3), M)
    for M in (1, 2):
        p = Q.qlin_gemv_plan(Q.Desc(320, 1280, 0, [6, 8, 4, 3, 8]), M)
        assert p["kernel"] == 2  # mixed widths


def test_gemv_tc_plan_invariants(lib):
    """Plans of the split-K tensor-core GEMV (M = 2..16, one width): one CTA
    per SM at most, shared memory within the opt-in limit, the workspace of
    the rotated x, and the code buffers holding whole 32-row tiles."""
    Ns = (1, 31, 32, 33, 148, 1000, 2560, 4096, 9728, 20000, 151936)
    for bits in (3, 4, 6, 8):
        for K in (128, 256, 384, 1280, 2560, 4096, 9728, 16384):
            for N in Ns:
                for M in (2, 4, 8, 9, 16):
                    d = Q.Desc(N, K, bits)
                    p = Q.qlin_gemv_plan(d, M)
                    if p["kernel"] == 2:
                        # at most 8 K slices (one cluster): 8-bit codes with very
                        # long K and M > 8 leave no shared-memory plan, and run on
                        # the other tensor-core kernel
                        assert bits == 8 and K >= 16384 and M > 8, (bits, K, N, M)
                        continue
                    assert p["kernel"] == 4, (bits, K, N, M)
                    assert p["threads"] == 256 and p["consumer_warps"] == 8
                    assert 1 <= p["grid"] <= 148 and p["smem_bytes"] <= 227 * 1024
                    assert p["rows_per_chunk"] == 32 and p["rows_per_cta"] % 32 == 0
                    assert p["stages"] in (1, 2) and p["chunks_in_flight"] >= 1
                    if p["stages"] == 1:  # one round: the buffer holds every tile of a CTA
                        assert p["chunks_in_flight"] * 32 == p["rows_per_cta"]
                    assert p["workspace_bytes"] == Q.qlin_gemv_workspace_bytes(d, M)
                    # workspace: x~ [G][NT][8][128] fp16 and its group sums [G][16]
                    # fp32; the K slices of a row part add their sums inside a
                    # thread-block cluster, with no workspace
                    G, NT = K // 128, (1 if M <= 8 else 2)
                    assert p["workspace_bytes"] == G * NT * 2048 + G * 64, (bits, K, N, M, p)


def test_gemv_plan_validation(lib):
    info = ctypes.create_string_buffer(64)
    assert lib.qlin_gemv_plan(Q.Desc(64, 128, 4).ref(), 17, info) == -3
    assert lib.qlin_gemv_plan(Q.Desc(64, 128, 4).ref(), 0, info) == -3
    assert lib.qlin_gemv_plan(Q.Desc(64, 128, 4).ref(), 1, None) == -1
    assert lib.qlin_gemv_plan(Q.Desc(64, 100, 4).ref(), 1, info) == -3
    assert lib.qlin_gemv_plan(None, 1, info) == -1


def test_linear_host_validation_returns_before_enqueue(lib):
    """qlin_linear_host checks every argument before its first copy: missing host
    buffers, a missing or small workspace and misaligned staging buffers are
    reported without a CUDA call (the pointers below are never dereferenced).
    Status codes: -1 invalid argument, -3 shape, -4 alignment, -6 workspace."""
    d = Q.Desc(2560, 9728, 3)
    dev = [ctypes.c_void_p(0x100000 * (i + 1)) for i in range(7)]  # 16-byte aligned stand-ins
    host = ctypes.c_void_p(0x7F0000000000)

    def call(M, x_host, y_host, x_dev, ws, ws_len):
        return lib.qlin_linear_host(d.ref(), dev[0], dev[1], dev[2], dev[3], x_host, y_host, x_dev, dev[4], M, ws,
                                    ws_len, None)

    assert call(1, None, host, dev[5], None, 0) == -1
    assert call(1, host, None, dev[5], None, 0) == -1
    assert call(0, host, host, dev[5], None, 0) == -3
    assert call(1, host, host, ctypes.c_void_p(0x100002), None, 0) == -4
    need = Q.qlin_gemv_workspace_bytes(d, 4)
    assert need > 0
    assert call(4, host, host, dev[5], None, 0) == -6
    assert call(4, host, host, dev[5], dev[6], need - 16) == -6
    assert call(32, host, host, dev[5], dev[6], 1024) == -6
