"""Benchmark of the quantised linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one call of the layer (rotation of x, load of the packed weight,
in-register/shared-memory dequantisation, contraction, fp16 store).  The
default workload is the decode gate/up-projection GEMV (M=1, K=2560, N=9728,
int4 codes, fp16 scale/zero per 128).  Inputs are seeded and synthetic.

Timing: W warm-up steps, then exactly K steps replayed from CUDA graphs that
rotate over enough copies of the packed weight to exceed twice the L2 cache,
bracketed by a barrier and a device synchronisation, measured with CUDA events
on the launching stream; the max over ranks is reported.  Under torchrun every
rank runs an independent replica of the workload (the layer is run on one GPU;
ranks do not exchange data).  ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time
from types import SimpleNamespace

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs/call and achieved HBM GB/s (fraction of ~8 TB/s) for quantised GEMV, M=1"
L2_BYTES = 126 * 1024 * 1024

WORKLOADS = {
    # name: (description, kind, params)
    "gateup": ("decode gate/up-proj GEMV: M=1, K=2560, N=9728, int4 g128 fp16 scale/zero, block-128 RHT", "gemv",
               dict(fn="gateup", M=1)),
    "tiny": ("tiny linear: M=1, K=256, N=512, int4 g128, block-128 RHT", "gemv", dict(fn="tiny", M=1)),
    "down1": ("decode down-proj GEMV: M=1, K=9728, N=2560, int3 g128, block-128 RHT", "gemv", dict(fn="down", M=1)),
    "down4": ("decode down-proj GEMV: M=4, K=9728, N=2560, int3 g128, block-128 RHT", "gemv", dict(fn="down", M=4)),
    "down16": ("decode down-proj GEMV: M=16, K=9728, N=2560, int3 g128, block-128 RHT", "gemv",
               dict(fn="down", M=16)),
    "stack": ("36-layer int6 g128 decoder linear stack + int8 lm_head, M=1 (253 GEMVs per step)", "stack", {}),
    "stack_fused": ("the same 36-layer int6 stack + int8 lm_head with q/k/v (2560->6144) and gate/up "
                    "(2560->19456) fused, each sharing one x, M=1 (145 GEMVs per step)", "stack", dict(fused=True)),
    "quantize": ("offline weight side: rotation (signs + block-128 FWHT, fp64) and RTN int4 g128 quantisation "
                 "of an fp16 weight, K=2560, N=9728", "quantize", dict(N=9728, K=2560, bits=4)),
    "gptq": ("offline weight side with error compensation: rotation (signs + block-128 FWHT) and GPTQ int6 g128 "
             "against a synthetic calibration Hessian (damped 1 %), gate/up-proj shape K=2560, N=9728", "gptq",
             dict(N=9728, K=2560, bits=6)),
    "mid32": ("mid-batch dequant-GEMM: M=32, K=2560, N=9728, mixed int6/int8 64-row blocks, block-128 RHT",
              "gemm", dict(M=32)),
    "prefill256": ("prefill dequant-GEMM: M=256, K=2560, N=9728, mixed int6/int8 64-row blocks, block-128 RHT",
                   "gemm", dict(M=256)),
    "prefill1024": ("prefill dequant-GEMM: M=1024, K=2560, N=9728, mixed int6/int8 64-row blocks, block-128 RHT",
                    "gemm", dict(M=1024)),
    "prefill2048": ("prefill dequant-GEMM: M=2048, K=2560, N=9728, mixed int6/int8 64-row blocks, block-128 RHT",
                    "gemm", dict(M=2048)),
}


# Default timed steps per workload kind: about a second of timed work (a
# gate/up call is ~5 us, a stack step ~2 ms, a prefill GEMM 40-150 us).
DEFAULT_STEPS = {"gemv": 100000, "stack": 500, "gemm": 10000, "quantize": 20000, "gptq": 20}

# fp32 instruction peak of the CUDA cores (nominal unit counts and clock: 148 SMs
# x 128 fp32 lanes x 1965 MHz), for work that may not fuse multiply and add.
FP32_ALU_TOPS = 148 * 128 * 1.965e9 / 1e12


# --------------------------------------------------------------------------- utils

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# The .cu file that defines each workload kind's dominant kernel.
KERNEL_FILE = {"gemv": ("qlin_gemv.cu", "qlin_gemv_imma.cu", "qlin_gemv_tc.cu"),
               "stack": ("qlin_gemv.cu", "qlin_gemv_imma.cu", "qlin_gemv_tc.cu"),
               "gemm": ("qlin_gemm.cu",), "quantize": ("qlin_quant.cu",), "gptq": ("qlin_gptq.cu", "qlin_quant.cu")}
QUANTIZE_METRIC = "µs/call and achieved HBM GB/s (fraction of ~8 TB/s) of the offline weight rotation + RTN quantisation"
GPTQ_METRIC = "µs/call and fp32 TFLOP/s (fraction of the CUDA cores' fp32 instruction rate) of rotation + GPTQ"


def kernel_source_hash(kind: str = None) -> str:
    """Hash of the sources of a workload kind's dominant kernel (its .cu file
    and the headers every kernel file includes), or of all of csrc/ when kind
    is None, so that counters taken on other sources are not reported."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dequant_gemv_packed_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cuh", ".h")) or (f.endswith(".cu") and (kind is None or f in KERNEL_FILE[kind])):
            h.update(f.encode())
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, kernel_hash: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")  # JSON text
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(workload)
    if not d or d.get("kernel_hash") != kernel_hash:
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.lines = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            t0 = time.time()
            while not self.lines and time.time() - t0 < 5:
                time.sleep(0.01)
        except FileNotFoundError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.06)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(backend: str | None = None):
    """One process per GPU under torchrun (RANK/LOCAL_RANK/WORLD_SIZE/MASTER_* from
    the environment): NCCL on GPUs; `backend="gloo"` runs the same plumbing on CPU."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        backend = backend or "nccl"
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
        return dist, dist.get_rank(), world, local
    return None, 0, 1, 0


def barrier(dist):
    if dist is not None:
        dist.barrier()


def max_over_ranks(dist, v: float) -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if dist is None:
        return v
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_step: int, steps: int, world: int, ms_max: float) -> float:
    """Weak scaling: every rank runs `steps` calls of `bytes_per_step`; the job's
    throughput is all ranks' bytes over the slowest rank's time."""
    return world * bytes_per_step * steps / (ms_max * 1e-3) / 1e9


# ------------------------------------------------------------------- workloads

class Case:
    """Device-resident inputs of one workload: C rotating copies of the weight."""

    def __init__(self, name: str, copies: int | None = None):
        from dequant_gemv_packed_b200 import qlin as Q
        from dequant_gemv_packed_b200 import workloads as W
        self.Q, self.name = Q, name
        desc, kind, p = WORKLOADS[name]
        self.desc_text, self.kind = desc, kind
        dev = "cuda"
        if kind == "stack":
            self.layers = []
            self.bytes = 0
            self.flops = 0
            for _, w, a in (W.stack_fused if p.get("fused") else W.stack)(device=dev):
                d = Q.Desc.of(w)
                packed = Q.qlin_pack(d, w.codes)
                del w.codes
                ws = torch.empty(max(Q.qlin_gemv_workspace_bytes(d, 1), 16), dtype=torch.uint8, device=dev)
                y = torch.empty(1, w.N, dtype=torch.float16, device=dev)
                self.layers.append((d, packed, w.scales, w.zeros, a.sign_bits, a.x, y, ws))
                self.bytes += Q.algorithmic_bytes(d)
                self.flops += 2 * w.N * w.K
            self.M, self.N, self.K, self.copies = 1, None, None, 1
            self.weight_bytes_total = self.bytes
            self.host_sample = None
            torch.cuda.synchronize()
            return
        if kind == "gptq":
            N, K, bits = p["N"], p["K"], p["bits"]
            self.M, self.N, self.K, self.bits, self.block_bits = 1, N, K, bits, None
            self.d = Q.Desc(N, K, bits)
            self.w = [W.draw_fp16_weight(N, K, device=dev)]
            a = W.draw_activation(1, K, device=dev)
            # the inverse-Hessian factor is an input: H = 2 X^T X / n of the
            # synthetic calibration draw, damped by 1 % of its mean diagonal,
            # U = chol((H + damp I)^-1)^T (fp64 library routines, then fp32)
            xc = W.draw_calibration(K, device=dev).double()
            H = (2.0 / xc.shape[0]) * (xc.T @ xc)
            H += 0.01 * torch.diagonal(H).mean() * torch.eye(K, dtype=torch.float64, device=dev)
            self.U = torch.linalg.cholesky(torch.linalg.inv(H)).T.contiguous().float()
            del xc, H
            G = K // 128
            self.bytes = N * K * 2 + N * K + 4 * N * G
            # algorithmic fp32 operations: every column's error updates every later
            # column of the row, one multiply and one subtraction each
            self.flops = N * K * (K - 1)
            self.copies = 1
            self.out = [(torch.empty(N, K, dtype=torch.uint8, device=dev),
                         torch.empty(N, G, dtype=torch.float16, device=dev),
                         torch.empty(N, G, dtype=torch.float16, device=dev))]
            self.ws = torch.empty(Q.qlin_gptq_workspace_bytes(self.d), dtype=torch.uint8, device=dev)
            self.weight_bytes_total = N * K * 2
            self.sign_bits, self.x = a.sign_bits, a.x
            self.host_sample = None
            torch.cuda.synchronize()
            return
        if kind == "quantize":
            N, K, bits = p["N"], p["K"], p["bits"]
            self.M, self.N, self.K, self.bits, self.block_bits = 1, N, K, bits, None
            self.d = Q.Desc(N, K, bits)
            w = W.draw_fp16_weight(N, K, device=dev)
            a = W.draw_activation(1, K, device=dev)
            G = K // 128
            # algorithmic bytes: read the fp16 weight, write codes (one byte each) and fp16 scale/zero
            self.bytes = N * K * 2 + N * K + 4 * N * G
            self.flops = 0
            self.copies = copies or max(1, math.ceil(2 * L2_BYTES / (N * K * 2)) + 1)
            self.w = [w.clone() for _ in range(self.copies)]
            self.out = [(torch.empty(N, K, dtype=torch.uint8, device=dev),
                         torch.empty(N, G, dtype=torch.float16, device=dev),
                         torch.empty(N, G, dtype=torch.float16, device=dev)) for _ in range(2)]
            self.weight_bytes_total = self.copies * N * K * 2
            self.sign_bits, self.x = a.sign_bits, a.x
            self.host_sample = (w.cpu().numpy(), a.sign_bits.cpu().numpy().view(np.uint32))
            del w
            torch.cuda.synchronize()
            return
        if kind == "gemv":
            fn = getattr(W, p["fn"])
            w, a = fn(device=dev, M=p["M"]) if p["fn"] != "tiny" else fn(device=dev)
        else:
            w, a = W.prefill(M=p["M"], device=dev)
        self.M, self.N, self.K = a.x.shape[0], w.N, w.K
        self.bits, self.block_bits = w.bits, w.block_bits
        self.d = Q.Desc.of(w)
        self.bytes = Q.algorithmic_bytes(self.d)
        self.flops = 2 * self.M * self.N * self.K
        packed = Q.qlin_pack(self.d, w.codes)
        if copies is None:
            copies = max(1, math.ceil(2 * L2_BYTES / self.bytes) + 1)
        self.copies = copies
        self.w = []
        for c in range(copies):
            self.w.append((packed.clone(), w.scales.clone(), w.zeros.clone()))
        self.weight_bytes_total = copies * self.bytes
        self.sign_bits, self.x = a.sign_bits, a.x
        self.y = [torch.empty(self.M, self.N, dtype=torch.float16, device=dev) for _ in range(copies)]
        ws_fn = Q.qlin_gemv_workspace_bytes if kind == "gemv" else Q.qlin_gemm_workspace_bytes
        self.ws = torch.empty(max(ws_fn(self.d, self.M), 16), dtype=torch.uint8, device=dev)
        self.call = Q.qlin_gemv if kind == "gemv" else Q.qlin_gemm
        # host copies for the oracle baseline (packed bytes as the oracle reads them)
        self.host_sample = (w.codes.cpu().numpy(), w.scales.cpu().numpy(), w.zeros.cpu().numpy(),
                            a.x.cpu().numpy(), a.sign_bits.cpu().numpy().view(np.uint32))
        del w
        torch.cuda.synchronize()

    def launches_per_step(self) -> int:
        from dequant_gemv_packed_b200 import qlin as Q
        if self.kind == "quantize":
            return 1  # uniform width: one launch
        if self.kind == "gptq":
            return 2 * (self.K // 128)  # the rotation, then per group a block and (but the last) a trailing kernel
        if self.kind == "stack":
            return sum(Q.kernel_launches_per_call("gemv", l[0], 1) for l in self.layers)
        return Q.kernel_launches_per_call(self.kind, self.d, self.M)

    def step(self, i: int):
        Q = self.Q
        if self.kind == "quantize":
            c, sc, z = self.out[i % 2]
            Q.qlin_quantize_rtn(self.d, self.w[i % self.copies], self.sign_bits, c, sc, z)
            return
        if self.kind == "gptq":
            c, sc, z = self.out[0]
            Q.qlin_quantize_gptq(self.d, self.w[0], self.sign_bits, self.U, c, sc, z, self.ws)
            return
        if self.kind == "stack":
            for (d, packed, s, z, sb, x, y, ws) in self.layers:
                Q.qlin_gemv(d, packed, s, z, sb, x, y, ws)
            return
        packed, s, z = self.w[i % self.copies]
        self.call(self.d, packed, s, z, self.sign_bits, self.x, self.y[i % self.copies], self.ws)


SPIN_CYCLES = 200_000  # ~0.1 ms at 1.9 GHz, longer than the host needs to queue the timed replays


def time_steps(case: Case, K: int, W: int, dist, stream, graph_len: int = 1024):
    """Warm up W steps, then time exactly K steps replayed from CUDA graphs."""
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(W):
            case.step(i)
    torch.cuda.synchronize()
    R = min(graph_len, K) if case.kind != "stack" else 1
    R = max(R, 1)
    graphs = []
    with torch.cuda.stream(stream):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(R):
                case.step(i)
        graphs.append((g, R))
        rem = K % R
        if rem:
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2, stream=stream):
                for i in range(rem):
                    case.step(R + i)
            graphs.append((g2, rem))
        # untimed replays of each graph (uploads the graph; warms clocks and caches)
        for _ in range(3):
            for g_, _ in graphs:
                g_.replay()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist)
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    with sampler:
        with torch.cuda.stream(stream):
            # A short device-side spin ahead of the start event: the host queues
            # the graph replays while it runs, so the timed region holds the K
            # steps back to back and no host enqueue gap (which a 20-step run
            # would otherwise spread over only 20 calls).
            torch.cuda._sleep(SPIN_CYCLES)
            torch.cuda.nvtx.range_push("qlin_timed")
            start.record(stream)
            for _ in range(K // R):
                graphs[0][0].replay()
            if len(graphs) > 1:
                graphs[1][0].replay()
            end.record(stream)
            torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
    barrier(dist)
    ms = start.elapsed_time(end)
    del graphs
    return max_over_ranks(dist, ms), sampler.summary()


def time_e2e(case: Case, K: int, W: int, stream):
    """Through the public binding, eager: per step copy x in from pinned host
    memory, run the layer, copy y back to pinned host memory."""
    if case.kind in ("stack", "gptq"):
        return None
    if case.kind == "quantize":
        return time_e2e_quantize(case, K, W, stream)
    n = min(K, 2000)
    xh = case.x.cpu().pin_memory()
    yh = torch.empty(case.M, case.N, dtype=torch.float16).pin_memory()
    xd = torch.empty_like(case.x)
    Q = case.Q
    with torch.cuda.stream(stream):
        def one(i):  # one C-ABI call: x in from pinned host memory, the layer, y back to pinned host memory
            packed, s, z = case.w[i % case.copies]
            Q.qlin_linear_host(case.d, packed, s, z, case.sign_bits, xh, yh, xd, case.y[i % case.copies], case.ws)
        for i in range(min(W, 50)):
            one(i)
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(n):
            one(i)
        end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / n
    return {"value": case.bytes / (ms * 1e-3) / 1e9, "unit": "GB/s", "us_per_call": ms * 1e3,
            "h2d_bytes_per_step": xh.numel() * 2, "d2h_bytes_per_step": yh.numel() * 2,
            "steps": n, "mode": "eager qlin_linear_host calls through the Python binding (host x in, host y out)"}


def time_e2e_quantize(case: Case, K: int, W: int, stream):
    """The offline tool through the public binding, eager: per step copy the fp16
    weight in from pinned host memory, quantise, copy codes, scales and zeros
    back to pinned host memory."""
    n = min(K, 200)
    wh = case.w[0].cpu().pin_memory()
    c, sc, z = case.out[0]
    ch, sh, zh = c.cpu().pin_memory(), sc.cpu().pin_memory(), z.cpu().pin_memory()
    wd = torch.empty_like(case.w[0])
    Q = case.Q
    with torch.cuda.stream(stream):
        def one():
            wd.copy_(wh, non_blocking=True)
            Q.qlin_quantize_rtn(case.d, wd, case.sign_bits, c, sc, z)
            ch.copy_(c, non_blocking=True)
            sh.copy_(sc, non_blocking=True)
            zh.copy_(z, non_blocking=True)
        for _ in range(min(W, 10)):
            one()
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(n):
            one()
        end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / n
    return {"value": case.bytes / (ms * 1e-3) / 1e9, "unit": "GB/s", "us_per_call": ms * 1e3,
            "h2d_bytes_per_step": wh.numel() * 2, "d2h_bytes_per_step": ch.numel() + 2 * sh.numel() * 2,
            "steps": n, "mode": "eager calls through the Python binding"}


def time_cublas(case: Case, stream, reps: int = 2000):
    """bf16 torch.nn.functional.linear (cuBLAS) of the same shape, same rotation."""
    if case.kind in ("stack", "quantize", "gptq"):
        return None
    copies = max(1, math.ceil(2 * L2_BYTES / (case.N * case.K * 2)) + 1)
    ws = [torch.randn(case.N, case.K, device="cuda", dtype=torch.bfloat16) for _ in range(copies)]
    x = case.x.to(torch.bfloat16)
    with torch.cuda.stream(stream):
        for i in range(10):
            torch.nn.functional.linear(x, ws[i % copies])
        g = torch.cuda.CUDAGraph()
        R = min(reps, 256)
        with torch.cuda.graph(g, stream=stream):
            for i in range(R):
                torch.nn.functional.linear(x, ws[i % copies])
        g.replay()
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = max(1, reps // R)
        start.record(stream)
        for _ in range(n):
            g.replay()
        end.record(stream)
    torch.cuda.synchronize()
    us = start.elapsed_time(end) * 1e3 / (n * R)
    del g, ws
    return us


def oracle_step(case_host, rows, bits, block_bits):
    """One oracle evaluation of the layer restricted to `rows` (from packed bytes)."""
    from oracle import qlin_oracle as O
    codes, s, z, x, sb = case_host
    N, K = codes.shape
    packed = case_host_packed(case_host, bits, block_bits)
    c = O.unpack(packed, N, K, bits or None, None if bits else block_bits, rows=rows)
    return O.linear64(x, c, s[rows], z[rows], sb)


_PACKED_CACHE = {}


def case_host_packed(case_host, bits, block_bits):
    key = id(case_host)
    if key not in _PACKED_CACHE:
        from oracle import qlin_oracle as O
        _PACKED_CACHE[key] = O.pack(case_host[0], bits or None, None if bits else block_bits)
    return _PACKED_CACHE[key]


def cpu_quantize_rate(case: Case, budget_s: float = 12.0, threads: int | None = 1):
    """Oracle throughput of the offline tool (GB/s of its algorithmic bytes) on
    row samples of the weight, BLAS limited to `threads` (None: all cores)."""
    from threadpoolctl import threadpool_limits
    from oracle import qlin_oracle as O
    w, sb = case.host_sample
    N = w.shape[0]
    per_row = case.bytes / N
    rng = np.random.default_rng(0)
    done_rows, t = 0, 0.0
    with threadpool_limits(limits=threads):
        while t < budget_s and done_rows < 32 * N:
            rows = np.sort(rng.choice(N, size=min(256, N), replace=False))
            t1 = time.perf_counter()
            O.quantize_rtn(w[rows], sb, case.bits)
            t += time.perf_counter() - t1
            done_rows += len(rows)
    return done_rows * per_row / t / 1e9, done_rows, t


def cpu_oracle_rate(case: Case, budget_s: float = 12.0, rows_per_step: int | None = None,
                    threads: int | None = 1):
    """Oracle throughput (GB/s of the layer's algorithmic bytes) on a bounded
    sample of the workload's weight rows, BLAS limited to `threads` (None: all
    cores)."""
    from threadpoolctl import threadpool_limits
    from oracle import qlin_oracle as O
    codes = case.host_sample[0]
    N, K = codes.shape
    bb = None if case.bits else np.asarray(case.block_bits)
    case_host_packed(case.host_sample, case.bits, bb)
    per_row = O.algorithmic_bytes(N, K, case.bits or None, bb) / N
    rng = np.random.default_rng(0)
    with threadpool_limits(limits=threads):
        t0 = time.perf_counter()
        rows = np.sort(rng.choice(N, size=min(64, N), replace=False))
        oracle_step(case.host_sample, rows, case.bits, bb)
        t_row = (time.perf_counter() - t0) / len(rows)
        if rows_per_step is None:
            rows_per_step = int(max(16, min(N, budget_s / max(t_row, 1e-9))))
        # samples of rows_per_step rows until the time budget is spent (at most 32 passes' worth)
        done_rows, t = 0, 0.0
        while t < budget_s and done_rows < 32 * N:
            rows = np.sort(rng.choice(N, size=min(rows_per_step, N), replace=False))
            t1 = time.perf_counter()
            oracle_step(case.host_sample, rows, case.bits, bb)
            t += time.perf_counter() - t1
            done_rows += len(rows)
    gbs = done_rows * per_row / t / 1e9
    return gbs, done_rows, t


# ------------------------------------------------------------- per-config table

# Every workload of the specification besides the headline one, each timed on
# its own short region (tens of ms) so that the default run stays short.
PER_CONFIG = (("tiny", 4000, 20), ("down1", 4000, 20), ("down4", 2000, 20), ("down16", 2000, 20),
              ("stack", 30, 3), ("stack_fused", 30, 3), ("mid32", 1000, 20), ("prefill256", 1000, 20),
              ("prefill1024", 400, 10), ("prefill2048", 200, 10), ("quantize", 1000, 20), ("gptq", 5, 3))


L2_POLICY = {
    "gemv": "inputs larger than L2: consecutive timed calls rotate over packed-weight copies totalling more than 2x L2",
    "gemm": "inputs larger than L2: consecutive timed calls rotate over packed-weight copies totalling more than 2x L2",
    "stack": "inputs larger than L2: one step streams every layer's packed weight (3.2 GB)",
    "quantize": "inputs larger than L2: consecutive timed calls rotate over fp16 weight copies totalling more than 2x L2",
    "gptq": "inputs larger than L2: the fp16 weight and its fp32 working copy",
}


def workload_config(case, world: int) -> dict:
    """What the workload is (identical in both arms): shapes, widths, inputs,
    and how the timed region keeps L2 from serving repeated inputs."""
    bits = getattr(case, "bits", None)
    return {"workload": case.desc_text, "M": case.M, "K": case.K, "N": case.N, "group": 128,
            "bits": ("mixed int6/int8" if bits == 0 else bits) if case.kind != "stack" else "int6 + int8 lm_head",
            "parallelism": f"replicas x{world}",
            "inputs": "seeded synthetic: weights N(0,0.02) with 0.1% x20 outliers, RTN g128 fp16 scale/zero; "
                      "activations N(0,1) fp16; random signs",
            "l2": L2_POLICY[case.kind]}


def roofline_of(case, ms_step: float, peaks: dict) -> dict:
    """HBM roofline below the ridge point (measured peak FLOP/s over measured HBM
    bytes/s), tensor roofline above it."""
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if case.kind == "gptq":
        achieved = case.flops / (ms_step * 1e-3) / 1e12
        return {"bound": "alu", "achieved": achieved, "peak": FP32_ALU_TOPS, "unit": "TFLOP/s",
                "frac": achieved / FP32_ALU_TOPS,
                "peak_source": "nominal fp32 instruction rate: 148 SMs x 128 lanes x 1965 MHz (no fused multiply-add)"}
    if case.kind == "gemm" and case.flops / case.bytes > ridge:
        achieved = case.flops / (ms_step * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"],
                "peak_source": f"{peaks['source']} dense bf16 cuBLAS burst (fp16 nominal ratio 1:1)"}
    achieved = case.bytes / (ms_step * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "peak_source": f"{peaks['source']} HBM copy bandwidth"}


def measure_per_config(stream, peaks: dict, skip: str) -> dict:
    """One short timed region per workload: us/call, roofline, cuBLAS bf16 of the
    same shape, and the clocks sampled during that region."""
    from dequant_gemv_packed_b200 import qlin as Q
    out = {}
    for name, steps, warmup in PER_CONFIG:
        if name == skip:
            continue
        case = Case(name)
        overlap = case.kind in ("gemv", "stack")
        prev = Q.qlin_set_overlap(overlap)
        try:
            ms, clocks = time_steps(case, steps, warmup, None, stream)
        finally:
            Q.qlin_set_overlap(prev)
        ms_step = ms / steps
        roof = roofline_of(case, ms_step, peaks)
        entry = {"us_per_call": ms_step * 1e3, "steps": steps, "bound": roof["bound"],
                 "achieved": roof["achieved"], "unit": roof["unit"], "frac": roof["frac"],
                 "algorithmic_bytes": case.bytes, "flops": case.flops,
                 "launches_per_step": case.launches_per_step(), "clocks": clocks,
                 "launch": "programmatic dependent launch" if overlap else "serial"}
        cub = time_cublas(case, stream, reps=512)
        if cub is not None:
            entry["cublas_bf16_us"] = cub
            entry["speedup_vs_cublas"] = cub / (ms_step * 1e3)
        out[name] = entry
        del case
        torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------------ main

def run_ours(args):
    dist, rank, world, local = dist_setup()
    torch.cuda.set_device(local)
    from dequant_gemv_packed_b200 import build
    if rank == 0:
        build.build()
    barrier(dist)
    case = Case(args.workload)
    stream = torch.cuda.Stream()
    from dequant_gemv_packed_b200 import qlin as Q
    overlap = case.kind in ("gemv", "stack") and not args.no_overlap
    no_overlap = None
    if overlap:
        # the same K steps with each call waiting for the previous one to finish
        Q.qlin_set_overlap(False)
        ms0, _ = time_steps(case, args.steps, args.warmup, dist, stream)
        no_overlap = {"ms_per_step": ms0 / args.steps,
                      "GB/s": case.bytes * args.steps / (ms0 * 1e-3) / 1e9}
    Q.qlin_set_overlap(overlap)
    ms, clocks = time_steps(case, args.steps, args.warmup, dist, stream)
    ms_step = ms / args.steps
    peaks = measured_peaks()
    value = whole_job_gbs(case.bytes, args.steps, world, ms)
    per_gpu_gbs = case.bytes / (ms_step * 1e-3) / 1e9
    khash = kernel_source_hash(case.kind)
    roof = roofline_of(case, ms_step, peaks)
    roof["traffic"] = ncu_traffic(args.workload, khash)
    roof["algorithmic_bytes_per_launch"] = case.bytes
    e2e = None if args.no_extras else time_e2e(case, args.steps, args.warmup, stream)
    cublas_us = time_cublas(case, stream) if rank == 0 and not args.no_extras else None
    cpu = cpu_all = None
    if rank == 0 and world == 1 and case.host_sample is not None and not args.no_cpu_baseline \
            and not args.no_extras:
        if case.kind == "quantize":
            gbs, rows, t = cpu_quantize_rate(case, budget_s=args.cpu_budget)
            what = "explicit-H fp64 rotation + fp32 RTN"
        else:
            gbs, rows, t = cpu_oracle_rate(case, budget_s=args.cpu_budget)
            what = "unpack + fp64 dequant + explicit-H rotation + fp64 matmul"
        cpu = {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"{rows} of {case.N} weight rows ({what}), {t:.1f} s, BLAS limited to 1 thread"}
        # the same oracle with BLAS on every host core (the unpack/dequant steps stay single-threaded numpy)
        ncores = os.cpu_count() or 1
        rate = cpu_quantize_rate if case.kind == "quantize" else cpu_oracle_rate
        gbs_all, rows_all, t_all = rate(case, budget_s=args.cpu_budget / 2, threads=None)
        cpu_all = {"value": gbs_all, "unit": "GB/s", "cores": ncores, "kind": "oracle",
                   "sample": f"{rows_all} of {case.N} weight rows ({what}), {t_all:.1f} s, BLAS on {ncores} threads"}
    per_config = None
    if rank == 0 and world == 1 and not args.no_extras and not args.no_per_config:
        per_config = measure_per_config(stream, peaks, args.workload)
    if rank == 0:
        us = ms_step * 1e3
        cfg = workload_config(case, world)
        timing = {"copies": case.copies,
                  "l2": (f"stack weights {case.weight_bytes_total / 1e9:.2f} GB > L2" if case.kind == "stack" else
                         f"fp16 weight {case.N * case.K * 2 / 1e6:.0f} MB + its fp32 working copy "
                         f"{case.N * case.K * 4 / 1e6:.0f} MB > L2" if case.kind == "gptq" else
                         f"rotating {case.copies} weight copies ({case.weight_bytes_total / 1e6:.0f} MB > 2x L2)"),
                  "accumulate": "fp64 rotation, fp32 quantiser" if case.kind == "quantize" else "fp32",
                  "kernel_hash": khash,
                  "launch": ("CUDA graph, consecutive calls overlapped by programmatic dependent launch "
                             "(qlin_set_overlap(1))") if overlap else "CUDA graph, serial launches",
                  "region": "device spin, start event, K steps from CUDA graphs, end event"}
        metric = {"quantize": QUANTIZE_METRIC, "gptq": GPTQ_METRIC}.get(case.kind, METRIC)
        if case.kind == "gptq":  # whole-job fp32 operations per second
            value, unit = world * case.flops * args.steps / (ms * 1e-3) / 1e12, "TFLOP/s"
        else:
            unit = "GB/s"
        out = {"metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": ms_step, "us_per_call": us,
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
               "dtype": {"quantize": "f64", "gptq": "f32"}.get(case.kind, "f16"), "data": "synthetic", "config": cfg, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
               "gpu_launches": case.launches_per_step() * args.steps, "clocks": clocks, "timing": timing}
        if cpu_all is not None:
            out["cpu_baseline_all_cores"] = cpu_all
        if cublas_us is not None:
            out["cublas_bf16"] = {"us_per_call": cublas_us, "speedup": cublas_us / us}
        if no_overlap is not None:
            out["no_overlap"] = no_overlap
        if per_config is not None:
            out["per_config"] = per_config
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_reference(args):
    """The CPU oracle as the reference arm: rank 0 only, bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from dequant_gemv_packed_b200 import workloads as W
    from oracle import qlin_oracle as O
    from threadpoolctl import threadpool_limits
    desc, kind, p = WORKLOADS[args.workload]
    if kind == "stack":
        print(json.dumps({"impl": "reference", "unavailable": "stack workload is not sampled by the CPU oracle arm"}))
        return
    if kind == "gptq":
        print(json.dumps({"impl": "reference", "unavailable": "the GPTQ workload is timed only on the GPU arm"}))
        return
    if kind == "quantize":
        run_reference_quantize(args, desc, p)
        return
    if kind == "gemv":
        fn = getattr(W, p["fn"])
        w, a = fn(M=p["M"]) if p["fn"] != "tiny" else fn()
    else:
        w, a = W.prefill(M=p["M"])
    N, K = w.N, w.K
    bb = None if w.bits else w.block_bits.numpy()
    codes, s, z = w.codes.numpy(), w.scales.numpy(), w.zeros.numpy()
    x, sb = a.x.numpy(), a.sign_bits.numpy().view(np.uint32)
    packed = O.pack(codes, w.bits or None, bb)
    per_row = O.algorithmic_bytes(N, K, w.bits or None, bb) / N
    rng = np.random.default_rng(0)
    total_budget = float(os.environ.get("QLIN_REFERENCE_BUDGET_S", "90"))
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        r = np.sort(rng.choice(N, size=min(32, N), replace=False))
        O.linear64(x, O.unpack(packed, N, K, w.bits or None, bb, rows=r), s[r], z[r], sb)
        t_row = (time.perf_counter() - t0) / len(r)
        rows_per_step = int(max(4, min(N, total_budget / max(args.steps + args.warmup, 1) / t_row)))
        def step():
            r = np.sort(rng.choice(N, size=rows_per_step, replace=False))
            O.linear64(x, O.unpack(packed, N, K, w.bits or None, bb, rows=r), s[r], z[r], sb)
        for _ in range(args.warmup):
            step()
        t1 = time.perf_counter()
        for _ in range(args.steps):
            step()
        t = time.perf_counter() - t1
    ms_step = t * 1e3 / args.steps
    value = rows_per_step * per_row * args.steps / t / 1e9
    sample = f"{rows_per_step} of {N} weight rows per step (unpack + fp64 dequant + explicit-H rotation + fp64 matmul)"
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": workload_config(SimpleNamespace(desc_text=desc, M=a.x.shape[0], K=K, N=N, bits=w.bits, kind=kind),
                                     int(os.environ.get("WORLD_SIZE", "1"))),
           "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_reference_quantize(args, desc, p):
    """Reference arm of the offline tool: the oracle on sampled rows per step."""
    from dequant_gemv_packed_b200 import workloads as W
    from oracle import qlin_oracle as O
    from threadpoolctl import threadpool_limits
    N, K, bits = p["N"], p["K"], p["bits"]
    w = W.draw_fp16_weight(N, K).numpy()
    sb = W.draw_activation(1, K).sign_bits.numpy().view(np.uint32)
    per_row = (N * K * 3 + 4 * N * (K // 128)) / N
    rng = np.random.default_rng(0)
    total_budget = float(os.environ.get("QLIN_REFERENCE_BUDGET_S", "90"))
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        O.quantize_rtn(w[:64], sb, bits)
        t_row = (time.perf_counter() - t0) / 64
        rows_per_step = int(max(4, min(N, total_budget / max(args.steps + args.warmup, 1) / t_row)))
        def step():
            O.quantize_rtn(w[np.sort(rng.choice(N, size=rows_per_step, replace=False))], sb, bits)
        for _ in range(args.warmup):
            step()
        t1 = time.perf_counter()
        for _ in range(args.steps):
            step()
        t = time.perf_counter() - t1
    value = rows_per_step * per_row * args.steps / t / 1e9
    sample = f"{rows_per_step} of {N} weight rows per step (explicit-H fp64 rotation + fp32 RTN)"
    out = {"impl": "reference", "metric": QUANTIZE_METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3 / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": workload_config(SimpleNamespace(desc_text=desc, M=1, K=K, N=N, bits=bits, kind="quantize"),
                                     int(os.environ.get("WORLD_SIZE", "1"))),
           "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: about a second of timed work for the workload; 20 for --impl reference)")
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--workload", default="gateup", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-overlap", action="store_true", help="serial launches only (no programmatic dependent launch)")
    ap.add_argument("--no-extras", action="store_true",
                    help="time the layer only (no e2e, cuBLAS, CPU-baseline or per-config legs), e.g. under a profiler")
    ap.add_argument("--no-per-config", action="store_true", help="skip the per-config table")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.steps is None:
        args.steps = 20 if args.impl == "reference" else DEFAULT_STEPS[WORKLOADS[args.workload][1]]
    if args.steps < 1:
        ap.error("--steps must be >= 1")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
