"""Summaries of Nsight Compute output used for the committed profiles.

    python -m dequant_gemv_packed_b200.ncu_summary launches <launches.csv> [regex]
        per kernel: launches, total device time and share of the listed time
        (only kernels whose short name matches regex, if given)
        (input: ncu --metrics gpu__time_duration.sum --csv --log-file ...)

    python -m dequant_gemv_packed_b200.ncu_summary report <file.ncu-rep> [regex]
        key counters of each captured launch (needs the ncu CLI to read the report)
"""
from __future__ import annotations

import collections
import csv
import io
import re
import subprocess
import sys

KEY_METRICS = (
    "gpu__time_duration.sum",
    "dram__bytes_read.sum",
    "dram__bytes_write.sum",
    "gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed",
    "sm__throughput.avg.pct_of_peak_sustained_elapsed",
    "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed",
    "smsp__inst_executed.sum",
    "smsp__issue_active.avg.pct_of_peak_sustained_active",
    "sm__warps_active.avg.pct_of_peak_sustained_active",
    "launch__registers_per_thread",
    "launch__grid_size",
    "launch__block_size",
    "smsp__average_warps_issue_stalled_long_scoreboard_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_short_scoreboard_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_wait_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_barrier_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_math_pipe_throttle_per_issue_active.ratio",
    "l1tex__data_bank_conflicts_pipe_lsu_mem_shared.sum",
)


def short_name(name: str) -> str:
    m = re.search(r"qlin::(?:[\w<>]+::)*?(\w+_kernel)(?:<([^>]*)>)?", name)
    if m:
        return m.group(1) + (f"<{m.group(2)}>" if m.group(2) else "")
    base = re.sub(r"\(.*", "", name)
    return base[:80]


def launches(path: str, only: str | None = None) -> str:
    rows = [r for r in csv.reader(open(path)) if len(r) > 10]
    hdr, data = rows[0], rows[1:]
    i_name, i_metric, i_val = hdr.index("Kernel Name"), hdr.index("Metric Name"), hdr.index("Metric Value")
    per = collections.OrderedDict()
    for r in data:
        if r[i_metric] != "gpu__time_duration.sum":
            continue
        k = short_name(r[i_name])
        if only and not re.search(only, k):
            continue
        n, t = per.get(k, (0, 0.0))
        per[k] = (n + 1, t + float(r[i_val].replace(",", "")))
    total = sum(t for _, t in per.values())
    out = io.StringIO()
    out.write(f"{'kernel':58s} {'launches':>8s} {'total_us':>11s} {'share':>7s}\n")
    for k, (n, t) in sorted(per.items(), key=lambda kv: -kv[1][1]):
        out.write(f"{k:58s} {n:8d} {t / 1e3:11.1f} {100 * t / total:6.1f}%\n")
    return out.getvalue()


def report(path: str, pattern: str = ".*") -> str:
    txt = subprocess.run(["ncu", "-i", path, "--page", "raw", "--csv"], capture_output=True, text=True).stdout
    rows = list(csv.reader(io.StringIO(txt)))
    hdr, data = rows[0], rows[2:]
    idx = {h: i for i, h in enumerate(hdr)}
    out = io.StringIO()
    for r in data:
        name = short_name(r[idx["Kernel Name"]])
        if not re.search(pattern, name):
            continue
        out.write(f"== {name}\n")
        for m in KEY_METRICS:
            if m in idx:
                out.write(f"  {m:80s} {r[idx[m]]}\n")
    return out.getvalue()


def main() -> None:
    if len(sys.argv) < 3 or sys.argv[1] not in ("launches", "report"):
        print(__doc__)
        sys.exit(2)
    if sys.argv[1] == "launches":
        print(launches(sys.argv[2], sys.argv[3] if len(sys.argv) > 3 else None), end="")
    else:
        print(report(sys.argv[2], sys.argv[3] if len(sys.argv) > 3 else ".*"), end="")


if __name__ == "__main__":
    main()
