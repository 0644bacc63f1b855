"""Short text summaries of Nsight Compute output for the profile notes.

Launch list (a `--metrics gpu__time_duration.sum --csv --log-file` run):

    python -m token_recurrent_decoding_b200.ncu_summary launches launches.csv [--match rlt::]

prints, per kernel (template arguments kept, parameter list dropped), the
launches, total time and share of the listed time. Per-launch times from ncu
are serialised and cold-cache, so shares are the figure to compare.

Raw page of a capture (`ncu -i report.ncu-rep --page raw --csv > raw.csv`):

    python -m token_recurrent_decoding_b200.ncu_summary raw raw.csv

prints, per captured launch, the duration, DRAM bytes read + written,
DRAM throughput, tensor-pipe activity, achieved occupancy, registers and the
top warp stall reasons.
"""
from __future__ import annotations

import argparse
import collections
import csv
import io
import re


def _rows(path):
    text = open(path, encoding="utf-8", errors="replace").read()
    start = text.find('"ID"')
    if start < 0:
        raise SystemExit(f"{path}: no CSV header")
    return list(csv.reader(io.StringIO(text[start:])))


def kernel_key(name: str) -> str:
    name = re.sub(r"^void\s+", "", name)
    depth, out = 0, []
    for ch in name:  # drop the parameter list, keep template arguments
        if ch == "(" and depth == 0:
            break
        depth += ch == "<"
        depth -= ch == ">"
        out.append(ch)
    return "".join(out).strip()


def launches(path, match=None):
    rows = _rows(path)
    hdr = rows[0]
    ki, mi, vi = hdr.index("Kernel Name"), hdr.index("Metric Name"), hdr.index("Metric Value")
    agg = collections.OrderedDict()
    for r in rows[1:]:
        if len(r) <= vi or r[mi] != "gpu__time_duration.sum":
            continue
        k = kernel_key(r[ki])
        if match and not re.search(match, k):
            continue
        v = float(r[vi].replace(",", ""))
        n, t = agg.get(k, (0, 0.0))
        agg[k] = (n + 1, t + v)
    tot = sum(t for _, t in agg.values()) or 1.0
    unit = hdr and "ns"
    lines = [f"{'kernel':<72} {'launches':>8} {'total us':>10} {'mean us':>9} {'share':>6}"]
    for k, (n, t) in sorted(agg.items(), key=lambda kv: -kv[1][1]):
        lines.append(f"{k[:72]:<72} {n:>8d} {t / 1e3:>10.1f} {t / n / 1e3:>9.2f} {t / tot:>6.3f}")
    lines.append(f"{'total':<72} {sum(n for n, _ in agg.values()):>8d} {tot / 1e3:>10.1f}")
    del unit
    return "\n".join(lines)


RAW = [
    ("duration", "gpu__time_duration.sum"),
    ("dram read", "dram__bytes_read.sum"),
    ("dram write", "dram__bytes_write.sum"),
    ("dram throughput % of peak", "gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed"),
    ("tensor pipe active %", "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active"),
    ("achieved occupancy %", "sm__warps_active.avg.pct_of_peak_sustained_active"),
    ("registers / thread", "launch__registers_per_thread"),
    ("grid size", "launch__grid_size"),
    ("block size", "launch__block_size"),
    ("dynamic smem / block", "launch__shared_mem_per_block_dynamic"),
]


def raw(path):
    rows = list(csv.reader(open(path, encoding="utf-8", errors="replace")))
    hdr = rows[0]
    units = rows[1] if len(rows) > 1 else [""] * len(hdr)
    data = [r for r in rows[2:] if len(r) == len(hdr)]
    col = {h: i for i, h in enumerate(hdr)}
    out = []
    for r in data:
        name = kernel_key(r[col["Kernel Name"]]) if "Kernel Name" in col else "?"
        out.append(f"launch {r[col['ID']] if 'ID' in col else '?'}: {name}")
        for label, m in RAW:
            if m in col:
                out.append(f"  {label:<28} {r[col[m]]} {units[col[m]]}".rstrip())
        rd = wr = None
        if "dram__bytes_read.sum" in col and "dram__bytes_write.sum" in col:
            rd = _bytes(r[col["dram__bytes_read.sum"]], units[col["dram__bytes_read.sum"]])
            wr = _bytes(r[col["dram__bytes_write.sum"]], units[col["dram__bytes_write.sum"]])
            out.append(f"  {'dram read + write (bytes)':<28} {rd + wr:.6g}")
        stalls = []
        for h, i in col.items():
            mm = re.match(r"smsp__average_warps_issue_stalled_(\w+)_per_issue_active\.ratio$", h)
            if mm:
                try:
                    stalls.append((float(r[i].replace(",", "")), mm.group(1)))
                except ValueError:
                    pass
        if stalls:
            top = ", ".join(f"{n} {v:.2f}" for v, n in sorted(stalls, reverse=True)[:6])
            out.append(f"  {'top stalls (per issue)':<28} {top}")
    return "\n".join(out)


def _bytes(v, unit):
    x = float(v.replace(",", ""))
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6,
             "GB": 1e9}.get(unit.strip(), 1)
    return x * scale


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("mode", choices=["launches", "raw"])
    ap.add_argument("path")
    ap.add_argument("--match", default=None, help="regex on the kernel name")
    a = ap.parse_args()
    print(launches(a.path, a.match) if a.mode == "launches" else raw(a.path))


if __name__ == "__main__":
    main()
