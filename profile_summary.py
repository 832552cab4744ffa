"""Short summaries of ncu captures for profiles/.

    python profile_summary.py kernel REPORT NAME --files F [F ...] --sources SOURCES.json \
        --command "CMD" --note "TEXT"
    python profile_summary.py launches LAUNCHES.csv NAME --command "CMD" --title "TEXT"

`kernel` reads one `ncu --set full` report (`ncu -i REPORT --page raw --csv`,
which works without a GPU) and writes profiles/NAME.md (the figures used:
duration, DRAM bytes and throughput, pipe and issue activity, occupancy,
registers, the top warp stalls) and profiles/NAME.json, the machine-readable
record the benchmark reads: the kernel's DRAM traffic per launch and a hash of
the CUDA sources it was built from.  SOURCES.json is the per-file hash list
that `bench.py --profile-case` writes on the GPU machine when the capture runs,
so the record names the sources of the capture itself; the benchmark reports
the traffic only while the current sources hash the same.

`launches` reads the CSV of an `ncu --metrics gpu__time_duration.sum` run and
writes profiles/NAME.md: launches, total time and share per kernel.
"""
from __future__ import annotations

import argparse
import collections
import csv
import io
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WANT = [("gpu__time_duration.sum", "duration"), ("dram__bytes_read.sum", "DRAM read"),
        ("dram__bytes_write.sum", "DRAM write"),
        ("gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed", "DRAM throughput % of peak"),
        ("lts__throughput.avg.pct_of_peak_sustained_elapsed", "L2 throughput % of peak"),
        ("sm__throughput.avg.pct_of_peak_sustained_elapsed", "SM throughput % of peak"),
        ("sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active", "tensor pipe active %"),
        ("sm__inst_executed_pipe_fma.avg.pct_of_peak_sustained_active", "FMA pipe %"),
        ("sm__inst_executed_pipe_alu.avg.pct_of_peak_sustained_active", "ALU pipe %"),
        ("smsp__issue_active.avg.pct_of_peak_sustained_active", "issue active %"),
        ("sm__warps_active.avg.pct_of_peak_sustained_active", "warps active % (occupancy)"),
        ("launch__grid_size", "grid"), ("launch__block_size", "block"),
        ("launch__registers_per_thread", "registers/thread"), ("smsp__inst_executed.sum", "warp instructions")]

BYTES = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
USEC = {"nsecond": 1e-3, "ns": 1e-3, "usecond": 1.0, "us": 1.0, "msecond": 1e3, "ms": 1e3}


def _raw(report):
    out = subprocess.run(["ncu", "-i", report, "--page", "raw", "--csv"], capture_output=True, text=True,
                         check=True).stdout
    rows = list(csv.reader(io.StringIO(out)))
    return rows[0], rows[1], rows[2:]


def kernel(args):
    import bench
    head, units, rows = _raw(args.report)
    if not rows:
        raise SystemExit("no kernel in the report")
    r = rows[0]
    lines = [f"# {args.name} -- ncu `--set full` summary", "", args.note, "",
             "Command (GPU box, committed files only):", "", "```", args.command, "```", "",
             "| metric | value |", "|---|---|"]
    got = {}
    for key, label in WANT:
        if key in head:
            i = head.index(key)
            lines.append(f"| {label} (`{key}`) | {r[i]} {units[i]} |")
            got[key] = (r[i], units[i])
    stalls = []
    for i, key in enumerate(head):
        if "stalled" in key and key.endswith("per_issue_active.ratio"):
            try:
                stalls.append((float(r[i]), key))
            except ValueError:
                pass
    lines += ["", "Top warp stall reasons (cycles per issued instruction):", ""]
    lines += [f"- `{k}`: {v:.2f}" for v, k in sorted(stalls, reverse=True)[:5]]

    def nbytes(key):
        v, u = got[key]
        return float(v.replace(",", "")) * BYTES.get(u, 1)

    traffic = int(nbytes("dram__bytes_read.sum") + nbytes("dram__bytes_write.sum"))
    with open(args.sources) as f:
        recorded = json.load(f)
    rec = {"kernel": args.name, "source_files": args.files,
           "source_hash": bench.source_hash(args.files, recorded),
           "traffic_bytes_per_launch": traffic,
           "duration_us": float(got["gpu__time_duration.sum"][0].replace(",", "")) *
           USEC.get(got["gpu__time_duration.sum"][1], 1.0),
           "command": args.command}
    lines += ["", f"DRAM traffic per launch (read + write): {traffic} bytes.",
              f"Sources of the capture: {', '.join(args.files)} (hash {rec['source_hash']}, also in "
              f"{args.name}.json)."]
    with open(os.path.join(ROOT, "profiles", args.name + ".md"), "w") as f:
        f.write("\n".join(lines) + "\n")
    with open(os.path.join(ROOT, "profiles", args.name + ".json"), "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    print("wrote", args.name)


def launches(args):
    rows = list(csv.reader(open(args.csv)))
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    head, data = rows[hi], rows[hi + 1:]
    ki, mi, ui = head.index("Kernel Name"), head.index("Metric Value"), head.index("Metric Unit")
    agg = collections.OrderedDict()
    for r in data:
        if len(r) <= mi:
            continue
        name = r[ki].split("(")[0]
        v = float(r[mi].replace(",", "")) * USEC.get(r[ui], 1.0)
        a = agg.setdefault(name, [0, 0.0])
        a[0] += 1
        a[1] += v
    tot = sum(v[1] for v in agg.values())
    lines = [f"# {args.title}", "",
             "Every kernel launch with its device time (`gpu__time_duration.sum`, one pass).  Times under ncu",
             "are cold-cache and serialised: compare the shares, not the absolute values (the factorization's",
             "streams run concurrently outside ncu).", "",
             "Command (GPU box, committed files only):", "", "```", args.command, "```", "",
             "| kernel | launches | total (us) | share | mean (us) |", "|---|---|---|---|---|"]
    for k, (n, t) in sorted(agg.items(), key=lambda x: -x[1][1]):
        lines.append(f"| `{k}` | {n} | {t:.1f} | {100 * t / tot:.1f}% | {t / n:.1f} |")
    lines.append(f"| total | {sum(v[0] for v in agg.values())} | {tot:.1f} | | |")
    with open(os.path.join(ROOT, "profiles", args.name + ".md"), "w") as f:
        f.write("\n".join(lines) + "\n")
    print("wrote", args.name)


def main():
    ap = argparse.ArgumentParser()
    sub = ap.add_subparsers(dest="what", required=True)
    k = sub.add_parser("kernel")
    k.add_argument("report")
    k.add_argument("name")
    k.add_argument("--files", nargs="+", required=True)
    k.add_argument("--sources", required=True)
    k.add_argument("--command", required=True)
    k.add_argument("--note", required=True)
    k.set_defaults(fn=kernel)
    ll = sub.add_parser("launches")
    ll.add_argument("csv")
    ll.add_argument("name")
    ll.add_argument("--command", required=True)
    ll.add_argument("--title", required=True)
    ll.set_defaults(fn=launches)
    args = ap.parse_args()
    args.fn(args)


if __name__ == "__main__":
    main()
