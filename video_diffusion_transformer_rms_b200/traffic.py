"""DRAM traffic records of the hot-path kernels, kept in profiles/traffic.json.

    python -m video_diffusion_transformer_rms_b200.traffic \
        --csv dram8.csv --captured-rows 32658 [--csv dram16.csv --captured-rows 65316] \
        --kernel qknorm_rope3d_tab --workload clip5s --command "<the commands>"

reads ncu CSV exports (`ncu --csv --log-file ...`) of dram__bytes_read.sum
and dram__bytes_write.sum for one kernel captured on slices of a workload,
averages them per launch and carries them to the workload's full row count.
Each kernel streams its rows once, so its traffic is a + b * rows: with two
slices of different sizes the line through them is evaluated at the full
size (the constant a holds the writes still in L2 when a launch ends, which
do not grow with the rows); with one slice the bytes are scaled by the rows.
The record keeps the sha256 of the sources the kernel is built from, and
`lookup` (bench.py's `roofline.traffic`) returns it only while those sources
are unchanged.
"""
import argparse
import csv
import hashlib
import json
import os

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
RECORDS = os.path.join(ROOT, "profiles", "traffic.json")

_COMMON = ["sol_device.cuh", "sol_launch.h", "sol_abi.cu"]
# the sources each kernel (as bench.py names it) is built from
KERNEL_SOURCES = {
    "rms_adaln": ["rms_adaln.cu"] + _COMMON,
    "gate_residual": ["gate_residual.cu"] + _COMMON,
    "qknorm_rope3d": ["qknorm_rope3d.cuh", "qknorm_rope3d_bf16.cu"] + _COMMON,
    "qknorm_rope3d_tab": ["qknorm_rope3d.cuh", "qknorm_rope3d_tab_bf16.cu", "rope_table.cu"]
    + _COMMON,
    "gate_residual_rms_adaln": ["rms_adaln.cu"] + _COMMON,
    "residual_change": ["residual_change.cu"] + _COMMON,
    "qknorm_rope3d_ex_bhsd_tab": ["qknorm_rope3d.cuh", "qknorm_rope3d_ex.cuh",
                                  "qknorm_rope3d_ex_tab_bf16.cu", "rope_table.cu"] + _COMMON,
    "qknorm_rope3d_ex_half_tab": ["qknorm_rope3d.cuh", "qknorm_rope3d_ex.cuh",
                                  "qknorm_rope3d_ex_tab_bf16.cu", "rope_table.cu"] + _COMMON,
    "qknorm_rope3d_ex_int8_tab": ["qknorm_rope3d.cuh", "qknorm_rope3d_ex.cuh",
                                  "qknorm_rope3d_ex_tab_int8.cu", "rope_table.cu"] + _COMMON,
    "gemm_gelu": ["gemm_gelu.cu"] + _COMMON,
}

_UNITS = {"byte": 1.0, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "tbyte": 1e12}


def source_sha(kernel, root=None):
    """sha256 over the kernel's source files, in order."""
    h = hashlib.sha256()
    csrc = os.path.join(root or ROOT, "video_diffusion_transformer_rms_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def parse_ncu_csv(path):
    """Per-launch (read, write) DRAM bytes from an ncu CSV export: a list of
    (kernel name, read bytes, write bytes), one entry per captured launch."""
    launches = {}
    with open(path, newline="") as fh:
        lines = [ln for ln in fh if ln.startswith('"')]  # drop ncu's ==PROF== chatter
    for row in csv.DictReader(lines):
        metric = row.get("Metric Name", "")
        if metric not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        scale = _UNITS.get(row.get("Metric Unit", "byte").strip().lower())
        if scale is None:
            raise ValueError(f"unknown unit {row.get('Metric Unit')!r} in {path}")
        value = float(row["Metric Value"].replace(",", "")) * scale
        entry = launches.setdefault(row["ID"], [row.get("Kernel Name", ""), 0.0, 0.0])
        entry[1 if metric.endswith("read.sum") else 2] += value
    return [tuple(v) for _, v in sorted(launches.items(), key=lambda kv: int(kv[0]))]


def make_record(captures, kernel, workload, full_rows, command, root=None):
    """captures: [(launches from parse_ncu_csv, captured rows)], one or two."""
    if not captures or any(not c[0] for c in captures):
        raise ValueError("the CSV holds no dram__bytes_read/write.sum rows")
    pts = []
    for launches, rows in captures:
        rd = sum(x[1] for x in launches) / len(launches)
        wr = sum(x[2] for x in launches) / len(launches)
        pts.append((rows, rd, wr))
    if len(pts) == 1:
        rows, rd, wr = pts[0]
        full_rd, full_wr = rd * full_rows / rows, wr * full_rows / rows
        how = f"x {full_rows / rows:.4f} = full rows / captured rows"
    else:
        (r0, rd0, wr0), (r1, rd1, wr1) = pts[:2]
        if r0 == r1:
            raise ValueError("two captures need different row counts")
        full_rd = rd0 + (rd1 - rd0) * (full_rows - r0) / (r1 - r0)
        full_wr = wr0 + (wr1 - wr0) * (full_rows - r0) / (r1 - r0)
        how = f"line through the {r0}- and {r1}-row captures, at {full_rows} rows"
    return {"workload": workload, "kernel_name": captures[0][0][0][0],
            "captures": [{"rows": r, "read_bytes": rd, "write_bytes": wr} for r, rd, wr in pts],
            "full_rows": full_rows, "read_bytes_per_launch": full_rd,
            "write_bytes_per_launch": full_wr,
            "traffic_bytes_per_launch": full_rd + full_wr, "scaling": how,
            "source_sha256": source_sha(kernel, root), "command": command}


def load(root=None):
    path = os.path.join(root, "profiles", "traffic.json") if root else RECORDS
    try:
        with open(path) as fh:
            return json.load(fh)
    except (OSError, ValueError):
        return {}


def lookup(kernel, workload, root=None):
    """DRAM bytes per full-size launch, or None if there is no record for this
    kernel and workload or a source changed since it was taken."""
    rec = load(root).get(kernel)
    if not rec or rec.get("workload") != workload or kernel not in KERNEL_SOURCES:
        return None
    if rec.get("source_sha256") != source_sha(kernel, root):
        return None
    return float(rec["traffic_bytes_per_launch"])


def main():
    from .workloads import WORKLOADS
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--csv", action="append", required=True)
    ap.add_argument("--captured-rows", type=int, action="append", required=True)
    ap.add_argument("--kernel", required=True, choices=sorted(KERNEL_SOURCES))
    ap.add_argument("--workload", default="clip5s", choices=sorted(WORKLOADS))
    ap.add_argument("--command", required=True)
    args = ap.parse_args()
    if len(args.csv) != len(args.captured_rows) or len(args.csv) > 2:
        raise SystemExit("give one or two --csv, each with its --captured-rows")
    caps = [(parse_ncu_csv(c), r) for c, r in zip(args.csv, args.captured_rows)]
    rec = make_record(caps, args.kernel, args.workload, WORKLOADS[args.workload].rows,
                      args.command)
    records = load()
    records[args.kernel] = rec
    os.makedirs(os.path.dirname(RECORDS), exist_ok=True)
    with open(RECORDS, "w") as fh:
        json.dump(records, fh, indent=1, sort_keys=True)
        fh.write("\n")
    print(json.dumps(rec, indent=1))


if __name__ == "__main__":
    main()
