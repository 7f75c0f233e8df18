"""DRAM traffic records of the hot-path kernels, kept in profiles/traffic.json.

    python -m video_diffusion_transformer_rms_b200.traffic \
        --csv dram.csv --kernel qknorm_rope3d_tab --workload clip5s \
        --captured-rows 32768 --command "<the ncu command that wrote dram.csv>"

reads an ncu CSV export (`ncu --csv --log-file ...`) of dram__bytes_read.sum
and dram__bytes_write.sum for one kernel captured on a slice of a workload,
averages them per launch, scales them to the workload's full row count (each
kernel streams its rows once, so its traffic grows in proportion to the rows)
and stores the record together with the sha256 of the sources the kernel is
built from.  `lookup` (bench.py's `roofline.traffic`) returns the record only
while those sources are unchanged.
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


def make_record(launches, kernel, workload, captured_rows, full_rows, command, root=None):
    if not launches:
        raise ValueError("the CSV holds no dram__bytes_read/write.sum rows")
    rd = sum(x[1] for x in launches) / len(launches)
    wr = sum(x[2] for x in launches) / len(launches)
    scale = full_rows / captured_rows
    return {"workload": workload, "kernel_name": launches[0][0], "launches": len(launches),
            "captured_rows": captured_rows, "full_rows": full_rows,
            "captured_read_bytes": rd, "captured_write_bytes": wr,
            "traffic_bytes_per_launch": (rd + wr) * scale,
            "scaling": f"x {scale:.4f} = full rows / captured rows (traffic grows with rows)",
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
    ap.add_argument("--csv", required=True)
    ap.add_argument("--kernel", required=True, choices=sorted(KERNEL_SOURCES))
    ap.add_argument("--workload", default="clip5s", choices=sorted(WORKLOADS))
    ap.add_argument("--captured-rows", type=int, required=True)
    ap.add_argument("--command", required=True)
    args = ap.parse_args()
    rec = make_record(parse_ncu_csv(args.csv), args.kernel, args.workload, args.captured_rows,
                      WORKLOADS[args.workload].rows, args.command)
    records = load()
    records[args.kernel] = rec
    os.makedirs(os.path.dirname(RECORDS), exist_ok=True)
    with open(RECORDS, "w") as fh:
        json.dump(records, fh, indent=1, sort_keys=True)
        fh.write("\n")
    print(json.dumps(rec, indent=1))


if __name__ == "__main__":
    main()
