#!/usr/bin/env python
"""Benchmark of the fused per-token DiT hot path on B200.

One step = one pass of all three kernels over one batch of the 5 s
1344x768 clip shape (126,552 tokens: 31x48x84 video latent patches + 1,560
audio tokens, D = 5120 = 40 heads x 128, bf16):
  RMS-AdaLN (x -> y), QKNorm + 3D RoPE (merged qkv -> q, k), gated residual
  (h, branch -> out).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 is launched by torchrun (one process per GPU); each rank processes its
own clip (weak scaling, no data exchange), the timed region is bracketed by
barriers and the time is the max over ranks.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the only other implementation
of these operations) on the host cores, one process per core, one bounded
sample of clip rows per process per step; under torchrun only rank 0 runs it.
"""
import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from video_diffusion_transformer_rms_b200 import dist, traffic  # noqa: E402
from video_diffusion_transformer_rms_b200.workloads import (WORKLOADS, activation,  # noqa: E402
                                                            make_inputs, to_oracle_array,
                                                            vectors)

METRIC = "tokens/s and achieved HBM GB/s (% of B200 peak) per fused kernel, 1 GPU"
WORKLOAD = "clip5s"
KERNELS = ("rms_adaln", "qknorm_rope3d", "gate_residual")
# Where the step's QKNorm + RoPE gets its (cos, sin): False = per row, on the
# fly (sol_qknorm_rope3d); True = a rotary table built once per clip shape
# (sol_qknorm_rope3d_tab).  The other one is timed beside the step.
QK_TABLE = True
# the traffic record (profiles/traffic.json) of the kernel each step name runs
TRAFFIC_NAME = {"rms_adaln": "rms_adaln", "gate_residual": "gate_residual",
                "qknorm_rope3d": "qknorm_rope3d_tab" if QK_TABLE else "qknorm_rope3d"}
# every config of the task, each step kernel timed on its own (clip5s is the
# headline step above)
PER_CONFIG = ("clip5s", "clip15s", "cfg5s", "cfg5s_d3072", "medium")
COOL_DOWN_S = 2.0  # idle seconds before the per-config block (outside every timed region)
L2_FLUSH_BYTES = 256 << 20   # written between reps where the inputs fit in L2
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
ORACLE_SECONDS_PER_ROW = 0.4e-3  # all three oracle ops on one clip row (estimate)


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="oracle time budget of the CPU baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def workload_config(w, n_gpus):
    return {
        "workload": (f"{w.name}: 5 s 1344x768 24 fps clip shape, B={w.B}, latent grid "
                     f"T={w.T} H={w.H} W={w.W} ({w.n_video} video tokens) + {w.n_audio} audio "
                     f"tokens = {w.L} tokens per sample, D={w.D} ({w.n_heads}x{w.head_dim} "
                     f"heads), merged QKV [{w.L}, {3 * w.D}], RoPE sections "
                     f"{'/'.join(map(str, w.sections))}, theta {w.theta:g}, eps {w.eps:g}"),
        "tokens_per_gpu": w.rows,
        "global_tokens_per_step": w.rows * n_gpus,
        "D": w.D,
        "io_dtype": w.dtype,
        "step": "rms_adaln + qknorm_rope3d" + ("_tab" if QK_TABLE else "") +
                " + gate_residual, one launch each",
        "l2": "no flush: every input is larger than the 126 MB L2 (1.3-3.9 GB per tensor)",
        "parallelism": f"{n_gpus} independent shards (one clip per GPU), no data-path collective",
        "inputs": "seeded synthetic N(0,1) activations with 1% outlier channels x20",
    }


# ----------------------------------------------------------------------------
# peaks, clocks, ncu traffic record
# ----------------------------------------------------------------------------

def load_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def traffic_record(kernel, workload):
    """DRAM bytes per full-size launch from profiles/traffic.json, or None if
    there is no record or the kernel's sources changed since it was taken."""
    return traffic.lookup(TRAFFIC_NAME.get(kernel, kernel), workload, ROOT)


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while running."""
    FIELDS = ("timestamp,index,uuid,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            pass
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "200"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.5)

    def mark(self):
        return time.time()

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": "nvidia-smi unavailable"}
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        lines = self.file.read().splitlines()
        os.unlink(self.file.name)
        return self.summarise(lines, self.uuid, t0, t1)

    @classmethod
    def summarise(cls, lines, uuid, t0, t1):
        """Median SM clock, max clock and the throttle reasons active in the
        samples of this GPU (uuid) taken within [t0 - 1, t1 + 1] (all of its
        samples if none fall inside)."""
        rows = []
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            if uuid and uuid not in parts[2] and parts[2] not in f"GPU-{uuid}":
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(parts[3]), float(parts[4]), parts[6:10]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 - 1 <= r[0] <= t1 + 1] or rows
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "no samples"}
        reasons = sorted({name for r in inside for name, v in zip(cls.REASONS, r[3])
                          if v.strip().lower() == "active"})
        return {"sm_mhz": float(np.median([r[1] for r in inside])),
                "sm_max_mhz": float(max(r[2] for r in inside)), "reasons": reasons,
                "samples": len(inside)}


# ----------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of clip rows
# ----------------------------------------------------------------------------

def oracle_sample_run(w, n_rows, seed, timer):
    """Run the three oracle ops on n_rows rows of the workload spread over the
    sequence (video and audio); returns oracle seconds (inputs drawn outside
    the timed part)."""
    import oracle
    ids = np.linspace(0, w.rows - 1, n_rows).round().astype(np.int64)
    bf = w.torch_dtype
    x = to_oracle_array(activation(n_rows, w.D, bf, "cpu", seed, w.outliers))
    h = to_oracle_array(activation(n_rows, w.D, bf, "cpu", seed + 1, w.outliers))
    br = to_oracle_array(activation(n_rows, w.D, bf, "cpu", seed + 2, w.outliers))
    qk = to_oracle_array(activation(n_rows, 2 * w.D, bf, "cpu", seed + 3, w.outliers))
    mod = to_oracle_array(vectors((w.B, 2, w.D), 0.0, 0.5, bf, "cpu", seed + 4))
    gq = to_oracle_array(vectors((w.head_dim,), 1.0, 0.1, bf, "cpu", seed + 5))
    t0 = timer()
    oracle.rms_adaln(x, mod, mod, w.L, w.n_video, w.eps, row_ids=ids)
    oracle.qknorm_rope3d(qk, w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim, w.sections,
                         w.eps, w.theta, gamma_q=gq, gamma_k=gq, row_ids=ids)
    oracle.gate_residual(h, br, mod, w.L, w.n_video, row_ids=ids)
    return timer() - t0


MAX_ORACLE_PROCS = 32  # bound on the all-cores leg of the CPU baseline


def _oracle_worker(arg):
    """Oracle rows of the named workload for about budget_s seconds of oracle
    time, starting at wall time start_at (if given): (rows done, oracle
    seconds, seconds started late).  Module level, so spawned workers can
    run it."""
    name, budget_s, seed, start_at = arg
    torch.set_num_threads(1)
    w = WORKLOADS[name]
    late = 0.0
    if start_at is not None:
        wait = start_at - time.time()
        if wait > 0:
            time.sleep(wait)
        late = max(0.0, -wait)
    done, spent, chunk = 0, 0.0, 256
    while spent < budget_s:
        spent += oracle_sample_run(w, chunk, seed, time.perf_counter)
        done += chunk
        seed += 10
    return done, spent, late


def cpu_baseline(w, budget_s):
    """The oracle as it stands on the host cores: one thread, then one
    spawned process per core (up to MAX_ORACLE_PROCS) each on its own rows,
    rates summed (the processes run side by side).  Spawned, not forked:
    this runs after the GPU work."""
    import multiprocessing
    from concurrent.futures import ProcessPoolExecutor
    done, spent, _ = _oracle_worker((w.name, budget_s, 900_000, None))
    single = done / spent
    n = max(1, min(os.cpu_count() or 1, MAX_ORACLE_PROCS))
    parts = []
    if n > 1:
        # all workers start their oracle loops at one wall time, after the
        # spawned interpreters have imported, so the loops run side by side;
        # a worker that dies raises BrokenProcessPool here instead of hanging
        start_at = time.time() + 20.0
        with ProcessPoolExecutor(n, mp_context=multiprocessing.get_context("spawn")) as ex:
            parts = list(ex.map(_oracle_worker,
                                [(w.name, budget_s / 2, 950_000 + 1000 * i, start_at)
                                 for i in range(n)], timeout=600))
    rate = sum(d / t for d, t, _ in parts) if parts else single
    rows_all = sum(d for d, _, _ in parts)
    late = max((x for _, _, x in parts), default=0.0)
    return {"value": rate, "unit": "tokens/s", "cores": n, "kind": "oracle",
            "single_thread_value": single,
            "cpu_model": cpu_model(),
            "sample": (f"rows of the {w.name} workload spread over video and audio, all three "
                       f"ops, fp64 oracle: {rows_all} rows in {n} processes side by side "
                       f"(~{budget_s / 2:.0f} s of oracle time each, started together, the "
                       f"latest {late:.1f} s late), and {done} rows in one thread "
                       f"({spent:.1f} s)")}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def run_ours(args):
    from video_diffusion_transformer_rms_b200 import _abi, api
    from video_diffusion_transformer_rms_b200 import build as libbuild

    rank, local_rank, world = dist.init("nccl", timeout_s=300.0)
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if rank == 0:
        libbuild.build()
    dist.barrier()
    _abi.lib()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOADS[WORKLOAD]
    D = w.D

    t = make_inputs(w, dev)
    x = t["x"].view(w.B, w.L, D)
    h = t["h"].view(w.B, w.L, D)
    br = t["branch"].view(w.B, w.L, D)
    qkv = t["qkv"].view(w.B, w.L, 3 * D)
    y = torch.empty_like(x)
    out = torch.empty_like(h)
    qk = torch.empty((w.B, w.L, 2 * D), dtype=qkv.dtype, device=dev)
    stream = torch.cuda.current_stream(dev)
    s = stream.cuda_stream
    dt = _abi.SOL_BF16
    st, sh_, sw = w.sections
    p = {k: v.data_ptr() for k, v in t.items()}
    ld_out = 2 * D

    def k_rms():
        return _abi.sol_rms_adaln(p["x"], y.data_ptr(), p["scale"], p["shift"], None, w.B, w.L,
                                  w.n_video, D, w.eps, dt, s)

    # rotary table of the clip's positions, built once per shape (like a
    # model's RoPE cache) before any timed step; its build is timed apart
    table = api.RopeTable.for_grid(w.T, w.H, w.W, w.n_audio, w.head_dim, sections=w.sections,
                                   theta=w.theta, device=dev)
    tab_ms = time_launches(lambda: _abi.sol_rope_table_build(table.desc, s), stream, 20)

    def k_qk_otf():
        return _abi.sol_qknorm_rope3d(p["qkv"], 3 * D, qk.data_ptr(), qk.data_ptr() + D * 2,
                                      ld_out, p["gamma_q"], p["gamma_k"], w.B, w.T, w.H, w.W,
                                      w.n_audio, w.n_heads, w.head_dim, st, sh_, sw, w.eps,
                                      w.theta, dt, s)

    def k_qk_tab():
        return _abi.sol_qknorm_rope3d_tab(p["qkv"], 3 * D, qk.data_ptr(), qk.data_ptr() + D * 2,
                                          ld_out, p["gamma_q"], p["gamma_k"], table.desc, w.B,
                                          w.T, w.H, w.W, w.n_audio, w.n_heads, w.eps, dt, s)

    k_qk = k_qk_tab if QK_TABLE else k_qk_otf

    def k_gate():
        return _abi.sol_gate_residual(p["h"], p["branch"], p["gate"], out.data_ptr(), w.B, w.L,
                                      w.n_video, D, dt, s)

    launch = {"rms_adaln": k_rms, "qknorm_rope3d": k_qk, "gate_residual": k_gate}

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        for i, name in enumerate(KERNELS):
            _abi.check(launch[name]())
            if ev is not None:
                ev[i + 1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(KERNELS) + 1)]
           for _ in range(K)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    clocks.start()
    dist.barrier()
    torch.cuda.synchronize()
    t0 = clocks.mark()
    start.record(stream)
    for i in range(K):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    t1 = clocks.mark()
    dist.barrier()
    clock_info = clocks.stop(t0, t1)
    elapsed_s = start.elapsed_time(end) / 1e3
    per_kernel_ms = {name: sum(e[i].elapsed_time(e[i + 1]) for e in evs) / K
                     for i, name in enumerate(KERNELS)}

    value, total_units, slowest = dist.job_throughput(w.rows * K, elapsed_s)
    per_kernel_ms = {k: dist.max_over_ranks(v) for k, v in per_kernel_ms.items()}

    # ---- next-row kernels, timed on their own after the step -------------
    ws = torch.empty(_abi.sol_residual_change_workspace_bytes(w.B), dtype=torch.uint8,
                     device=dev)
    rc_out = torch.empty((w.B + 1, 3), dtype=torch.float64, device=dev)
    # QKNorm+RoPE epilogue variants write into the step's q/k buffer (q in its
    # first half, k in the second) or, for INT8, into code and scale buffers
    half_bytes = w.rows * D * w.esize
    q8 = torch.empty(2 * w.rows * D, dtype=torch.int8, device=dev)
    s8 = torch.empty(2 * w.rows * w.n_heads, dtype=torch.float32, device=dev)
    hd = w.head_dim
    lay_bhsd = _abi.QkLayout(w.L * D, hd, w.L * hd, 0, 0, None, None)
    lay_half = _abi.QkLayout(w.L * D, D, hd, 1, 0, None, None)
    lay_int8 = _abi.QkLayout(w.L * D, D, hd, 0, 1, s8.data_ptr(),
                             s8.data_ptr() + w.rows * w.n_heads * 4)
    v8 = torch.empty(w.rows * D, dtype=torch.int8, device=dev)
    vs8 = torch.empty(w.rows * w.n_heads, dtype=torch.float32, device=dev)
    lay_int8_v = _abi.QkLayout(w.L * D, D, hd, 0, 1, s8.data_ptr(),
                               s8.data_ptr() + w.rows * w.n_heads * 4, 0, 0, v8.data_ptr(),
                               vs8.data_ptr())

    def k_qk_ex(lay, q_ptr, k_ptr, use_table=QK_TABLE):
        if use_table:
            return lambda: _abi.sol_qknorm_rope3d_ex_tab(
                p["qkv"], 3 * D, q_ptr, k_ptr, lay, p["gamma_q"], p["gamma_k"], table.desc, w.B,
                w.T, w.H, w.W, w.n_audio, w.n_heads, w.eps, dt, s)
        return lambda: _abi.sol_qknorm_rope3d_ex(
            p["qkv"], 3 * D, q_ptr, k_ptr, lay, p["gamma_q"], p["gamma_k"], w.B, w.T, w.H, w.W,
            w.n_audio, w.n_heads, hd, st, sh_, sw, w.eps, w.theta, dt, s)

    row = D * w.esize  # bytes of one D-wide bf16 row
    extra = {
        # the other source of (cos, sin) for the step's QKNorm + RoPE: per row,
        # on the fly (fp64 angle reduction, sincosf, a CTA barrier per stage)
        ("qknorm_rope3d_table" if not QK_TABLE else "qknorm_rope3d_otf"):
            (4 * row, k_qk_otf if QK_TABLE else k_qk_tab),
        # h_out = h + gate*branch and y = RMS-AdaLN(h_out) in one pass: 4 D-wide rows
        "gate_residual_rms_adaln": (4 * row, lambda: _abi.sol_gate_residual_rms_adaln(
            p["h"], p["branch"], p["gate"], out.data_ptr(), y.data_ptr(), p["scale"],
            p["shift"], None, w.B, w.L, w.n_video, D, w.eps, dt, s)),
        # First-Block-Cache change of h against branch (stand-ins for two steps'
        # residuals): 2 D-wide rows read; with the cache refresh 3
        "residual_change": (2 * row, lambda: _abi.sol_residual_change(
            p["h"], p["branch"], None, w.B, w.L, D, rc_out.data_ptr(), ws.data_ptr(),
            ws.numel(), dt, s)),
        "residual_change_refresh": (3 * row, lambda: _abi.sol_residual_change(
            p["h"], p["branch"], out.data_ptr(), w.B, w.L, D, rc_out.data_ptr(),
            ws.data_ptr(), ws.numel(), dt, s)),
        # q, k read and written (4 rows) in attention's [B, H, L, hd] layout
        "qknorm_rope3d_ex_bhsd": (4 * row, k_qk_ex(lay_bhsd, qk.data_ptr(),
                                                   qk.data_ptr() + half_bytes)),
        # half-split rotary pairs
        "qknorm_rope3d_ex_half": (4 * row, k_qk_ex(lay_half, qk.data_ptr(),
                                                   qk.data_ptr() + half_bytes)),
        # INT8 codes (2D bytes) + fp32 scales per (row, head) for q and k
        "qknorm_rope3d_ex_int8": (2 * row + 2 * D + 2 * w.n_heads * 4,
                                  k_qk_ex(lay_int8, q8.data_ptr(), q8.data_ptr() + w.rows * D)),
        # the same, plus v quantised as it stands (a second launch): q, k, v read,
        # three sets of codes and scales written
        "qknorm_rope3d_ex_int8_qkv": (3 * row + 3 * D + 3 * w.n_heads * 4,
                                      k_qk_ex(lay_int8_v, q8.data_ptr(),
                                              q8.data_ptr() + w.rows * D)),
    }
    # the epilogue variants with the other (cos, sin) source too
    other = "_otf" if QK_TABLE else "_table"
    for name, lay, qp, kp, bpr_ in (
            ("qknorm_rope3d_ex_bhsd", lay_bhsd, qk.data_ptr(), qk.data_ptr() + half_bytes,
             4 * row),
            ("qknorm_rope3d_ex_half", lay_half, qk.data_ptr(), qk.data_ptr() + half_bytes,
             4 * row),
            ("qknorm_rope3d_ex_int8", lay_int8, q8.data_ptr(), q8.data_ptr() + w.rows * D,
             2 * row + 2 * D + 2 * w.n_heads * 4)):
        extra[name + other] = (bpr_, k_qk_ex(lay, qp, kp, not QK_TABLE))
    next_rows = {}
    for name, (bytes_per_row, fn) in extra.items():
        ms = dist.max_over_ranks(time_launches(fn, stream, 200))
        nbytes = bytes_per_row * w.rows
        next_rows[name] = {"ms": round(ms, 4), "tokens_per_s": round(w.rows / (ms / 1e3)),
                           "bytes_per_token": bytes_per_row,
                           "GB_per_s": round(nbytes / (ms / 1e3) / 1e9, 1)}
    del ws, q8, s8, v8, vs8

    # ---- every config: each step kernel on its own (before the GEMM: it runs
    # at the power cap, and the kernels right after it ran slow).  An idle
    # pause first: the next rows' 200-launch loops leave the GPU at its power
    # cap, and the first config timed right after them dipped in some runs.
    peak, peak_kind = load_peak()
    torch.cuda.synchronize()
    time.sleep(COOL_DOWN_S)
    configs = {c: time_config(WORKLOADS[c], dev, stream, peak) for c in PER_CONFIG}

    next_rows["gemm_gelu"] = time_gemm_gelu(w, D, dev, stream)


    # ---- end to end through the public API, host buffers ------------------
    e2e = run_e2e(args, w, t, stream, api, table if QK_TABLE else None)
    e2e_value, _, _ = dist.job_throughput(w.rows * e2e["steps"], e2e["seconds"])

    bpr = w.bytes_per_row()
    kernels = {}
    for name in KERNELS:
        ms = per_kernel_ms[name]
        gbs = bpr[name] * w.rows / (ms / 1e3) / 1e9
        kernels[name] = {"ms": round(ms, 4), "tokens_per_s": round(w.rows / (ms / 1e3)),
                         "bytes_per_token": bpr[name], "GB_per_s": round(gbs, 1),
                         f"frac_of_{peak_kind}_hbm": round(gbs / peak, 4),
                         "frac_of_8TBs_nominal": round(gbs / NOMINAL_HBM_GBS, 4)}
    dominant = max(KERNELS, key=lambda k: per_kernel_ms[k])
    traffic = traffic_record(dominant, WORKLOAD)
    roofline = {"kernel": dominant, "bound": "hbm",
                "achieved": kernels[dominant]["GB_per_s"], "peak": peak, "unit": "GB/s",
                "frac": round(kernels[dominant]["GB_per_s"] / peak, 4),
                "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6.65 TB/s",
                "traffic": traffic,
                "algorithmic_bytes_per_launch": bpr[dominant] * w.rows}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": round(slowest * 1e3 / K, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; no dataset or weights involved)",
            "config": workload_config(w, world),
            "roofline": roofline, "kernels": kernels, "next_rows": next_rows,
            "configs": configs,
            "rope_table": {"n_pos": table.n_pos, "bytes": table.n_pos * w.head_dim * 4,
                           "build_ms": round(tab_ms, 4),
                           "note": "built once per clip shape before the timed steps (a "
                                   "RoPE cache); the step's QKNorm + RoPE reads it"
                           if QK_TABLE else "not used by the step"},
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s",
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                    "steps": e2e["steps"],
                    "path": "pinned host inputs -> H2D -> api.rms_adaln / api.qknorm_rope3d"
                            + (" (rotary table built once, outside the steps)" if QK_TABLE
                               else "") + " / "
                            "api.gate_residual -> D2H of y, q, k, out; of the merged QKV rows "
                            "only the q and k columns the step reads are copied (one pitched "
                            "copy); copy-in, kernels and copy-out on three streams ordered by "
                            "events; CUDA events"},
            "gpu_launches": len(KERNELS) * K,
            "clocks": clock_info,
        }
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.shutdown()


def time_launches(fn, stream, n, warmup=5):
    """Mean ms of n back-to-back launches of fn on `stream` (CUDA events)."""
    from video_diffusion_transformer_rms_b200 import _abi
    for _ in range(warmup):
        _abi.check(fn())
    ea = torch.cuda.Event(enable_timing=True)
    eb = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ea.record(stream)
    for _ in range(n):
        _abi.check(fn())
    eb.record(stream)
    torch.cuda.synchronize()
    return ea.elapsed_time(eb) / n


def time_config(w, dev, stream, peak, reps=30, warmup=10):
    """The step's three kernels on one config, each timed on its own: CUDA
    events around every launch, median over `reps` after `warmup` launches.  Where an activation is
    under 1 GB (the medium case, whose tensors are L2-sized), the reps are
    separated by an L2 flush: 256 MB written, then another 256 MB read, so the
    timed launch starts with no lines of its inputs and no dirty lines in L2.
    The larger configs stream several GB per launch and need no flush."""
    from video_diffusion_transformer_rms_b200 import _abi, api
    t = make_inputs(w, dev)
    D = w.D
    p = {k: v.data_ptr() for k, v in t.items()}
    y = torch.empty_like(t["x"])
    out = torch.empty_like(t["h"])
    qk = torch.empty((w.rows, 2 * D), dtype=t["qkv"].dtype, device=dev)
    table = api.RopeTable.for_grid(w.T, w.H, w.W, w.n_audio, w.head_dim, sections=w.sections,
                                   theta=w.theta, device=dev)
    dt = _abi.SOL_BF16 if w.dtype == "bf16" else _abi.SOL_F32
    s = stream.cuda_stream
    st, sh, sw = w.sections
    fns = {
        "rms_adaln": lambda: _abi.sol_rms_adaln(p["x"], y.data_ptr(), p["scale"], p["shift"],
                                                None, w.B, w.L, w.n_video, D, w.eps, dt, s),
        "qknorm_rope3d": (lambda: _abi.sol_qknorm_rope3d_tab(
            p["qkv"], 3 * D, qk.data_ptr(), qk.data_ptr() + 2 * D, 2 * D, p["gamma_q"],
            p["gamma_k"], table.desc, w.B, w.T, w.H, w.W, w.n_audio, w.n_heads, w.eps, dt, s))
        if QK_TABLE else (lambda: _abi.sol_qknorm_rope3d(
            p["qkv"], 3 * D, qk.data_ptr(), qk.data_ptr() + 2 * D, 2 * D, p["gamma_q"],
            p["gamma_k"], w.B, w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim, st, sh, sw,
            w.eps, w.theta, dt, s)),
        "gate_residual": lambda: _abi.sol_gate_residual(p["h"], p["branch"], p["gate"],
                                                        out.data_ptr(), w.B, w.L, w.n_video, D,
                                                        dt, s),
    }
    flush = w.rows * D * w.esize < (1 << 30)
    if flush:
        fw = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        fr = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    bpr = w.bytes_per_row()
    res = {"tokens": w.rows, "B": w.B, "D": D, "l2_flush": bool(flush), "reps": reps,
           "kernels": {}}
    for name, fn in fns.items():
        for _ in range(warmup):
            _abi.check(fn())
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        for a, b in evs:
            if flush:
                fw.fill_(1.0)
                fr.sum()
            a.record(stream)
            _abi.check(fn())
            b.record(stream)
        torch.cuda.synchronize()
        ms = float(np.median([a.elapsed_time(b) for a, b in evs]))
        ms = dist.max_over_ranks(ms)
        gbs = bpr[name] * w.rows / (ms / 1e3) / 1e9
        res["kernels"][name] = {"ms": round(ms, 4), "tokens_per_s": round(w.rows / (ms / 1e3)),
                                "GB_per_s": round(gbs, 1), "frac_of_peak": round(gbs / peak, 4),
                                "frac_of_8TBs_nominal": round(gbs / NOMINAL_HBM_GBS, 4)}
    del t, y, out, qk, table
    if flush:
        del fw, fr
    torch.cuda.empty_cache()
    return res


def load_tensor_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


def time_gemm_gelu(w, D, dev, stream):
    """The MLP up-projection of one block, GELU fused in the epilogue: A = the
    step's normalised tokens [rows, D], W1 [4D, D], bias [4D].  Compute bound:
    2*rows*4D*D flops per launch, against the bf16 tensor peak."""
    from video_diffusion_transformer_rms_b200 import _abi
    M, N, K = w.rows, 4 * D, D
    g = torch.Generator(device=dev).manual_seed(77)
    A = torch.randn((M, K), generator=g, device=dev).to(torch.bfloat16)
    Wt = (torch.randn((N, K), generator=g, device=dev) * K ** -0.5).to(torch.bfloat16)
    bias = (0.1 * torch.randn((N,), generator=g, device=dev)).to(torch.bfloat16)
    C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    need = _abi.sol_gemm_gelu_workspace_bytes(M, N, K)
    gws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    s = stream.cuda_stream

    def fn():
        return _abi.sol_gemm_gelu(A.data_ptr(), Wt.data_ptr(), bias.data_ptr(), C.data_ptr(),
                                  M, N, K, gws.data_ptr(), need, s)

    for _ in range(3):
        _abi.check(fn())
    n_it = 10
    ea = torch.cuda.Event(enable_timing=True)
    eb = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ea.record(stream)
    for _ in range(n_it):
        _abi.check(fn())
    eb.record(stream)
    torch.cuda.synchronize()
    ms = dist.max_over_ranks(ea.elapsed_time(eb) / n_it)
    flops = 2.0 * M * N * K
    tflops = flops / (ms / 1e3) / 1e12
    burst, sustained, kind = load_tensor_peaks()
    del A, Wt, bias, C, gws
    return {"ms": round(ms, 3), "M": M, "N": N, "K": K, "flops_per_launch": flops,
            "TFLOP_per_s": round(tflops, 1), "bound": "tensor",
            f"frac_of_{kind}_bf16_burst": round(tflops / burst, 4),
            f"frac_of_{kind}_bf16_sustained": round(tflops / sustained, 4),
            "tokens_per_s": round(M / (ms / 1e3))}


def run_e2e(args, w, t, stream, api, table=None):
    """Same step through the public tensor API, inputs copied every step
    from pinned host memory and every output copied back.

    Three streams: host-to-device copies, the kernels, device-to-host
    copies.  Each kernel waits for its own inputs and each output copy for
    its kernel, so the two PCIe directions and the kernels overlap; the
    next step's copy into a buffer waits for the kernel that read it, and a
    kernel's write waits for the copy-out of its previous result."""
    D = w.D
    groups = {  # inputs of each kernel, in launch order
        "rms_adaln": ("scale", "shift", "x"),
        "qknorm_rope3d": ("gamma_q", "gamma_k", "qkv"),
        "gate_residual": ("gate", "h", "branch"),
    }
    names = [n for g in groups.values() for n in g]
    host = {n: torch.empty(t[n].shape, dtype=t[n].dtype, pin_memory=True) for n in names}
    for n in names:
        host[n].copy_(t[n])
    dev = {n: torch.empty_like(t[n]) for n in names}
    # merged QKV: the step reads only the q and k columns, so one pitched copy
    # brings those (2D of every 3D-wide host row) into a packed [rows, 2D]
    # device buffer, which the API takes as merged rows with ld_qkv = 2D
    from cuda.bindings import runtime as cudart
    rows, esize = w.rows, t["qkv"].element_size()
    dev["qkv"] = torch.empty((rows, 2 * D), dtype=t["qkv"].dtype, device=t["qkv"].device)

    def copy_in(n):
        if n != "qkv":
            dev[n].copy_(host[n], non_blocking=True)
            return
        err, = cudart.cudaMemcpy2DAsync(dev[n].data_ptr(), 2 * D * esize, host[n].data_ptr(),
                                        3 * D * esize, 2 * D * esize, rows,
                                        cudart.cudaMemcpyKind.cudaMemcpyHostToDevice,
                                        s_in.cuda_stream)
        if err != cudart.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaMemcpy2DAsync: {err}")
    y = torch.empty((w.B, w.L, D), dtype=t["x"].dtype, device=t["x"].device)
    qk = torch.empty((w.B, w.L, 2 * D), dtype=t["x"].dtype, device=t["x"].device)
    out = torch.empty_like(y)
    results = {"rms_adaln": y, "qknorm_rope3d": qk, "gate_residual": out}
    host_out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
                for k, v in results.items()}
    h2d = sum(dev[n].numel() * dev[n].element_size() for n in names)  # bytes copied in
    d2h = sum(v.numel() * v.element_size() for v in host_out.values())
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    read_done = {k: None for k in groups}   # kernel k finished reading its inputs
    copied_out = {k: None for k in groups}  # result of kernel k is on the host

    def kernel(k):
        if k == "rms_adaln":
            api.rms_adaln(dev["x"].view(w.B, w.L, D), dev["scale"], dev["shift"], w.n_video,
                          eps=w.eps, out=y, stream=stream)
        elif k == "qknorm_rope3d":
            api.qknorm_rope3d(dev["qkv"].view(w.B, w.L, 2 * D), w.T, w.H, w.W, w.n_audio,
                              w.n_heads, w.head_dim, w.sections, dev["gamma_q"],
                              dev["gamma_k"], w.eps, w.theta, q_out=qk[..., :D],
                              k_out=qk[..., D:], stream=stream, table=table)
        else:
            api.gate_residual(dev["h"].view(w.B, w.L, D), dev["branch"].view(w.B, w.L, D),
                              dev["gate"], w.n_video, out=out, stream=stream)

    def step():
        for k, g in groups.items():
            if read_done[k] is not None:
                s_in.wait_event(read_done[k])
            with torch.cuda.stream(s_in):
                for n in g:
                    copy_in(n)
            arrived = ev()
            arrived.record(s_in)
            stream.wait_event(arrived)
            if copied_out[k] is not None:
                stream.wait_event(copied_out[k])
            kernel(k)
            done = ev()
            done.record(stream)
            read_done[k] = done
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                host_out[k].copy_(results[k], non_blocking=True)
            c = ev()
            c.record(s_out)
            copied_out[k] = c

    step()
    torch.cuda.synchronize()
    n = max(1, args.e2e_steps)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    a.record(s_in)
    for _ in range(n):
        step()
    for c in copied_out.values():
        stream.wait_event(c)
    b.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    secs = a.elapsed_time(b) / 1e3
    del host, host_out, dev
    return {"seconds": secs, "steps": n, "h2d": h2d, "d2h": d2h}


# ----------------------------------------------------------------------------
# reference arm: the oracle on the host cores
# ----------------------------------------------------------------------------

def _oracle_rows(arg):
    """Oracle seconds for one sample of n_rows rows (a spawned worker's task)."""
    name, n_rows, seed = arg
    torch.set_num_threads(1)
    return oracle_sample_run(WORKLOADS[name], n_rows, seed, time.perf_counter)


def run_reference(args):
    """The fp64 oracle as it stands on the host cores: one spawned process per
    core (up to MAX_ORACLE_PROCS), each step one sample of clip rows per
    process, the processes side by side; a step lasts as long as its slowest
    process's oracle time."""
    import multiprocessing
    from concurrent.futures import ProcessPoolExecutor
    rank, _, world = dist.env_world()
    if rank != 0:
        return  # only rank 0 times the CPU reference
    w = WORKLOADS[WORKLOAD]
    n = max(1, min(os.cpu_count() or 1, MAX_ORACLE_PROCS))
    total_steps = args.steps + args.warmup
    per_proc = int(90.0 / max(1, total_steps) / ORACLE_SECONDS_PER_ROW)
    per_proc = max(8, min(2048, per_proc))
    spent, done = 0.0, 0
    with ProcessPoolExecutor(n, mp_context=multiprocessing.get_context("spawn")) as ex:
        # start the workers (imports, oracle load) outside the timed steps
        list(ex.map(_oracle_rows, [(w.name, 8, 1) for _ in range(n)], timeout=600))
        for i in range(total_steps):
            secs = list(ex.map(_oracle_rows,
                               [(w.name, per_proc, 700_000 + 10 * i + 100_000 * j)
                                for j in range(n)], timeout=600))
            if i >= args.warmup:
                spent += max(secs)
                done += per_proc * n
    value = done / spent
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(spent * 1e3 / max(1, args.steps), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, 1),
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": n,
                         "kind": "oracle", "cpu_model": cpu_model(),
                         "sample": f"{per_proc} rows of {w.name} per process per step, {n} "
                                   f"processes side by side, all three ops, fp64 oracle"},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
