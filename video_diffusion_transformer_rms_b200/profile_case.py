"""Run each hot-path kernel a few times on a seeded slice of a clip workload,
for profilers (ncu) that should capture a small, self-contained case.

    python -m video_diffusion_transformer_rms_b200.profile_case \
        [--workload clip5s] [--frames 4] [--launches 1]
        [--kernel norm|rms|gate|qk|qk_tab|gemm|qk_bhsd|qk_half|qk_int8|qk_all|next] [--table]

The slice keeps the clip's H x W latent grid, D and head layout, takes the
first `--frames` latent frames (T) and scales the audio rows by the same
fraction.  Inputs are larger than L2 at the default 4 frames (16,384 rows:
168 MB per activation, 503 MB of merged QKV), so DRAM counters stay
meaningful while the device footprint stays near 1.5 GB.  `--kernel gemm`
runs the MLP up-projection with fused GELU on the same slice instead
(A [rows, D], W1 [4D, D], C [rows, 4D]: about 1 GB at 4 frames), and
`--kernel qk_*` one QKNorm+RoPE epilogue variant ([B, H, L, hd] output,
half-split pairs, INT8 output; qk_all runs the first two and INT8 with the
quantised v, one launch each), and `--kernel next` the fused residual +
RMS-AdaLN and the change detector (read-only, then with the cache refresh).
`--kernel norm` runs the step's three kernels; `rms`, `gate`, `qk` (per-row
cos/sin) and `qk_tab` (rotary table) one of them alone, for captures that
must hold a single kernel.  `--table` makes the qk_* variants read a rotary
table too.  The slice prints its row count (the scale factor to the full
workload's traffic).
"""
import argparse
import dataclasses

import torch

from . import _abi, api
from .workloads import WORKLOADS, make_inputs


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="clip5s", choices=sorted(WORKLOADS))
    ap.add_argument("--frames", type=int, default=4)
    ap.add_argument("--launches", type=int, default=1)
    ap.add_argument("--kernel", default="norm",
                    choices=["norm", "rms", "gate", "qk", "qk_tab", "gemm", "qk_bhsd", "qk_half",
                             "qk_int8", "qk_all", "next"])
    ap.add_argument("--table", action="store_true",
                    help="QKNorm+RoPE variants read a precomputed rotary table")
    args = ap.parse_args()
    full = WORKLOADS[args.workload]
    T = max(1, min(full.T, args.frames))
    n_audio = full.n_audio * T // full.T
    w = dataclasses.replace(full, name=f"{full.name}_slice{T}", T=T, n_audio=n_audio)
    if args.kernel == "gemm":
        return gemm_case(w, args.launches)
    t = make_inputs(w, "cuda")
    D = w.D
    x = t["x"].view(w.B, w.L, D)
    h = t["h"].view(w.B, w.L, D)
    br = t["branch"].view(w.B, w.L, D)
    qkv = t["qkv"].view(w.B, w.L, 3 * D)
    y = torch.empty_like(x)
    out = torch.empty_like(h)
    qk = torch.empty((w.B, w.L, 2 * D), dtype=qkv.dtype, device=qkv.device)
    table = None
    if args.table or args.kernel == "qk_tab":
        table = api.RopeTable.for_grid(w.T, w.H, w.W, w.n_audio, w.head_dim, sections=w.sections,
                                       theta=w.theta, device=qkv.device)
    if args.kernel in ("rms", "gate", "qk", "qk_tab"):
        for _ in range(args.launches):
            if args.kernel == "rms":
                api.rms_adaln(x, t["scale"], t["shift"], w.n_video, eps=w.eps, out=y)
            elif args.kernel == "gate":
                api.gate_residual(h, br, t["gate"], w.n_video, out=out)
            else:
                api.qknorm_rope3d(qkv, w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim,
                                  w.sections, t["gamma_q"], t["gamma_k"], w.eps, w.theta,
                                  q_out=qk[..., :D], k_out=qk[..., D:],
                                  table=table if args.kernel == "qk_tab" else None)
        torch.cuda.synchronize()
        print(f"{w.name}: {w.rows} rows, D={D}, {args.launches} launch(es) of {args.kernel}")
        return
    if args.kernel == "next":
        ws = torch.empty(_abi.sol_residual_change_workspace_bytes(w.B), dtype=torch.uint8,
                         device=x.device)
        for _ in range(args.launches):
            api.gate_residual_rms_adaln(h, br, t["gate"], t["scale"], t["shift"], w.n_video,
                                        h_out=out, y=y, eps=w.eps)
            api.residual_change(h, br, workspace=ws)
            api.residual_change(h, br, prev_out=out, workspace=ws)
        torch.cuda.synchronize()
        print(f"{w.name}: {w.rows} rows, D={D}, {args.launches} launch(es) of the next rows")
        return
    if args.kernel.startswith("qk_"):
        variants = {"qk_bhsd": [{"layout": "bhsd"}], "qk_half": [{"half_split": True}],
                    "qk_int8": [{"int8": True}],
                    "qk_all": [{"layout": "bhsd"}, {"half_split": True},
                               {"int8": True, "quantize_v": True}]}[args.kernel]
        for _ in range(args.launches):
            for opts in variants:
                if table is not None and opts.get("per_axis_freq"):
                    raise SystemExit("per-axis variants need a per-axis table")
                api.qknorm_rope3d_ex(qkv, w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim,
                                     w.sections, t["gamma_q"], t["gamma_k"], w.eps, w.theta,
                                     table=table, **opts)
        torch.cuda.synchronize()
        print(f"{w.name}: {w.rows} rows, D={D}, {args.launches} launch(es) of {args.kernel}")
        return
    for _ in range(args.launches):
        api.rms_adaln(x, t["scale"], t["shift"], w.n_video, eps=w.eps, out=y)
        api.qknorm_rope3d(qkv, w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim, w.sections,
                          t["gamma_q"], t["gamma_k"], w.eps, w.theta, q_out=qk[..., :D],
                          k_out=qk[..., D:], table=table)
        api.gate_residual(h, br, t["gate"], w.n_video, out=out)
    torch.cuda.synchronize()
    print(f"{w.name}: {w.rows} rows, D={D}, {args.launches} launch(es) of each kernel")


def gemm_case(w, launches):
    M, N, K = w.rows, 4 * w.D, w.D
    g = torch.Generator(device="cuda").manual_seed(77)
    A = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    W1 = (torch.randn((N, K), generator=g, device="cuda") * K ** -0.5).to(torch.bfloat16)
    bias = (0.1 * torch.randn((N,), generator=g, device="cuda")).to(torch.bfloat16)
    C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for _ in range(launches):
        api.gemm_gelu(A, W1, bias, out=C)
    torch.cuda.synchronize()
    print(f"{w.name}: gemm_gelu M={M} N={N} K={K}, {launches} launch(es)")


if __name__ == "__main__":
    main()
