"""Build libsol.so (the CUDA kernels + C ABI) in-tree for sm_100a.

    python -m video_diffusion_transformer_rms_b200.build [--force] [-v]

nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically, so it only needs the driver at run time.  Objects go to
_build/ next to the repository root; the .so lands inside the package.
"""
import argparse
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsol.so")

SOURCES = ["sol_abi.cu", "rms_adaln.cu", "gate_residual.cu", "qknorm_rope3d_bf16.cu",
           "qknorm_rope3d_f32.cu", "qknorm_rope3d_tab_bf16.cu", "qknorm_rope3d_tab_f32.cu",
           "qknorm_rope3d_ex_bf16.cu", "qknorm_rope3d_ex_int8.cu", "qknorm_rope3d_ex_tab_bf16.cu",
           "qknorm_rope3d_ex_tab_int8.cu", "residual_change.cu", "quantize_heads.cu",
           "rope_table.cu", "gemm_gelu.cu"]
# sources built against the CUTLASS / CuTe headers (the sm100 GEMM templates)
CUTLASS_SOURCES = {"gemm_gelu.cu"}
HEADERS = ["sol_device.cuh", "sol_launch.h", "qknorm_rope3d.cuh", "qknorm_rope3d_ex.cuh"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr"]


def _nvcc():
    for c in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libsol")


# The GEMM + GELU kernel is assembled from CUTLASS's sm100 collective
# templates (CTA-pair tcgen05 MMA, TMA, TMEM); it was built and measured with
# CUTLASS 4.5.0.  Older trees lack parts of the sm100 builders it uses.
CUTLASS_MIN = (4, 0)


def _cutlass_version(root):
    """(major, minor, patch) from include/cutlass/version.h, or None."""
    import re
    try:
        with open(os.path.join(root, "include", "cutlass", "version.h")) as fh:
            text = fh.read()
    except OSError:
        return None
    v = [re.search(rf"#define CUTLASS_{k}\s+(\d+)", text) for k in ("MAJOR", "MINOR", "PATCH")]
    return tuple(int(m.group(1)) for m in v) if all(v) else None


def _cutlass_root():
    """The CUTLASS / CuTe header tree the GEMM + GELU kernel is built against:
    $SOL_CUTLASS_DIR if set (a CUTLASS checkout: include/cute and
    include/cutlass), else the tree vendored inside the installed flashinfer
    package (flashinfer/data/cutlass; headers only, flashinfer is not
    imported).  Fails with the path it looked at."""
    env = os.environ.get("SOL_CUTLASS_DIR")
    if env:
        candidates, where = [env], f"SOL_CUTLASS_DIR={env}"
    else:
        import importlib.util
        spec = importlib.util.find_spec("flashinfer")
        bases = (spec.submodule_search_locations if spec else None) or []
        candidates = [os.path.join(b, "data", "cutlass") for b in bases]
        where = ("flashinfer/data/cutlass (" + ", ".join(candidates) + ")" if candidates
                 else "flashinfer/data/cutlass (flashinfer is not installed)")
    for root in candidates:
        if os.path.isdir(os.path.join(root, "include", "cute")):
            ver = _cutlass_version(root)
            if ver is None or ver[:2] < CUTLASS_MIN:
                raise RuntimeError(f"CUTLASS at {root} is version {ver}; gemm_gelu.cu needs "
                                   f">= {CUTLASS_MIN[0]}.{CUTLASS_MIN[1]} (set SOL_CUTLASS_DIR)")
            return root
    raise RuntimeError(f"CUTLASS headers not found at {where}: gemm_gelu.cu needs a CUTLASS "
                       f">= {CUTLASS_MIN[0]}.{CUTLASS_MIN[1]} tree; set SOL_CUTLASS_DIR to one")


def cutlass_info():
    """(root, 'major.minor.patch') of the CUTLASS tree the build uses."""
    root = _cutlass_root()
    return root, ".".join(map(str, _cutlass_version(root)))


def _digest():
    h = hashlib.sha256()
    for f in SOURCES + HEADERS:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    with open(os.path.join(INCLUDE, "sol.h"), "rb") as fh:
        h.update(fh.read())
    h.update(" ".join(ARCH + FLAGS).encode())
    root, ver = cutlass_info()
    h.update(f"cutlass {ver} {root}".encode())
    return h.hexdigest()


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu for sm_100a and link libsol.so; skip if up to date."""
    stamp = LIB + ".sha256"
    digest = _digest()
    if not force and os.path.exists(LIB) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == digest:
                return LIB
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    objs = []
    procs = []
    for src in SOURCES:
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        cmd = [nvcc, *ARCH, *FLAGS, "-I", INCLUDE, "-I", CSRC, "-c",
               os.path.join(CSRC, src), "-o", obj]
        if src in CUTLASS_SOURCES:
            cut = _cutlass_root()
            cmd[1:1] = ["-I", os.path.join(cut, "include"), "-I",
                        os.path.join(cut, "tools", "util", "include"),
                        "-diag-suppress", "20012"]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                            stderr=subprocess.STDOUT, text=True)))
        objs.append(obj)
    failed = False
    for src, p in procs:
        out, _ = p.communicate()
        if verbose or p.returncode != 0:
            sys.stderr.write(f"--- {src}\n{out}")
        failed |= p.returncode != 0
    if failed:
        raise RuntimeError("nvcc failed while building libsol")
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs],
                   check=True)
    os.replace(tmp, LIB)
    with open(stamp, "w") as f:
        f.write(digest + "\n")
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true", help="print ptxas resource usage")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose))
