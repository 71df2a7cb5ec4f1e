"""Build libkda.so in-tree with nvcc for sm_100a (B200).

    python -m gated_delta_rule_144_b200.build [--force] [--verbose]

Each csrc/*.cu is compiled separately (in parallel) into _build/, then linked into
gated_delta_rule_144_b200/libkda.so with the static CUDA runtime, so the library only needs the
driver (libcuda) at run time. ptxas register/spill reports go to _build/ptxas.log.
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
BUILD = ROOT / "_build"
LIB = PKG / "libkda.so"

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v",
         "--expt-relaxed-constexpr", "-I", str(INCLUDE), "-I", str(CSRC)]


# Per-file flags. The chunked kernels evaluate one exponential and one reciprocal per operand
# element through the MUFU unit, the prologue two per element (its SiLU); flushing subnormals lets
# those intrinsics compile without their subnormal fix-ups (14 % fewer instructions in the
# intra-chunk kernel). Nothing they compute is meant to be subnormal: chunks whose decay products
# fall below 1e-30 take the direct path, and a prologue output below 1.2e-38 is zero to any
# tolerance the inputs' precision allows.
FILE_FLAGS = {
    "kda_intra.cu": ["-ftz=true"],
    "kda_chunk64.cu": ["-ftz=true"],
    "kda_conv.cu": ["-ftz=true"],
}


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise RuntimeError("nvcc not found: the CUDA 12.9 toolkit is required to build libkda.so")


def _sources():
    return sorted(CSRC.glob("*.cu"))


def _deps():
    return _sources() + sorted(CSRC.glob("*.cuh")) + sorted(INCLUDE.glob("*.h"))


def up_to_date() -> bool:
    if not LIB.exists():
        return False
    t = LIB.stat().st_mtime
    return all(p.stat().st_mtime <= t for p in _deps()) and Path(__file__).stat().st_mtime <= t


def _compile(src: Path, verbose: bool) -> tuple[Path, str]:
    obj = BUILD / (src.stem + ".o")
    cmd = [nvcc(), *ARCH, *FLAGS, *FILE_FLAGS.get(src.name, []), "-c", str(src), "-o", str(obj)]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed on %s:\n%s%s" % (src.name, r.stdout, r.stderr))
    return obj, r.stderr


def build(force: bool = False, verbose: bool = False) -> Path:
    if not force and up_to_date():
        return LIB
    BUILD.mkdir(exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda s: _compile(s, verbose), _sources()))
    (BUILD / "ptxas.log").write_text("".join(log for _, log in results))
    tmp = LIB.with_suffix(".so.tmp%d" % os.getpid())
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", str(tmp),
           *[str(o) for o, _ in results]]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s%s" % (r.stdout, r.stderr))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
    sys.exit(0)
