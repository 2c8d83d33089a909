"""Build libmoe.so (the layer) and libmoe_synth.so (device input generator) in-tree for sm_100a.

    python -m expert_ffn_token_b200.build [--force]

nvcc cross-compiles without a GPU.  Objects go to expert_ffn_token_b200/_build/ and the shared
libraries next to this file, so that they travel with the source tree.
"""
from __future__ import annotations

import argparse
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
BUILD = PKG / "_build"
INCLUDE = ROOT / "include"
LIB = PKG / "libmoe.so"
SYNTH_LIB = PKG / "libmoe_synth.so"

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", f"-I{INCLUDE}", f"-I{CSRC}"]

LIB_SOURCES = ["k_route.cu", "k_ffn.cu", "k_decode.cu", "k_gateup_tc.cu", "k_gateup_i8.cu",
               "k_down_tc.cu", "k_router.cu", "moe_api.cu", "moe_noalloc.cu"]
OPTIONAL_SOURCES: list[str] = []
SYNTH_SOURCES = ["synth_fill.cu"]


def _sources(names):
    out = [CSRC / n for n in names if (CSRC / n).exists()]
    return out


def _stale(target: Path, deps) -> bool:
    if not target.exists():
        return True
    t = target.stat().st_mtime
    return any(d.stat().st_mtime > t for d in deps)


def _compile(src: Path, verbose: bool) -> Path:
    obj = BUILD / (src.stem + ".o")
    deps = [src, *CSRC.glob("*.cuh"), *INCLUDE.glob("*.h")]
    if _stale(obj, deps):
        cmd = [NVCC, *ARCH, *FLAGS, "-c", str(src), "-o", str(obj)]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
    return obj


def _link(objs, target: Path) -> None:
    if _stale(target, objs):
        tmp = target.with_suffix(f".so.{os.getpid()}")
        subprocess.run([NVCC, *ARCH, "-shared", "-cudart", "static", "-o", str(tmp), *map(str, objs)],
                       check=True)
        os.replace(tmp, target)


def build(force: bool = False, verbose: bool = False) -> Path:
    BUILD.mkdir(exist_ok=True)
    if force:
        for o in BUILD.glob("*.o"):
            o.unlink()
    srcs = _sources(LIB_SOURCES + OPTIONAL_SOURCES)
    ssrcs = _sources(SYNTH_SOURCES)
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose), srcs))
        sobjs = list(ex.map(lambda s: _compile(s, verbose), ssrcs))
    _link(objs, LIB)
    _link(sobjs, SYNTH_LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="ptxas register/spill report")
    a = ap.parse_args()
    print(build(a.force, a.verbose))
