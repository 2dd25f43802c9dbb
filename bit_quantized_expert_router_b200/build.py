"""Build step: compile the CUDA engine (libfmoe.so) for sm_100a, in-tree.

Run ``python -m bit_quantized_expert_router_b200.build``.  The shared library
is written next to this file so that it travels with the source tree.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared"]

ENGINE_SRC = os.path.join(HERE, "csrc", "fmoe_api.cu")
ENGINE_DEPS = [os.path.join(HERE, "csrc", f) for f in
               ("common.cuh", "dequant.cuh", "layer_kernel.cuh", "route_quant_kernels.cuh", "grouped_kernels.cuh", "tc.cuh", "shared_tc.cuh",
                "deltanet.cuh", "expert_cache.h")] + \
              [os.path.join(ROOT, "include", "fmoe.h")]
ENGINE_SO = os.path.join(HERE, "libfmoe.so")


def _stale(target: str, sources: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def compile_so(src: str, out: str, deps: list[str], extra: list[str] | None = None,
               force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale(out, [src] + deps):
        return out
    cmd = [NVCC, *ARCH, *FLAGS, *(extra or []), src, "-o", out + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(out + ".tmp", out)
    return out


def build_engine(force: bool = False, verbose: bool = False) -> str:
    return compile_so(ENGINE_SRC, ENGINE_SO, ENGINE_DEPS, force=force, verbose=verbose)


if __name__ == "__main__":
    print(build_engine(force="--force" in sys.argv, verbose="-v" in sys.argv))
