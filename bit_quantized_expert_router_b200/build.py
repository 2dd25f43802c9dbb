"""Build step: compile the CUDA engine (libfmoe.so) for sm_100a, in-tree.

Run ``python -m bit_quantized_expert_router_b200.build``.  The shared library
is written next to this file so that it travels with the source tree.
"""
from __future__ import annotations

import hashlib
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
                "deltanet.cuh", "expert_cache.h", "streamer.cuh")] + \
              [os.path.join(ROOT, "include", "fmoe.h")]
ENGINE_SO = os.path.join(HERE, "libfmoe.so")


def build_key(sources: list[str], cmd: list[str]) -> str:
    """Hash of the sources' bytes and the compiler command: a library is rebuilt
    whenever this differs from the key stored beside it (file times are not
    trusted: a copied tree can carry a stale library with a fresh time)."""
    h = hashlib.sha256()
    for c in cmd:
        h.update(c.encode() + b"\0")
    for s in sources:
        h.update(os.path.basename(s).encode() + b"\0")
        with open(s, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _stale(target: str, key: str) -> bool:
    try:
        with open(target + ".key") as f:
            return not os.path.exists(target) or f.read().strip() != key
    except OSError:
        return True


def compile_so(src: str, out: str, deps: list[str], extra: list[str] | None = None,
               force: bool = False, verbose: bool = False) -> str:
    cmd = [NVCC, *ARCH, *FLAGS, *(extra or []), src, "-o", out + ".tmp"]
    key = build_key([src] + deps, cmd)
    if not force and not _stale(out, key):
        return out
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(out + ".tmp", out)
    with open(out + ".key.tmp", "w") as f:
        f.write(key + "\n")
    os.replace(out + ".key.tmp", out + ".key")
    return out


def build_engine(force: bool = False, verbose: bool = False) -> str:
    return compile_so(ENGINE_SRC, ENGINE_SO, ENGINE_DEPS, force=force, verbose=verbose)


if __name__ == "__main__":
    print(build_engine(force="--force" in sys.argv, verbose="-v" in sys.argv))
