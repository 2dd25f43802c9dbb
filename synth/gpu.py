"""Device-side synthetic inputs: ctypes wrapper of synth/libfmoe_synth.so.

Draws expert blobs directly in HBM with the same counter-based definition as
``synth.code_words`` / ``synth.sb_words`` (the test suite checks byte
equality), and uploads the host-drawn router, shared-gate and token vectors.
The blob section offsets are passed in by the caller; nothing here knows the
layer's arithmetic.
"""
from __future__ import annotations

import ctypes
import hashlib
import os
import subprocess

import numpy as np
import torch

import synth as S

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "synth.cu")
SO = os.path.join(HERE, "libfmoe_synth.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

_lib = None


def build(force: bool = False) -> str:
    """Compile synth.cu in-tree; rebuilt whenever the hash of its source and
    command differs from the one stored beside the library."""
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-Xcompiler",
           "-fPIC", "-shared", SRC, "-o", SO + ".tmp"]
    h = hashlib.sha256()
    for c in cmd:
        h.update(c.encode() + b"\0")
    with open(SRC, "rb") as f:
        h.update(f.read())
    key = h.hexdigest()
    try:
        with open(SO + ".key") as f:
            stale = f.read().strip() != key or not os.path.exists(SO)
    except OSError:
        stale = True
    if force or stale:
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {SRC}:\n{r.stdout}\n{r.stderr}")
        os.replace(SO + ".tmp", SO)
        with open(SO + ".key.tmp", "w") as f:
            f.write(key + "\n")
        os.replace(SO + ".key.tmp", SO + ".key")
    return SO


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(SO):
            raise RuntimeError(f"{SO} is missing; run synth.gpu.build()")
        L = ctypes.CDLL(SO)
        vp, i, ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
        L.synth_fill_experts.argtypes = [vp, ll, ctypes.POINTER(ll), i, i, i, i, i, ctypes.c_ulonglong, i, i, vp]
        L.synth_fill_experts.restype = i
        _lib = L
    return _lib


def fill_experts(dst: torch.Tensor, stride: int, offsets, first_expert: int, n_experts: int, hidden: int,
                 inter: int, bits: int, seed: int, layer: int, expert_id_override: int = -1):
    """Write n_experts synthetic blobs at dst (uint8, device), blob e at e*stride."""
    assert dst.is_cuda and dst.dtype == torch.uint8
    assert dst.numel() >= (n_experts - 1) * stride + offsets[5] + inter * (hidden // 64) * 4
    off = (ctypes.c_longlong * 6)(*[int(o) for o in offsets])
    rc = lib().synth_fill_experts(dst.data_ptr(), stride, off, first_expert, n_experts, hidden, inter, bits,
                                  seed, layer, expert_id_override, torch.cuda.current_stream().cuda_stream)
    if rc != 0:
        raise RuntimeError(f"synth_fill_experts failed: cudaError {rc}")


def bf16_tensor(bits_u16: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits_u16).view(np.int16)).to(device)


def make_layer(seed: int, layer: int, hidden: int, inter: int, n_experts: int, bits: int, shared_bits: int,
               offsets_fn, expert_bytes_fn, device, with_shared: bool = True, with_sgate: bool = True,
               experts_out: torch.Tensor | None = None):
    """Synthetic weights of one layer on `device`.

    offsets_fn(hidden, inter, bits) -> 6 section offsets and expert_bytes_fn(...)
    -> blob bytes come from the caller (the engine's layout functions).
    Returns dict(experts [E][stride] uint8, shared uint8|None, w_router int16
    [E][H], w_sgate int16 [H] | None, stride).
    """
    eb = expert_bytes_fn(hidden, inter, bits)
    stride = (eb + 255) // 256 * 256
    experts = experts_out if experts_out is not None else torch.empty(
        n_experts, stride, dtype=torch.uint8, device=device)
    fill_experts(experts, stride, offsets_fn(hidden, inter, bits), 0, n_experts, hidden, inter, bits, seed, layer)
    shared = None
    if with_shared:
        sb = expert_bytes_fn(hidden, inter, shared_bits)
        shared = torch.empty((sb + 255) // 256 * 256, dtype=torch.uint8, device=device)
        fill_experts(shared, sb, offsets_fn(hidden, inter, shared_bits), 0, 1, hidden, inter, shared_bits, seed,
                     layer, S.SHARED_EXPERT_ID)
    w_router = bf16_tensor(S.router_bf16(seed, layer, n_experts, hidden), device)
    w_sgate = bf16_tensor(S.sgate_bf16(seed, layer, hidden), device) if with_sgate else None
    return dict(experts=experts, shared=shared, w_router=w_router, w_sgate=w_sgate, stride=stride)
