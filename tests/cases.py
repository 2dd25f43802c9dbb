"""Seeded layer cases shared by the GPU parity tests, the smoke check and the bench's CPU leg.

The workloads follow the layer shapes of the Flash-MoE pages (512 experts,
K = 4 plus one shared expert, hidden 4096; expert intermediate 1024, the size
that gives the printed 6.75 MB per 4-bit expert) and a tiny variant for fast
checks.  Inputs come from ``synth`` (no layer arithmetic); expected values come
only from ``oracle``.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

import oracle as O
import synth as S

NEAR_TIE = 1e-4  # minimum gap between adjacent top-(K+1) router logits of a parity input


@dataclass(frozen=True)
class Shape:
    name: str
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    bits: int
    shared_bits: int = 4


TINY = Shape("tiny_h512_i128_e16_4bit", 512, 128, 16, 4, 4)
FULL4 = Shape("full_h4096_i1024_e512_4bit", 4096, 1024, 512, 4, 4)
FULL2 = Shape("full_h4096_i1024_e512_2bit_routed", 4096, 1024, 512, 4, 2, 4)


def cpu_blob(seed: int, layer: int, expert: int, hidden: int, inter: int, bits: int) -> np.ndarray:
    """An expert blob assembled on the host from the seeded generator (oracle layout)."""
    return O.assemble_blob(S.expert_parts(seed, layer, expert, hidden, inter, bits), hidden, inter, bits)


def parity_x(seed: int, layer: int, step: int, w_router_bf16: np.ndarray, top_k: int, hidden: int,
             n_tokens: int = 1, norm_w=None, norm_eps: float = 1e-6) -> np.ndarray:
    """Token vectors whose router logits have no near-tie among the top K+1.

    A token is redrawn from an independent substream until the smallest gap
    between adjacent logits among its K+1 largest is at least NEAR_TIE, so that
    the selected experts are the same in any precision.
    """
    out = np.empty((n_tokens, hidden), dtype=np.float32)
    for t in range(n_tokens):
        for redraw in range(1000):
            x = S.token_x(seed, layer, step * 64 + t, 1, hidden, redraw)[0]
            xr = x if norm_w is None else O.rms_norm(x, norm_w, norm_eps)  # what the router sees
            lg = O.router_logits(w_router_bf16, xr)
            if O.top5_min_gap(lg, top_k) >= NEAR_TIE:
                out[t] = x
                break
        else:
            raise RuntimeError("could not draw a token without near-ties")
    return out


def oracle_layer(seed: int, layer: int, shape: Shape, x: np.ndarray, residual: np.ndarray,
                 with_shared: bool = True, with_sgate: bool = True, norm_w=None, norm_eps: float = 1e-6) -> dict:
    """Oracle output of one token through a synthetic layer."""
    H, I = shape.hidden, shape.inter
    w_router = S.router_bf16(seed, layer, shape.n_experts, H)
    w_sg = S.sgate_bf16(seed, layer, H) if with_sgate else None
    shared = cpu_blob(seed, layer, S.SHARED_EXPERT_ID, H, I, shape.shared_bits) if with_shared else None
    cache = {}

    def get(e):
        if e not in cache:
            cache[e] = cpu_blob(seed, layer, e, H, I, shape.bits)
        return cache[e]

    return O.layer_decode(w_router, w_sg, get, shared, x, residual, shape.top_k, H, I, shape.bits,
                          shape.shared_bits, norm_w_bf16=norm_w, norm_eps=norm_eps)


def errors(got: np.ndarray, want: np.ndarray) -> tuple[float, float]:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    d = got - want
    return float(np.max(np.abs(d))), float(np.linalg.norm(d) / max(np.linalg.norm(want), 1e-300))


# Tolerance for fp32 outputs against the fp64 oracle: max-abs <= 2e-3 and
# relative L2 <= 1e-4.
MAX_ABS = 2e-3
REL_L2 = 1e-4


def assert_close(got, want, what: str = "", max_abs: float = MAX_ABS, rel_l2: float = REL_L2):
    ma, rl = errors(got, want)
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max-abs {ma:.3e} (<= {max_abs}), rel-L2 {rl:.3e} (<= {rel_l2})"
