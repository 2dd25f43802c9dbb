"""Seeded synthetic inputs for the quantised MoE layer (host side).

This module draws the inputs that both the CPU oracle and the CUDA engine
consume.  It holds none of the layer's arithmetic: no dequantisation, no
GEMV, no routing, no activation.  It only produces

* packed 4-bit / 2-bit code words (uniform codes, so every code word is a
  uniform 32-bit integer),
* per-group bf16 (scale, bias) pairs drawn from the workload's value
  distributions (scale ~ U(1e-3, 4e-3), bias = -m * scale * (1 + U(-0.1, 0.1))
  with m = 8 at 4 bits and m = 1.5 at 2 bits),
* bf16 router rows and the bf16 shared-gate vector ~ N(0, 0.02),
* fp32 token vectors x and residual ~ N(0, 1);
* for the linear-attention state update: an fp32 state ~ N(0, 0.1^2) per
  element, and per token and head a key of unit length (a standard normal
  vector divided by its length), a query ~ N(0, 1/dk) per element, a value
  ~ N(0, 1), a decay gate alpha ~ U(0.9, 1) and a write gate beta ~ U(0, 1).

Code words and (scale, bias) pairs come from a counter-based generator: the
i-th output of SplitMix64 (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014; output mix with the constants of
Vigna's public-domain ``splitmix64.c``) seeded with a key that chains the tuple
(tag, seed, layer, expert, matrix).  ``synth/synth.cu`` implements the same
definition on the GPU so that multi-GB layers can be drawn in HBM; the test
suite checks that both produce identical bytes.

Router weights and token vectors are drawn on the host with NumPy's PCG64 and
uploaded.  A ``redraw`` counter selects an independent substream, used by the
tests to redraw a token whose router logits have a near-tie.
"""
from __future__ import annotations

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB

# Stream tags (arbitrary distinct constants).
TAG_CODES = 0xC0DE5
TAG_SB = 0x5CA1E
TAG_ROUTER = 0x20073
TAG_X = 0x7E5
TAG_RES = 0x2E5
TAG_SGATE = 0x5647E
TAG_DENSE = 0xDE45E
TAG_NORM = 0x40235
TAG_DSTATE = 0xD57A7
TAG_DTOK = 0xD70C5

GROUP = 64  # quantisation group length along the input dimension

# Matrix ids inside one expert.
MAT_GATE, MAT_UP, MAT_DOWN = 0, 1, 2


def _mix_scalar(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX1) & MASK64
    z = ((z ^ (z >> 27)) * MIX2) & MASK64
    return z ^ (z >> 31)


def _mix_array(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= np.uint64(MIX1)
        z ^= z >> np.uint64(27)
        z *= np.uint64(MIX2)
        z ^= z >> np.uint64(31)
    return z


def stream_key(tag: int, seed: int, layer: int, expert: int, matrix: int) -> int:
    """64-bit key for one (tag, seed, layer, expert, matrix) stream."""
    k = 0
    for part in (tag, seed, layer, expert, matrix):
        k = _mix_scalar((k ^ (part & MASK64)) + GAMMA)
    return k


def splitmix64_outputs(key: int, start: int, count: int) -> np.ndarray:
    """Outputs start..start+count-1 of SplitMix64 seeded with ``key``.

    Output i is mix(key + (i + 1) * GAMMA) (mod 2^64).
    """
    i = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        state = np.uint64(key) + (i + np.uint64(1)) * np.uint64(GAMMA)
    return _mix_array(state)


def bf16_bits_rne(f32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(f32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint32) << np.uint32(16)).view(np.float32)


def code_words(seed: int, layer: int, expert: int, matrix: int, n_rows: int,
               n_in: int, bits: int) -> np.ndarray:
    """uint32 [n_rows][n_in*bits/32]: uniform packed codes of one matrix."""
    wpr = n_in * bits // 32
    key = stream_key(TAG_CODES, seed, layer, expert, matrix)
    h = splitmix64_outputs(key, 0, n_rows * wpr)
    return (h >> np.uint64(32)).astype(np.uint32).reshape(n_rows, wpr)


def bias_multiplier(bits: int) -> float:
    return {4: 8.0, 2: 1.5}[bits]


def sb_words(seed: int, layer: int, expert: int, matrix: int, n_rows: int,
             n_in: int, bits: int) -> np.ndarray:
    """uint32 [n_rows][n_in/64]: bf16 scale in bits 0..15, bf16 bias in 16..31."""
    ng = n_in // GROUP
    key = stream_key(TAG_SB, seed, layer, expert, matrix)
    h = splitmix64_outputs(key, 0, n_rows * ng)
    two24 = np.float32(1.0 / 16777216.0)
    u = (h >> np.uint64(40)).astype(np.float32) * two24
    u2 = ((h >> np.uint64(16)) & np.uint64(0xFFFFFF)).astype(np.float32) * two24
    s32 = (np.float32(3e-3) * u).astype(np.float32) + np.float32(1e-3)
    s_bits = bf16_bits_rne(s32)
    s_f = bf16_bits_to_f32(s_bits)
    fac = (np.float32(0.2) * u2).astype(np.float32) + np.float32(0.9)
    neg_ms = (np.float32(-bias_multiplier(bits)) * s_f).astype(np.float32)
    b32 = (neg_ms * fac).astype(np.float32)
    b_bits = bf16_bits_rne(b32)
    w = s_bits.astype(np.uint32) | (b_bits.astype(np.uint32) << np.uint32(16))
    return w.reshape(n_rows, ng)


def matrix_shape(matrix: int, hidden: int, inter: int) -> tuple[int, int]:
    """(rows, inputs) of gate / up ([I][H]) and down ([H][I])."""
    return (inter, hidden) if matrix in (MAT_GATE, MAT_UP) else (hidden, inter)


def expert_parts(seed: int, layer: int, expert: int, hidden: int, inter: int,
                 bits: int) -> dict:
    """Code words and (scale, bias) words of the three matrices of one expert."""
    out = {}
    for m, name in ((MAT_GATE, "gate"), (MAT_UP, "up"), (MAT_DOWN, "down")):
        n, k = matrix_shape(m, hidden, inter)
        out[name] = (code_words(seed, layer, expert, m, n, k, bits),
                     sb_words(seed, layer, expert, m, n, k, bits))
    return out


# Expert id used for the shared expert's streams (distinct from routed ids).
SHARED_EXPERT_ID = 0xFFFFF


def _rng(*parts: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([p & 0xFFFFFFFF for p in parts])))


def router_bf16(seed: int, layer: int, n_experts: int, hidden: int) -> np.ndarray:
    """uint16 [E][H] bf16 bit patterns, ~N(0, 0.02)."""
    g = _rng(seed, TAG_ROUTER, layer)
    w = g.normal(0.0, 0.02, size=(n_experts, hidden)).astype(np.float32)
    return bf16_bits_rne(w).reshape(n_experts, hidden)


def sgate_bf16(seed: int, layer: int, hidden: int) -> np.ndarray:
    """uint16 [H] bf16 bit patterns of the shared-expert gate vector, ~N(0, 0.02)."""
    g = _rng(seed, TAG_SGATE, layer)
    w = g.normal(0.0, 0.02, size=hidden).astype(np.float32)
    return bf16_bits_rne(w)


def norm_bf16(seed: int, layer: int, hidden: int) -> np.ndarray:
    """uint16 [H] bf16 bit patterns of an RMS-norm weight, ~N(1, 0.1)."""
    g = _rng(seed, TAG_NORM, layer)
    w = g.normal(1.0, 0.1, size=hidden).astype(np.float32)
    return bf16_bits_rne(w)


def token_x(seed: int, layer: int, step: int, n_tokens: int, hidden: int,
            redraw: int = 0) -> np.ndarray:
    """fp32 [T][H] ~ N(0, 1)."""
    g = _rng(seed, TAG_X, layer, step, redraw)
    return g.standard_normal((n_tokens, hidden), dtype=np.float32)


TAG_STREAM = 0x57E4


def token_stream(seed: int, n_tokens: int, hidden: int, rho: float) -> np.ndarray:
    """fp32 [T][H]: a first-order autoregressive token sequence, each row
    N(0, 1) per element, consecutive rows correlated by rho
    (x_t = rho x_{t-1} + sqrt(1 - rho^2) z_t), a stand-in for the temporal
    locality of a decoded text (consecutive tokens tend to pick the same
    experts)."""
    g = _rng(seed, TAG_STREAM, n_tokens, hidden)
    z = g.standard_normal((n_tokens, hidden), dtype=np.float32)
    out = np.empty_like(z)
    out[0] = z[0]
    c = np.float32(np.sqrt(1.0 - rho * rho))
    for t in range(1, n_tokens):
        out[t] = np.float32(rho) * out[t - 1] + c * z[t]
    return out


def token_residual(seed: int, layer: int, step: int, n_tokens: int,
                   hidden: int) -> np.ndarray:
    g = _rng(seed, TAG_RES, layer, step)
    return g.standard_normal((n_tokens, hidden), dtype=np.float32)


def dense_matrix(seed: int, tag: int, n_rows: int, n_in: int, std: float = 0.02) -> np.ndarray:
    """fp32 dense matrix ~ N(0, std) (input for the quantiser)."""
    g = _rng(seed, TAG_DENSE, tag)
    return (g.standard_normal((n_rows, n_in), dtype=np.float32) * np.float32(std)).astype(np.float32)


def delta_state(seed: int, layer: int, heads: int, dv: int, dk: int) -> np.ndarray:
    """fp32 [heads][dv][dk] ~ N(0, 0.1^2)."""
    g = _rng(seed, TAG_DSTATE, layer)
    return (g.standard_normal((heads, dv, dk), dtype=np.float32) * np.float32(0.1)).astype(np.float32)


def delta_tokens(seed: int, layer: int, step: int, n_tokens: int, heads: int, dk: int, dv: int) -> dict:
    """fp32 inputs of n_tokens state updates: q, k [T][heads][dk], v [T][heads][dv],
    alpha, beta [T][heads] (distributions in the module docstring)."""
    g = _rng(seed, TAG_DTOK, layer, step)
    k = g.standard_normal((n_tokens, heads, dk))
    k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
    q = (g.standard_normal((n_tokens, heads, dk)) / np.sqrt(dk)).astype(np.float32)
    v = g.standard_normal((n_tokens, heads, dv), dtype=np.float32)
    alpha = g.uniform(0.9, 1.0, (n_tokens, heads)).astype(np.float32)
    beta = g.uniform(0.0, 1.0, (n_tokens, heads)).astype(np.float32)
    return {"q": q, "k": k, "v": v, "alpha": alpha, "beta": beta}
