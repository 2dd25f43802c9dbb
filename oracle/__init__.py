"""CPU oracle for the single-token quantised MoE layer (test infrastructure).

THIS IS TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import it.  The CUDA engine never calls it and
shares no code with it: no kernels, headers, helpers, tables or constants.

It is plain and slow on purpose: every weight is dequantised to fp64 and every
product is an ordinary matrix-vector product (numpy), with no blocking, fusion
or reordering beyond what the definitions below state.

Sources (the web pages about Flash-MoE), cited as [Pn "section"]:

* [P1] "397B MoE en MacBook: Motor Flash-MoE a 4,4 t/s" (aibit.im)
* [P2] "Flash-MoE: Ausführen eines 397B-Parameter-Qwen-Modells auf dem MacBook
  Pro mit reinem C/Metal" (openclawradar.com)
* [P3] "Flash-MoE - Executando um modelo de 397 bilhões de parâmetros em um
  notebook" (news.hada.io)
* [P4] "Flash-MoE: modello AI da 397 miliardi di parametri funziona localmente
  su MacBook a 4,4 token/sec" (aipulse.it)
* [P5] "Flash-MoE : un modèle de 397 milliards de paramètres qui tourne sur un
  MacBook" (mondary.design)

What the layer computes, per token (definitions restated, not copied):

1. Router: one logit per expert, the dot product of the expert's router row
   with the MoE input ([P2 "Pipeline-Leistung"]: routing runs inside the
   second command buffer; [P2 "Technische Implementierung"]: 512 experts,
   K = 4 active per token plus one shared expert, hidden size 4096).
2. Softmax over the logits, the K largest, and their weights renormalised to
   sum to one ([P2 "Pipeline-Leistung"]: "Softmax + TopK-Routing").
3. Every selected expert and the shared expert runs gate and up projections,
   SwiGLU, then the down projection ([P2 "Metal-Compute-Shader"]: fused SwiGLU,
   4-bit and 2-bit dequantised matrix-vector products).
4. Weights are affine group-quantised: a weight equals nibble * scale + bias
   ([P1 "Técnicas innovadoras" §2], [P2 "FMA-optimierter Dequant-Kernel"],
   [P3 "Kernel de dequantização otimizado com FMA"]).  The engine evaluates
   fma(nibble, scale*x, bias*x); that rearrangement is exact algebra, so the
   oracle evaluates the plain form (nibble*scale + bias) * x.
5. The layer ends with one fused step: the weighted sum of the expert outputs,
   the residual add and the sigmoid-gated shared expert
   ([P2 "Metal-Compute-Shader"]: "MoE-Kombination + Rest + Sigmoid-Gate").

Readings where the pages are silent (each one is listed in the design notes):

* group length 64 along the input dimension; bf16 scale and bias per group;
* codes packed LSB-first: element k of a row sits in 32-bit word k // (32/b)
  at bit b * (k mod 32/b);
* a blob per expert = [gate codes | gate (s,b) | up codes | up (s,b) |
  down codes | down (s,b)], gate/up stored [I][H], down stored [H][I];
* K = 4 routed experts *plus* one shared expert;
* the shared gate is a scalar sigmoid(w_sg . x) multiplying the shared
  expert's output; with no gate vector the shared expert is ungated (factor 1);
* top-K order: descending logit, lower expert index first on exact ties;
* the quantiser (not described by the pages) is affine min/max per group in
  IEEE fp32: s = bf16(fl(fl(max - min) / (2^b - 1))), bias = bf16(min),
  q = clamp(rint(fl(fl(w - bias) / s)), 0, 2^b - 1), q = 0 when s == 0.

A second, independent step: the gated delta-rule update of the linear-
attention state (delta_update, at the end of this file).

Parity status: every function here is pinned by the CPU tests against closed
forms, exact rational arithmetic, brute force and the expert size the pages
print (6.75 MB per 4-bit expert).  Agreement with the pages' own engine
outputs is unpinned: those need the trained model, which is out of scope.
"""
from __future__ import annotations

import numpy as np

GROUP = 64


# ---------------------------------------------------------------------------
# bf16 helpers (the oracle's own; round to nearest even)
# ---------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp64 exactly."""
    u32 = np.asarray(bits, dtype=np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16, nearest even, returning the bit patterns."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    return ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# Packed expert format
# ---------------------------------------------------------------------------

def section_bytes(rows: int, n_in: int, bits: int) -> tuple[int, int]:
    """(code bytes, scale/bias bytes) of one quantised matrix."""
    return rows * n_in * bits // 8, rows * (n_in // GROUP) * 4


def blob_layout(hidden: int, inter: int, bits: int) -> dict:
    """Byte offsets of the six sections of an expert blob.

    Gate and up are [inter][hidden] (rows = intermediate units); down is
    [hidden][inter].  Each matrix stores its codes, then its (scale, bias)
    words.
    """
    off = 0
    lay = {}
    for name, rows, n_in in (("gate", inter, hidden), ("up", inter, hidden),
                             ("down", hidden, inter)):
        cb, sb = section_bytes(rows, n_in, bits)
        lay[name] = (off, off + cb, rows, n_in)
        off += cb + sb
    lay["total"] = off
    return lay


def expert_bytes(hidden: int, inter: int, bits: int, group: int = GROUP) -> int:
    """Bytes of one expert: 3*H*I weights at b/8 bytes plus 4 bytes per group.

    [P1 "Técnicas innovadoras" §1], [P2 "SSD-Experten-Streaming"]: about
    6.75 MB per 4-bit expert, which this formula gives exactly (in MiB) for
    H = 4096, I = 1024, g = 64.
    """
    assert group == GROUP
    return 3 * hidden * inter * bits // 8 + 3 * hidden * inter // group * 4


def unpack_codes(words: np.ndarray, bits: int) -> np.ndarray:
    """uint32 [N][W] -> uint8 [N][W*32/b]; element k at bits b*(k mod 32/b)."""
    words = np.asarray(words, dtype=np.uint32)
    per = 32 // bits
    mask = np.uint32((1 << bits) - 1)
    shifts = (np.arange(per, dtype=np.uint32) * np.uint32(bits))
    codes = (words[..., :, None] >> shifts) & mask
    return codes.reshape(*words.shape[:-1], words.shape[-1] * per).astype(np.uint8)


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of unpack_codes."""
    codes = np.asarray(codes, dtype=np.uint32)
    per = 32 // bits
    n_in = codes.shape[-1]
    assert n_in % per == 0
    c = codes.reshape(*codes.shape[:-1], n_in // per, per)
    shifts = (np.arange(per, dtype=np.uint32) * np.uint32(bits))
    return np.bitwise_or.reduce(c << shifts, axis=-1).astype(np.uint32)


def unpack_scale_bias(sb: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """uint32 (scale | bias << 16) words -> (scale, bias) as exact fp64."""
    sb = np.asarray(sb, dtype=np.uint32)
    return bf16_to_f64(sb & np.uint32(0xFFFF)), bf16_to_f64(sb >> np.uint32(16))


def dequantize(words: np.ndarray, sb: np.ndarray, bits: int) -> np.ndarray:
    """Dense fp64 weights: W[r, k] = q[r, k] * s[r, k // 64] + b[r, k // 64].

    [P1 "Técnicas innovadoras" §2], [P2 "FMA-optimierter Dequant-Kernel"]:
    a weight is nibble * scale + bias.
    """
    q = unpack_codes(words, bits).astype(np.float64)
    s, b = unpack_scale_bias(sb)
    s_full = np.repeat(s, GROUP, axis=-1)
    b_full = np.repeat(b, GROUP, axis=-1)
    return q * s_full + b_full


def split_blob(blob: np.ndarray, hidden: int, inter: int, bits: int) -> dict:
    """Views of the (codes, sb) word arrays of the three matrices of a blob."""
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    lay = blob_layout(hidden, inter, bits)
    assert blob.size >= lay["total"], "blob too small"
    out = {}
    for name in ("gate", "up", "down"):
        c_off, s_off, rows, n_in = lay[name]
        cb, sbb = section_bytes(rows, n_in, bits)
        codes = blob[c_off:c_off + cb].view(np.uint32).reshape(rows, n_in * bits // 32)
        sb = blob[s_off:s_off + sbb].view(np.uint32).reshape(rows, n_in // GROUP)
        out[name] = (codes, sb)
    return out


def assemble_blob(parts: dict, hidden: int, inter: int, bits: int) -> np.ndarray:
    """Build a blob (uint8) from {'gate'|'up'|'down': (codes, sb)} word arrays."""
    lay = blob_layout(hidden, inter, bits)
    blob = np.zeros(lay["total"], dtype=np.uint8)
    for name in ("gate", "up", "down"):
        c_off, s_off, rows, n_in = lay[name]
        codes, sb = parts[name]
        codes = np.ascontiguousarray(codes, dtype=np.uint32)
        sb = np.ascontiguousarray(sb, dtype=np.uint32)
        assert codes.shape == (rows, n_in * bits // 32) and sb.shape == (rows, n_in // GROUP)
        blob[c_off:c_off + codes.nbytes] = codes.view(np.uint8).ravel()
        blob[s_off:s_off + sb.nbytes] = sb.view(np.uint8).ravel()
    return blob


def expert_matrices(blob: np.ndarray, hidden: int, inter: int, bits: int):
    """(Wg [I][H], Wu [I][H], Wd [H][I]) dequantised to fp64."""
    p = split_blob(blob, hidden, inter, bits)
    return tuple(dequantize(*p[n], bits) for n in ("gate", "up", "down"))


# ---------------------------------------------------------------------------
# Activations
# ---------------------------------------------------------------------------

def sigmoid(z):
    """1 / (1 + exp(-z)) in fp64 (evaluated without overflow)."""
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def silu(z):
    """z * sigmoid(z): the gate activation of SwiGLU ([P2 "Metal-Compute-Shader"])."""
    z = np.asarray(z, dtype=np.float64)
    return z * sigmoid(z)


# ---------------------------------------------------------------------------
# Expert forward
# ---------------------------------------------------------------------------

def expert_forward(blob: np.ndarray, hidden: int, inter: int, bits: int,
                   x: np.ndarray) -> np.ndarray:
    """y = Wd (silu(Wg x) * (Wu x)), all in fp64.

    [P2 "Metal-Compute-Shader"]: dequantised matrix-vector products and a fused
    SwiGLU; [P2 "Pipeline-Leistung"]: the expert forward pass of the third
    command buffer.
    """
    wg, wu, wd = expert_matrices(blob, hidden, inter, bits)
    x = np.asarray(x, dtype=np.float64)
    g = wg @ x
    u = wu @ x
    a = silu(g) * u
    return wd @ a


# ---------------------------------------------------------------------------
# Routing
# ---------------------------------------------------------------------------

def router_logits(w_router_bf16: np.ndarray, x: np.ndarray) -> np.ndarray:
    """logits[e] = sum_h W_r[e, h] * x[h] with bf16 weights widened exactly."""
    return bf16_to_f64(w_router_bf16) @ np.asarray(x, dtype=np.float64)


def softmax(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(z - z.max())
    return e / e.sum()


def top_k_order(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits, descending; lower index first on ties."""
    order = np.argsort(-np.asarray(logits, dtype=np.float64), kind="stable")
    return order[:k].astype(np.int32)


def route(w_router_bf16: np.ndarray, w_sgate_bf16, x: np.ndarray, top_k: int) -> dict:
    """Router logits -> softmax -> top-K -> renormalised weights, plus the shared gate.

    [P2 "Pipeline-Leistung"]: router projection then "Softmax + TopK-Routing";
    [P2 "Technische Implementierung"]: K = 4 per token plus one shared expert;
    [P2 "Metal-Compute-Shader"]: the shared expert enters through a sigmoid gate.
    """
    logits = router_logits(w_router_bf16, x)
    p = softmax(logits)
    idx = top_k_order(logits, top_k)
    w = p[idx] / p[idx].sum()
    if w_sgate_bf16 is None:
        sg = 1.0
    else:
        sg = float(sigmoid(bf16_to_f64(w_sgate_bf16) @ np.asarray(x, dtype=np.float64)))
    return {"logits": logits, "p": p, "idx": idx, "w": w, "sg": sg}


def top5_min_gap(logits: np.ndarray, k: int = 4) -> float:
    """Smallest gap between adjacent logits among the k+1 largest (near-tie test)."""
    s = np.sort(np.asarray(logits, dtype=np.float64))[::-1][: k + 1]
    return float(np.min(s[:-1] - s[1:])) if s.size > 1 else np.inf


# ---------------------------------------------------------------------------
# The layer
# ---------------------------------------------------------------------------

def rms_norm(x, w_bf16, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * w, in fp64 with the bf16 weight widened exactly.

    The pages name the step only ("combine + norm" feeding the next layer,
    [P2 "Verzögerte GPU-Experten-Berechnung"]); this is the plain RMS
    normalisation with a per-element weight.
    """
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x) + eps) * bf16_to_f64(w_bf16)


def layer_decode(w_router_bf16, w_sgate_bf16, get_expert_blob, shared_blob,
                 x, residual, top_k: int, hidden: int, inter: int, bits: int,
                 shared_bits: int = 4, norm_w_bf16=None, norm_eps: float = 1e-6) -> dict:
    """One MoE layer for one token.

    out = residual + sum_k w_k * y_{idx_k} + sg * y_shared
    ([P2 "Metal-Compute-Shader"]: "MoE-Kombination + Rest + Sigmoid-Gate").
    ``get_expert_blob(e)`` returns expert e's blob; ``shared_blob`` may be None.
    With ``norm_w_bf16`` the layer's input is first ``rms_norm(x, norm_w, eps)``
    (the residual is not normalised).
    """
    if norm_w_bf16 is not None:
        x = rms_norm(x, norm_w_bf16, norm_eps)
    r = route(w_router_bf16, w_sgate_bf16, x, top_k)
    out = np.asarray(residual, dtype=np.float64).copy()
    ys = []
    for k, e in enumerate(r["idx"]):
        y = expert_forward(get_expert_blob(int(e)), hidden, inter, bits, x)
        ys.append(y)
        out += r["w"][k] * y
    y_sh = None
    if shared_blob is not None:
        y_sh = expert_forward(shared_blob, hidden, inter, shared_bits, x)
        out += r["sg"] * y_sh
    r.update(out=out, y_routed=ys, y_shared=y_sh)
    return r


# ---------------------------------------------------------------------------
# Quantiser (offline; the pages do not describe it, see module docstring)
# ---------------------------------------------------------------------------

def quantize_matrix(w: np.ndarray, bits: int) -> tuple[np.ndarray, np.ndarray]:
    """fp32 W [N][K] -> (codes uint32 [N][K*b/32], sb uint32 [N][K/64]).

    Every step is an IEEE fp32 operation in this order, per group of 64:
    mn, mx = min, max; s32 = (mx - mn) / (2^b - 1); s = bf16(s32);
    bb = bf16(mn); q = clamp(rint((w - bb) / s), 0, 2^b - 1), q = 0 if s == 0.
    """
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, kdim = w.shape
    assert kdim % GROUP == 0
    g = w.reshape(n, kdim // GROUP, GROUP)
    mn = g.min(axis=-1)
    mx = g.max(axis=-1)
    levels = np.float32((1 << bits) - 1)
    s32 = (mx - mn).astype(np.float32) / levels
    s_bits = f32_to_bf16_bits(s32)
    bb_bits = f32_to_bf16_bits(mn)
    s_f = (s_bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    bb_f = (bb_bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    diff = (g - bb_f[..., None]).astype(np.float32)
    safe = np.where(s_f == 0, np.float32(1), s_f)
    ratio = (diff / safe[..., None]).astype(np.float32)
    q = np.clip(np.rint(ratio), 0, (1 << bits) - 1)
    q = np.where((s_f == 0)[..., None], 0, q).astype(np.uint32)
    codes = pack_codes(q.reshape(n, kdim), bits)
    sb = s_bits.astype(np.uint32) | (bb_bits.astype(np.uint32) << np.uint32(16))
    return codes, sb


def quantize_expert(w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray,
                    bits: int) -> np.ndarray:
    """Quantise and pack one expert into a blob (uint8)."""
    inter, hidden = w_gate.shape
    assert w_up.shape == (inter, hidden) and w_down.shape == (hidden, inter)
    parts = {name: quantize_matrix(m, bits)
             for name, m in (("gate", w_gate), ("up", w_up), ("down", w_down))}
    return assemble_blob(parts, hidden, inter, bits)


# ---------------------------------------------------------------------------
# The linear-attention state update (a second, independent decode step)
# ---------------------------------------------------------------------------

def delta_update(state, q, k, v, alpha, beta):
    """Gated delta-rule recurrence of a multi-head state, T tokens in turn.

    The pages name the routines only: the GatedDeltaNet recurrence updates a
    64-head x 128x128 state matrix with single-precision scale, matrix-vector
    and rank-1-update calls ([P2 "Accelerate-BLAS für lineare
    Aufmerksamkeit"], [P1 "Técnicas innovadoras" §5], [P3 "Uso do
    Accelerate BLAS"], [P5 "Points clés du projet"]).  Read in that order,
    per head and token:

      S <- alpha * S                  (scale)
      u <- S k                        (matrix-vector)
      S <- S + beta * (v - u) k^T     (rank-1 update)
      o <- S q                        (matrix-vector: the readout)

    which is the gated delta rule S' = alpha S (I - beta k k^T) + beta v k^T,
    o = S' q.  Shapes: state [heads][dv][dk] (row i of a head holds the dk
    key coefficients of value i), q and k [T][heads][dk], v [T][heads][dv],
    alpha and beta [T][heads].  Each token is computed in fp64 from the fp32
    state; the state is stored back in fp32 after every token (single
    precision, as the pages' routines are).  Returns (state' as float32,
    o [T][heads][dv] as float64); the input state is not modified.
    """
    S = np.array(state, dtype=np.float32)
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    alpha = np.asarray(alpha, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    T, heads = alpha.shape
    dv = S.shape[1]
    o = np.empty((T, heads, dv), dtype=np.float64)
    for t in range(T):
        for h in range(heads):
            Sh = S[h].astype(np.float64)
            Sh = alpha[t, h] * Sh
            u = Sh @ k[t, h]
            Sh = Sh + beta[t, h] * np.outer(v[t, h] - u, k[t, h])
            o[t, h] = Sh @ q[t, h]
            S[h] = Sh.astype(np.float32)
    return S, o
