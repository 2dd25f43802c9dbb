"""Plant plausible mistakes in the oracle (on the CPU) and check a pin catches each.

Every mutant below is a one-line slip someone could make while writing the
oracle: a wrong nibble order, a dropped bias, a wrong group index, a
transposed operand, a missing renormalisation, and so on.  For each, at least
one pin in ``oracle_pins`` must fail; otherwise the pins would not be strong
enough to trust the oracle.
"""
import numpy as np
import pytest

import oracle as O
from tests import oracle_pins as P


def _msb_first_unpack(words, bits):
    words = np.asarray(words, dtype=np.uint32)
    per = 32 // bits
    mask = np.uint32((1 << bits) - 1)
    shifts = (np.arange(per, dtype=np.uint32)[::-1] * np.uint32(bits))
    codes = (words[..., :, None] >> shifts) & mask
    return codes.reshape(*words.shape[:-1], words.shape[-1] * per).astype(np.uint8)


def _dequant_no_bias(words, sb, bits):
    q = O.unpack_codes(words, bits).astype(np.float64)
    s, b = O.unpack_scale_bias(sb)
    return q * np.repeat(s, 64, axis=-1)


def _dequant_group32(words, sb, bits):
    q = O.unpack_codes(words, bits).astype(np.float64)
    s, b = O.unpack_scale_bias(sb)
    k = q.shape[-1]
    gi = np.minimum(np.arange(k) // 32, s.shape[-1] - 1)
    return q * s[..., gi] + b[..., gi]


def _dequant_swapped_sb(words, sb, bits):
    q = O.unpack_codes(words, bits).astype(np.float64)
    s, b = O.unpack_scale_bias(sb)
    return q * np.repeat(b, 64, axis=-1) + np.repeat(s, 64, axis=-1)


def _dequant_centered(words, sb, bits):
    # symmetric-code slip: (q - 2^(b-1)) * s + b
    q = O.unpack_codes(words, bits).astype(np.float64) - (1 << (bits - 1))
    s, b = O.unpack_scale_bias(sb)
    return q * np.repeat(s, 64, axis=-1) + np.repeat(b, 64, axis=-1)


def _forward_transposed_down(blob, hidden, inter, bits, x):
    wg, wu, wd = O.expert_matrices(blob, hidden, inter, bits)
    a = O.silu(wg @ x) * (wu @ x)
    # slip: use the down matrix as if it were stored [I][H]
    return wd.reshape(inter, hidden).T @ a


def _forward_swapped_gate_up(blob, hidden, inter, bits, x):
    wg, wu, wd = O.expert_matrices(blob, hidden, inter, bits)
    return wd @ (O.silu(wu @ x) * (wg @ x))


def _silu_wrong(z):
    z = np.asarray(z, dtype=np.float64)
    return z * O.sigmoid(-z)


def _top_k_ascending(logits, k):
    return np.argsort(np.asarray(logits), kind="stable")[:k].astype(np.int32)


def _top_k_ties_high(logits, k):
    l = np.asarray(logits, dtype=np.float64)
    order = np.lexsort((-np.arange(l.size), -l))
    return order[:k].astype(np.int32)


def _route_no_renorm(w_router_bf16, w_sgate_bf16, x, top_k):
    r = ORIG_ROUTE(w_router_bf16, w_sgate_bf16, x, top_k)
    r["w"] = r["p"][r["idx"]]
    return r


def _route_sg_no_sigmoid(w_router_bf16, w_sgate_bf16, x, top_k):
    r = ORIG_ROUTE(w_router_bf16, w_sgate_bf16, x, top_k)
    if w_sgate_bf16 is not None:
        r["sg"] = float(O.bf16_to_f64(w_sgate_bf16) @ np.asarray(x, dtype=np.float64))
    return r


def _layer_no_residual(w_router_bf16, w_sgate_bf16, get_blob, shared_blob, x, residual, *a, **kw):
    return ORIG_LAYER(w_router_bf16, w_sgate_bf16, get_blob, shared_blob, x,
                      np.zeros_like(np.asarray(residual, dtype=np.float64)), *a, **kw)


def _expert_bytes_bf16_once(hidden, inter, bits, group=64):
    # slip: one 2-byte scale per group and no bias
    return 3 * hidden * inter * bits // 8 + 3 * hidden * inter // group * 2


def _quantize_bias_max(w, bits):
    codes, sb = ORIG_QUANT(w, bits)
    g = np.asarray(w, dtype=np.float32).reshape(w.shape[0], -1, 64)
    mx_bits = O.f32_to_bf16_bits(g.max(-1))
    return codes, (sb & np.uint32(0xFFFF)) | (mx_bits.astype(np.uint32) << np.uint32(16))


def _quantize_floor(w, bits):
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, kdim = w.shape
    g = w.reshape(n, kdim // 64, 64)
    mn, mx = g.min(-1), g.max(-1)
    s32 = (mx - mn).astype(np.float32) / np.float32((1 << bits) - 1)
    sbits = O.f32_to_bf16_bits(s32)
    bbits = O.f32_to_bf16_bits(mn)
    s_f = (sbits.astype(np.uint32) << 16).view(np.float32)
    b_f = (bbits.astype(np.uint32) << 16).view(np.float32)
    q = np.clip(np.floor((g - b_f[..., None]) / s_f[..., None]), 0, (1 << bits) - 1).astype(np.uint32)
    return O.pack_codes(q.reshape(n, kdim), bits), sbits.astype(np.uint32) | (bbits.astype(np.uint32) << 16)


def _rms_norm_mean_abs(x, w_bf16, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / (np.mean(np.abs(x)) + eps) * O.bf16_to_f64(w_bf16)


def _rms_norm_no_sqrt(x, w_bf16, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / (np.mean(x * x) + eps) * O.bf16_to_f64(w_bf16)


def _rms_norm_no_weight(x, w_bf16, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x) + eps)


def _layer_ignores_norm(*a, **kw):
    kw.pop("norm_w_bf16", None)
    kw.pop("norm_eps", None)
    return ORIG_LAYER(*a, **kw)


def _delta_variant(order):
    """A delta-rule oracle with one slip, chosen by `order`."""
    def step(Sh, a_, b_, kk, vv, qq):
        if order == "gemv_before_scale":
            u = Sh @ kk
            Sn = a_ * Sh + b_ * np.outer(vv - u, kk)
        elif order == "correction_sign":
            Sa = a_ * Sh
            Sn = Sa - b_ * np.outer(vv - Sa @ kk, kk)
        elif order == "scale_after_update":
            Sn = a_ * (Sh + b_ * np.outer(vv - Sh @ kk, kk))
        elif order == "no_beta":
            Sa = a_ * Sh
            Sn = Sa + np.outer(vv - Sa @ kk, kk)
        elif order == "transposed_outer":
            Sa = a_ * Sh
            Sn = Sa + b_ * np.outer(kk, vv - Sa @ kk)
        else:  # readout_before_update
            Sa = a_ * Sh
            return Sa + b_ * np.outer(vv - Sa @ kk, kk), Sh @ qq
        return Sn, Sn @ qq

    def fn(state, q, k, v, alpha, beta):
        S = np.array(state, dtype=np.float32)
        q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
        alpha, beta = np.asarray(alpha, dtype=np.float64), np.asarray(beta, dtype=np.float64)
        T, heads = alpha.shape
        o = np.empty((T, heads, S.shape[1]))
        for t in range(T):
            for h in range(heads):
                Sn, o[t, h] = step(S[h].astype(np.float64), alpha[t, h], beta[t, h], k[t, h], v[t, h], q[t, h])
                S[h] = Sn.astype(np.float32)
        return S, o
    return fn


def _bf16_truncate(f):
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


def _bf16_half_up(f):
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + np.uint64(0x8000)) >> np.uint64(16)).astype(np.uint16)


def _quantize_variant(kind):
    """The stated quantiser with one slip: an fp64 quotient, or halves rounded up."""
    def fn(w, bits):
        w = np.ascontiguousarray(w, dtype=np.float32)
        n, kdim = w.shape
        g = w.reshape(n, kdim // 64, 64)
        mn, mx = g.min(-1), g.max(-1)
        s32 = (mx - mn).astype(np.float32) / np.float32((1 << bits) - 1)
        sbits = O.f32_to_bf16_bits(s32)
        bbits = O.f32_to_bf16_bits(mn)
        s_f = (sbits.astype(np.uint32) << 16).view(np.float32)
        b_f = (bbits.astype(np.uint32) << 16).view(np.float32)
        safe = np.where(s_f == 0, np.float32(1), s_f)
        if kind == "fp64_quotient":
            ratio = (g.astype(np.float64) - b_f[..., None].astype(np.float64)) / safe[..., None].astype(np.float64)
            q = np.rint(ratio)
        else:  # half_up
            ratio = ((g - b_f[..., None]).astype(np.float32) / safe[..., None]).astype(np.float32)
            q = np.floor(ratio + np.float32(0.5))
        q = np.clip(q, 0, (1 << bits) - 1)
        q = np.where((s_f == 0)[..., None], 0, q).astype(np.uint32)
        return O.pack_codes(q.reshape(n, kdim), bits), sbits.astype(np.uint32) | (bbits.astype(np.uint32) << 16)
    return fn


def _gap_never_near(logits, k=4):
    return np.inf


def _gap_top_k_only(logits, k=4):
    s = np.sort(np.asarray(logits, dtype=np.float64))[::-1][:k]
    return float(np.min(s[:-1] - s[1:])) if s.size > 1 else np.inf


ORIG_ROUTE = O.route
ORIG_LAYER = O.layer_decode
ORIG_QUANT = O.quantize_matrix

MUTANTS = {
    "msb_first_packing": ("unpack_codes", _msb_first_unpack),
    "dropped_bias": ("dequantize", _dequant_no_bias),
    "group_index_32": ("dequantize", _dequant_group32),
    "scale_bias_swapped": ("dequantize", _dequant_swapped_sb),
    "centered_codes": ("dequantize", _dequant_centered),
    "transposed_down": ("expert_forward", _forward_transposed_down),
    "gate_up_swapped": ("expert_forward", _forward_swapped_gate_up),
    "silu_sign": ("silu", _silu_wrong),
    "topk_ascending": ("top_k_order", _top_k_ascending),
    "topk_ties_high_index": ("top_k_order", _top_k_ties_high),
    "no_renormalisation": ("route", _route_no_renorm),
    "shared_gate_no_sigmoid": ("route", _route_sg_no_sigmoid),
    "no_residual": ("layer_decode", _layer_no_residual),
    "expert_bytes_wrong": ("expert_bytes", _expert_bytes_bf16_once),
    "quantizer_bias_is_max": ("quantize_matrix", _quantize_bias_max),
    "quantizer_floor": ("quantize_matrix", _quantize_floor),
    "rms_norm_mean_abs": ("rms_norm", _rms_norm_mean_abs),
    "rms_norm_no_sqrt": ("rms_norm", _rms_norm_no_sqrt),
    "rms_norm_no_weight": ("rms_norm", _rms_norm_no_weight),
    "layer_ignores_norm": ("layer_decode", _layer_ignores_norm),
    "delta_gemv_before_scale": ("delta_update", _delta_variant("gemv_before_scale")),
    "delta_correction_sign": ("delta_update", _delta_variant("correction_sign")),
    "delta_scale_after_update": ("delta_update", _delta_variant("scale_after_update")),
    "delta_no_beta": ("delta_update", _delta_variant("no_beta")),
    "delta_transposed_outer": ("delta_update", _delta_variant("transposed_outer")),
    "delta_readout_before_update": ("delta_update", _delta_variant("readout_before_update")),
    "bf16_truncation": ("f32_to_bf16_bits", _bf16_truncate),
    "bf16_round_half_up": ("f32_to_bf16_bits", _bf16_half_up),
    "quantizer_fp64_quotient": ("quantize_matrix", _quantize_variant("fp64_quotient")),
    "quantizer_round_half_up": ("quantize_matrix", _quantize_variant("half_up")),
    "near_tie_gap_never_near": ("top5_min_gap", _gap_never_near),
    "near_tie_gap_top_k_only": ("top5_min_gap", _gap_top_k_only),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for pin in P.ALL_PINS:
        try:
            pin(O)
        except AssertionError:
            failed.append(pin.__name__)
        except Exception as e:  # a crash also counts as caught
            failed.append(f"{pin.__name__}:{type(e).__name__}")
    assert failed, f"mutant {name} survived every pin"
