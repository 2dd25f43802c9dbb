"""Checks that pin the oracle to facts outside itself.

Each ``pin_*`` function takes the oracle module and raises AssertionError when
the oracle disagrees with a value the pages print, a closed form, exact
rational arithmetic or a brute-force evaluation written differently from the
oracle (bit strings, Python loops, Fractions).  ``test_oracle_pins.py`` runs
them on the real oracle; ``test_oracle_mutations.py`` plants plausible mistakes
in the oracle and checks that some pin fails for each.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
from scipy.special import expit, softmax as sp_softmax

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------------------
# Independent helpers (bit strings and Fractions; nothing shared with the oracle)
# ---------------------------------------------------------------------------

def code_from_bitstring(word: int, bits: int, j: int) -> int:
    """Code j of a 32-bit word by reading the word's binary string."""
    s = format(int(word) & 0xFFFFFFFF, "032b")[::-1]  # s[i] = bit i
    return int(s[bits * j: bits * j + bits][::-1], 2)


def bf16_exact(bits16: int) -> Fraction:
    """Exact value of a bf16 bit pattern (finite)."""
    b = int(bits16) & 0xFFFF
    sign = -1 if b >> 15 else 1
    exp = (b >> 7) & 0xFF
    man = b & 0x7F
    if exp == 0:
        return sign * Fraction(man, 128) * Fraction(2) ** (-126)
    return sign * (1 + Fraction(man, 128)) * Fraction(2) ** (exp - 127)


def bf16_bits_of_dyadic(v: Fraction) -> int:
    """bf16 bit pattern of a dyadic value that bf16 represents exactly."""
    if v == 0:
        return 0
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    man = (a - 1) * 128
    assert man.denominator == 1, "not exactly representable in bf16"
    return sign | ((e + 127) << 7) | int(man)


def load_packing_golden():
    rows = []
    with open(os.path.join(GOLDEN, "packing.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            rows.append((int(parts[0]), int(parts[1], 16), [int(c) for c in parts[2:]]))
    return rows


def rand_words(rng, shape):
    return rng.integers(0, 2**32, size=shape, dtype=np.uint64).astype(np.uint32)


def dyadic_sb(rng, n_rows, n_groups, bits):
    """bf16-exact dyadic scales k/256 and biases -j/64, as (sb words, exact values)."""
    sb = np.zeros((n_rows, n_groups), dtype=np.uint32)
    exact = {}
    for r in range(n_rows):
        for g in range(n_groups):
            s = Fraction(int(rng.integers(1, 16)), 256)
            b = -Fraction(int(rng.integers(0, 64)), 64)
            sb[r, g] = bf16_bits_of_dyadic(s) | (bf16_bits_of_dyadic(b) << 16)
            exact[r, g] = (s, b)
    return sb, exact


# ---------------------------------------------------------------------------
# Pins
# ---------------------------------------------------------------------------

def pin_expert_size(O):
    """The pages print about 6.75 MB per 4-bit expert at hidden 4096."""
    with open(os.path.join(GOLDEN, "pages_sizes.json")) as f:
        g = json.load(f)
    h = g["hidden"]
    # I = 1024 is the only intermediate size that gives the printed figure.
    sizes = {i: O.expert_bytes(h, i, 4) for i in range(64, 4097, 64)}
    hits = [i for i, b in sizes.items() if b == int(g["expert_size_mb_4bit"] * 2**20)]
    assert hits == [1024], hits
    assert O.blob_layout(h, 1024, 4)["total"] == 7_077_888
    assert O.expert_bytes(h, 1024, 2) == 3 * h * 1024 * 2 // 8 + 3 * h * 1024 // 64 * 4 == 3_932_160
    # Section sizes add up and each section starts on a 256-byte boundary.
    for bits in (2, 4):
        for (h2, i2) in ((512, 128), (4096, 1024), (64, 64)):
            lay = O.blob_layout(h2, i2, bits)
            assert lay["total"] == O.expert_bytes(h2, i2, bits)
            for name in ("gate", "up", "down"):
                assert lay[name][0] % 256 == 0 and lay[name][1] % 256 == 0


def pin_packing_golden(O):
    for bits, word, codes in load_packing_golden():
        got = O.unpack_codes(np.array([[word]], dtype=np.uint32), bits)[0].tolist()
        assert got == codes, (bits, hex(word), got, codes)
        back = O.pack_codes(np.array([codes], dtype=np.uint8), bits)
        assert int(back[0, 0]) == word
    rng = np.random.default_rng(7)
    for bits in (2, 4):
        w = rand_words(rng, (5, 12))
        c = O.unpack_codes(w, bits)
        for r in range(5):
            for k in range(c.shape[1]):
                per = 32 // bits
                assert int(c[r, k]) == code_from_bitstring(w[r, k // per], bits, k % per)
        assert np.array_equal(O.pack_codes(c, bits), w)


def _exact_gemv_fma_form(words, exact_sb, bits, x_frac):
    """sum_k fma(q, s*x_k, b*x_k) in exact rationals (the pages' rearrangement)."""
    per = 32 // bits
    n_rows, n_words = words.shape
    out = []
    for r in range(n_rows):
        acc = Fraction(0)
        for k in range(n_words * per):
            q = code_from_bitstring(words[r, k // per], bits, k % per)
            s, b = exact_sb[r, k // 64]
            acc += q * (s * x_frac[k]) + (b * x_frac[k])
        out.append(acc)
    return out


def pin_fma_identity_exact(O):
    """Dequantised GEMV equals the pages' fma(q, s*x, b*x) form exactly.

    Scales, biases and x are dyadic with few bits, so the fp64 oracle makes no
    rounding error and must equal the rational result bit for bit.
    """
    rng = np.random.default_rng(11)
    for bits in (4, 2):
        n_rows, n_in = 6, 192
        words = rand_words(rng, (n_rows, n_in * bits // 32))
        sb, exact = dyadic_sb(rng, n_rows, n_in // 64, bits)
        xi = rng.integers(-32, 33, size=n_in)
        x = xi.astype(np.float64) / 8.0
        x_frac = [Fraction(int(v), 8) for v in xi]
        got = O.dequantize(words, sb, bits) @ x
        want = _exact_gemv_fma_form(words, exact, bits, x_frac)
        for r in range(n_rows):
            assert Fraction(float(got[r])) == want[r], (bits, r, got[r], float(want[r]))


def pin_constant_codes(O):
    """All-zero codes give sum_G b_G * sum(x_G); all-max codes give (qmax*s + b) * sum(x_G)."""
    rng = np.random.default_rng(12)
    for bits in (4, 2):
        n_rows, n_in = 4, 256
        sb, exact = dyadic_sb(rng, n_rows, n_in // 64, bits)
        xi = rng.integers(-64, 65, size=n_in)
        x = xi / 16.0
        gs = [Fraction(int(xi[g * 64:(g + 1) * 64].sum()), 16) for g in range(n_in // 64)]
        qmax = (1 << bits) - 1
        for fill, q in ((0x00000000, 0), (0xFFFFFFFF, qmax)):
            words = np.full((n_rows, n_in * bits // 32), fill, dtype=np.uint32)
            got = O.dequantize(words, sb, bits) @ x
            for r in range(n_rows):
                want = sum((q * exact[r, g][0] + exact[r, g][1]) * gs[g] for g in range(len(gs)))
                assert Fraction(float(got[r])) == want, (bits, fill, r)


def pin_one_hot(O):
    """x = e_k picks out the single weight q[r,k]*s[r,k//64] + b[r,k//64]."""
    rng = np.random.default_rng(13)
    for bits in (4, 2):
        per = 32 // bits
        n_rows, n_in = 3, 192
        words = rand_words(rng, (n_rows, n_in // per))
        sb, exact = dyadic_sb(rng, n_rows, n_in // 64, bits)
        w = O.dequantize(words, sb, bits)
        for k in list(range(0, n_in, 7)) + [n_in - 1]:
            x = np.zeros(n_in)
            x[k] = 1.0
            got = w @ x
            for r in range(n_rows):
                q = code_from_bitstring(words[r, k // per], bits, k % per)
                s, b = exact[r, k // 64]
                assert Fraction(float(got[r])) == q * s + b, (bits, r, k)


def _blob_from_matrices(O, qs, s_b, hidden, inter, bits):
    """Build a blob from integer code matrices and one exact (s, b) per matrix."""
    parts = {}
    for name, q in qs.items():
        rows, n_in = q.shape
        s, b = s_b[name]
        sbw = np.full((rows, n_in // 64), bf16_bits_of_dyadic(s) | (bf16_bits_of_dyadic(b) << 16),
                      dtype=np.uint32)
        per = 32 // bits
        words = np.zeros((rows, n_in // per), dtype=np.uint32)
        for r in range(rows):
            for k in range(n_in):
                words[r, k // per] |= np.uint32(int(q[r, k]) << (bits * (k % per)))
        parts[name] = (words, sbw)
    return O.assemble_blob(parts, hidden, inter, bits)


def pin_permutation_expert(O):
    """Scaled permutation matrices give y = Pd (silu(Pg x) * (Pu x)) by index moves alone."""
    rng = np.random.default_rng(14)
    hidden, inter, bits = 128, 64, 4
    perm_g = rng.permutation(hidden)[:inter]   # gate row i reads x[perm_g[i]]
    perm_u = rng.permutation(hidden)[:inter]
    perm_d = rng.permutation(hidden)           # down row h reads a[perm_d[h] % inter]
    cg = rng.integers(1, 16, size=inter)
    cu = rng.integers(1, 16, size=inter)
    cd = rng.integers(1, 16, size=hidden)
    qg = np.zeros((inter, hidden), dtype=np.int64)
    qu = np.zeros((inter, hidden), dtype=np.int64)
    qd = np.zeros((hidden, inter), dtype=np.int64)
    for i in range(inter):
        qg[i, perm_g[i]] = cg[i]
        qu[i, perm_u[i]] = cu[i]
    for h in range(hidden):
        qd[h, perm_d[h] % inter] = cd[h]
    one = Fraction(1)
    blob = _blob_from_matrices(O, {"gate": qg, "up": qu, "down": qd},
                               {"gate": (one / 4, Fraction(0)), "up": (one / 8, Fraction(0)),
                                "down": (one / 2, Fraction(0))}, hidden, inter, bits)
    x = rng.standard_normal(hidden)
    y = O.expert_forward(blob, hidden, inter, bits, x)
    a = np.empty(inter)
    for i in range(inter):
        g = cg[i] * 0.25 * x[perm_g[i]]
        u = cu[i] * 0.125 * x[perm_u[i]]
        a[i] = g * expit(g) * u
    want = np.array([cd[h] * 0.5 * a[perm_d[h] % inter] for h in range(hidden)])
    np.testing.assert_allclose(y, want, rtol=1e-13, atol=1e-15)


def pin_dense_bruteforce(O):
    """A tiny expert matches Python loops over bit-string-decoded weights."""
    rng = np.random.default_rng(15)
    hidden, inter = 64, 64
    for bits in (4, 2):
        per = 32 // bits
        parts = {}
        dense = {}
        for name, rows, n_in in (("gate", inter, hidden), ("up", inter, hidden), ("down", hidden, inter)):
            words = rand_words(rng, (rows, n_in // per))
            s16 = (rng.integers(0x3A00, 0x3B80, size=(rows, n_in // 64))).astype(np.uint32)
            b16 = (rng.integers(0xBB00, 0xBC80, size=(rows, n_in // 64))).astype(np.uint32)
            parts[name] = (words, s16 | (b16 << 16))
            m = [[0.0] * n_in for _ in range(rows)]
            for r in range(rows):
                for k in range(n_in):
                    q = code_from_bitstring(words[r, k // per], bits, k % per)
                    s = float(bf16_exact(s16[r, k // 64]))
                    b = float(bf16_exact(b16[r, k // 64]))
                    m[r][k] = q * s + b
            dense[name] = m
        blob = O.assemble_blob(parts, hidden, inter, bits)
        x = rng.standard_normal(hidden).tolist()
        g = [math.fsum(dense["gate"][i][k] * x[k] for k in range(hidden)) for i in range(inter)]
        u = [math.fsum(dense["up"][i][k] * x[k] for k in range(hidden)) for i in range(inter)]
        a = [g[i] / (1.0 + math.exp(-g[i])) * u[i] for i in range(inter)]
        want = [math.fsum(dense["down"][h][i] * a[i] for i in range(inter)) for h in range(hidden)]
        got = O.expert_forward(blob, hidden, inter, bits, np.array(x))
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)


def pin_activations(O):
    assert O.silu(0.0) == 0.0
    assert O.sigmoid(0.0) == 0.5
    z = np.linspace(-30, 30, 601)
    np.testing.assert_allclose(O.sigmoid(z), expit(z), rtol=1e-15, atol=0)
    np.testing.assert_allclose(O.silu(z), z * expit(z), rtol=1e-15, atol=1e-300)
    # silu tends to the identity for large z and to 0 for very negative z.
    assert abs(O.silu(40.0) - 40.0) < 1e-12 and abs(O.silu(-40.0)) < 1e-15


def pin_routing(O):
    rng = np.random.default_rng(16)
    E, H = 24, 128
    for trial in range(20):
        w16 = rng.integers(0, 2**16, size=(E, H)).astype(np.uint16)
        # keep finite, modest weights: random sign, exponent near 2^-6
        w16 = ((w16 & 0x807F) | 0x3C00).astype(np.uint16)
        x = rng.standard_normal(H)
        for k in (1, 4, 7):
            r = O.route(w16, None, x, k)
            # logits by Fractions/floats in a loop
            logits = [math.fsum(float(bf16_exact(w16[e, h])) * x[h] for h in range(H)) for e in range(E)]
            want_idx = sorted(range(E), key=lambda e: (-logits[e], e))[:k]
            assert r["idx"].tolist() == want_idx
            assert abs(r["w"].sum() - 1.0) < 1e-15
            p = sp_softmax(np.array(logits))
            np.testing.assert_allclose(r["w"], p[want_idx] / p[want_idx].sum(), rtol=1e-12)
            assert np.all(np.diff(r["w"]) <= 0)
            assert r["sg"] == 1.0
        # K = E reduces to the full softmax
        r = O.route(w16, None, x, E)
        np.testing.assert_allclose(np.sort(r["w"]), np.sort(sp_softmax(np.array(logits))), rtol=1e-12)
    # equal logits: uniform weights and the lowest indices
    r = O.route(np.zeros((E, H), dtype=np.uint16), np.zeros(H, dtype=np.uint16), rng.standard_normal(H), 4)
    assert r["idx"].tolist() == [0, 1, 2, 3]
    assert np.all(r["w"] == 0.25)
    assert r["sg"] == 0.5
    # shared gate = sigmoid(w_sg . x)
    sg16 = np.array([bf16_bits_of_dyadic(Fraction(1, 32))] * H, dtype=np.uint16)
    x = rng.standard_normal(H)
    r = O.route(np.zeros((E, H), dtype=np.uint16), sg16, x, 2)
    assert abs(r["sg"] - expit(math.fsum(x) / 32)) < 1e-15


def pin_layer(O):
    """Layer-level identities: combine weights, residual and the shared gate."""
    rng = np.random.default_rng(17)
    hidden, inter, bits, E = 128, 64, 4, 6
    per = 32 // bits

    def rand_blob(b=bits):
        parts = {}
        for name, rows, n_in in (("gate", inter, hidden), ("up", inter, hidden), ("down", hidden, inter)):
            pw = 32 // b
            words = rand_words(rng, (rows, n_in // pw))
            s16 = rng.integers(0x3A00, 0x3B80, size=(rows, n_in // 64)).astype(np.uint32)
            b16 = rng.integers(0xBB00, 0xBC80, size=(rows, n_in // 64)).astype(np.uint32)
            parts[name] = (words, s16 | (b16 << 16))
        return O.assemble_blob(parts, hidden, inter, b)

    same = rand_blob()
    shared = rand_blob()
    x = rng.standard_normal(hidden)
    res = rng.standard_normal(hidden)
    wr = rng.integers(0x3C00, 0x3C7F, size=(E, hidden)).astype(np.uint16)
    y = O.expert_forward(same, hidden, inter, bits, x)
    ysh = O.expert_forward(shared, hidden, inter, bits, x)
    # (a) K = E with identical experts: the weights sum to one -> res + y + sg*y_sh
    r = O.layer_decode(wr, np.zeros(hidden, dtype=np.uint16), lambda e: same, shared, x, res, E,
                       hidden, inter, bits)
    np.testing.assert_allclose(r["out"], res + y + 0.5 * ysh, rtol=1e-12, atol=1e-12)
    # (b) no shared expert and one routed expert: out = res + y_e (w = 1)
    blobs = [rand_blob() for _ in range(E)]
    r = O.layer_decode(wr, None, lambda e: blobs[e], None, x, res, 1, hidden, inter, bits)
    e0 = int(r["idx"][0])
    np.testing.assert_allclose(r["out"], res + O.expert_forward(blobs[e0], hidden, inter, bits, x),
                               rtol=1e-12, atol=1e-12)
    # (c) a router row aligned with x wins: make expert 4's row the bf16 sign pattern of x
    wr2 = np.zeros((E, hidden), dtype=np.uint16)
    wr2[4] = np.where(x >= 0, 0x3F80, 0xBF80).astype(np.uint16)   # +-1
    wr2[2] = np.where(x >= 0, 0x3F00, 0xBF00).astype(np.uint16)   # +-0.5
    r = O.layer_decode(wr2, None, lambda e: blobs[e], shared, x, res, 2, hidden, inter, bits)
    assert r["idx"].tolist() == [4, 2]
    lg = [np.abs(x).sum(), 0.5 * np.abs(x).sum()]
    w4 = 1.0 / (1.0 + math.exp(lg[1] - lg[0]))
    want = res + w4 * O.expert_forward(blobs[4], hidden, inter, bits, x) \
        + (1 - w4) * O.expert_forward(blobs[2], hidden, inter, bits, x) + ysh
    np.testing.assert_allclose(r["out"], want, rtol=1e-12, atol=1e-12)
    # (d) mixed widths: a 2-bit routed expert with a 4-bit shared expert
    b2 = rand_blob(2)
    r = O.layer_decode(wr, None, lambda e: b2, shared, x, res, 1, hidden, inter, 2, shared_bits=4)
    np.testing.assert_allclose(r["out"], res + O.expert_forward(b2, hidden, inter, 2, x) + ysh,
                               rtol=1e-12, atol=1e-12)
    # (e) input RMS norm (unit weight, eps 0): the layer sees x / rms(x), so scaling
    # x by a power of two leaves the decision and the MoE output unchanged,
    # and the result equals the un-normalised layer on x / rms(x)
    ones = np.full(hidden, 0x3F80, dtype=np.uint16)
    zero = np.zeros(hidden)
    rn = O.layer_decode(wr, None, lambda e: blobs[e], shared, x, zero, 2, hidden, inter, bits,
                        norm_w_bf16=ones, norm_eps=0.0)
    rs = O.layer_decode(wr, None, lambda e: blobs[e], shared, x * 8.0, zero, 2, hidden, inter, bits,
                        norm_w_bf16=ones, norm_eps=0.0)
    assert rn["idx"].tolist() == rs["idx"].tolist()
    np.testing.assert_allclose(rs["out"], rn["out"], rtol=1e-12, atol=1e-12)
    xn = x / math.sqrt(float(np.mean(x * x)))
    r0 = O.layer_decode(wr, None, lambda e: blobs[e], shared, xn, zero, 2, hidden, inter, bits)
    np.testing.assert_allclose(rn["out"], r0["out"], rtol=1e-12, atol=1e-12)
    assert np.max(np.abs(rn["out"] - O.layer_decode(wr, None, lambda e: blobs[e], shared, x, zero, 2, hidden,
                                                    inter, bits)["out"])) > 1e-6  # the norm matters here


def pin_quantizer(O):
    rng = np.random.default_rng(18)
    for bits in (4, 2):
        qmax = (1 << bits) - 1
        w = (rng.standard_normal((8, 256)) * 0.02).astype(np.float32)
        codes, sb = O.quantize_matrix(w, bits)
        assert codes.shape == (8, 256 * bits // 32) and sb.shape == (8, 4)
        wh = O.dequantize(codes, sb, bits)
        s = np.array([[float(bf16_exact(v & 0xFFFF)) for v in row] for row in sb])
        b = np.array([[float(bf16_exact(v >> 16)) for v in row] for row in sb])
        g = w.astype(np.float64).reshape(8, 4, 64)
        mn, mx = g.min(-1), g.max(-1)
        s32 = (mx - mn) / qmax
        # bias is mn rounded to bf16, scale is the range / qmax rounded to bf16
        assert np.all(np.abs(b - mn) <= np.abs(mn) * 2.0**-8)
        assert np.all(np.abs(s - s32) <= s32 * 2.0**-8 + 1e-30)
        bound = s / 2 + np.abs(b - mn) + qmax * np.abs(s - s32)
        err = np.abs(wh.reshape(8, 4, 64) - g)
        assert np.all(err <= bound[..., None] * (1 + 1e-5) + 1e-12)
        # a group already on the grid re-quantises to the same codes
        q = rng.integers(0, qmax + 1, size=(4, 128))
        q[:, 0] = 0
        q[:, 64] = 0
        q[:, 1] = qmax
        q[:, 65] = qmax
        s_grid = Fraction(3, 1024)
        b_grid = -Fraction(5, 128)
        wg = np.array([[float(int(v) * s_grid + b_grid) for v in row] for row in q], dtype=np.float32)
        c2, sb2 = O.quantize_matrix(wg, bits)
        assert np.array_equal(O.unpack_codes(c2, bits), q.astype(np.uint8))
        assert np.all(sb2 == (bf16_bits_of_dyadic(s_grid) | (bf16_bits_of_dyadic(b_grid) << 16)))
        # a constant group: scale 0, codes 0, bias = the constant
        wc = np.full((2, 64), 0.375, dtype=np.float32)
        c3, sb3 = O.quantize_matrix(wc, bits)
        assert np.all(c3 == 0) and np.all(sb3 == (bf16_bits_of_dyadic(Fraction(3, 8)) << 16))
    # quantise_expert builds a blob whose matrices dequantise to the quantised values
    wg_ = (rng.standard_normal((64, 128)) * 0.02).astype(np.float32)
    wu_ = (rng.standard_normal((64, 128)) * 0.02).astype(np.float32)
    wd_ = (rng.standard_normal((128, 64)) * 0.02).astype(np.float32)
    blob = O.quantize_expert(wg_, wu_, wd_, 4)
    assert blob.size == O.expert_bytes(128, 64, 4)
    mg, mu, md = O.expert_matrices(blob, 128, 64, 4)
    for m, ref in ((mg, wg_), (mu, wu_), (md, wd_)):
        assert np.max(np.abs(m - ref)) < 0.02 * 8 / 15


def load_bf16_golden():
    rows = []
    with open(os.path.join(GOLDEN, "bf16_rounding.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                a, b = line.split()[:2]
                rows.append((int(a, 16), int(b, 16)))
    return rows


def _bf16_nearest_even(u32: int) -> int:
    """bf16 pattern nearest to the finite fp32 pattern u32 by exact comparison
    of the two neighbouring bf16 values (ties to the even mantissa)."""
    x = Fraction(float(np.array([u32], dtype=np.uint32).view(np.float32)[0]))
    lo = u32 >> 16  # the bf16 pattern of the same sign toward zero
    hi = lo + 1     # the next bf16 pattern away from zero
    d_lo = abs(x - bf16_exact(lo))
    d_hi = abs(bf16_exact(hi) - x) if (hi & 0x7FFF) < 0x7F80 else None
    if d_hi is None or d_lo < d_hi:
        return lo
    if d_hi < d_lo:
        return hi
    return lo if lo % 2 == 0 else hi


def pin_bf16_rne(O):
    """fp32 -> bf16 is round to nearest, ties to even: hand-worked bit patterns
    (ties both ways, just above and below a tie, a carry into the exponent,
    subnormals; tests/golden/bf16_rounding.txt) and, on random finite values,
    the nearest bf16 neighbour found by exact rational comparison."""
    gold = load_bf16_golden()
    assert len(gold) >= 16
    src = np.array([a for a, _ in gold], dtype=np.uint32).view(np.float32)
    got = O.f32_to_bf16_bits(src)
    for (a, want), g in zip(gold, got.tolist()):
        assert g == want, (hex(a), hex(g), hex(want))
    rng = np.random.default_rng(22)
    u = rng.integers(0, 2**32, size=3000, dtype=np.uint64).astype(np.uint32)
    u = u[(u & 0x7F800000) < 0x7F000000]  # finite, clear of bf16 overflow
    # every exact tie pattern of these exponents too
    u = np.concatenate([u, (u & np.uint32(0xFFFF0000)) | np.uint32(0x8000)])
    got = O.f32_to_bf16_bits(u.view(np.float32))
    for a, g in zip(u.tolist(), got.tolist()):
        assert g == _bf16_nearest_even(a), hex(a)


def load_quantizer_ties():
    groups = []
    with open(os.path.join(GOLDEN, "quantizer_ties.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0] == "group":
                groups.append((int(parts[1]), int(parts[2], 16), [], []))
            else:
                groups[-1][2].append(int(parts[0], 16))
                groups[-1][3].append(int(parts[1]))
    return groups


def pin_quantizer_ties(O):
    """Groups whose fp32 quotient (w - bias) / s is an exact half only after
    the fp32 subtraction rounds: the hand-worked codes (round half to even on
    the fp32 quotient, tests/golden/quantizer_ties.txt) separate the stated
    fp32 op order from an fp64 division and from rounding halves up."""
    groups = load_quantizer_ties()
    assert [g[0] for g in groups] == [4, 2]
    for bits, sbw, wbits, codes in groups:
        assert len(wbits) == 64
        w = np.array(wbits, dtype=np.uint32).view(np.float32).reshape(1, 64)
        got_codes, got_sb = O.quantize_matrix(w, bits)
        assert int(got_sb[0, 0]) == sbw, (bits, hex(int(got_sb[0, 0])))
        words = [int(v) for v in got_codes[0]]
        per = 32 // bits
        dec = [code_from_bitstring(words[k // per], bits, k % per) for k in range(64)]
        assert dec == codes, (bits, dec, codes)
    # on every quotient: the fp32 subtraction, the fp32 division and ties to
    # even, evaluated one element at a time with Python floats narrowed to fp32
    rng = np.random.default_rng(23)
    f32 = lambda v: float(np.float32(v))
    for bits in (4, 2):
        qmax = (1 << bits) - 1
        w = (rng.standard_normal((4, 128)) * 0.02).astype(np.float32)
        got_codes, got_sb = O.quantize_matrix(w, bits)
        for r in range(4):
            for gi in range(2):
                grp = [float(v) for v in w[r, gi * 64:(gi + 1) * 64]]
                sbw = int(got_sb[r, gi])
                s = float(bf16_exact(sbw & 0xFFFF))
                b = float(bf16_exact(sbw >> 16))
                for j, v in enumerate(grp):
                    quot = f32(f32(v - b) / s)
                    want = min(max(round(quot), 0), qmax)  # Python round: ties to even
                    k = gi * 64 + j
                    got = code_from_bitstring(int(got_codes[r, k // (32 // bits)]), bits, k % (32 // bits))
                    assert got == want, (bits, r, k, quot)


def pin_near_tie_gap(O):
    """The near-tie screen is the smallest gap between adjacent values among
    the k + 1 largest logits (descending order), ties giving 0."""
    # top-5 of (9, 7, 5, 3, 3 - 2^-7, -4): gaps 2, 2, 2, 2^-7
    assert O.top5_min_gap(np.array([3.0, 9.0, -4.0, 5.0, 3.0 - 2.0**-7, 7.0]), 4) == 2.0**-7
    # a small gap just outside the k + 1 largest does not count
    assert O.top5_min_gap(np.array([10.0, 8.0, 6.0, 4.0, 2.0, 2.0 - 2.0**-10]), 4) == 2.0
    # an exact tie among the largest
    assert O.top5_min_gap(np.array([1.0, 5.0, 5.0, 0.0, -1.0]), 4) == 0.0
    # k = 1 looks at the two largest only
    assert O.top5_min_gap(np.array([0.0, 4.0, 3.5, 3.4]), 1) == 0.5
    # against a plain sort on random vectors
    rng = np.random.default_rng(24)
    for _ in range(50):
        v = rng.standard_normal(40)
        k = int(rng.integers(1, 8))
        top = sorted(v.tolist(), reverse=True)[: k + 1]
        assert O.top5_min_gap(v, k) == min(a - b for a, b in zip(top, top[1:]))


def pin_rms_norm(O):
    """RMS normalisation against closed forms (eps = 0 unless stated)."""
    one = np.full(8, 0x3F80, dtype=np.uint16)  # bf16 1.0
    # a constant vector normalises to +-1 exactly
    assert np.array_equal(O.rms_norm(np.full(8, -3.0), one, 0.0), np.full(8, -1.0))
    # (3, 4): mean of squares 12.5, so the result is (3, 4) / sqrt(12.5) = (3, 4) * sqrt(2) / 5
    got = O.rms_norm(np.array([3.0, 4.0]), one[:2], 0.0)
    np.testing.assert_allclose(got, np.array([3.0, 4.0]) * np.sqrt(2.0) / 5.0, rtol=1e-15, atol=0)
    # scale invariance by powers of two (exact), and mean of squares 1 with unit weight
    rng = np.random.default_rng(21)
    x = rng.standard_normal(256)
    y = O.rms_norm(x, np.full(256, 0x3F80, dtype=np.uint16), 0.0)
    assert np.array_equal(O.rms_norm(x * 2.0**-7, np.full(256, 0x3F80, dtype=np.uint16), 0.0), y)
    assert abs(np.mean(y * y) - 1.0) < 1e-14
    # the weight multiplies element by element (bf16 2.0 = 0x4000, 0.5 = 0x3F00)
    w = np.where(np.arange(256) % 2 == 0, 0x4000, 0x3F00).astype(np.uint16)
    yw = O.rms_norm(x, w, 0.0)
    assert np.array_equal(yw[0::2], 2.0 * y[0::2]) and np.array_equal(yw[1::2], 0.5 * y[1::2])
    # eps keeps a zero input finite (zero)
    assert np.array_equal(O.rms_norm(np.zeros(4), one[:4], 1e-6), np.zeros(4))
    # eps enters under the root: x = (1, 1), eps = 3 -> 1 / sqrt(4) = 0.5
    assert np.array_equal(O.rms_norm(np.ones(2), one[:2], 3.0), np.full(2, 0.5))


def _delta_inputs(rng, T, heads, dk, dv, unit_k=True):
    S = (0.1 * rng.standard_normal((heads, dv, dk))).astype(np.float32)
    q = rng.standard_normal((T, heads, dk))
    k = rng.standard_normal((T, heads, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, heads, dv))
    alpha = rng.uniform(0.8, 1.0, (T, heads))
    beta = rng.uniform(0.0, 1.0, (T, heads))
    return S, q, k, v, alpha, beta


def pin_delta_rule(O):
    """The delta-rule update against its defining properties and an exact
    brute force (the stepwise oracle is checked against the matrix form
    alpha S (I - beta k k^T) + beta v k^T, computed differently)."""
    rng = np.random.default_rng(31)
    # (a) matrix form, one token, several heads: S' and o = S' q
    S, q, k, v, alpha, beta = _delta_inputs(rng, 1, 3, 16, 12)
    got_S, got_o = O.delta_update(S, q, k, v, alpha, beta)
    for h in range(3):
        S64 = S[h].astype(np.float64)
        M = alpha[0, h] * S64 @ (np.eye(16) - beta[0, h] * np.outer(k[0, h], k[0, h])) \
            + beta[0, h] * np.outer(v[0, h], k[0, h])
        np.testing.assert_allclose(got_S[h], M.astype(np.float32), rtol=2e-7, atol=1e-7)
        np.testing.assert_allclose(got_o[0, h], M @ q[0, h], rtol=1e-12, atol=1e-12)
    # (b) beta = 0 is a pure decay: S' = fl32(alpha S), o = alpha S q
    S, q, k, v, alpha, _ = _delta_inputs(rng, 1, 2, 8, 8)
    got_S, got_o = O.delta_update(S, q, k, v, alpha, np.zeros((1, 2)))
    for h in range(2):
        assert np.array_equal(got_S[h], (alpha[0, h] * S[h].astype(np.float64)).astype(np.float32))
        np.testing.assert_allclose(got_o[0, h], alpha[0, h] * S[h].astype(np.float64) @ q[0, h], rtol=1e-13)
    # (c) alpha = beta = 1 with a unit key writes v at k: S' k = v (the rule's
    # defining property), and leaves every direction orthogonal to k alone
    S, q, k, v, _, _ = _delta_inputs(rng, 1, 1, 32, 20)
    got_S, _ = O.delta_update(S, q, k, v, np.ones((1, 1)), np.ones((1, 1)))
    np.testing.assert_allclose(got_S[0].astype(np.float64) @ k[0, 0], v[0, 0], rtol=0, atol=2e-6)
    w = rng.standard_normal(32)
    w -= (w @ k[0, 0]) * k[0, 0]
    np.testing.assert_allclose(got_S[0].astype(np.float64) @ w, S[0].astype(np.float64) @ w, rtol=0, atol=2e-6)
    # (d) exact brute force on small integers and dyadic gates (every value
    # and intermediate exact in fp64 and the state exact in fp32), two tokens
    from fractions import Fraction as Fr
    heads, dk, dv, T = 2, 3, 2, 2
    Si = rng.integers(-4, 5, (heads, dv, dk))
    qi = rng.integers(-3, 4, (T, heads, dk))
    ki = rng.integers(-2, 3, (T, heads, dk))
    vi = rng.integers(-5, 6, (T, heads, dv))
    al = np.array([[0.5, 1.0], [0.75, 0.5]])
    be = np.array([[0.25, 0.5], [1.0, 0.125]])
    got_S, got_o = O.delta_update(Si.astype(np.float32), qi, ki, vi, al, be)
    for h in range(heads):
        M = [[Fr(int(Si[h, i, j])) for j in range(dk)] for i in range(dv)]
        for t in range(T):
            a_, b_ = Fr(al[t, h]), Fr(be[t, h])
            M = [[a_ * M[i][j] for j in range(dk)] for i in range(dv)]
            u = [sum(M[i][j] * int(ki[t, h, j]) for j in range(dk)) for i in range(dv)]
            M = [[M[i][j] + b_ * (int(vi[t, h, i]) - u[i]) * int(ki[t, h, j]) for j in range(dk)]
                 for i in range(dv)]
            for i in range(dv):
                assert got_o[t, h, i] == float(sum(M[i][j] * int(qi[t, h, j]) for j in range(dk))), (t, h, i)
        for i in range(dv):
            for j in range(dk):
                assert got_S[h, i, j] == np.float32(float(M[i][j])), (h, i, j)
    # (e) heads are independent and the state rows are the value dimension:
    # permuting the heads, or the values (rows of S and entries of v), permutes
    # the results the same way
    S, q, k, v, alpha, beta = _delta_inputs(rng, 2, 4, 8, 6)
    ref_S, ref_o = O.delta_update(S, q, k, v, alpha, beta)
    ph = np.array([2, 0, 3, 1])
    pS, po = O.delta_update(S[ph], q[:, ph], k[:, ph], v[:, ph], alpha[:, ph], beta[:, ph])
    assert np.array_equal(pS, ref_S[ph]) and np.array_equal(po, ref_o[:, ph])
    pr = np.array([5, 3, 1, 0, 2, 4])
    pS, po = O.delta_update(S[:, pr], q, k, v[:, :, pr], alpha, beta)
    # (the library's matrix-vector product may sum a row in another order at
    # another position: equal to rounding)
    np.testing.assert_allclose(pS, ref_S[:, pr], rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(po, ref_o[:, :, pr], rtol=1e-12, atol=1e-12)
    # (f) the input state is left as it was
    S0 = S.copy()
    O.delta_update(S, q, k, v, alpha, beta)
    assert np.array_equal(S, S0)


ALL_PINS = [pin_expert_size, pin_packing_golden, pin_fma_identity_exact, pin_constant_codes,
            pin_one_hot, pin_permutation_expert, pin_dense_bruteforce, pin_activations,
            pin_routing, pin_layer, pin_quantizer, pin_rms_norm, pin_delta_rule, pin_bf16_rne,
            pin_quantizer_ties, pin_near_tie_gap]
