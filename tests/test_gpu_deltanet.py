"""The gated delta-rule state update on the GPU against the oracle.

Every case draws seeded inputs (synth), runs `fmoe_delta_update` through the
C ABI and compares the updated state and the readouts element by element with
the fp64 oracle, within a bound from an fp32 rounding model written here (not
in the oracle): unit roundoff u = 2^-24; a dot product of dk terms is off by at
most (dk + 2) u times the sum of its absolute terms; each stored value adds u
of itself; a state error carries into the next token scaled by alpha and
through the rank-1 update, so the per-token bounds add up.  The bound is that
model times 2.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth as S

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


@pytest.fixture(scope="module")
def F():
    from bit_quantized_expert_router_b200 import build as B
    B.build_engine()
    import bit_quantized_expert_router_b200 as F
    F.lib()
    return F


def dev():
    return torch.device("cuda:0")


def error_bounds(state, q, k, v, alpha, beta):
    """Elementwise bounds on |kernel - oracle| for the state and the readouts."""
    Sx = state.astype(np.float64)
    bS = np.zeros_like(Sx)
    T, heads = alpha.shape
    dk = Sx.shape[2]
    bo = np.zeros((T, heads, Sx.shape[1]))
    for t in range(T):
        for h in range(heads):
            kk, qq = k[t, h].astype(np.float64), q[t, h].astype(np.float64)
            a_, b_ = float(alpha[t, h]), float(beta[t, h])
            Sa = a_ * Sx[h]
            ui = Sa @ kk
            e_u = (dk + 2) * U * (np.abs(Sa) @ np.abs(kk)) + a_ * (bS[h] @ np.abs(kk))
            c = b_ * (v[t, h] - ui)
            e_c = abs(b_) * (U * np.abs(v[t, h] - ui) + e_u) + U * np.abs(c)
            Sn = Sa + np.outer(c, kk)
            eS = a_ * bS[h] + 2 * U * np.abs(Sa) + np.outer(e_c, np.abs(kk)) + 2 * U * np.abs(Sn)
            bo[t, h] = (dk + 2) * U * (np.abs(Sn) @ np.abs(qq)) + eS @ np.abs(qq)
            bS[h] = eS
            Sx[h] = Sn
    return 2 * bS, 2 * bo


def run_case(F, heads, dk, dv, T, seed=41, layer=0, beta_zero=False):
    st = S.delta_state(seed, layer, heads, dv, dk)
    tk = S.delta_tokens(seed, layer, 0, T, heads, dk, dv)
    if beta_zero:
        tk["beta"] = np.zeros_like(tk["beta"])
    d = {n: torch.from_numpy(a).to(dev()) for n, a in tk.items()}
    sd = torch.from_numpy(st).to(dev())
    o = F.delta_update(sd, d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    torch.cuda.synchronize()
    got_S, got_o = sd.cpu().numpy(), o.cpu().numpy()
    ref_S, ref_o = O.delta_update(st, tk["q"], tk["k"], tk["v"], tk["alpha"], tk["beta"])
    bS, bo = error_bounds(st, tk["q"], tk["k"], tk["v"], tk["alpha"], tk["beta"])
    eS = np.abs(got_S.astype(np.float64) - ref_S.astype(np.float64))
    eo = np.abs(got_o.astype(np.float64) - ref_o)
    assert np.isfinite(got_S).all() and np.isfinite(got_o).all()
    assert (eS <= bS).all(), f"state: worst excess {np.max(eS - bS):.3e}, max err {eS.max():.3e}"
    assert (eo <= bo).all(), f"readout: worst excess {np.max(eo - bo):.3e}, max err {eo.max():.3e}"
    return st, tk, got_S, got_o, ref_S


def test_full_size_one_token(F):
    """The pages' state: 64 heads x 128x128, one token (the bench's call)."""
    run_case(F, 64, 128, 128, 1)


def test_several_tokens_in_turn(F):
    run_case(F, 64, 128, 128, 4, seed=42)


@pytest.mark.parametrize("heads,dk,dv,T", [(1, 128, 1, 1), (3, 256, 37, 2), (2, 384, 5, 3), (2, 512, 64, 1),
                                           (5, 128, 13, 5)],
                         ids=["one_row", "ragged_rows_dk256", "dk384_dv5", "dk512", "five_tokens"])
def test_edge_shapes(F, heads, dk, dv, T):
    """Single row, row counts that leave the last CTA partly empty, every key width."""
    run_case(F, heads, dk, dv, T, seed=43)


def test_zero_write_gate_is_pure_decay(F):
    """beta = 0: the state is only scaled, so it equals fl32(alpha * S) exactly."""
    st, tk, got_S, _, ref_S = run_case(F, 8, 128, 128, 1, seed=44, beta_zero=True)
    want = (tk["alpha"][0][:, None, None] * st).astype(np.float32)  # one fp32 product per element
    assert np.array_equal(got_S, want)
    assert np.array_equal(ref_S, want)


def test_deterministic_and_in_place(F):
    heads, dk, dv = 64, 128, 128
    st = S.delta_state(45, 0, heads, dv, dk)
    tk = {n: torch.from_numpy(a).to(dev()) for n, a in S.delta_tokens(45, 0, 0, 2, heads, dk, dv).items()}
    outs = []
    for _ in range(2):
        sd = torch.from_numpy(st).to(dev())
        ptr = sd.data_ptr()
        o = F.delta_update(sd, tk["q"], tk["k"], tk["v"], tk["alpha"], tk["beta"])
        assert sd.data_ptr() == ptr
        outs.append((sd.clone(), o.clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_rejects_bad_arguments(F):
    sd = torch.zeros(2, 4, 128, device=dev())
    tk = {n: torch.from_numpy(a).to(dev()) for n, a in S.delta_tokens(46, 0, 0, 1, 2, 128, 4).items()}
    with pytest.raises(F.FmoeError):  # the readout may not alias the state
        F.delta_update(sd, tk["q"], tk["k"], tk["v"], tk["alpha"], tk["beta"], o=sd.view(-1)[:8].view(1, 2, 4))
    with pytest.raises(ValueError):
        F.delta_update(sd, tk["q"], tk["k"], tk["v"][:, :1], tk["alpha"], tk["beta"])
