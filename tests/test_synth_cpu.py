"""The host-side synthetic generator: determinism and value distributions."""
import numpy as np

import synth as S


def test_splitmix64_reference_values():
    # SplitMix64 seeded with 0: the first outputs of the published generator.
    out = S.splitmix64_outputs(0, 0, 3)
    assert [int(v) for v in out] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_codes_uniform_and_deterministic():
    a = S.code_words(1, 0, 3, S.MAT_GATE, 64, 512, 4)
    b = S.code_words(1, 0, 3, S.MAT_GATE, 64, 512, 4)
    c = S.code_words(1, 0, 4, S.MAT_GATE, 64, 512, 4)
    assert a.shape == (64, 64) and np.array_equal(a, b) and not np.array_equal(a, c)
    nib = ((a[..., None] >> (np.arange(8, dtype=np.uint32) * 4)) & 15).ravel()
    counts = np.bincount(nib, minlength=16)
    assert counts.min() > 0.8 * nib.size / 16 and counts.max() < 1.2 * nib.size / 16


def test_scale_bias_distribution():
    for bits, m in ((4, 8.0), (2, 1.5)):
        sb = S.sb_words(5, 2, 7, S.MAT_DOWN, 256, 1024, bits)
        s = S.bf16_bits_to_f32(sb & 0xFFFF).astype(np.float64)
        b = S.bf16_bits_to_f32(sb >> 16).astype(np.float64)
        assert s.min() >= 1e-3 * (1 - 2**-8) and s.max() <= 4e-3 * (1 + 2**-8)
        ratio = -b / (m * s)
        assert ratio.min() >= 0.9 * (1 - 2**-7) and ratio.max() <= 1.1 * (1 + 2**-7)
        assert abs(ratio.mean() - 1.0) < 0.01


def test_router_and_tokens():
    w = S.router_bf16(3, 0, 16, 512)
    f = S.bf16_bits_to_f32(w).astype(np.float64)
    assert w.shape == (16, 512) and abs(f.std() - 0.02) < 0.002
    x = S.token_x(3, 0, 0, 2, 512)
    assert x.dtype == np.float32 and x.shape == (2, 512) and abs(x.std() - 1) < 0.1
    assert not np.array_equal(S.token_x(3, 0, 0, 1, 512, redraw=1), x[:1])


def test_delta_inputs_seeded_and_shaped():
    """The delta-rule inputs: deterministic per (seed, layer, step), the stated
    shapes and distributions (unit keys, gates in their ranges)."""
    a = S.delta_tokens(7, 2, 3, 4, 5, 128, 96)
    b = S.delta_tokens(7, 2, 3, 4, 5, 128, 96)
    c = S.delta_tokens(7, 2, 4, 4, 5, 128, 96)
    for n in a:
        assert a[n].dtype == np.float32 and np.array_equal(a[n], b[n])
        assert not np.array_equal(a[n], c[n])
    assert a["q"].shape == a["k"].shape == (4, 5, 128) and a["v"].shape == (4, 5, 96)
    assert a["alpha"].shape == a["beta"].shape == (4, 5)
    np.testing.assert_allclose(np.linalg.norm(a["k"].astype(np.float64), axis=-1), 1.0, rtol=1e-6)
    assert (a["alpha"] >= 0.9).all() and (a["alpha"] <= 1.0).all()
    assert (a["beta"] >= 0.0).all() and (a["beta"] <= 1.0).all()
    st = S.delta_state(7, 2, 5, 96, 128)
    assert st.shape == (5, 96, 128) and st.dtype == np.float32
    assert np.array_equal(st, S.delta_state(7, 2, 5, 96, 128))
    assert abs(float(st.std()) - 0.1) < 0.005
