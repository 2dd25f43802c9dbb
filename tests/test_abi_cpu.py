"""The C-ABI library on a machine without a GPU: it builds, loads, exports every
declared entry point, and rejects invalid arguments on the host."""
import ctypes
import os
import re
import subprocess

import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def F():
    from bit_quantized_expert_router_b200 import build as B
    B.build_engine()
    import bit_quantized_expert_router_b200 as F
    F.lib()
    return F


def declared_functions():
    src = open(os.path.join(ROOT, "include", "fmoe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fmoe_[a-z_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("fmoe_quantize_expert", "fmoe_route", "fmoe_expert_forward", "fmoe_layer_decode"):
        assert n in names


def test_every_declared_symbol_is_exported(F):
    out = subprocess.run(["nm", "-D", "--defined-only", F.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (fmoe_[a-z_]+)\b", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(F.lib(), n)
    assert sorted(F.EXPORTED) == declared_functions()


def test_layout_agrees_with_oracle(F):
    for (h, i) in ((4096, 1024), (512, 128), (320, 192), (64, 64)):
        for bits in (2, 4):
            assert F.expert_bytes(h, i, bits) == O.expert_bytes(h, i, bits)
            lay = O.blob_layout(h, i, bits)
            assert F.blob_offsets(h, i, bits) == [lay["gate"][0], lay["gate"][1], lay["up"][0], lay["up"][1],
                                                  lay["down"][0], lay["down"][1]]
    assert F.expert_bytes(4096, 1024, 4) == 7_077_888


def test_invalid_arguments_rejected_on_host(F):
    L = F.lib()
    assert L.fmoe_expert_bytes(4096, 1024, 3) == 0
    assert L.fmoe_expert_bytes(100, 1024, 4) == 0
    assert L.fmoe_expert_bytes(4096, 0, 4) == 0
    off = (ctypes.c_int64 * 6)()
    assert L.fmoe_blob_offsets(4096, 1024, 8, off) == F.FMOE_EINVAL
    # null pointers
    assert L.fmoe_expert_forward(None, 4096, 1024, 4, None, None, None, 0, None) == F.FMOE_EINVAL
    assert L.fmoe_layer_decode(None, None, None, None, 1, None, 0, None, None, None) == F.FMOE_EINVAL
    assert L.fmoe_route(None, None, None, 1, 4096, 512, 4, None, None, None, None, None, 0, None) == F.FMOE_EINVAL
    assert L.fmoe_quantize_expert(None, None, None, 4096, 1024, 4, 64, None, 0, None) == F.FMOE_EINVAL
    fake = 1 << 20  # aligned non-null stand-ins; validation fails before any use
    base = dict(w_router=fake, w_sgate=fake, experts=fake, expert_stride=7077888 + 256 - 7077888 % 256,
                shared=fake, hidden=4096, inter=1024, n_experts=512, top_k=4, bits=4, shared_bits=4, group=64)

    def decode(T=1, ws_bytes=1 << 20, x=fake, out=fake * 2, **kw):
        c = F.FmoeLayerC(**{**base, **kw})
        return L.fmoe_layer_decode(ctypes.byref(c), x, None, out, T, fake, ws_bytes, None, None, None)

    assert decode(bits=3) == F.FMOE_EINVAL
    assert decode(shared_bits=8) == F.FMOE_EINVAL
    assert decode(group=32) == F.FMOE_EINVAL
    assert decode(hidden=4000) == F.FMOE_EINVAL
    assert decode(inter=100) == F.FMOE_EINVAL
    assert decode(top_k=9) == F.FMOE_EINVAL
    assert decode(top_k=0) == F.FMOE_EINVAL
    assert decode(n_experts=3, top_k=4) == F.FMOE_EINVAL
    assert decode(n_experts=2048) == F.FMOE_EINVAL
    assert decode(T=0) == F.FMOE_EINVAL
    assert decode(T=17) == F.FMOE_EINVAL
    assert decode(expert_stride=1000) == F.FMOE_EINVAL
    assert decode(expert_stride=7077888 + 16) == F.FMOE_EINVAL  # not a multiple of 256
    assert decode(experts=fake + 16) == F.FMOE_EINVAL  # blobs must be 256-byte aligned
    assert decode(x=fake + 4) == F.FMOE_EINVAL
    assert decode(x=fake, out=fake) == F.FMOE_EINVAL  # out may not alias x
    assert decode(ws_bytes=16) == F.FMOE_ENOMEM
    assert decode(inter=4096) == F.FMOE_EINVAL  # (K+1)*I above the staging limit
    c = F.FmoeLayerC(**base)
    # workspace header: 256 B of counters, then the tagged router logits sized
    # for the most experts (1025 words of 8 B, rounded to 256): 8448 B; then
    # the tagged activations sized for the largest (K+1)*I (10240 words of
    # 8 B): 81920 B.  A single-token decode uses the header alone.
    header = 256 + (1025 * 8 + 255) // 256 * 256 + 10240 * 8
    assert header == 90624
    assert L.fmoe_workspace_bytes(ctypes.byref(c), 1) == header
    assert L.fmoe_expert_workspace_bytes(4096, 1024) == header
    # a grouped workspace serves single-token calls of the layer too
    assert L.fmoe_workspace_bytes(ctypes.byref(c), 16) > L.fmoe_workspace_bytes(ctypes.byref(c), 1)
    small = F.FmoeLayerC(**{**base, "n_experts": 16, "inter": 128})
    assert L.fmoe_workspace_bytes(ctypes.byref(small), 1) == header  # independent of the layer's shape
    # the given-routing entry point checks its arguments on the host too
    blobs = (ctypes.c_void_p * 4)(fake, fake, fake, fake)
    wts = (ctypes.c_float * 4)(0.25, 0.25, 0.25, 0.25)
    assert L.fmoe_experts_decode(ctypes.byref(c), None, wts, 1.0, fake, None, fake * 2, fake, 1 << 20, None) \
        == F.FMOE_EINVAL
    bad = (ctypes.c_void_p * 4)(fake, fake + 16, fake, fake)  # a blob off the 256-byte grid
    assert L.fmoe_experts_decode(ctypes.byref(c), bad, wts, 1.0, fake, None, fake * 2, fake, 1 << 20, None) \
        == F.FMOE_EINVAL
    assert L.fmoe_experts_decode(ctypes.byref(c), blobs, wts, 1.0, fake, None, fake * 2, fake, 16, None) \
        == F.FMOE_ENOMEM
    # the allocation-free entry point serves single tokens only
    assert L.fmoe_layer_decode_noalloc(ctypes.byref(c), fake, None, fake * 2, 2, None, None, None) == F.FMOE_EINVAL
    assert L.fmoe_workspace_bytes(ctypes.byref(c), 0) == 0
    assert L.fmoe_route_workspace_bytes(17, 512) == 0
    # the expert streamer checks its layers on the host before any CUDA call
    def streamer(layers, hosts=None, slots=fake, n_slots=8):
        arr = (F.FmoeLayerC * len(layers))(*layers)
        hp = (ctypes.c_void_p * len(layers))(*(hosts or [fake] * len(layers)))
        h = ctypes.c_void_p(123)
        rc = L.fmoe_streamer_create(arr, len(layers), hp, slots, n_slots, ctypes.byref(h))
        assert not h.value  # nothing is created on an error
        return rc
    assert streamer([c], n_slots=3) == F.FMOE_EINVAL  # fewer slots than top_k
    assert streamer([c], slots=fake + 16) == F.FMOE_EINVAL  # slots off the 256-byte grid
    assert streamer([c], hosts=[fake + 8]) == F.FMOE_EINVAL  # host blobs off the grid
    assert streamer([F.FmoeLayerC(**{**base, "norm_weight": fake})]) == F.FMOE_EINVAL  # routing reads x as given
    assert streamer([c, F.FmoeLayerC(**{**base, "inter": 512})]) == F.FMOE_EINVAL  # layers of different shapes
    assert streamer([F.FmoeLayerC(**{**base, "expert_stride": 1000})]) == F.FMOE_EINVAL
    assert L.fmoe_streamer_decode(None, 0, fake, None, fake * 2, fake, 1 << 20, None, None, None, None) \
        == F.FMOE_EINVAL
    assert L.fmoe_streamer_destroy(None) == F.FMOE_OK
    # delta-rule update: shapes, alignment and overlap are checked on the host.
    # The defaults are disjoint stand-ins (the 64 x 128 x 128 state spans 4 MiB
    # from 1 MiB; every other buffer lies beyond it); only variants with one
    # fault each are called, so no call gets past validation.
    MiB = 1 << 20

    def delta(state=MiB, q=8 * MiB, k=9 * MiB, v=10 * MiB, alpha=11 * MiB, beta=12 * MiB, o=13 * MiB,
              heads=64, dk=128, dv=128, T=1):
        return L.fmoe_delta_update(state, q, k, v, alpha, beta, o, heads, dk, dv, T, None)

    for kw in (dict(state=None), dict(o=None), dict(alpha=None),
               dict(dk=64), dict(dk=640), dict(dk=200), dict(heads=0), dict(dv=0), dict(T=0),
               dict(heads=65537), dict(state=MiB + 8), dict(q=8 * MiB + 4), dict(v=10 * MiB + 2),
               dict(o=MiB + 4096),           # readout inside the state
               dict(q=MiB + 1024),           # an input inside the state
               dict(o=10 * MiB + 256)):      # readout overlapping v
        assert delta(**kw) == F.FMOE_EINVAL, kw
    # launch-mode switch: only 0 and 1, nothing changes otherwise
    prev = ctypes.c_int(-1)
    assert L.fmoe_set_dependent_launch(2, ctypes.byref(prev)) == F.FMOE_EINVAL and prev.value == -1
    assert L.fmoe_set_dependent_launch(0, ctypes.byref(prev)) == F.FMOE_OK and prev.value == 1
    assert L.fmoe_set_dependent_launch(1, ctypes.byref(prev)) == F.FMOE_OK and prev.value == 0
    for code in range(5):
        assert len(F.strerror(code)) >= 2 and F.strerror(code) != F.strerror(99)
