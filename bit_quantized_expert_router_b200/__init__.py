"""Python binding of libfmoe.so (the single-token quantised MoE layer on B200).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  If the
shared library is missing the import of any entry point fails loudly; there is
no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfmoe.so")

FMOE_OK, FMOE_EINVAL, FMOE_ENOMEM, FMOE_ECUDA, FMOE_EDEVICE = range(5)
GROUP = 64
MAX_TOKENS = 16
MAX_TOPK = 8

EXPORTED = [
    "fmoe_expert_bytes", "fmoe_blob_offsets", "fmoe_quantize_expert", "fmoe_route_workspace_bytes",
    "fmoe_route", "fmoe_expert_workspace_bytes", "fmoe_expert_forward", "fmoe_workspace_bytes",
    "fmoe_workspace_init", "fmoe_layer_decode", "fmoe_get_status", "fmoe_strerror", "fmoe_last_cuda_error",
    "fmoe_layer_decode_noalloc", "fmoe_set_wait_limit_ns", "fmoe_set_dependent_launch", "fmoe_delta_update",
    "fmoe_cache_create", "fmoe_cache_destroy", "fmoe_cache_lookup", "fmoe_cache_stats", "fmoe_cache_reset",
    "fmoe_experts_decode", "fmoe_streamer_create", "fmoe_streamer_decode", "fmoe_streamer_stats",
    "fmoe_streamer_destroy", "fmoe_streamer_prepare", "fmoe_streamer_finish",
]


class FmoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        extra = ""
        if code == FMOE_ECUDA:
            extra = f", cudaError {lib().fmoe_last_cuda_error()}"
        super().__init__(f"{what}: {strerror(code)} (code {code}{extra})")


class FmoeLayerC(ctypes.Structure):
    """Mirror of the C struct fmoe_layer."""
    _fields_ = [
        ("w_router", ctypes.c_void_p), ("w_sgate", ctypes.c_void_p), ("experts", ctypes.c_void_p),
        ("expert_stride", ctypes.c_int64), ("shared", ctypes.c_void_p), ("hidden", ctypes.c_int),
        ("inter", ctypes.c_int), ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int),
        ("bits", ctypes.c_int), ("shared_bits", ctypes.c_int), ("group", ctypes.c_int),
        ("norm_weight", ctypes.c_void_p), ("norm_eps", ctypes.c_float),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libfmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                           "`python -m bit_quantized_expert_router_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.fmoe_expert_bytes.argtypes = [i, i, i]
    L.fmoe_expert_bytes.restype = sz
    L.fmoe_blob_offsets.argtypes = [i, i, i, ctypes.POINTER(ctypes.c_int64)]
    L.fmoe_quantize_expert.argtypes = [vp, vp, vp, i, i, i, i, vp, sz, vp]
    L.fmoe_route_workspace_bytes.argtypes = [i, i]
    L.fmoe_route_workspace_bytes.restype = sz
    L.fmoe_route.argtypes = [vp, vp, vp, i, i, i, i, vp, vp, vp, vp, vp, sz, vp]
    L.fmoe_expert_workspace_bytes.argtypes = [i, i]
    L.fmoe_expert_workspace_bytes.restype = sz
    L.fmoe_expert_forward.argtypes = [vp, i, i, i, vp, vp, vp, sz, vp]
    L.fmoe_workspace_bytes.argtypes = [ctypes.POINTER(FmoeLayerC), i]
    L.fmoe_workspace_bytes.restype = sz
    L.fmoe_workspace_init.argtypes = [vp, sz, vp]
    L.fmoe_layer_decode.argtypes = [ctypes.POINTER(FmoeLayerC), vp, vp, vp, i, vp, sz, vp, vp, vp]
    L.fmoe_layer_decode_noalloc.argtypes = [ctypes.POINTER(FmoeLayerC), vp, vp, vp, i, vp, vp, vp]
    L.fmoe_experts_decode.argtypes = [ctypes.POINTER(FmoeLayerC), ctypes.POINTER(vp), ctypes.POINTER(ctypes.c_float),
                                      ctypes.c_float, vp, vp, vp, vp, sz, vp]
    L.fmoe_get_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint)]
    L.fmoe_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong, ctypes.POINTER(ctypes.c_ulonglong)]
    L.fmoe_set_dependent_launch.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
    L.fmoe_delta_update.argtypes = [vp] * 7 + [i, i, i, i, vp]
    L.fmoe_cache_create.argtypes = [i, ctypes.POINTER(vp)]
    L.fmoe_cache_destroy.argtypes = [vp]
    L.fmoe_cache_lookup.argtypes = [vp, i, vp, i, vp, vp, ctypes.POINTER(i)]
    u64p = ctypes.POINTER(ctypes.c_uint64)
    L.fmoe_cache_stats.argtypes = [vp, u64p, u64p, u64p]
    L.fmoe_cache_reset.argtypes = [vp]
    L.fmoe_streamer_create.argtypes = [ctypes.POINTER(FmoeLayerC), i, ctypes.POINTER(vp), vp, i, ctypes.POINTER(vp)]
    L.fmoe_streamer_decode.argtypes = [vp, i, vp, vp, vp, vp, sz, vp, vp, vp, vp]
    L.fmoe_streamer_prepare.argtypes = [vp, i, vp, vp, vp, vp, vp]
    L.fmoe_streamer_finish.argtypes = [vp, i, vp, vp, vp, vp, sz, vp]
    L.fmoe_streamer_stats.argtypes = [vp, u64p, u64p, u64p]
    L.fmoe_streamer_destroy.argtypes = [vp]
    L.fmoe_last_cuda_error.argtypes = []
    L.fmoe_last_cuda_error.restype = i
    L.fmoe_strerror.argtypes = [i]
    L.fmoe_strerror.restype = ctypes.c_char_p
    for name in ("fmoe_blob_offsets", "fmoe_quantize_expert", "fmoe_route", "fmoe_expert_forward",
                 "fmoe_workspace_init", "fmoe_layer_decode", "fmoe_get_status", "fmoe_layer_decode_noalloc",
                 "fmoe_experts_decode", "fmoe_streamer_create", "fmoe_streamer_decode", "fmoe_streamer_stats",
                 "fmoe_streamer_destroy", "fmoe_streamer_prepare", "fmoe_streamer_finish"):
        getattr(L, name).restype = i
    _lib = L
    return L


def strerror(code: int) -> str:
    return lib().fmoe_strerror(code).decode()


def _check(rc: int, what: str):
    if rc != FMOE_OK:
        raise FmoeError(rc, what)


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dev_tensor(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


# ---------------------------------------------------------------------------

def expert_bytes(hidden: int, inter: int, bits: int) -> int:
    return int(lib().fmoe_expert_bytes(hidden, inter, bits))


def blob_offsets(hidden: int, inter: int, bits: int) -> list[int]:
    off = (ctypes.c_int64 * 6)()
    _check(lib().fmoe_blob_offsets(hidden, inter, bits, off), "fmoe_blob_offsets")
    return list(off)


def workspace_init(ws: torch.Tensor, stream=None):
    _check(lib().fmoe_workspace_init(ws.data_ptr(), ws.numel() * ws.element_size(), _stream(stream)),
           "fmoe_workspace_init")


def _alloc_ws(nbytes: int, device) -> torch.Tensor:
    return torch.zeros(max(256, (nbytes + 255) // 256 * 256), dtype=torch.uint8, device=device)


def quantize_expert(w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor, bits: int,
                    out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Quantise fp32 (gate [I][H], up [I][H], down [H][I]) into a packed blob (uint8)."""
    for t, n in ((w_gate, "w_gate"), (w_up, "w_up"), (w_down, "w_down")):
        _dev_tensor(t, torch.float32, n)
    inter, hidden = w_gate.shape
    nbytes = expert_bytes(hidden, inter, bits)
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=w_gate.device)
    _check(lib().fmoe_quantize_expert(w_gate.data_ptr(), w_up.data_ptr(), w_down.data_ptr(), hidden, inter,
                                      bits, GROUP, out.data_ptr(), out.numel(), _stream(stream)),
           "fmoe_quantize_expert")
    return out


def route(w_router: torch.Tensor, w_sgate: torch.Tensor | None, x: torch.Tensor, top_k: int,
          want_logits: bool = False, stream=None):
    """Router for T tokens: returns (idx int32 [T][K], w fp32 [T][K], sgate fp32 [T], logits|None)."""
    _dev_tensor(w_router, torch.int16, "w_router")
    if w_sgate is not None:
        _dev_tensor(w_sgate, torch.int16, "w_sgate")
    _dev_tensor(x, torch.float32, "x")
    x2 = x.view(-1, x.shape[-1])
    T, H = x2.shape
    E = w_router.shape[0]
    dev = x.device
    idx = torch.empty(T, top_k, dtype=torch.int32, device=dev)
    w = torch.empty(T, top_k, dtype=torch.float32, device=dev)
    sg = torch.empty(T, dtype=torch.float32, device=dev)
    logits = torch.empty(T, E, dtype=torch.float32, device=dev) if want_logits else None
    nws = int(lib().fmoe_route_workspace_bytes(T, E))
    ws = _alloc_ws(nws, dev)
    _check(lib().fmoe_route(w_router.data_ptr(), _ptr(w_sgate), x2.data_ptr(), T, H, E, top_k, idx.data_ptr(),
                            w.data_ptr(), sg.data_ptr(), _ptr(logits), ws.data_ptr(), ws.numel(),
                            _stream(stream)), "fmoe_route")
    return idx, w, sg, logits


def expert_workspace(hidden: int, inter: int, device) -> torch.Tensor:
    return _alloc_ws(int(lib().fmoe_expert_workspace_bytes(hidden, inter)), device)


def expert_forward(blob: torch.Tensor, hidden: int, inter: int, bits: int, x: torch.Tensor,
                   out: torch.Tensor | None = None, ws: torch.Tensor | None = None, stream=None):
    """One expert for one token: y = Wd (silu(Wg x) * (Wu x))."""
    _dev_tensor(blob, torch.uint8, "blob")
    _dev_tensor(x, torch.float32, "x")
    if out is None:
        out = torch.empty(hidden, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = expert_workspace(hidden, inter, x.device)
    _check(lib().fmoe_expert_forward(blob.data_ptr(), hidden, inter, bits, x.data_ptr(), out.data_ptr(),
                                     ws.data_ptr(), ws.numel(), _stream(stream)), "fmoe_expert_forward")
    return out


@dataclass
class Layer:
    """Device-resident weights of one MoE layer (all tensors on one GPU).

    experts: uint8 [E][stride] packed routed experts; shared: uint8 blob or None;
    w_router: int16 [E][H] bf16 bits; w_sgate: int16 [H] bf16 bits or None;
    norm_weight: int16 [H] bf16 bits or None (input RMS norm with norm_eps).
    """
    w_router: torch.Tensor
    w_sgate: torch.Tensor | None
    experts: torch.Tensor
    shared: torch.Tensor | None
    hidden: int
    inter: int
    top_k: int
    bits: int = 4
    shared_bits: int = 4
    norm_weight: torch.Tensor | None = None
    norm_eps: float = 1e-6

    def __post_init__(self):
        _dev_tensor(self.w_router, torch.int16, "w_router")
        if self.norm_weight is not None:
            _dev_tensor(self.norm_weight, torch.int16, "norm_weight")
        if self.w_sgate is not None:
            _dev_tensor(self.w_sgate, torch.int16, "w_sgate")
        _dev_tensor(self.experts, torch.uint8, "experts")
        if self.shared is not None:
            _dev_tensor(self.shared, torch.uint8, "shared")
        self.n_experts = self.w_router.shape[0]
        self.c = FmoeLayerC(
            w_router=self.w_router.data_ptr(), w_sgate=_ptr(self.w_sgate), experts=self.experts.data_ptr(),
            expert_stride=self.experts.stride(0) if self.experts.dim() == 2 else expert_bytes(
                self.hidden, self.inter, self.bits),
            shared=_ptr(self.shared), hidden=self.hidden, inter=self.inter, n_experts=self.n_experts,
            top_k=self.top_k, bits=self.bits, shared_bits=self.shared_bits, group=GROUP,
            norm_weight=_ptr(self.norm_weight), norm_eps=float(self.norm_eps))
        self._ws = None

    def workspace_bytes(self, T: int = 1) -> int:
        return int(lib().fmoe_workspace_bytes(ctypes.byref(self.c), T))

    def workspace(self, T: int = 1) -> torch.Tensor:
        if self._ws is None or self._ws.numel() < self.workspace_bytes(T):
            self._ws = _alloc_ws(self.workspace_bytes(T), self.experts.device)
        return self._ws

    def decode(self, x: torch.Tensor, residual: torch.Tensor | None = None, out: torch.Tensor | None = None,
               idx_out: torch.Tensor | None = None, w_out: torch.Tensor | None = None,
               ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """out[t] = residual[t] + sum_k w[t,k] E_idx(x[t]) + sgate[t] E_shared(x[t]), T = x rows."""
        _dev_tensor(x, torch.float32, "x")
        x2 = x.view(-1, self.hidden)
        T = x2.shape[0]
        if residual is not None:
            _dev_tensor(residual, torch.float32, "residual")
        if out is None:
            out = torch.empty_like(x2)
        if ws is None:
            ws = self.workspace(T)
        _check(lib().fmoe_layer_decode(ctypes.byref(self.c), x2.data_ptr(), _ptr(residual), out.data_ptr(), T,
                                       ws.data_ptr(), ws.numel(), _ptr(idx_out), _ptr(w_out), _stream(stream)),
               "fmoe_layer_decode")
        return out


def experts_decode(layer: "Layer", blobs, weights, shared_gate: float, x: torch.Tensor,
                   residual: torch.Tensor | None = None, out: torch.Tensor | None = None,
                   ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The layer's expert path for one token with the routing given: blobs are
    the top_k routed experts' device addresses (ints or uint8 tensors, e.g.
    expert-cache slots), weights their combine weights, shared_gate the
    shared expert's factor.  out = residual + sum_k w_k E_k(x) + g E_shared(x)."""
    _dev_tensor(x, torch.float32, "x")
    x1 = x.view(layer.hidden)
    if residual is not None:
        _dev_tensor(residual, torch.float32, "residual")
    if out is None:
        out = torch.empty_like(x1)
    if ws is None:
        ws = layer.workspace(1)
    K = layer.top_k
    ptrs = [b if isinstance(b, int) else b.data_ptr() for b in blobs]
    if len(ptrs) != K or len(weights) != K:
        raise ValueError(f"experts_decode: need {K} blobs and weights")
    pa = (ctypes.c_void_p * K)(*ptrs)
    wa = (ctypes.c_float * K)(*[float(w) for w in weights])
    _check(lib().fmoe_experts_decode(ctypes.byref(layer.c), pa, wa, ctypes.c_float(float(shared_gate)),
                                     x1.data_ptr(), _ptr(residual), out.data_ptr(), ws.data_ptr(), ws.numel(),
                                     _stream(stream)), "fmoe_experts_decode")
    return out


def layer_decode_noalloc(layer: "Layer", x: torch.Tensor, residual: torch.Tensor | None = None,
                         out: torch.Tensor | None = None, idx_out: torch.Tensor | None = None,
                         w_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Layer.decode without a workspace argument: the library's fixed device
    scratch is used instead (see fmoe_layer_decode_noalloc in include/fmoe.h)."""
    _dev_tensor(x, torch.float32, "x")
    x2 = x.view(-1, layer.hidden)
    if out is None:
        out = torch.empty_like(x2)
    _check(lib().fmoe_layer_decode_noalloc(ctypes.byref(layer.c), x2.data_ptr(), _ptr(residual), out.data_ptr(),
                                           x2.shape[0], _ptr(idx_out), _ptr(w_out), _stream(stream)),
           "fmoe_layer_decode_noalloc")
    return out


def set_wait_limit_ns(limit_ns: int) -> int:
    """Set the time limit of the kernels' device-side waits; returns the previous limit."""
    prev = ctypes.c_ulonglong(0)
    rc = lib().fmoe_set_wait_limit_ns(ctypes.c_ulonglong(int(limit_ns)), ctypes.byref(prev))
    if rc != FMOE_OK:
        raise FmoeError(rc, "fmoe_set_wait_limit_ns")
    return int(prev.value)


def delta_update(state: torch.Tensor, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor,
                 beta: torch.Tensor, o: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Gated delta-rule update of `state` [heads][dv][dk] (in place) for the T
    tokens of q, k [T][heads][dk], v [T][heads][dv], alpha, beta [T][heads];
    returns the readouts o [T][heads][dv] (all fp32, on one GPU)."""
    for name, t in (("state", state), ("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta)):
        _dev_tensor(t, torch.float32, name)
    heads, dv, dk = state.shape
    T = alpha.shape[0]
    if q.shape != (T, heads, dk) or k.shape != (T, heads, dk) or v.shape != (T, heads, dv) or \
            alpha.shape != (T, heads) or beta.shape != (T, heads):
        raise ValueError("delta_update: inconsistent shapes")
    if o is None:
        o = torch.empty(T, heads, dv, dtype=torch.float32, device=state.device)
    _dev_tensor(o, torch.float32, "o")
    _check(lib().fmoe_delta_update(state.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(), alpha.data_ptr(),
                                   beta.data_ptr(), o.data_ptr(), heads, dk, dv, T, _stream(stream)),
           "fmoe_delta_update")
    return o


class ExpertCache:
    """Host directory of a device expert cache of n_slots slots (see
    fmoe_cache_lookup in include/fmoe.h): which selected experts are in a
    slot and which slot each miss goes to (least recently used)."""

    def __init__(self, n_slots: int):
        h = ctypes.c_void_p()
        _check(lib().fmoe_cache_create(int(n_slots), ctypes.byref(h)), "fmoe_cache_create")
        self._h = h
        self.n_slots = int(n_slots)

    def lookup(self, layer: int, idx) -> tuple[np.ndarray, np.ndarray]:
        """(slots, misses) for the experts idx selected in `layer`."""
        idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(-1))
        slot = np.empty_like(idx)
        miss = np.empty_like(idx)
        n = ctypes.c_int(0)
        _check(lib().fmoe_cache_lookup(self._h, int(layer), idx.ctypes.data, idx.size, slot.ctypes.data,
                                       miss.ctypes.data, ctypes.byref(n)), "fmoe_cache_lookup")
        return slot, miss

    def stats(self) -> dict:
        v = [ctypes.c_uint64(0) for _ in range(3)]
        _check(lib().fmoe_cache_stats(self._h, *(ctypes.byref(x) for x in v)), "fmoe_cache_stats")
        return {"hits": v[0].value, "misses": v[1].value, "evictions": v[2].value}

    def reset(self) -> None:
        _check(lib().fmoe_cache_reset(self._h), "fmoe_cache_reset")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.fmoe_cache_destroy(h)
            self._h = None


class Streamer:
    """Routed experts streamed from page-locked host memory into n_slots device
    slots (see fmoe_streamer_create in include/fmoe.h).  `layers`: Layer
    objects of one shape (their `experts` tables are not used); `host_experts`:
    per layer a pinned CPU uint8 tensor [n_experts, expert_stride]; `slots`: a
    CUDA uint8 tensor [n_slots, expert_stride]."""

    def __init__(self, layers, host_experts, slots: torch.Tensor):
        if len(layers) != len(host_experts) or not layers:
            raise ValueError("one host expert table per layer")
        for h in host_experts:
            if not isinstance(h, torch.Tensor) or h.is_cuda or not h.is_pinned() or h.dtype != torch.uint8:
                raise ValueError("host_experts must be pinned CPU uint8 tensors")
        _dev_tensor(slots, torch.uint8, "slots")
        self.layers = list(layers)
        self._keep = (list(host_experts), slots)
        arr = (FmoeLayerC * len(layers))(*[L.c for L in layers])
        hp = (ctypes.c_void_p * len(layers))(*[h.data_ptr() for h in host_experts])
        h = ctypes.c_void_p()
        _check(lib().fmoe_streamer_create(arr, len(layers), hp, slots.data_ptr(), slots.shape[0], ctypes.byref(h)),
               "fmoe_streamer_create")
        self._h = h

    def decode(self, layer: int, x: torch.Tensor, residual: torch.Tensor | None = None,
               out: torch.Tensor | None = None, ws: torch.Tensor | None = None, stream=None, copy_stream=None,
               return_routing: bool = False):
        L = self.layers[layer]
        x = _dev_tensor(x, torch.float32, "x")
        if out is None:
            out = torch.empty_like(x)
        if ws is None:
            ws = L.workspace(1)
        K = L.top_k
        idx = np.empty(K, dtype=np.int32)
        w = np.empty(K, dtype=np.float32)
        cs = _stream(stream)
        ks = cs if copy_stream is None else copy_stream.cuda_stream
        _check(lib().fmoe_streamer_decode(self._h, int(layer), x.data_ptr(), _ptr(residual), out.data_ptr(),
                                          ws.data_ptr(), ws.numel(), cs, ks, idx.ctypes.data, w.ctypes.data),
               "fmoe_streamer_decode")
        return (out, idx, w) if return_routing else out

    def prepare(self, layer: int, x: torch.Tensor, route_stream=None, copy_stream=None):
        """Route x for `layer` and start its misses' copies; returns the
        routing decision (host arrays idx, w)."""
        L = self.layers[layer]
        x = _dev_tensor(x, torch.float32, "x")
        idx = np.empty(L.top_k, dtype=np.int32)
        w = np.empty(L.top_k, dtype=np.float32)
        rs = _stream(route_stream)
        ks = rs if copy_stream is None else copy_stream.cuda_stream
        _check(lib().fmoe_streamer_prepare(self._h, int(layer), x.data_ptr(), rs, ks, idx.ctypes.data, w.ctypes.data),
               "fmoe_streamer_prepare")
        return idx, w

    def finish(self, layer: int, x: torch.Tensor, residual: torch.Tensor | None = None,
               out: torch.Tensor | None = None, ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """Decode the oldest prepared layer (`layer`, with the same x)."""
        L = self.layers[layer]
        x = _dev_tensor(x, torch.float32, "x")
        if out is None:
            out = torch.empty_like(x)
        if ws is None:
            ws = L.workspace(1)
        _check(lib().fmoe_streamer_finish(self._h, int(layer), x.data_ptr(), _ptr(residual), out.data_ptr(),
                                          ws.data_ptr(), ws.numel(), _stream(stream)), "fmoe_streamer_finish")
        return out

    def stats(self) -> dict:
        v = [ctypes.c_uint64(0) for _ in range(3)]
        _check(lib().fmoe_streamer_stats(self._h, *(ctypes.byref(x) for x in v)), "fmoe_streamer_stats")
        return {"hits": v[0].value, "misses": v[1].value, "h2d_bytes": v[2].value}

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.fmoe_streamer_destroy(h)
            self._h = None


def set_dependent_launch(enable: bool) -> bool:
    """Launch the single-token layer kernel as a programmatic dependent launch
    (True, the default: it overlaps the previous kernel's end) or as a
    cooperative launch (False); the grouped decode's kernels follow the same
    switch (dependent or plain launches).  Returns the previous setting."""
    prev = ctypes.c_int(0)
    rc = lib().fmoe_set_dependent_launch(1 if enable else 0, ctypes.byref(prev))
    if rc != FMOE_OK:
        raise FmoeError(rc, "fmoe_set_dependent_launch")
    return bool(prev.value)


def get_status(stream=None) -> int:
    """Synchronise the stream, read and clear the device status word (0 = clean)."""
    bits = ctypes.c_uint(0)
    rc = lib().fmoe_get_status(_stream(stream), ctypes.byref(bits))
    if rc not in (FMOE_OK, FMOE_EDEVICE):
        raise FmoeError(rc, "fmoe_get_status")
    return int(bits.value)
