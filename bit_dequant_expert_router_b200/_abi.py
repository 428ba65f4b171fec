"""ctypes binding of libfmoe.so (include/fmoe.h, fmoe_gdn.h, fmoe_cache.h): argument marshalling only.

Every function takes torch tensors that already live on the GPU, passes their
device pointers and the current torch stream to the C ABI, and raises
FmoeError on a non-OK status.  No step of the block runs in Python; if the
shared library is missing the import of a function fails loudly.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
SO_PATH = os.path.join(_HERE, "libfmoe.so")

FMOE_OK = 0
STATUS_NAMES = {0: "FMOE_OK", 1: "FMOE_ERR_INVALID_ARG", 2: "FMOE_ERR_ALIGNMENT", 3: "FMOE_ERR_UNSUPPORTED",
                4: "FMOE_ERR_WORKSPACE", 5: "FMOE_ERR_CUDA", 6: "FMOE_ERR_DEVICE_TIMEOUT", 7: "FMOE_ERR_DEVICE_BOUNDS"}


class FmoeError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class FmoeBank(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("group_size", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("inter", ctypes.c_int32), ("num_experts", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("base", ctypes.c_void_p), ("stride", ctypes.c_int64), ("off", ctypes.c_int64 * 9)]


class FmoeLayer(ctypes.Structure):
    _fields_ = [("routed", FmoeBank), ("shared", FmoeBank), ("w_router", ctypes.c_void_p),
                ("router_bias", ctypes.c_void_p), ("w_shared_gate", ctypes.c_void_p), ("gamma", ctypes.c_void_p),
                ("eps", ctypes.c_float), ("top_k", ctypes.c_int32)]


class FmoeExpertCache(ctypes.Structure):
    _fields_ = [("host_base", ctypes.c_void_p), ("host_stride", ctypes.c_int64), ("slots", ctypes.c_void_p),
                ("slot_stride", ctypes.c_int64), ("record_bytes", ctypes.c_int64), ("num_experts", ctypes.c_int32),
                ("num_slots", ctypes.c_int32), ("state", ctypes.c_void_p)]


_lib = None

# (name, restype, argtypes) of every entry point declared in include/fmoe.h
_vp, _i, _sz, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
SIGNATURES = [
    ("fmoe_bank_layout", _i, [_i, _i, _i, _i, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64)]),
    ("fmoe_rmsnorm", _i, [_vp, _vp, _f, _i, _i, _vp, _vp]),
    ("fmoe_router_topk", _i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    ("fmoe_router_topk_workspace_size", _sz, [_i, _i]),
    ("fmoe_expert_ffn", _i, [ctypes.POINTER(FmoeBank), _i, _vp, _vp, _vp, _sz, _vp]),
    ("fmoe_expert_ffn_workspace_size", _sz, [ctypes.POINTER(FmoeBank)]),
    ("fmoe_moe_layer", _i, [ctypes.POINTER(FmoeLayer), _vp, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    ("fmoe_moe_layer_workspace_size", _sz, [ctypes.POINTER(FmoeLayer), _i]),
    ("fmoe_moe_layer_static", _i, [ctypes.POINTER(FmoeLayer), _vp, _i, _vp, _vp, _vp, _vp, _vp]),
    ("fmoe_moe_layer_routed", _i, [ctypes.POINTER(FmoeLayer), _vp, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    ("fmoe_wait_flag", _i, [_vp, ctypes.c_uint32, ctypes.c_int64, _vp, _vp]),
    ("fmoe_gdn_step", _i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, ctypes.c_uint32, _vp]),
    ("fmoe_expert_cache_state_size", _sz, [_i, _i]),
    ("fmoe_expert_cache_reset", _i, [ctypes.POINTER(FmoeExpertCache), _vp]),
    ("fmoe_expert_cache_fetch", _i, [ctypes.POINTER(FmoeExpertCache), _vp, _i, _vp, _vp]),
    ("fmoe_expert_cache_stats", _i, [ctypes.POINTER(FmoeExpertCache), ctypes.POINTER(ctypes.c_int64),
                                     ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64), _vp]),
    ("fmoe_moe_layer_cached", _i, [ctypes.POINTER(FmoeLayer), ctypes.POINTER(FmoeExpertCache), _vp, _i, _vp, _vp, _vp,
                                   _vp, _sz, _vp]),
    ("fmoe_moe_stack", _i, [ctypes.POINTER(FmoeLayer), _i, _vp, _i, _vp, _vp, _sz, _vp]),
    ("fmoe_trace_next_layer", _i, [ctypes.POINTER(ctypes.c_void_p), _i]),
    ("fmoe_workspace_init", _i, [_vp, _sz, _vp]),
    ("fmoe_workspace_check", _i, [_vp, _vp]),
    ("fmoe_last_error", ctypes.c_char_p, []),
    ("fmoe_status_string", ctypes.c_char_p, [_i]),
    ("fmoe_version", _i, []),
    ("fmoe_debug_bounds", _i, []),
]


def lib():
    """Loads libfmoe.so (built in-tree by build.py; FMOE_SO may name its debug build,
    libfmoe_debug.so, instead); raises if it is missing."""
    global _lib
    if _lib is None:
        so = os.environ.get("FMOE_SO") or SO_PATH
        if not os.path.exists(so):
            raise RuntimeError(f"{so} is missing: build it with `python -m bit_dequant_expert_router_b200.build` "
                               "(there is no fallback implementation)")
        L = ctypes.CDLL(so)
        for name, res, args in SIGNATURES:
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status):
    if status != FMOE_OK:
        raise FmoeError(status, lib().fmoe_last_error().decode())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t, dtype=None, what="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def bank_layout(bits, hidden, inter, group_size=64):
    """Canonical record layout: (record_bytes, [9 offsets])."""
    nb = ctypes.c_int64()
    off = (ctypes.c_int64 * 9)()
    _check(lib().fmoe_bank_layout(bits, group_size, hidden, inter, ctypes.byref(nb), off))
    return nb.value, list(off)


class Bank:
    """A bank of expert records held in one device tensor (uint8)."""

    def __init__(self, storage, bits, hidden, inter, num_experts, stride, off, group_size=64):
        self.storage = storage   # None: the records live elsewhere (an expert cache's host store)
        base = None if storage is None else _ptr(storage, torch.uint8, "bank storage").value
        self.s = FmoeBank(bits, group_size, hidden, inter, num_experts, 0, base, stride, (ctypes.c_int64 * 9)(*off))


class Layer:
    """One MoE layer: routed and shared banks, router (bf16 bits as int16/uint16), shared gate, gamma, bias."""

    def __init__(self, routed, shared, w_router, w_shared_gate, gamma=None, router_bias=None, eps=1e-6, top_k=4):
        self.routed, self.shared = routed, shared
        self.tensors = (w_router, w_shared_gate, gamma, router_bias)
        self.s = FmoeLayer(routed.s, shared.s, _ptr(w_router, None, "w_router"), _ptr(router_bias, torch.float32,
                           "router_bias"), _ptr(w_shared_gate, None, "w_shared_gate"), _ptr(gamma, torch.float32, "gamma"),
                           eps, top_k)

    @property
    def hidden(self):
        return self.s.routed.hidden

    @property
    def top_k(self):
        return self.s.top_k


def trace_next_layer(events):
    """Makes the next moe_layer call record 4 torch.cuda.Events around its kernels (None cancels)."""
    if events is None:
        _check(lib().fmoe_trace_next_layer(None, 0))
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(lib().fmoe_trace_next_layer(arr, len(events)))


def workspace(nbytes, device=None, stream=None):
    """Allocates a zero-initialised workspace tensor of `nbytes` (torch allocations are 512-byte aligned)."""
    ws = torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device or "cuda")
    workspace_init(ws, stream)
    return ws


def workspace_init(ws, stream=None):
    _check(lib().fmoe_workspace_init(_ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def workspace_check(ws, stream=None):
    _check(lib().fmoe_workspace_check(_ptr(ws, torch.uint8, "ws"), _stream(stream)))


def rmsnorm(h, gamma, eps, out=None, stream=None):
    T, H = h.shape
    out = torch.empty_like(h) if out is None else out
    _check(lib().fmoe_rmsnorm(_ptr(h, torch.float32, "h"), _ptr(gamma, torch.float32, "gamma"), eps, T, H,
                              _ptr(out, torch.float32, "out"), _stream(stream)))
    return out


def router_topk_workspace_size(T, E):
    return lib().fmoe_router_topk_workspace_size(T, E)


def router_topk(x, w_router, top_k, logit_bias=None, idx=None, w=None, probs=None, ws=None, stream=None):
    T, H = x.shape
    E = w_router.shape[0]
    idx = torch.empty((T, top_k), dtype=torch.int32, device=x.device) if idx is None else idx
    w = torch.empty((T, top_k), dtype=torch.float32, device=x.device) if w is None else w
    if ws is None:
        ws = workspace(router_topk_workspace_size(T, E), x.device, stream)
    _check(lib().fmoe_router_topk(_ptr(x, torch.float32, "x"), _ptr(w_router, None, "w_router"),
                                  _ptr(logit_bias, torch.float32, "logit_bias"), T, H, E, top_k,
                                  _ptr(idx, torch.int32, "idx"), _ptr(w, torch.float32, "w"),
                                  _ptr(probs, torch.float32, "probs"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
                                  _stream(stream)))
    return idx, w


def expert_ffn_workspace_size(bank):
    return lib().fmoe_expert_ffn_workspace_size(ctypes.byref(bank.s))


def expert_ffn(bank, expert, x, y=None, ws=None, stream=None):
    y = torch.empty_like(x) if y is None else y
    if ws is None:
        ws = workspace(expert_ffn_workspace_size(bank), x.device, stream)
    _check(lib().fmoe_expert_ffn(ctypes.byref(bank.s), expert, _ptr(x, torch.float32, "x"),
                                 _ptr(y, torch.float32, "y"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
                                 _stream(stream)))
    return y


def moe_layer_workspace_size(layer, T=1):
    return lib().fmoe_moe_layer_workspace_size(ctypes.byref(layer.s), T)


def moe_layer(layer, h, out=None, topk_idx=None, topk_w=None, ws=None, stream=None):
    T = h.shape[0] if h.dim() == 2 else 1
    out = torch.empty_like(h) if out is None else out
    if ws is None:
        ws = workspace(moe_layer_workspace_size(layer, T), h.device, stream)
    _check(lib().fmoe_moe_layer(ctypes.byref(layer.s), _ptr(h, torch.float32, "h"), T,
                                _ptr(out, torch.float32, "out"), _ptr(topk_idx, torch.int32, "topk_idx"),
                                _ptr(topk_w, torch.float32, "topk_w"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
                                _stream(stream)))
    return out


def moe_layer_static(layer, h, out=None, topk_idx=None, topk_w=None, dev_err=None, stream=None):
    """fmoe_moe_layer on the library's static scratch (no workspace argument)."""
    T = h.shape[0] if h.dim() == 2 else 1
    out = torch.empty_like(h) if out is None else out
    _check(lib().fmoe_moe_layer_static(ctypes.byref(layer.s), _ptr(h, torch.float32, "h"), T,
                                       _ptr(out, torch.float32, "out"), _ptr(topk_idx, torch.int32, "topk_idx"),
                                       _ptr(topk_w, torch.float32, "topk_w"), _ptr(dev_err, torch.int32, "dev_err"),
                                       _stream(stream)))
    return out


def moe_layer_routed(layer, h, topk_idx, topk_w, out=None, ws=None, stream=None):
    """The block with the caller's routing (int32 [T][K] experts, fp32 [T][K] weights)."""
    T = h.shape[0] if h.dim() == 2 else 1
    out = torch.empty_like(h) if out is None else out
    if ws is None:
        ws = workspace(moe_layer_workspace_size(layer, 1), h.device, stream)
    _check(lib().fmoe_moe_layer_routed(ctypes.byref(layer.s), _ptr(h, torch.float32, "h"), T,
                                       _ptr(topk_idx, torch.int32, "topk_idx"), _ptr(topk_w, torch.float32, "topk_w"),
                                       _ptr(out, torch.float32, "out"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
                                       _stream(stream)))
    return out


def wait_flag(flag, value, limit_ns, ws, stream=None):
    """Bounded stream-ordered wait until flag (int32/uint32 device tensor of one element) == value."""
    _check(lib().fmoe_wait_flag(_ptr(flag, None, "flag"), int(value), int(limit_ns), _ptr(ws, torch.uint8, "ws"),
                                _stream(stream)))


GDN_STATE_EARLY = 1


def gdn_step(state, q, k, v, alpha, beta, o=None, early=False, stream=None):
    """One Gated DeltaNet decode step of n heads (fmoe_gdn_step): state fp32 [n][dv][dk] is
    updated in place; q, k [n][dk], v [n][dv], alpha, beta [n]; returns o [n][dv].
    early: the previous launch on the stream does not write `state` (FMOE_GDN_STATE_EARLY)."""
    n, dv, dk = state.shape
    o = torch.empty((n, dv), dtype=torch.float32, device=state.device) if o is None else o
    f32 = torch.float32
    _check(lib().fmoe_gdn_step(_ptr(state, f32, "state"), _ptr(q, f32, "q"), _ptr(k, f32, "k"), _ptr(v, f32, "v"),
                               _ptr(alpha, f32, "alpha"), _ptr(beta, f32, "beta"), _ptr(o, f32, "o"), n, dk, dv,
                               GDN_STATE_EARLY if early else 0, _stream(stream)))
    return o


class ExpertCache:
    """An HBM cache of `num_slots` expert records in front of `host_records`, a pinned host
    tensor (uint8) holding `num_experts` records at `stride` bytes (fmoe_cache.h)."""

    def __init__(self, host_records, num_experts, stride, record_bytes, num_slots, device=None, stream=None):
        if host_records.is_cuda or not host_records.is_pinned():
            raise ValueError("host_records must be a pinned host tensor")
        if host_records.dtype != torch.uint8 or not host_records.is_contiguous():
            raise TypeError("host_records must be a contiguous uint8 tensor")
        if host_records.numel() < num_experts * stride:
            raise ValueError("host_records holds fewer than num_experts records")
        device = device or "cuda"
        self.host = host_records
        self.slots = torch.empty(num_slots * stride, dtype=torch.uint8, device=device)
        self.state = torch.empty(max(1, lib().fmoe_expert_cache_state_size(num_experts, num_slots)),
                                 dtype=torch.uint8, device=device)
        self.s = FmoeExpertCache(host_records.data_ptr(), stride, self.slots.data_ptr(), stride, record_bytes,
                                 num_experts, num_slots, self.state.data_ptr())
        self.reset(stream)

    def reset(self, stream=None):
        _check(lib().fmoe_expert_cache_reset(ctypes.byref(self.s), _stream(stream)))

    def fetch(self, idx, slot=None, stream=None):
        """One lookup of the experts idx (device int32 [K]); returns their slots (device int32 [K])."""
        slot = torch.empty_like(idx) if slot is None else slot
        _check(lib().fmoe_expert_cache_fetch(ctypes.byref(self.s), _ptr(idx, torch.int32, "idx"), idx.numel(),
                                             _ptr(slot, torch.int32, "slot"), _stream(stream)))
        return slot

    def stats(self, stream=None):
        """(hits, misses, bytes copied) since the last reset; synchronises the stream."""
        h, m, b = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(lib().fmoe_expert_cache_stats(ctypes.byref(self.s), ctypes.byref(h), ctypes.byref(m), ctypes.byref(b),
                                             _stream(stream)))
        return h.value, m.value, b.value


def moe_layer_cached(layer, cache, h, out=None, topk_idx=None, topk_w=None, ws=None, stream=None):
    """fmoe_moe_layer_cached: the block with the routed experts behind `cache`."""
    T = h.shape[0] if h.dim() == 2 else 1
    out = torch.empty_like(h) if out is None else out
    if ws is None:
        ws = workspace(moe_layer_workspace_size(layer, 1), h.device, stream)
    _check(lib().fmoe_moe_layer_cached(ctypes.byref(layer.s), ctypes.byref(cache.s), _ptr(h, torch.float32, "h"), T,
                                       _ptr(out, torch.float32, "out"), _ptr(topk_idx, torch.int32, "topk_idx"),
                                       _ptr(topk_w, torch.float32, "topk_w"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
                                       _stream(stream)))
    return out


def moe_stack(layers, h, out=None, ws=None, stream=None):
    T = h.shape[0] if h.dim() == 2 else 1
    out = torch.empty_like(h) if out is None else out
    arr = (FmoeLayer * len(layers))(*[l.s for l in layers])
    if ws is None:
        ws = workspace(max(moe_layer_workspace_size(l, T) for l in layers), h.device, stream)
    _check(lib().fmoe_moe_stack(arr, len(layers), _ptr(h, torch.float32, "h"), T, _ptr(out, torch.float32, "out"),
                                _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))
    return out
