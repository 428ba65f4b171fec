"""CPU oracle of the routed-MoE decode block and of the Gated DeltaNet state update
(fp64, plain C) -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  It shares no code with the CUDA path; inputs are numpy arrays in
host memory (bf16 values as uint16 bit patterns).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


class OrMatrix(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("group", ctypes.c_int), ("rows", ctypes.c_int), ("cols", ctypes.c_int),
                ("qw", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("bias", ctypes.c_void_p)]


class OrBank(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("group", ctypes.c_int), ("hidden", ctypes.c_int), ("inter", ctypes.c_int),
                ("num_experts", ctypes.c_int), ("base", ctypes.c_void_p), ("stride", ctypes.c_int64),
                ("off", ctypes.c_int64 * 9), ("records", ctypes.c_void_p)]


class OrLayer(ctypes.Structure):
    _fields_ = [("routed", OrBank), ("shared", OrBank), ("w_router", ctypes.c_void_p),
                ("router_bias", ctypes.c_void_p), ("w_shared_gate", ctypes.c_void_p), ("gamma", ctypes.c_void_p),
                ("eps", ctypes.c_double), ("top_k", ctypes.c_int)]


def lib():
    global _lib
    if _lib is None:
        # FMOE_ORACLE_SO: load another build of the oracle source instead (the mutation
        # tests point it at copies with a planted mistake, to show that the pins fail)
        so = os.environ.get("FMOE_ORACLE_SO")
        if not so:
            _build.build()
            so = _build.SO
        L = ctypes.CDLL(so)
        vp, ci, cd = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.or_bf16.restype = cd
        L.or_bf16.argtypes = [ctypes.c_uint16]
        L.or_code.restype = ctypes.c_uint
        L.or_code.argtypes = [vp, ci, ci]
        L.or_weight.restype = cd
        L.or_weight.argtypes = [ctypes.POINTER(OrMatrix), ci, ci]
        L.or_matvec.argtypes = [ctypes.POINTER(OrMatrix), vp, vp]
        L.or_rmsnorm.argtypes = [vp, vp, cd, ci, vp]
        L.or_router_logits.argtypes = [vp, vp, vp, ci, ci, vp]
        L.or_softmax.argtypes = [vp, ci, vp]
        L.or_topk.argtypes = [vp, ci, ci, vp]
        L.or_expert_ffn.argtypes = [ctypes.POINTER(OrBank), ci, vp, vp, vp]
        L.or_moe_layer.argtypes = [ctypes.POINTER(OrLayer), vp, ci, vp, vp, vp, vp, vp, vp, vp]
        L.or_gdn_step.argtypes = [ci, ci, ci, vp, vp, vp, vp, vp, vp, vp]
        L.or_set_threads.argtypes = [ci]
        L.or_get_threads.restype = ci
        L.or_max_threads.restype = ci
        _lib = L
    return _lib


def set_threads(n):
    lib().or_set_threads(int(n))


def get_threads():
    return lib().or_get_threads()


def max_threads():
    return lib().or_max_threads()


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def bf16(v):
    return lib().or_bf16(int(v))


def code(words, bits, c):
    w = _c(words, np.uint32)
    return lib().or_code(w.ctypes.data, bits, c)


def matrix(qw, scale, bias, bits, rows, cols, group=64):
    """Wraps numpy arrays as one packed matrix; keep the returned tuple alive while using it."""
    qw, scale, bias = _c(qw, np.uint32), _c(scale, np.uint16), _c(bias, np.uint16)
    m = OrMatrix(bits, group, rows, cols, qw.ctypes.data, scale.ctypes.data, bias.ctypes.data)
    return m, (qw, scale, bias)


def weight(m, r, c):
    return lib().or_weight(ctypes.byref(m[0]), r, c)


def matvec(m, x):
    x = _c(x, np.float64)
    y = np.empty(m[0].rows, dtype=np.float64)
    lib().or_matvec(ctypes.byref(m[0]), x.ctypes.data, y.ctypes.data)
    return y


def rmsnorm(h, gamma, eps):
    h = _c(h, np.float32)
    gamma = _c(gamma, np.float32)
    x = np.empty(h.shape[-1], dtype=np.float64)
    lib().or_rmsnorm(h.ctypes.data, _p(gamma), eps, h.shape[-1], x.ctypes.data)
    return x


def router_logits(w_router, bias, x):
    w_router = _c(w_router, np.uint16)
    bias = _c(bias, np.float32)
    x = _c(x, np.float64)
    E, H = w_router.shape
    out = np.empty(E, dtype=np.float64)
    lib().or_router_logits(w_router.ctypes.data, _p(bias), x.ctypes.data, E, H, out.ctypes.data)
    return out


def softmax(l):
    l = _c(l, np.float64)
    p = np.empty_like(l)
    lib().or_softmax(l.ctypes.data, l.size, p.ctypes.data)
    return p


def topk(p, k):
    p = _c(p, np.float64)
    idx = np.empty(k, dtype=np.int32)
    lib().or_topk(p.ctypes.data, p.size, k, idx.ctypes.data)
    return idx


def bank(base, bits, hidden, inter, num_experts, stride, off, group=64):
    """Wraps a uint8 array of `num_experts` records (record e at e*stride), or a dict
    {expert id: uint8 record} holding only some records (the others must not be selected)."""
    if isinstance(base, dict):
        keep = {e: np.ascontiguousarray(r, dtype=np.uint8) for e, r in base.items()}
        table = (ctypes.c_void_p * num_experts)(*[keep[e].ctypes.data if e in keep else None
                                                   for e in range(num_experts)])
        b = OrBank(bits, group, hidden, inter, num_experts, None, stride, (ctypes.c_int64 * 9)(*off),
                   ctypes.cast(table, ctypes.c_void_p))
        return b, (keep, table)
    base = np.ascontiguousarray(base, dtype=np.uint8)
    b = OrBank(bits, group, hidden, inter, num_experts, base.ctypes.data, stride, (ctypes.c_int64 * 9)(*off), None)
    return b, base


def expert_ffn(bk, e, x, want_act=False):
    x = _c(x, np.float64)
    y = np.empty(bk[0].hidden, dtype=np.float64)
    a = np.empty(bk[0].inter, dtype=np.float64) if want_act else None
    lib().or_expert_ffn(ctypes.byref(bk[0]), e, x.ctypes.data, y.ctypes.data, _p(a))
    return (y, a) if want_act else y


class Layer:
    """A layer for the oracle: routed bank [E][record], shared record, router, shared gate, gamma, bias."""

    def __init__(self, routed, shared, w_router, w_shared_gate, gamma, router_bias, bits, hidden, inter, top_k,
                 stride, off, eps=1e-6, group=64):
        E = w_router.shape[0]
        self.routed = bank(routed if isinstance(routed, dict) else routed.reshape(-1), bits, hidden, inter, E,
                           stride, off, group)
        self.shared = bank(shared.reshape(-1), bits, hidden, inter, 1, stride, off, group)
        self.w_router = _c(w_router, np.uint16)
        self.w_shared_gate = _c(w_shared_gate, np.uint16)
        self.gamma = _c(gamma, np.float32)
        self.router_bias = _c(router_bias, np.float32)
        self.E, self.H, self.K = E, hidden, top_k
        self.s = OrLayer(self.routed[0], self.shared[0], self.w_router.ctypes.data, _p(self.router_bias),
                         self.w_shared_gate.ctypes.data, _p(self.gamma), eps, top_k)

    def forward(self, h, force_idx=None):
        """Returns dict(out [T][H], idx [T][K], w [T][K], probs [T][E], logits [T][E], sigma [T])."""
        h = _c(h, np.float32).reshape(-1, self.H)
        T = h.shape[0]
        out = np.empty((T, self.H), dtype=np.float64)
        idx = np.empty((T, self.K), dtype=np.int32)
        w = np.empty((T, self.K), dtype=np.float64)
        probs = np.empty((T, self.E), dtype=np.float64)
        logits = np.empty((T, self.E), dtype=np.float64)
        sigma = np.empty(T, dtype=np.float64)
        fi = None if force_idx is None else _c(force_idx, np.int32).reshape(T, self.K)
        lib().or_moe_layer(ctypes.byref(self.s), h.ctypes.data, T, _p(fi), out.ctypes.data, idx.ctypes.data,
                           w.ctypes.data, probs.ctypes.data, logits.ctypes.data, sigma.ctypes.data)
        return dict(out=out, idx=idx, w=w, probs=probs, logits=logits, sigma=sigma)


def gdn_step(S, q, k, v, alpha, beta):
    """One gated-delta-rule step of n heads (or_gdn_step): S [n][dv][dk], q/k [n][dk], v [n][dv],
    alpha/beta [n], any float dtype (widened to fp64).  Returns (new state, o [n][dv]) in fp64;
    the inputs are not modified."""
    S = np.array(S, dtype=np.float64, order="C", copy=True)
    n, dv, dk = S.shape
    q, k = _c(q, np.float64).reshape(n, dk), _c(k, np.float64).reshape(n, dk)
    v = _c(v, np.float64).reshape(n, dv)
    alpha, beta = _c(alpha, np.float64).reshape(n), _c(beta, np.float64).reshape(n)
    o = np.empty((n, dv), dtype=np.float64)
    lib().or_gdn_step(n, dk, dv, S.ctypes.data, q.ctypes.data, k.ctypes.data, v.ctypes.data, alpha.ctypes.data,
                      beta.ctypes.data, o.ctypes.data)
    return S, o
