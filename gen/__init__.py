"""Seeded synthetic inputs for the routed-MoE block and the Gated DeltaNet state update:
shapes, layouts and generators.

Both the CPU oracle (through the host library) and the GPU path (through the
device library) consume the bytes drawn here; this module holds none of the
block's own arithmetic.  Workload shapes follow the Flash-MoE pages' model
description (Qwen3.5-397B-A17B: hidden 4096, 512 routed experts, top-4 plus
one shared expert, 4-bit or 2-bit group-64 affine experts).

Input recipe (all synthetic, no dataset and no trained weights):
  * expert weights N(0, 0.02), quantised per group of 64 along the input dim
    (min/max affine, bf16 scale and bias, codes packed LSB-first);
  * router N(0, 0.02) bf16 (tiny layer: N(0, 1/H) so that logits are ~N(0,1));
  * shared-expert gate vector N(0, 0.02) bf16;
  * RMSNorm weight gamma = 1 (tests also draw gamma = 1 + 0.1 N(0,1));
  * token hidden states N(0, 1) fp32, a fresh seeded draw per token;
  * Zipf-routed variant: per-expert logit bias ln p_pi(e), p_r ~ r^-1.1.
"""
import ctypes
import dataclasses
import math
import os

import numpy as np

from . import build as _build

GROUP = 64
KIND_GATE, KIND_UP, KIND_DOWN, KIND_ROUTER, KIND_SHARED_GATE, KIND_GAMMA, KIND_PERM = range(7)
EXPERT_SHARED = 0xFFFFFFF
EXPERT_LAYER = 0xFFFFFFE
WEIGHT_SEED = 0
TOKEN_SEED = 1

_host = None
_cuda = None


def host_lib():
    global _host
    if _host is None:
        _build.build()
        lib = ctypes.CDLL(_build.HOST_SO)
        u64, i64, f32 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_float
        vp = ctypes.c_void_p
        lib.fg_host_key.restype = u64
        lib.fg_host_key.argtypes = [u64, u64]
        lib.fg_host_stream_id.restype = u64
        lib.fg_host_stream_id.argtypes = [u64, u64, u64]
        lib.fg_host_normal_f32.argtypes = [u64, f32, i64, vp]
        lib.fg_host_normal_bf16.argtypes = [u64, f32, i64, vp]
        lib.fg_host_uniform_u32.argtypes = [u64, ctypes.c_uint32, i64, vp]
        lib.fg_host_packed.argtypes = [u64, f32, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp]
        _host = lib
    return _host


def cuda_lib():
    global _cuda
    if _cuda is None:
        _build.build()
        lib = ctypes.CDLL(_build.CUDA_SO)
        u64, i64, f32, i32, vp = ctypes.c_uint64, ctypes.c_longlong, ctypes.c_float, ctypes.c_int, ctypes.c_void_p
        lib.fg_cuda_packed_bank.restype = i32
        lib.fg_cuda_packed_bank.argtypes = [u64, u64, u64, i32, i32, f32, i32, i32, i32, i32, vp, i64, i64, i64, i64,
                                            vp]
        lib.fg_cuda_normal_f32.restype = i32
        lib.fg_cuda_normal_f32.argtypes = [u64, f32, i64, vp, vp]
        lib.fg_cuda_normal_bf16.restype = i32
        lib.fg_cuda_normal_bf16.argtypes = [u64, f32, i64, vp, vp]
        _cuda = lib
    return _cuda


def key(seed, layer, expert, kind):
    lib = host_lib()
    return int(lib.fg_host_key(seed, lib.fg_host_stream_id(layer, expert, kind)))


def token_key(t):
    """Key of token t's hidden state (seed 1, stream t)."""
    return int(host_lib().fg_host_key(TOKEN_SEED, t))


# ----------------------------------------------------------------------------------------------- shapes


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    """One routed-MoE layer: hidden H, E routed experts of intermediate I, top-K, code width."""
    hidden: int
    experts: int
    inter: int
    top_k: int
    bits: int
    group: int = GROUP
    eps: float = 1e-6
    weight_std: float = 0.02
    router_std: float = 0.02
    shared_gate_std: float = 0.02
    zipf: float = 0.0          # > 0: per-expert logit bias ln p_pi(e), p_r ~ r^-zipf
    random_gamma: bool = False  # False: gamma = 1


def tiny_layer(bits=4):
    """Tiny layer: hidden 256, 8 experts of intermediate 128, top-2; router N(0, 1/H)."""
    return LayerSpec(hidden=256, experts=8, inter=128, top_k=2, bits=bits, router_std=1.0 / math.sqrt(256))


def small_layer(bits=4, experts=16, top_k=4):
    """Small layer for batched-path tests: hidden 512, intermediate 512 (8 groups of 64 per row)."""
    return LayerSpec(hidden=512, experts=experts, inter=512, top_k=top_k, bits=bits,
                     router_std=1.0 / math.sqrt(512))


def qwen397_layer(bits=4, zipf=0.0):
    """Qwen3.5-397B-A17B-shaped MoE layer: hidden 4096, 512 experts of intermediate 1024, top-4 + shared."""
    return LayerSpec(hidden=4096, experts=512, inter=1024, top_k=4, bits=bits, zipf=zipf)


def _align16(n):
    return (n + 15) // 16 * 16


def record_layout(bits, hidden, inter, group=GROUP):
    """Byte layout of one expert record: gate{qw,scale,bias} | up{...} | down{...}.

    A packed [out][in] matrix is qw uint32[out][in*bits/32] (code j of a word at
    bits [bits*j, bits*j+bits)) followed by scale and bias bf16[out][in/group];
    every sub-array starts on a 16-byte boundary.  Returns (record_bytes, off[9]).
    """
    off = []
    pos = 0
    for out_dim, in_dim in ((inter, hidden), (inter, hidden), (hidden, inter)):
        for nbytes in (out_dim * in_dim * bits // 8, out_dim * (in_dim // group) * 2, out_dim * (in_dim // group) * 2):
            off.append(pos)
            pos = _align16(pos + nbytes)
    return pos, off


def record_bytes(spec):
    return record_layout(spec.bits, spec.hidden, spec.inter, spec.group)[0]


def matrix_shapes(spec):
    """(rows, cols) of gate, up, down."""
    return ((spec.inter, spec.hidden), (spec.inter, spec.hidden), (spec.hidden, spec.inter))


def algorithmic_bytes_per_token(spec):
    """Bytes one token must read: K routed + 1 shared expert records (packed codes + scales + biases) + router."""
    return (spec.top_k + 1) * _payload_bytes(spec) + spec.experts * spec.hidden * 2


def _payload_bytes(spec):
    total = 0
    for rows, cols in matrix_shapes(spec):
        total += rows * cols * spec.bits // 8 + 2 * rows * (cols // spec.group) * 2
    return total


# ----------------------------------------------------------------------------------------------- host generation


def host_record(spec, seed, layer, expert_id):
    """One expert record (numpy uint8) drawn on the host."""
    lib = host_lib()
    nbytes, off = record_layout(spec.bits, spec.hidden, spec.inter, spec.group)
    rec = np.zeros(nbytes, dtype=np.uint8)
    base = rec.ctypes.data
    for m, (rows, cols) in enumerate(matrix_shapes(spec)):
        k = key(seed, layer, expert_id, m)
        lib.fg_host_packed(k, spec.weight_std, spec.bits, spec.group, rows, cols, base + off[3 * m],
                           base + off[3 * m + 1], base + off[3 * m + 2])
    return rec


def host_normal_f32(k, std, n):
    out = np.empty(n, dtype=np.float32)
    host_lib().fg_host_normal_f32(k, std, n, out.ctypes.data)
    return out


def host_normal_bf16(k, std, n):
    out = np.empty(n, dtype=np.uint16)
    host_lib().fg_host_normal_bf16(k, std, n, out.ctypes.data)
    return out


def zipf_logit_bias(spec, seed, layer):
    """Per-expert logit bias ln p_pi(e) with p_r ~ r^-zipf over ranks 1..E and pi a seeded permutation."""
    E = spec.experts
    draws = np.empty(E, dtype=np.uint32)
    lib = host_lib()
    k = key(seed, layer, EXPERT_LAYER, KIND_PERM)
    # Fisher-Yates with draw i choosing among E - i remaining positions.
    perm = np.arange(E)
    for i in range(E - 1, 0, -1):
        lib.fg_host_uniform_u32(lib.fg_host_key(k, i), i + 1, 1, draws.ctypes.data)
        j = int(draws[0])
        perm[i], perm[j] = perm[j], perm[i]
    ranks = np.arange(1, E + 1, dtype=np.float64)
    p = ranks ** (-spec.zipf)
    p /= p.sum()
    return np.log(p[perm]).astype(np.float32)


@dataclasses.dataclass
class HostLayer:
    spec: LayerSpec
    routed: dict            # expert id -> uint8 record
    shared: np.ndarray      # uint8 record
    w_router: np.ndarray    # uint16 (bf16 bits) [E][H]
    w_shared_gate: np.ndarray  # uint16 [H]
    gamma: np.ndarray       # float32 [H]
    logit_bias: object      # float32 [E] or None


def host_gamma(spec, seed, layer):
    if spec.random_gamma:
        return (1.0 + host_normal_f32(key(seed, layer, EXPERT_LAYER, KIND_GAMMA), 0.1, spec.hidden)).astype(np.float32)
    return np.ones(spec.hidden, dtype=np.float32)


def host_layer(spec, seed=WEIGHT_SEED, layer=0, experts=None):
    """Draws a layer on the host; `experts` limits which routed records are drawn (default: all)."""
    ids = range(spec.experts) if experts is None else sorted(set(int(e) for e in experts))
    routed = {e: host_record(spec, seed, layer, e) for e in ids}
    shared = host_record(spec, seed, layer, EXPERT_SHARED)
    wr = host_normal_bf16(key(seed, layer, EXPERT_LAYER, KIND_ROUTER), spec.router_std,
                          spec.experts * spec.hidden).reshape(spec.experts, spec.hidden)
    wsg = host_normal_bf16(key(seed, layer, EXPERT_LAYER, KIND_SHARED_GATE), spec.shared_gate_std, spec.hidden)
    bias = zipf_logit_bias(spec, seed, layer) if spec.zipf > 0 else None
    return HostLayer(spec, routed, shared, wr, wsg, host_gamma(spec, seed, layer), bias)


def host_tokens(t0, T, hidden):
    """Hidden states of tokens t0..t0+T-1: fresh N(0,1) fp32 draws, shape [T][H]."""
    out = np.empty((T, hidden), dtype=np.float32)
    for i in range(T):
        out[i] = host_normal_f32(token_key(t0 + i), 1.0, hidden)
    return out


def bank_array(hl):
    """All routed records of a fully drawn host layer as one [E][record] uint8 array."""
    E = hl.spec.experts
    if len(hl.routed) != E:
        raise ValueError("layer was drawn with a subset of experts")
    return np.stack([hl.routed[e] for e in range(E)])


# ----------------------------------------------------------------------------------------------- device generation


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what}: CUDA error {rc}")


def device_fill_bank(spec, seed, layer, expert_id0, n, dst, stream_ptr):
    """Draws records expert_id0 .. expert_id0+n-1 into device buffer `dst` (torch uint8 [n*record])."""
    lib = cuda_lib()
    nbytes, off = record_layout(spec.bits, spec.hidden, spec.inter, spec.group)
    assert dst.numel() >= n * nbytes
    for m, (rows, cols) in enumerate(matrix_shapes(spec)):
        _check(lib.fg_cuda_packed_bank(seed, layer, expert_id0, n, m, spec.weight_std, spec.bits, spec.group, rows,
                                       cols, dst.data_ptr(), nbytes, off[3 * m], off[3 * m + 1], off[3 * m + 2],
                                       stream_ptr), "fg_cuda_packed_bank")


def device_normal_f32(k, std, dst, stream_ptr):
    _check(cuda_lib().fg_cuda_normal_f32(k, std, dst.numel(), dst.data_ptr(), stream_ptr), "fg_cuda_normal_f32")


def device_normal_bf16(k, std, dst, stream_ptr):
    _check(cuda_lib().fg_cuda_normal_bf16(k, std, dst.numel(), dst.data_ptr(), stream_ptr), "fg_cuda_normal_bf16")


# ----------------------------------------------------------------------------------------------- device layers


@dataclasses.dataclass
class DeviceLayer:
    spec: LayerSpec
    bank: object          # torch uint8 [E * record]
    shared: object        # torch uint8 [record]
    w_router: object      # torch int16 (bf16 bits) [E][H]
    w_shared_gate: object  # torch int16 [H]
    gamma: object         # torch float32 [H]
    logit_bias: object    # torch float32 [E] or None


def upload_layer(hl, device="cuda"):
    """Copies a fully drawn host layer to the device."""
    import torch
    spec = hl.spec
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return DeviceLayer(spec, t(gen_bank_bytes(hl)), t(hl.shared), t(hl.w_router.view(np.int16)),
                       t(hl.w_shared_gate.view(np.int16)), t(hl.gamma),
                       None if hl.logit_bias is None else t(hl.logit_bias))


def gen_bank_bytes(hl):
    return bank_array(hl).reshape(-1)


def device_layer(spec, seed=WEIGHT_SEED, layer=0, device="cuda"):
    """Draws a whole layer directly in device memory (same bytes as host_layer)."""
    import torch
    stream = torch.cuda.current_stream().cuda_stream
    nbytes = record_bytes(spec)
    bank = torch.empty(spec.experts * nbytes, dtype=torch.uint8, device=device)
    shared = torch.empty(nbytes, dtype=torch.uint8, device=device)
    device_fill_bank(spec, seed, layer, 0, spec.experts, bank, stream)
    device_fill_bank(spec, seed, layer, EXPERT_SHARED, 1, shared, stream)
    wr = torch.empty((spec.experts, spec.hidden), dtype=torch.int16, device=device)
    device_normal_bf16(key(seed, layer, EXPERT_LAYER, KIND_ROUTER), spec.router_std, wr, stream)
    wsg = torch.empty(spec.hidden, dtype=torch.int16, device=device)
    device_normal_bf16(key(seed, layer, EXPERT_LAYER, KIND_SHARED_GATE), spec.shared_gate_std, wsg, stream)
    gamma = torch.from_numpy(host_gamma(spec, seed, layer)).to(device)
    bias = None
    if spec.zipf > 0:
        bias = torch.from_numpy(zipf_logit_bias(spec, seed, layer)).to(device)
    return DeviceLayer(spec, bank, shared, wr, wsg, gamma, bias)


def binding_layer(dl, top_k=None, use_gamma=True):
    """Wraps a DeviceLayer as a layer of the product binding."""
    import bit_dequant_expert_router_b200 as fmoe
    spec = dl.spec
    nbytes, off = record_layout(spec.bits, spec.hidden, spec.inter, spec.group)
    routed = fmoe.Bank(dl.bank, spec.bits, spec.hidden, spec.inter, spec.experts, nbytes, off, spec.group)
    shared = fmoe.Bank(dl.shared, spec.bits, spec.hidden, spec.inter, 1, nbytes, off, spec.group)
    return fmoe.Layer(routed, shared, dl.w_router, dl.w_shared_gate, dl.gamma if use_gamma else None, dl.logit_bias,
                      spec.eps, spec.top_k if top_k is None else top_k)


def device_tokens(t0, T, hidden, device="cuda"):
    """Token hidden states drawn on the device (same values as host_tokens)."""
    import torch
    out = torch.empty((T, hidden), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream().cuda_stream
    for i in range(T):
        device_normal_f32(token_key(t0 + i), 1.0, out[i], stream)
    return out


# ----------------------------------------------------------------------------------------------- Gated DeltaNet
# Inputs of the linear-attention state update (64 heads x 128 x 128 in the Qwen3.5-397B-A17B
# description of the Flash-MoE pages).  Recipe: state entries N(0, 0.1^2) fp32; k a fresh
# N(0,1) draw per head scaled to unit L2 norm; q the same, times dk^-1/2; v N(0,1); the
# decay gate alpha uniform in [0.8, 1.0) and the write strength beta uniform in [0, 1),
# both on a 2^-24 grid.  Every token draws fresh q, k, v, alpha, beta.

GDN_SEED = 2
GDN_Q, GDN_K, GDN_V, GDN_ALPHA, GDN_BETA, GDN_STATE = range(6)


@dataclasses.dataclass(frozen=True)
class GdnSpec:
    """n independent heads (batch x heads), each a dv x dk fp32 state."""
    heads: int
    dk: int
    dv: int
    state_std: float = 0.1


def gdn_qwen397(batch=1):
    """Qwen3.5-397B-A17B linear-attention layer: 64 heads of 128 x 128, `batch` sequences."""
    return GdnSpec(heads=64 * batch, dk=128, dv=128)


def gdn_key(layer, t, kind):
    return int(host_lib().fg_host_key(GDN_SEED, (int(layer) << 40) | (int(t) << 4) | int(kind)))


def _gdn_uniform(k, n):
    u = np.empty(n, dtype=np.uint32)
    host_lib().fg_host_uniform_u32(k, 1 << 24, n, u.ctypes.data)
    return u.astype(np.float32) * np.float32(2.0 ** -24)


def _unit_rows(a):
    return (a / np.sqrt(np.sum(a.astype(np.float64) ** 2, axis=1, keepdims=True))).astype(np.float32)


def host_gdn_state(spec, layer=0):
    """Initial state of one layer: fp32 [heads][dv][dk]."""
    n = spec.heads * spec.dv * spec.dk
    return host_normal_f32(gdn_key(layer, 0, GDN_STATE), spec.state_std, n).reshape(spec.heads, spec.dv, spec.dk)


def host_gdn_token(spec, layer, t):
    """Token t's inputs to one layer: q, k fp32 [heads][dk], v [heads][dv], alpha, beta [heads]."""
    n, dk, dv = spec.heads, spec.dk, spec.dv
    k = _unit_rows(host_normal_f32(gdn_key(layer, t, GDN_K), 1.0, n * dk).reshape(n, dk))
    q = (_unit_rows(host_normal_f32(gdn_key(layer, t, GDN_Q), 1.0, n * dk).reshape(n, dk))
         * np.float32(1.0 / math.sqrt(dk))).astype(np.float32)
    v = host_normal_f32(gdn_key(layer, t, GDN_V), 1.0, n * dv).reshape(n, dv)
    alpha = (np.float32(0.8) + np.float32(0.2) * _gdn_uniform(gdn_key(layer, t, GDN_ALPHA), n)).astype(np.float32)
    beta = _gdn_uniform(gdn_key(layer, t, GDN_BETA), n)
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta)


def device_gdn_state(spec, layer=0, device="cuda"):
    """The same initial state as host_gdn_state, drawn on the device."""
    import torch
    out = torch.empty((spec.heads, spec.dv, spec.dk), dtype=torch.float32, device=device)
    device_normal_f32(gdn_key(layer, 0, GDN_STATE), spec.state_std, out, torch.cuda.current_stream().cuda_stream)
    return out
