"""Test-side helpers: an independent numpy packer/dequantiser, the error metric and layer marshalling."""
import math

import numpy as np

import gen


def f32_to_bf16_exact(v):
    """bf16 bit pattern of values that are exactly representable in bf16 (asserts it)."""
    a = np.asarray(v, dtype=np.float32)
    u = a.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exactly representable in bf16"
    return (u >> 16).astype(np.uint16)


def bf16_to_f64(b):
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def np_pack(codes, bits):
    """Packs unsigned codes [rows][cols] into uint32 words, field j of a word at bits [bits*j, bits*j+bits)."""
    per = 32 // bits
    rows, cols = codes.shape
    w = codes.astype(np.uint64).reshape(rows, cols // per, per)
    shifts = (np.arange(per, dtype=np.uint64) * np.uint64(bits))
    return np.bitwise_or.reduce(w << shifts, axis=-1).astype(np.uint32)


def np_unpack(words, bits, cols):
    """Inverse of np_pack, vectorised over whole words."""
    per = 32 // bits
    w = np.asarray(words, dtype=np.uint32).astype(np.uint64)
    rows = w.shape[0]
    shifts = (np.arange(per, dtype=np.uint64) * np.uint64(bits))
    c = (w[..., None] >> shifts) & np.uint64((1 << bits) - 1)
    return c.reshape(rows, -1)[:, :cols].astype(np.int64)


def dense_from_record(rec, spec_bits, hidden, inter, group=64):
    """Dense fp64 gate, up, down of one record, via whole-array unpacking (independent of the oracle's decoder)."""
    nbytes, off = gen.record_layout(spec_bits, hidden, inter, group)
    rec = np.asarray(rec, dtype=np.uint8)
    out = []
    for m, (rows, cols) in enumerate(((inter, hidden), (inter, hidden), (hidden, inter))):
        nw = rows * cols * spec_bits // 32
        ng = rows * cols // group
        qw = rec[off[3 * m]:off[3 * m] + 4 * nw].view(np.uint32).reshape(rows, -1)
        s = bf16_to_f64(rec[off[3 * m + 1]:off[3 * m + 1] + 2 * ng].view(np.uint16)).reshape(rows, -1)
        b = bf16_to_f64(rec[off[3 * m + 2]:off[3 * m + 2] + 2 * ng].view(np.uint16)).reshape(rows, -1)
        codes = np_unpack(qw, spec_bits, cols).astype(np.float64)
        out.append(codes * np.repeat(s, group, axis=1) + np.repeat(b, group, axis=1))
    return out


def max_rel_err(got, ref, floor=1e-2, slack=None):
    """max_i (|g_i - r_i| - slack_i)+ / max(|r_i|, floor * rms(r)) over the last axis, maximised over rows.

    `slack` is an absolute allowance per element (default 0), used when `got` was
    recovered from a stored fp32 value: out - h cannot be closer than one fp32 ulp of out."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    den = np.maximum(np.abs(ref), floor * rms)
    den = np.where(den > 0, den, 1.0)
    diff = np.abs(got - ref)
    if slack is not None:
        diff = np.maximum(diff - np.asarray(slack, dtype=np.float64), 0.0)
    return float(np.max(diff / den)) if got.size else 0.0


def ulp32(a):
    """One fp32 ulp of each element."""
    return np.spacing(np.abs(np.asarray(a, dtype=np.float32))).astype(np.float64)


def oracle_layer(hl, top_k=None, gamma=True):
    """Marshals a gen.HostLayer (all routed experts drawn) into an oracle.Layer."""
    import oracle
    spec = hl.spec
    nbytes, off = gen.record_layout(spec.bits, spec.hidden, spec.inter, spec.group)
    return oracle.Layer(gen.bank_array(hl), hl.shared, hl.w_router, hl.w_shared_gate,
                        hl.gamma if gamma else None, hl.logit_bias, spec.bits, spec.hidden, spec.inter,
                        top_k if top_k is not None else spec.top_k, nbytes, off, eps=spec.eps, group=spec.group)


def oracle_layer_sparse(hl, top_k=None):
    """Oracle layer over a host layer drawn with a subset of experts (only those may be selected)."""
    import oracle
    spec = hl.spec
    nbytes, off = gen.record_layout(spec.bits, spec.hidden, spec.inter, spec.group)
    return oracle.Layer(dict(hl.routed), hl.shared, hl.w_router, hl.w_shared_gate, hl.gamma, hl.logit_bias,
                        spec.bits, spec.hidden, spec.inter, top_k if top_k is not None else spec.top_k, nbytes, off,
                        eps=spec.eps, group=spec.group)


def silu(z):
    return z / (1.0 + np.exp(-z))


U32 = 2.0 ** -24


def routing_margin(w_router_bf16, xhat, logit_bias=None, safety=8.0):
    """Per-token bound on how far an fp32 logit may sit from the exact one: safety * u * sqrt(H) * sum_i |w x|.

    Returns (exact logits [E] in fp64 from the fp64 x, delta)."""
    W = bf16_to_f64(w_router_bf16)
    l = W @ xhat + (0.0 if logit_bias is None else np.asarray(logit_bias, np.float64))
    s = np.abs(W) @ np.abs(xhat)
    return l, safety * U32 * math.sqrt(W.shape[1]) * float(s.max())


def check_routing(gpu_idx, logits, K, delta):
    """Compares one token's GPU top-K with the exact logits.

    Returns True when the exact top K+1 logits are separated by more than delta (the
    selection must then match exactly, in order); otherwise checks that every selected
    expert is within delta of the exact K-th logit (a valid near-tie choice) and returns False."""
    order = np.argsort(-logits, kind="stable")
    top = logits[order[:K + 1]] if len(logits) > K else np.append(logits[order[:K]], -np.inf)
    gaps = top[:-1] - top[1:]
    gpu_idx = [int(i) for i in gpu_idx]
    if np.all(gaps > delta):
        assert gpu_idx == order[:K].tolist(), (gpu_idx, order[:K].tolist())
        return True
    assert len(set(gpu_idx)) == K
    kth = logits[order[K - 1]]
    for i in gpu_idx:
        assert logits[i] >= kth - delta, (i, logits[i], kth)
    sel = logits[gpu_idx]
    assert np.all(sel[:-1] >= sel[1:] - delta)  # descending up to the near-tie margin
    return False
