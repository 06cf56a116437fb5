"""Helpers for the GPU tests: load a generated workload into a KV layer
through the C ABI, run the attention, and compare with the oracle."""
import numpy as np
import torch

import oracle
from shared_context_decode_b200.workloads import bf16_bits
from tests.flat import decode_slots, decode_queries, prefill_slots, prefill_queries

# Tolerances on o (bf16 inputs, fp32 accumulation), the method's acceptance
# bar for this path: max |err| <= 1e-2, mean <= 1e-3.
O_MAX, O_MEAN = 1e-2, 1e-3
# lse is fp32 from fp32 scores of exact bf16 products.
LSE_MAX = 5e-3


def pp():
    from shared_context_decode_b200 import ppattn
    return ppattn


def doc_tags(N, device):
    return (torch.zeros(N, dtype=torch.int16, device=device),
            torch.arange(N, dtype=torch.int32, device=device))


def load_decode(W, L, device, S_cap=None, P_max=None, doc_cap=None):
    """Fresh KV layer holding layer L of decode workload W, with the decode
    tokens already appended (the cache state at the attention call)."""
    m = pp()
    layer = m.KVLayer(W.H, W.d, doc_cap or max(W.N, 1), P_max or W.P, S_cap or W.S_need, device)
    if W.N:
        sid, pos = doc_tags(W.N, device)
        m.kv_append(layer, L.doc_k, L.doc_v, sid, pos)
    if L.suf_sid.numel():
        m.kv_append(layer, L.suf_k, L.suf_v, L.suf_sid, L.suf_pos)
    m.kv_append(layer, L.new_k, L.new_v, L.q_sid, L.q_pos)
    return layer


def load_prefill(W, L, device, S_cap=None):
    m = pp()
    S = S_cap or int(W.q_len.max())
    layer = m.KVLayer(W.H, W.d, max(W.N, 1), W.P, S, device)
    sid, pos = doc_tags(W.N, device)
    m.kv_append(layer, L.doc_k, L.doc_v, sid, pos)
    m.kv_append(layer, L.qk, L.qv, L.sid, L.pos)
    return layer


def oracle_decode(W, L, rows=None):
    k, v, ks, kp = decode_slots(L, W.N)
    q, qs, qp = decode_queries(L)
    if rows is not None:
        q, qs, qp = q[rows], qs[rows], qp[rows]
    return oracle.masked_attention(q, qs, qp, k, v, ks, kp, W.scale)


def oracle_prefill(W, L, rows=None):
    k, v, ks, kp = prefill_slots(L, W.N)
    q, qs, qp = prefill_queries(L)
    if rows is not None:
        q, qs, qp = q[rows], qs[rows], qp[rows]
    return oracle.masked_attention(q, qs, qp, k, v, ks, kp, W.scale)


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """Element-wise comparison against the oracle within the stated bar."""
    og = o_gpu.float().cpu().numpy().astype(np.float64)
    err = np.abs(og - o_ref)
    assert np.isfinite(og).all(), f"{what}: non-finite output"
    assert err.max() <= O_MAX, f"{what}: max |o err| {err.max():.3e}"
    assert err.mean() <= O_MEAN, f"{what}: mean |o err| {err.mean():.3e}"
    if lse_gpu is not None:
        lg = lse_gpu.cpu().numpy().astype(np.float64)
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lg), fin), f"{what}: lse finiteness differs"
        if fin.any():
            e2 = np.abs(lg[fin] - lse_ref[fin])
            assert e2.max() <= LSE_MAX, f"{what}: max |lse err| {e2.max():.3e}"
    return float(err.max()), float(err.mean())
