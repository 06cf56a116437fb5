"""Flatten generated workloads into the oracle's tagged-slot list.

Pure bookkeeping (concatenation of rows and their stream/position tags);
no attention arithmetic.  The decode token's own K/V is part of the list:
it is appended before the attention of its step.
"""
import numpy as np
import torch

from shared_context_decode_b200.workloads import bf16_bits


def _np(t):
    return t.detach().cpu().numpy() if isinstance(t, torch.Tensor) else np.asarray(t)


def decode_slots(L, N):
    """(k, v, k_sid, k_pos) for one DecodeLayer: document, cached stream
    rows, then the decode tokens."""
    k = np.concatenate([bf16_bits(L.doc_k), bf16_bits(L.suf_k), bf16_bits(L.new_k)])
    v = np.concatenate([bf16_bits(L.doc_v), bf16_bits(L.suf_v), bf16_bits(L.new_v)])
    sid = np.concatenate([np.zeros(N, np.int32), _np(L.suf_sid).astype(np.int32),
                          _np(L.q_sid).astype(np.int32)])
    pos = np.concatenate([np.arange(N, dtype=np.int32), _np(L.suf_pos).astype(np.int32),
                          _np(L.q_pos).astype(np.int32)])
    return k, v, sid, pos


def decode_queries(L):
    return bf16_bits(L.q), _np(L.q_sid).astype(np.int32), _np(L.q_pos).astype(np.int32)


def prefill_slots(L, N):
    k = np.concatenate([bf16_bits(L.doc_k), bf16_bits(L.qk)])
    v = np.concatenate([bf16_bits(L.doc_v), bf16_bits(L.qv)])
    sid = np.concatenate([np.zeros(N, np.int32), _np(L.sid).astype(np.int32)])
    pos = np.concatenate([np.arange(N, dtype=np.int32), _np(L.pos).astype(np.int32)])
    return k, v, sid, pos


def prefill_queries(L):
    return bf16_bits(L.q), _np(L.sid).astype(np.int32), _np(L.pos).astype(np.int32)
