"""numpy fp64 brute force -- TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The project page "Read Once, Answer Many" (section "How it works") claims
that with the stream mask and shared positions every answer is the same as
decoding its question alone.  This module computes that "alone" result
directly: for one stream it concatenates the document with that stream's own
question and answer tokens, orders them by position, and runs ordinary causal
softmax attention (a query at position p sees every token at position <= p).
No stream ids appear anywhere in this computation.
"""
import numpy as np


def bf16_bits_to_f64(a):
    """Exact bf16 -> float64: a bf16 value is the top half of a binary32."""
    a = np.asarray(a, dtype=np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def causal_attention(q, q_pos, k, v, k_pos, scale):
    """Plain causal attention of one sequence.

    q [nq,H,d], k/v [nk,H,d] float64; q_pos [nq], k_pos [nk].
    Returns o [nq,H,d] and lse [nq,H] (natural log); an empty visible set
    gives o = 0, lse = -inf.
    """
    nq, H, d = q.shape
    o = np.zeros((nq, H, d))
    lse = np.full((nq, H), -np.inf)
    for i in range(nq):
        sel = np.nonzero(np.asarray(k_pos) <= q_pos[i])[0]
        if sel.size == 0:
            continue
        for h in range(H):
            x = scale * (k[sel, h, :] @ q[i, h, :])
            m = x.max()
            w = np.exp(x - m)
            z = w.sum()
            o[i, h] = (w @ v[sel, h, :]) / z
            lse[i, h] = m + np.log(z)
    return o, lse


def per_stream_causal(doc_k, doc_v, streams, scale):
    """Answer every stream as if its question were the only one.

    doc_k, doc_v: bf16 bits [N,H,d] (document token i has position i).
    streams: list of dicts with bf16-bit arrays 'k', 'v' [L,H,d] and int
    'pos' [L] for the stream's own cached tokens, and 'q' [nq,H,d] with
    'q_pos' [nq] for its queries.
    Returns a list of (o, lse) per stream.
    """
    N = np.asarray(doc_k).shape[0]
    dk, dv = bf16_bits_to_f64(doc_k), bf16_bits_to_f64(doc_v)
    out = []
    for st in streams:
        sk, sv = bf16_bits_to_f64(st["k"]), bf16_bits_to_f64(st["v"])
        order = np.argsort(np.asarray(st["pos"]), kind="stable")
        k = np.concatenate([dk, sk[order]], axis=0)
        v = np.concatenate([dv, sv[order]], axis=0)
        kpos = np.concatenate([np.arange(N), np.asarray(st["pos"])[order]])
        out.append(causal_attention(bf16_bits_to_f64(st["q"]), np.asarray(st["q_pos"]),
                                    k, v, kpos, scale))
    return out
