"""Pins of the oracle against things other than itself (CPU only).

Every test here checks oracle/ against a closed form, an invariant, a hand
example from the project page "Read Once, Answer Many", an independent
brute force, or a library routine -- chosen so that a dropped term, a wrong
sign or index, a leaked stream or a transposed operand fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from oracle.append import AppendReplay
from shared_context_decode_b200 import workloads as wl
from shared_context_decode_b200.workloads import bf16_bits
from tests.flat import decode_slots, decode_queries, prefill_slots, prefill_queries

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def f2bits(x):
    """float values exactly representable in bf16 -> bf16 bit patterns."""
    t = torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.tensor(np.asarray(x, np.float32))), "not exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


def small_decode(seed=0, **kw):
    shape = dict(layers=1, H=2, d=16, N=37, P=5, q=(2, 6), a=(0, 4))
    shape.update(kw)
    return wl.make_decode(seed=seed, **shape)


def run_oracle_decode(W, L):
    k, v, ks, kp = decode_slots(L, W.N)
    q, qs, qp = decode_queries(L)
    return oracle.masked_attention(q, qs, qp, k, v, ks, kp, W.scale)


# ---------------------------------------------------------------- pin 6 ----
def test_hand_two_token_example():
    g = json.load(open(os.path.join(GOLD, "two_token.json")))
    k = f2bits(np.array(g["k"]).reshape(-1, 1, 1))
    v = f2bits(np.array(g["v"]).reshape(-1, 1, 1))
    q = f2bits(np.array(g["q"]).reshape(1, 1, 1))
    o, lse, nvis = oracle.masked_attention(q, g["q_sid"], g["q_pos"], k, v,
                                           g["k_sid"], g["k_pos"], g["scale"])
    assert abs(o[0, 0, 0] - g["o"]) < 1e-15
    assert abs(lse[0, 0] - g["lse"]) < 1e-15
    assert nvis[0] == 2
    assert abs(o[0, 0, 0] - g["o_if_leaked"]) > 1.0


def test_hand_two_token_leak_would_be_caught():
    """The same example with stream 2 relabelled as stream 1 (a planted leak)
    gives the leaked value, so the pin above has teeth."""
    g = json.load(open(os.path.join(GOLD, "two_token.json")))
    k = f2bits(np.array(g["k"]).reshape(-1, 1, 1))
    v = f2bits(np.array(g["v"]).reshape(-1, 1, 1))
    q = f2bits(np.array(g["q"]).reshape(1, 1, 1))
    o, _, _ = oracle.masked_attention(q, g["q_sid"], g["q_pos"], k, v,
                                      [0, 1, 1], g["k_pos"], g["scale"])
    assert abs(o[0, 0, 0] - g["o_if_leaked"]) < 1e-12


# ---------------------------------------------------------------- pin 5 ----
def test_mask_figure_hand_matrix():
    g = json.load(open(os.path.join(GOLD, "mask_figure.json")))
    m = oracle.visibility(g["q_sid"], g["q_pos"], g["k_sid"], g["k_pos"])
    assert m.tolist() == g["mask"]


def test_visibility_count_closed_form_decode():
    W = small_decode(seed=3, P=9, q=(1, 7), a=(0, 5))
    L = W.layer(0)
    _, _, nvis = run_oracle_decode(W, L)
    expect = W.N + W.q_len + W.a_len + 1
    assert np.array_equal(nvis, expect.astype(np.int32))


def test_visibility_count_closed_form_prefill():
    W = wl.make_prefill(layers=1, H=1, d=8, N=11, P=6, q=(1, 9), seed=2)
    L = W.layer(0)
    k, v, ks, kp = prefill_slots(L, W.N)
    q, qs, qp = prefill_queries(L)
    _, _, nvis = oracle.masked_attention(q, qs, qp, k, v, ks, kp, W.scale)
    off = L.row_off.numpy()
    expect = np.concatenate([W.N + np.arange(n) + 1 for n in W.q_len])
    assert np.array_equal(nvis, expect)
    assert off[-1] == W.R


def test_inactive_rows_and_doc_queries():
    """Inactive rows (sid -1) see nothing; a document query (sid 0) is
    causal over the document and sees no stream token."""
    m = oracle.visibility([-1, 0, 0], [9, 0, 2], [0, 0, 0, 1, -1], [0, 1, 2, 3, 3])
    assert m.tolist() == [[0, 0, 0, 0, 0], [1, 0, 0, 0, 0], [1, 1, 1, 0, 0]]


# ---------------------------------------------------------------- pin 1 ----
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_equals_per_stream_causal_brute_force(seed):
    W = small_decode(seed=seed)
    L = W.layer(0)
    o, lse, _ = run_oracle_decode(W, L)
    streams = []
    sid = L.suf_sid.numpy()
    for s in range(1, W.P + 1):
        rows = np.nonzero(sid == s)[0]
        i = s - 1
        streams.append(dict(
            k=np.concatenate([bf16_bits(L.suf_k)[rows], bf16_bits(L.new_k)[i:i + 1]]),
            v=np.concatenate([bf16_bits(L.suf_v)[rows], bf16_bits(L.new_v)[i:i + 1]]),
            pos=np.concatenate([L.suf_pos.numpy()[rows], L.q_pos.numpy()[i:i + 1]]),
            q=bf16_bits(L.q)[i:i + 1], q_pos=L.q_pos.numpy()[i:i + 1]))
    ref = brute.per_stream_causal(bf16_bits(L.doc_k), bf16_bits(L.doc_v), streams, W.scale)
    for s in range(W.P):
        np.testing.assert_allclose(o[s], ref[s][0][0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[s], ref[s][1][0], rtol=0, atol=1e-11)


def test_tiny_config_equals_brute_force():
    W = wl.make_decode("tiny")
    L = W.layer(0)
    o, lse, nvis = run_oracle_decode(W, L)
    assert np.all(nvis == 256 + 8 + 3 + 1)
    sid = L.suf_sid.numpy()
    for s in range(1, W.P + 1):
        rows = np.nonzero(sid == s)[0]
        i = s - 1
        st = dict(k=np.concatenate([bf16_bits(L.suf_k)[rows], bf16_bits(L.new_k)[i:i + 1]]),
                  v=np.concatenate([bf16_bits(L.suf_v)[rows], bf16_bits(L.new_v)[i:i + 1]]),
                  pos=np.concatenate([L.suf_pos.numpy()[rows], L.q_pos.numpy()[i:i + 1]]),
                  q=bf16_bits(L.q)[i:i + 1], q_pos=L.q_pos.numpy()[i:i + 1])
        (ro, rl), = brute.per_stream_causal(bf16_bits(L.doc_k), bf16_bits(L.doc_v), [st], W.scale)
        np.testing.assert_allclose(o[i], ro[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[i], rl[0], rtol=0, atol=1e-11)


def test_prefill_equals_brute_force():
    W = wl.make_prefill(layers=1, H=2, d=16, N=29, P=4, q=(1, 7), seed=5)
    L = W.layer(0)
    k, v, ks, kp = prefill_slots(L, W.N)
    q, qs, qp = prefill_queries(L)
    o, lse, _ = oracle.masked_attention(q, qs, qp, k, v, ks, kp, W.scale)
    off = L.row_off.numpy()
    for s in range(W.P):
        r = slice(off[s], off[s + 1])
        st = dict(k=bf16_bits(L.qk)[r], v=bf16_bits(L.qv)[r], pos=L.pos.numpy()[r],
                  q=bf16_bits(L.q)[r], q_pos=L.pos.numpy()[r])
        (ro, rl), = brute.per_stream_causal(bf16_bits(L.doc_k), bf16_bits(L.doc_v), [st], W.scale)
        np.testing.assert_allclose(o[r], ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[r], rl, rtol=0, atol=1e-11)


def test_brute_force_catches_a_leak():
    """Planted mistake (in the oracle's inputs, on the CPU): collapse all
    stream ids into one stream.  The brute force must then disagree."""
    W = small_decode(seed=4)
    L = W.layer(0)
    k, v, ks, kp = decode_slots(L, W.N)
    q, qs, qp = decode_queries(L)
    ks_leak = np.where(ks > 0, 1, ks)
    qs_leak = np.where(qs > 0, 1, qs)
    o_leak, _, _ = oracle.masked_attention(q, qs_leak, qp, k, v, ks_leak, kp, W.scale)
    o, _, _ = oracle.masked_attention(q, qs, qp, k, v, ks, kp, W.scale)
    assert np.abs(o_leak - o).max() > 1e-3


# ---------------------------------------------------------------- pin 2 ----
def test_stream_permutation_equivariance():
    W = small_decode(seed=7, P=7)
    L = W.layer(0)
    k, v, ks, kp = decode_slots(L, W.N)
    q, qs, qp = decode_queries(L)
    o, lse, _ = oracle.masked_attention(q, qs, qp, k, v, ks, kp, W.scale)
    rng = np.random.default_rng(11)
    perm = rng.permutation(W.P) + 1                # stream s -> perm[s-1]
    relabel = np.concatenate([[0], perm])
    ks2 = np.where(ks > 0, relabel[np.maximum(ks, 0)], ks)
    order = rng.permutation(len(ks))               # shuffle the slot order too
    qorder = rng.permutation(W.P)                  # and the query rows
    qs2 = relabel[qs[qorder]]
    o2, lse2, _ = oracle.masked_attention(q[qorder], qs2, qp[qorder], k[order], v[order],
                                          ks2[order], kp[order], W.scale)
    np.testing.assert_allclose(o2, o[qorder], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse[qorder], rtol=0, atol=1e-11)


# ---------------------------------------------------------------- pin 3 ----
def test_constant_v_rows_give_that_row():
    W = small_decode(seed=8)
    L = W.layer(0)
    k, v, ks, kp = decode_slots(L, W.N)
    q, qs, qp = decode_queries(L)
    c = f2bits(np.array([[0.5, -1.25, 3.0, 0.0625] * (W.d // 4)] * W.H))   # [H,d]
    v_const = np.broadcast_to(c, v.shape).copy()
    o, _, _ = oracle.masked_attention(q, qs, qp, k, v_const, ks, kp, W.scale)
    cf = brute.bf16_bits_to_f64(c)
    for i in range(W.P):
        np.testing.assert_allclose(o[i], cf, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- pin 4 ----
def test_identical_keys_give_mean_of_visible_v():
    W = small_decode(seed=9)
    L = W.layer(0)
    k, v, ks, kp = decode_slots(L, W.N)
    q, qs, qp = decode_queries(L)
    k_same = np.broadcast_to(k[0], k.shape).copy()
    o, lse, nvis = oracle.masked_attention(q, qs, qp, k_same, v, ks, kp, W.scale)
    vf = brute.bf16_bits_to_f64(v)
    kf = brute.bf16_bits_to_f64(k[0])
    qf = brute.bf16_bits_to_f64(q)
    for i in range(W.P):
        vis = (ks == 0) | ((ks == qs[i]) & (kp <= qp[i]))
        assert vis.sum() == nvis[i]
        np.testing.assert_allclose(o[i], vf[vis].mean(axis=0), rtol=0, atol=1e-12)
        x = W.scale * np.einsum("hd,hd->h", qf[i], kf)
        np.testing.assert_allclose(lse[i], x + math.log(nvis[i]), rtol=0, atol=1e-11)


# ---------------------------------------------------------------- pin 7 ----
def test_single_stream_no_suffix_is_plain_sdpa():
    W = wl.make_decode(layers=1, H=3, d=32, N=50, P=1, q=(0, 0), a=(0, 0), seed=12)
    L = W.layer(0)
    o, lse, nvis = run_oracle_decode(W, L)
    assert nvis[0] == W.N + 1
    kk = torch.cat([L.doc_k, L.new_k]).double()     # [N+1,H,d]
    vv = torch.cat([L.doc_v, L.new_v]).double()
    qq = L.q.double()                               # [1,H,d]
    ref = torch.nn.functional.scaled_dot_product_attention(
        qq.permute(1, 0, 2)[None], kk.permute(1, 0, 2)[None], vv.permute(1, 0, 2)[None],
        scale=W.scale)[0].permute(1, 0, 2)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
    ref_lse = torch.logsumexp(W.scale * torch.einsum("hd,nhd->hn", qq[0], kk), dim=1)
    np.testing.assert_allclose(lse[0], ref_lse.numpy(), rtol=0, atol=1e-11)


def test_empty_visible_set():
    q = f2bits(np.ones((1, 1, 2)))
    k = f2bits(np.ones((1, 1, 2)))
    o, lse, nvis = oracle.masked_attention(q, [2], [5], k, k, [1], [0], 1.0)
    assert nvis[0] == 0 and np.all(o == 0) and lse[0, 0] == -np.inf


# ------------------------------------------------------- append replay -----
def test_append_replay_hand_fixture():
    g = json.load(open(os.path.join(GOLD, "append_replay.json")))
    R = AppendReplay(g["P_max"], g["S_cap"], g["doc_cap"])
    for call in g["calls"]:
        n = len(call["sid"])
        rows = np.array(call["tag"], np.int64).reshape(n, 1, 1)
        R.append(rows, -rows, call["sid"], call["pos"])
    for s_str, slots in g["segments"].items():
        s = int(s_str)
        got = [[int(t[0][0, 0]), int(t[2]), int(t[3])] for t in R.seg[s]]
        assert got == slots, (s, got)
        assert all(int(t[1][0, 0]) == -int(t[0][0, 0]) for t in R.seg[s])
    assert {int(p): int(kv[0][0, 0]) for p, kv in R.doc.items()} == \
        {int(p): t for p, t in g["doc"].items()}
    assert sorted(R.flags) == sorted(g["flags"])


def test_append_replay_invariants():
    """Random calls: per stream, stored rows are the accepted rows in call
    order; totals add up; nothing is invented."""
    rng = np.random.default_rng(3)
    P, S, D = 6, 9, 20
    R = AppendReplay(P, S, D)
    sent = {s: [] for s in range(1, P + 1)}
    tag = 0
    for _ in range(12):
        n = int(rng.integers(0, 8))
        sid = rng.integers(-1, P + 1, size=n)
        pos = rng.integers(0, D, size=n)
        rows = np.arange(tag, tag + n).reshape(n, 1, 1)
        tag += n
        R.append(rows, rows, sid, pos)
        for i in range(n):
            if sid[i] >= 1:
                sent[int(sid[i])].append(int(rows[i, 0, 0]))
    for s in range(1, P + 1):
        got = [int(t[0][0, 0]) for t in R.seg[s]]
        assert got == sent[s][:S]
        assert R.length(s) == min(len(sent[s]), S)
    assert ("segment_overflow" in R.flags) == any(len(sent[s]) > S for s in sent)


def test_document_queries_equal_causal_brute_force():
    """Document prefill (project page "Read Once, Answer Many", section "How
    it works": the document is encoded once): a document token (stream 0)
    attends to the document tokens at or before its position -- ordinary
    causal attention, checked against the stream-free brute force."""
    rng = np.random.default_rng(7)
    N, H, d = 37, 2, 8

    def rbits(shape):   # random values rounded to bf16
        t = torch.tensor(rng.standard_normal(shape), dtype=torch.float32).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16)

    k, v, q = rbits((N, H, d)), rbits((N, H, d)), rbits((N, H, d))
    pos = np.arange(N, dtype=np.int32)
    # a stream token that no document query may see
    k2 = np.concatenate([k, rbits((1, H, d))])
    v2 = np.concatenate([v, f2bits(100.0 * np.ones((1, H, d)))])
    ks = np.concatenate([np.zeros(N, np.int32), [1]])
    kp = np.concatenate([pos, [N]])
    o, lse, nvis = oracle.masked_attention(q, np.zeros(N, np.int32), pos, k2, v2, ks, kp, 0.3)
    ref_o, ref_lse = brute.causal_attention(brute.bf16_bits_to_f64(q), pos,
                                            brute.bf16_bits_to_f64(k), brute.bf16_bits_to_f64(v),
                                            pos, 0.3)
    np.testing.assert_allclose(o, ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-11)
    assert nvis.tolist() == list(range(1, N + 1))


def test_append_replay_refill_hand_case():
    """Refill rule by hand: after stream 2 is reset its next row lands in slot
    0 again, other streams keep their slots, -1 is ignored and an id outside
    1..P_max raises bad_stream."""
    R = AppendReplay(3, 4, 8)
    rows = np.arange(1, 7, dtype=np.int64).reshape(6, 1, 1)
    R.append(rows, -rows, [1, 2, 2, 3, 2, 1], [10, 10, 11, 10, 12, 11])
    assert [R.length(s) for s in (1, 2, 3)] == [2, 3, 1]
    R.reset_streams([2, -1])
    assert [R.length(s) for s in (1, 2, 3)] == [2, 0, 1] and not R.flags
    R.append(np.array([[[7]]]), np.array([[[-7]]]), [2], [10])
    assert [(int(t[0][0, 0]), t[2], t[3]) for t in R.seg[2]] == [(7, 2, 10)]
    assert [int(t[0][0, 0]) for t in R.seg[1]] == [1, 6]
    R.reset_streams([4])
    assert R.flags == {"bad_stream"}
