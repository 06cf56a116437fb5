"""GPU integer bookkeeping, bit-exact: appended K/V bits, slot tags and
lengths against the append replay, and the kernels' visibility predicate
against the oracle's mask rule."""
import numpy as np
import pytest
import torch

import oracle
from oracle.append import AppendReplay
from shared_context_decode_b200 import workloads as wl
from shared_context_decode_b200.workloads import bf16_bits
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_append_matches_replay_bit_exact():
    m = gu.pp()
    H, d, P_max, S_cap, doc_cap = 3, 64, 6, 7, 50
    layer = m.KVLayer(H, d, doc_cap, P_max, S_cap, DEV)
    m.kv_reset(layer)
    R = AppendReplay(P_max, S_cap, doc_cap)
    rng = np.random.default_rng(5)
    for call in range(10):
        n = int(rng.integers(1, 12))
        sid = rng.integers(-1, P_max + 2, size=n).astype(np.int16)   # includes bad ids
        pos = rng.integers(-2, doc_cap + 3, size=n).astype(np.int32)  # includes out of range
        k = wl.randn_bf16((n, H, d), 100 + call, DEV)
        v = wl.randn_bf16((n, H, d), 200 + call, DEV)
        m.kv_append(layer, k, v, torch.from_numpy(sid).to(DEV), torch.from_numpy(pos).to(DEV))
        R.append(bf16_bits(k), bf16_bits(v), sid, pos)
    torch.cuda.synchronize()
    ln = layer.len.cpu().numpy()
    ks, vs = bf16_bits(layer.k_suf), bf16_bits(layer.v_suf)     # [P_max, H, S_cap, d]
    tag_s, tag_p = layer.sid.cpu().numpy(), layer.pos.cpu().numpy()
    for s in range(1, P_max + 1):
        assert ln[s - 1] == R.length(s)
        for t, (kk, vv, ss, pp_) in enumerate(R.seg[s]):
            assert np.array_equal(ks[s - 1, :, t, :], kk)
            assert np.array_equal(vs[s - 1, :, t, :], vv)
            assert tag_s[s - 1, t] == ss and tag_p[s - 1, t] == pp_
    kd, vd = bf16_bits(layer.k_doc), bf16_bits(layer.v_doc)     # [H, doc_cap, d]
    for p, (kk, vv) in R.doc.items():
        assert np.array_equal(kd[:, p, :], kk) and np.array_equal(vd[:, p, :], vv)
    flags = {"segment_overflow": m.PP_DEV_SEGMENT_OVERFLOW,
             "doc_out_of_range": m.PP_DEV_DOC_OUT_OF_RANGE, "bad_stream": m.PP_DEV_BAD_STREAM}
    expect = 0
    for f in R.flags:
        expect |= flags[f]
    assert m.device_status(layer) == expect


@pytest.mark.parametrize("n", [300, 3000, 20000])
def test_large_mixed_calls_match_replay_bit_exact(n):
    """Calls large enough that one CTA takes many rows (up to 64): stream,
    document, inactive and out-of-range rows mixed, streams repeated, some
    segments overflowing."""
    m = gu.pp()
    H, d, P_max, doc_cap = 1, 64, 37, 400
    S_cap = max(8, n // (2 * P_max))
    layer = m.KVLayer(H, d, doc_cap, P_max, S_cap, DEV)
    m.kv_reset(layer)
    R = AppendReplay(P_max, S_cap, doc_cap)
    rng = np.random.default_rng(n)
    for call in range(2):
        sid = rng.integers(-1, P_max + 3, size=n).astype(np.int16)
        pos = rng.integers(-2, doc_cap + 2, size=n).astype(np.int32)
        # document rows of one call take distinct positions (two rows of a
        # call at one document position are the caller's error)
        doc_rows = np.nonzero(sid == 0)[0]
        free = rng.permutation(np.arange(-2, doc_cap + 2)).astype(np.int32)
        take = min(len(doc_rows), len(free))
        pos[doc_rows[:take]] = free[:take]
        sid[doc_rows[take:]] = -1
        k = wl.randn_bf16((n, H, d), 300 + call, DEV)
        v = wl.randn_bf16((n, H, d), 400 + call, DEV)
        m.kv_append(layer, k, v, torch.from_numpy(sid).to(DEV), torch.from_numpy(pos).to(DEV))
        R.append(bf16_bits(k), bf16_bits(v), sid, pos)
    torch.cuda.synchronize()
    ln = layer.len.cpu().numpy()
    ks, vs = bf16_bits(layer.k_suf), bf16_bits(layer.v_suf)
    tag_s, tag_p = layer.sid.cpu().numpy(), layer.pos.cpu().numpy()
    for s in range(1, P_max + 1):
        assert ln[s - 1] == R.length(s)
        seg = R.seg[s]
        if seg:
            assert np.array_equal(ks[s - 1, :, :len(seg), :], np.stack([x[0] for x in seg], 1))
            assert np.array_equal(vs[s - 1, :, :len(seg), :], np.stack([x[1] for x in seg], 1))
            assert np.array_equal(tag_s[s - 1, :len(seg)], [x[2] for x in seg])
            assert np.array_equal(tag_p[s - 1, :len(seg)], [x[3] for x in seg])
    kd, vd = bf16_bits(layer.k_doc), bf16_bits(layer.v_doc)
    for p_, (kk, vv) in R.doc.items():
        assert np.array_equal(kd[:, p_, :], kk) and np.array_equal(vd[:, p_, :], vv)
    flags = {"segment_overflow": m.PP_DEV_SEGMENT_OVERFLOW,
             "doc_out_of_range": m.PP_DEV_DOC_OUT_OF_RANGE, "bad_stream": m.PP_DEV_BAD_STREAM}
    expect = 0
    for f in R.flags:
        expect |= flags[f]
    assert expect & m.PP_DEV_SEGMENT_OVERFLOW
    assert m.device_status(layer) == expect


def test_append_many_rows_per_stream_keeps_call_order():
    m = gu.pp()
    H, d, P_max, S_cap = 2, 128, 4, 300
    layer = m.KVLayer(H, d, 8, P_max, S_cap, DEV)
    n = 1000
    rng = np.random.default_rng(6)
    sid = rng.integers(1, P_max + 1, size=n).astype(np.int16)
    pos = np.arange(n, dtype=np.int32)
    k = wl.randn_bf16((n, H, d), 7, DEV)
    m.kv_append(layer, k, k, torch.from_numpy(sid).to(DEV), torch.from_numpy(pos).to(DEV))
    R = AppendReplay(P_max, S_cap, 8)
    R.append(bf16_bits(k), bf16_bits(k), sid, pos)
    torch.cuda.synchronize()
    tag_p = layer.pos.cpu().numpy()
    for s in range(1, P_max + 1):
        want = [t[3] for t in R.seg[s]]
        assert layer.len[s - 1].item() == len(want)
        assert np.array_equal(tag_p[s - 1, :len(want)], want)
    assert m.device_status(layer) == (m.PP_DEV_SEGMENT_OVERFLOW if R.flags else 0)


@pytest.mark.parametrize("seed", [0, 1])
def test_visibility_matches_oracle_bit_exact(seed):
    m = gu.pp()
    W = wl.make_decode(layers=1, H=1, d=64, N=37, P=11, q=(1, 9), a=(0, 6), seed=seed, device=DEV)
    active = np.arange(W.P) % 4 != 3
    L = W.layer(0, active=active)
    S_cap = W.S_need + 2
    layer = gu.load_decode(W, L, DEV, S_cap=S_cap)
    # queries: every decode token plus every cached token of every stream
    # (positions inside the stream see only a prefix of it)
    q_sid = np.concatenate([L.q_sid.cpu().numpy(), L.suf_sid.cpu().numpy(), [0, 12, -1]])
    q_pos = np.concatenate([L.q_pos.cpu().numpy(), L.suf_pos.cpu().numpy(), [5, 40, 40]])
    qs_t = torch.from_numpy(q_sid.astype(np.int16)).to(DEV)
    qp_t = torch.from_numpy(q_pos.astype(np.int32)).to(DEV)
    count, mask = m.debug_visibility(layer, W.N, qs_t, qp_t)
    torch.cuda.synchronize()
    # oracle over the segment slots in layout order; unused slots get sid -1
    slot_sid = np.full((W.P, S_cap), -1, np.int32)
    slot_pos = np.zeros((W.P, S_cap), np.int32)
    suf_sid, suf_pos = L.suf_sid.cpu().numpy(), L.suf_pos.cpu().numpy()
    for s in range(1, W.P + 1):
        rows = list(suf_pos[suf_sid == s])
        if active[s - 1]:
            rows.append(int(L.q_pos[s - 1]))
        slot_sid[s - 1, :len(rows)] = s
        slot_pos[s - 1, :len(rows)] = rows
    ref = oracle.visibility(q_sid, q_pos, slot_sid.ravel(), slot_pos.ravel())
    # stream queries (sid 1..P_max) only: document queries and bad ids are
    # served by no kernel and report nothing
    sq = (q_sid >= 1) & (q_sid <= W.P)
    got = mask.cpu().numpy()
    assert np.array_equal(got[sq], ref[sq])
    assert not got[~sq].any()
    # counts include the document, and equal the oracle's visible-set sizes
    k_sid = np.concatenate([np.zeros(W.N, np.int32), slot_sid.ravel()])
    k_pos = np.concatenate([np.arange(W.N, dtype=np.int32), slot_pos.ravel()])
    full = oracle.visibility(q_sid, q_pos, k_sid, k_pos)
    c = count.cpu().numpy()
    assert np.array_equal(c[sq], full[sq].sum(axis=1))
    assert np.all(c[~sq] == 0)
    # closed form for the decode tokens: N + q_s + a_s + 1
    dec = np.nonzero(active)[0]
    assert np.array_equal(c[dec], (W.N + W.q_len + W.a_len + 1)[dec])
