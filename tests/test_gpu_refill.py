"""Continuous-batching refill on the GPU: pp_kv_reset_streams frees a finished
stream's segment for a new question.  Bookkeeping bit-exact against the
append replay; attention after a refill against the oracle; the refill inside
a fixed-shape CUDA graph."""
import numpy as np
import pytest
import torch

import oracle
from oracle.append import AppendReplay
from shared_context_decode_b200 import workloads as wl
from shared_context_decode_b200.workloads import bf16_bits
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0) if torch.cuda.is_available() else None


def test_resets_between_appends_match_replay_bit_exact():
    m = gu.pp()
    H, d, P_max, S_cap, doc_cap = 2, 64, 5, 9, 16
    layer = m.KVLayer(H, d, doc_cap, P_max, S_cap, DEV)
    R = AppendReplay(P_max, S_cap, doc_cap)
    rng = np.random.default_rng(8)
    for call in range(14):
        if call % 3 == 2:
            ids = rng.integers(-1, P_max + 2, size=3).astype(np.int16)   # includes -1 and bad ids
            m.kv_reset_streams(layer, torch.from_numpy(ids).to(DEV))
            R.reset_streams(ids)
            continue
        n = int(rng.integers(1, 10))
        sid = rng.integers(1, P_max + 1, size=n).astype(np.int16)
        pos = rng.integers(0, 100, size=n).astype(np.int32)
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
        for t, (kk, vv, ss, pp_) in enumerate(R.seg[s]):
            assert np.array_equal(ks[s - 1, :, t, :], kk) and np.array_equal(vs[s - 1, :, t, :], vv)
            assert tag_s[s - 1, t] == ss and tag_p[s - 1, t] == pp_
    bits = {"segment_overflow": m.PP_DEV_SEGMENT_OVERFLOW,
            "doc_out_of_range": m.PP_DEV_DOC_OUT_OF_RANGE, "bad_stream": m.PP_DEV_BAD_STREAM}
    expect = 0
    for f in R.flags:
        expect |= bits[f]
    assert "bad_stream" in R.flags          # the random resets did include a bad id
    assert m.device_status(layer) == expect


def refill_case(H=2, d=128, N=300, seed=0):
    """Three streams decode; stream 2 finishes, its segment is refilled with a
    new 6-token question, then every stream decodes one more token."""
    m = gu.pp()
    P, S_cap = 3, 24
    rnd = lambda shape, tag: wl.randn_bf16(shape, wl.seed_of("refill", tag, seed), DEV)
    layer = m.KVLayer(H, d, N, P, S_cap, DEV)
    doc_k, doc_v = rnd((N, H, d), "dk"), rnd((N, H, d), "dv")
    sid, pos = gu.doc_tags(N, DEV)
    m.kv_append(layer, doc_k, doc_v, sid, pos)
    lens = [5, 7, 4]                      # question + cached answer tokens per stream
    slots = []                            # (k, v, sid, pos) visible at the end
    for s, n in enumerate(lens, start=1):
        k, v = rnd((n, H, d), f"s{s}k"), rnd((n, H, d), f"s{s}v")
        sd = torch.full((n,), s, dtype=torch.int16, device=DEV)
        ps = torch.arange(N, N + n, dtype=torch.int32, device=DEV)
        m.kv_append(layer, k, v, sd, ps)
        if s != 2:
            slots.append((k, v, sd, ps))
    m.kv_reset_streams(layer, torch.tensor([2, -1], dtype=torch.int16, device=DEV))
    nk, nv = rnd((6, H, d), "newk"), rnd((6, H, d), "newv")
    sd = torch.full((6,), 2, dtype=torch.int16, device=DEV)
    ps = torch.arange(N, N + 6, dtype=torch.int32, device=DEV)
    m.kv_append(layer, nk, nv, sd, ps)
    slots.append((nk, nv, sd, ps))
    # the decode token of every stream
    qk, qv, q = rnd((P, H, d), "qk"), rnd((P, H, d), "qv"), rnd((P, H, d), "q")
    q_sid = torch.arange(1, P + 1, dtype=torch.int16, device=DEV)
    q_pos = torch.tensor([N + 5, N + 6, N + 4], dtype=torch.int32, device=DEV)
    m.kv_append(layer, qk, qv, q_sid, q_pos)
    slots.append((qk, qv, q_sid, q_pos))
    keys = [(doc_k, doc_v, sid, pos)] + slots
    k = np.concatenate([bf16_bits(a[0]) for a in keys])
    v = np.concatenate([bf16_bits(a[1]) for a in keys])
    ks = np.concatenate([a[2].cpu().numpy().astype(np.int32) for a in keys])
    kp = np.concatenate([a[3].cpu().numpy() for a in keys])
    return layer, q, q_sid, q_pos, (k, v, ks, kp), N


def test_attention_after_refill_matches_oracle():
    m = gu.pp()
    layer, q, q_sid, q_pos, (k, v, ks, kp), N = refill_case()
    assert layer.len.cpu().tolist() == [6, 7, 5]
    scale = 0.09
    lse = torch.empty((3, 2), dtype=torch.float32, device=DEV)
    o = m.decode_attn(layer, N, q, q_sid, q_pos, scale, lse=lse)
    torch.cuda.synchronize()
    assert m.device_status(layer) == 0
    ref_o, ref_lse, nvis = oracle.masked_attention(bf16_bits(q), q_sid.cpu().numpy(),
                                                   q_pos.cpu().numpy(), k, v, ks, kp, scale)
    # stream 2 sees the document, its new question and its decode token only
    assert nvis.tolist() == [N + 6, N + 7, N + 5]
    err = np.abs(o.float().cpu().numpy() - ref_o)
    assert err.max() <= gu.O_MAX and err.mean() <= gu.O_MEAN
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=gu.LSE_MAX)


def test_refill_inside_a_fixed_shape_graph():
    """One captured step = reset the listed streams, append, decode.  The list
    is a device tensor updated between replays (-1 = no refill)."""
    m = gu.pp()
    H, d, N, P, S_cap = 2, 64, 130, 4, 8
    layer = m.KVLayer(H, d, N, P, S_cap, DEV)
    dk = wl.randn_bf16((N, H, d), 1, DEV)
    dv = wl.randn_bf16((N, H, d), 2, DEV)
    sid, pos = gu.doc_tags(N, DEV)
    m.kv_append(layer, dk, dv, sid, pos)
    refill = torch.full((P,), -1, dtype=torch.int16, device=DEV)
    q_sid = torch.arange(1, P + 1, dtype=torch.int16, device=DEV)
    q_pos = torch.full((P,), N, dtype=torch.int32, device=DEV)
    nk = wl.randn_bf16((P, H, d), 3, DEV)
    nv = wl.randn_bf16((P, H, d), 4, DEV)
    q = wl.randn_bf16((P, H, d), 5, DEV)
    o = torch.empty_like(q)
    ws = m.workspace(m.decode_workspace_bytes(P, H, d, N), DEV)

    def body():
        m.kv_reset_streams(layer, refill)
        m.kv_append(layer, nk, nv, q_sid, q_pos)
        m.decode_attn(layer, N, q, q_sid, q_pos, 0.125, o=o, ws=ws)

    body()
    torch.cuda.synchronize()
    m.kv_reset(layer)
    m.kv_append(layer, dk, dv, sid, pos)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(DEV)
    s.wait_stream(torch.cuda.current_stream(DEV))
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            body()
    torch.cuda.current_stream(DEV).wait_stream(s)
    torch.cuda.synchronize()
    for step in range(3):               # streams grow by one token per step
        g.replay()
    torch.cuda.synchronize()
    assert layer.len.cpu().tolist() == [3, 3, 3, 3]
    refill.copy_(torch.tensor([3, -1, 1, -1], dtype=torch.int16))
    g.replay()                          # streams 1 and 3 restart: reset, then one token
    torch.cuda.synchronize()
    assert layer.len.cpu().tolist() == [1, 4, 1, 4]
    assert m.device_status(layer) == 0
