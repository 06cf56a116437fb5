"""pp_decode_step (append + attention in one call, the append inside the
document pass launch) against the two separate calls it replaces, and
against the oracle.

The separate calls are pp_kv_append (project page "Read Once, Answer Many",
section "How it works": each decode step appends one token per stream) and
pp_decode_attn; the step must leave the same slots, tags, lengths and device
flags and produce the same outputs bit for bit (the attention kernels are the
same; only where the append runs differs)."""
import numpy as np
import pytest
import torch

from oracle.append import AppendReplay
from shared_context_decode_b200 import workloads as wl
from shared_context_decode_b200.workloads import bf16_bits
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0) if torch.cuda.is_available() else None


def cached_layer(W, L, S_cap=None, P_max=None):
    """Layer l of decode workload W before the step: document and cached
    stream rows, not the decode tokens."""
    m = gu.pp()
    layer = m.KVLayer(W.H, W.d, max(W.N, 1), P_max or W.P, S_cap or W.S_need, DEV)
    if W.N:
        sid, pos = gu.doc_tags(W.N, DEV)
        m.kv_append(layer, L.doc_k, L.doc_v, sid, pos)
    if L.suf_sid.numel():
        m.kv_append(layer, L.suf_k, L.suf_v, L.suf_sid, L.suf_pos)
    return layer


def same_state(a, b):
    m = gu.pp()
    assert torch.equal(a.len, b.len)
    assert torch.equal(a.sid, b.sid) and torch.equal(a.pos, b.pos)
    assert torch.equal(a.k_suf.view(torch.int16), b.k_suf.view(torch.int16))
    assert torch.equal(a.v_suf.view(torch.int16), b.v_suf.view(torch.int16))
    assert torch.equal(a.k_doc.view(torch.int16), b.k_doc.view(torch.int16))
    assert m.device_status(a) == m.device_status(b)


def step_vs_separate(W, L, k, v, q, q_sid, q_pos, opt=None, S_cap=None, P_max=None):
    """Runs both ways on fresh copies of the cache; returns (o, lse, layer) of
    the step after checking it against the separate calls."""
    m = gu.pp()
    P = q_sid.shape[0]
    a = cached_layer(W, L, S_cap, P_max)
    b = cached_layer(W, L, S_cap, P_max)
    lse_a = torch.empty((P, W.H), dtype=torch.float32, device=DEV)
    lse_b = torch.empty_like(lse_a)
    # the step writes no document rows: the separate append gets them as -1
    sid_sep = torch.where(q_sid == 0, torch.full_like(q_sid, -1), q_sid)
    m.kv_append(a, k, v, sid_sep, q_pos)
    o_a = m.decode_attn(a, W.N, q, q_sid, q_pos, W.scale, lse=lse_a, opt=opt)
    o_b = m.decode_step(b, W.N, k, v, q, q_sid, q_pos, W.scale, lse=lse_b, opt=opt)
    torch.cuda.synchronize()
    same_state(a, b)
    assert torch.equal(o_a.view(torch.int16), o_b.view(torch.int16))
    assert torch.equal(lse_a, lse_b)
    return o_b, lse_b, b


@pytest.mark.parametrize("case", ["tiny", "ragged", "d64", "single"])
def test_step_equals_append_then_attend(case):
    W = {"tiny": lambda: wl.make_decode("tiny", device=DEV),
         "ragged": lambda: wl.make_decode(layers=1, H=4, d=128, N=1000, P=200, q=(1, 20),
                                          a=(0, 10), seed=1, device=DEV),
         "d64": lambda: wl.make_decode(layers=1, H=3, d=64, N=777, P=130, q=(2, 12), a=(0, 7),
                                       seed=3, device=DEV),
         "single": lambda: wl.make_decode(layers=1, H=2, d=128, N=129, P=1, q=(3, 3), a=(1, 1),
                                          seed=4, device=DEV)}[case]()
    L = W.layer(0)
    o, lse, _ = step_vs_separate(W, L, L.new_k, L.new_v, L.q, L.q_sid, L.q_pos)
    ref_o, ref_lse, _ = gu.oracle_decode(W, L)
    gu.compare(o, lse, ref_o, ref_lse, case)


@pytest.mark.parametrize("name", ["doc8k_p64", "doc16k_p256"])
def test_full_size_step_whole_layer(name):
    """The fused step at full size: every row and head of one layer."""
    W = wl.make_decode(name, layers=1, device=DEV)
    L = W.layer(0)
    o, lse, _ = step_vs_separate(W, L, L.new_k, L.new_v, L.q, L.q_sid, L.q_pos)
    ref_o, ref_lse, _ = gu.oracle_decode(W, L)
    gu.compare(o, lse, ref_o, ref_lse, f"{name} step")


def test_duplicates_overflow_and_bad_rows_bit_exact():
    """Two rows of one stream (ranks 0 and 1), a stream one slot short of full
    (its second row overflows), inactive rows, a stream-0 row and a stream
    past P_max: bookkeeping against the append replay, flags and outputs
    against the separate calls."""
    m = gu.pp()
    W = wl.make_decode(layers=1, H=2, d=128, N=300, P=6, q=(2, 5), a=(0, 2), seed=11, device=DEV)
    L = W.layer(0)
    S_cap = int(L.suf_sid.numel())   # generous; stream 4 is filled to S_cap - 1 below
    S_cap = max(S_cap, 16)
    # fill stream 4 up to S_cap - 1 before the step
    n4 = int((L.suf_sid == 4).sum().item())
    extra = S_cap - 1 - n4
    P_max = 10                       # room for the 10 rows; stream 11 is out of range
    sid_rows = torch.tensor([1, 2, 2, -1, 4, 4, 0, 11, 3, -1], dtype=torch.int16, device=DEV)
    R = sid_rows.shape[0]
    base_pos = {s: W.N + int((L.suf_sid == s).sum().item()) for s in range(1, W.P + 1)}
    pos_list, seen = [], {}
    for s in sid_rows.tolist():
        p = base_pos.get(s, 5000) + (extra if s == 4 else 0) + seen.get(s, 0)
        seen[s] = seen.get(s, 0) + 1
        pos_list.append(p)
    q_pos = torch.tensor(pos_list, dtype=torch.int32, device=DEV)
    k = wl.randn_bf16((R, W.H, W.d), 71, DEV)
    v = wl.randn_bf16((R, W.H, W.d), 72, DEV)
    q = wl.randn_bf16((R, W.H, W.d), 73, DEV)

    def prepared():
        lay = cached_layer(W, L, S_cap=S_cap, P_max=P_max)
        if extra > 0:
            m.kv_append(lay, wl.randn_bf16((extra, W.H, W.d), 74, DEV),
                        wl.randn_bf16((extra, W.H, W.d), 75, DEV),
                        torch.full((extra,), 4, dtype=torch.int16, device=DEV),
                        torch.arange(base_pos[4], base_pos[4] + extra, dtype=torch.int32,
                                     device=DEV))
        return lay

    a, b = prepared(), prepared()
    torch.cuda.synchronize()
    before = a.len.cpu().numpy().copy()
    sid_sep = torch.where(sid_rows == 0, torch.full_like(sid_rows, -1), sid_rows)
    m.kv_append(a, k, v, sid_sep, q_pos)
    o_a = m.decode_attn(a, W.N, q, sid_rows, q_pos, W.scale)
    o_b = m.decode_step(b, W.N, k, v, q, sid_rows, q_pos, W.scale)
    torch.cuda.synchronize()
    same_state(a, b)
    assert torch.equal(o_a.view(torch.int16), o_b.view(torch.int16))
    # the append replay from the cache state before the step
    R_ = AppendReplay(P_max, S_cap, max(W.N, 1))
    for s in range(1, P_max + 1):
        R_.seg[s] = [None] * int(before[s - 1])
    R_.append(bf16_bits(k), bf16_bits(v), sid_sep.cpu().numpy(), q_pos.cpu().numpy())
    ln = b.len.cpu().numpy()
    for s in range(1, P_max + 1):
        assert ln[s - 1] == R_.length(s)
    assert ln[1] == before[1] + 2 and ln[3] == S_cap          # duplicates; saturated at S_cap
    st = m.device_status(b)
    assert st & m.PP_DEV_SEGMENT_OVERFLOW and st & m.PP_DEV_BAD_STREAM
    # both rows of stream 2 landed in consecutive slots, in call order
    tags = b.pos.cpu().numpy()
    assert tags[1, before[1]] == pos_list[1] and tags[1, before[1] + 1] == pos_list[2]


@pytest.mark.parametrize("which", ["no_document", "ablation", "sibling_scan"])
def test_fallback_paths_equal_separate_calls(which):
    m = gu.pp()
    N = 0 if which == "no_document" else 500
    W = wl.make_decode(layers=1, H=2, d=128, N=N, P=20, q=(1, 9), a=(0, 6), seed=12, device=DEV)
    L = W.layer(0)
    opt = {"no_document": None, "ablation": m.Options(ablation_doc_per_stream=1),
           "sibling_scan": m.Options(sibling_scan=1)}[which]
    o, lse, _ = step_vs_separate(W, L, L.new_k, L.new_v, L.q, L.q_sid, L.q_pos, opt=opt)
    ref_o, ref_lse, _ = gu.oracle_decode(W, L)
    gu.compare(o, lse, ref_o, ref_lse, which)


def test_more_rows_than_the_fused_append_takes():
    # 4100 rows: the append kernels run first (the fused append stops at 4096)
    W = wl.make_decode(layers=1, H=1, d=64, N=130, P=4100, q=(1, 2), a=(0, 1), seed=13, device=DEV)
    L = W.layer(0)
    o, lse, _ = step_vs_separate(W, L, L.new_k, L.new_v, L.q, L.q_sid, L.q_pos)
    rows = np.array([0, 1, 2047, 4095, 4096, 4099])
    ref_o, ref_lse, _ = gu.oracle_decode(W, L, rows)
    gu.compare(o[rows], lse[rows], ref_o, ref_lse, "4100 rows")


def test_steps_in_a_graph_match_separate_calls():
    """Three decode steps captured once and replayed: the lengths the suffix
    pass stores are what the next replay's append reads."""
    m = gu.pp()
    W = wl.make_decode(layers=1, H=2, d=64, N=260, P=8, q=(1, 4), a=(0, 2), seed=14, device=DEV)
    L = W.layer(0)
    S_cap = W.S_need + 8
    a = cached_layer(W, L, S_cap=S_cap)
    b = cached_layer(W, L, S_cap=S_cap)
    pos = L.q_pos.clone()
    o_a, o_b = torch.empty_like(L.q), torch.empty_like(L.q)
    ws = m.workspace(m.decode_workspace_bytes(W.P, W.H, W.d, W.N), DEV)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(DEV)
    s.wait_stream(torch.cuda.current_stream(DEV))
    with torch.cuda.stream(s):
        m.decode_step(b, W.N, L.new_k, L.new_v, L.q, L.q_sid, pos, W.scale, o=o_b, ws=ws)
        torch.cuda.synchronize()
    b = cached_layer(W, L, S_cap=S_cap)   # warm-up done: start again from the cached state
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            m.decode_step(b, W.N, L.new_k, L.new_v, L.q, L.q_sid, pos, W.scale, o=o_b, ws=ws)
    torch.cuda.current_stream(DEV).wait_stream(s)
    torch.cuda.synchronize()
    for step in range(3):
        m.kv_append(a, L.new_k, L.new_v, L.q_sid, pos)
        m.decode_attn(a, W.N, L.q, L.q_sid, pos, W.scale, o=o_a)
        g.replay()
        torch.cuda.synchronize()
        same_state(a, b)
        assert torch.equal(o_a.view(torch.int16), o_b.view(torch.int16))
        pos += 1
