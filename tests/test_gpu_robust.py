"""GPU robustness: a bounded in-kernel wait that is made to expire returns
an error status instead of hanging and leaves the context usable; a
captured decode step replays bit-identically; empty calls launch nothing."""
import numpy as np
import pytest
import torch

from shared_context_decode_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
DEV = "cuda"


def small():
    return wl.make_decode(layers=1, H=2, d=128, N=600, P=150, q=(1, 9), a=(0, 5), seed=11,
                          device=DEV)


def test_injected_timeout_reports_status_and_recovers():
    m = gu.pp()
    W = small()
    L = W.layer(0)
    layer = gu.load_decode(W, L, DEV)
    opt = m.Options(debug_inject_timeout=1, wait_limit_log2=22)   # ~2^22 cycles per wait
    m.decode_attn(layer, W.N, L.q, L.q_sid, L.q_pos, W.scale, opt=opt)
    torch.cuda.synchronize()
    rc, word = m.device_status_code(layer)
    assert word & m.PP_DEV_TIMEOUT and rc == m.PP_ERR_DEVICE_TIMEOUT
    # the context is intact: a normal call on the same layer is correct
    layer.status.zero_()
    lse = torch.empty((W.P, W.H), dtype=torch.float32, device=DEV)
    o = m.decode_attn(layer, W.N, L.q, L.q_sid, L.q_pos, W.scale, lse=lse)
    torch.cuda.synchronize()
    assert m.device_status_code(layer) == (m.PP_OK, 0)
    o_ref, lse_ref, _ = gu.oracle_decode(W, L)
    gu.compare(o, lse, o_ref, lse_ref, "after timeout")


def test_graph_replay_is_bit_identical():
    m = gu.pp()
    W = small()
    L = W.layer(0)
    layer = gu.load_decode(W, L, DEV)
    # cache state before the step's own append: undo the decode tokens
    len_after = layer.len.clone()
    len_before = len_after - (L.q_sid > 0).to(torch.int32)
    ws = m.workspace(m.decode_workspace_bytes(W.P, W.H, W.d, W.N), DEV)
    o = torch.empty_like(L.q)
    layer.len.copy_(len_before)
    m.kv_append(layer, L.new_k, L.new_v, L.q_sid, L.q_pos)
    m.decode_attn(layer, W.N, L.q, L.q_sid, L.q_pos, W.scale, o=o, ws=ws)
    torch.cuda.synchronize()
    eager = o.clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            layer.len.copy_(len_before)
            m.kv_append(layer, L.new_k, L.new_v, L.q_sid, L.q_pos)
            m.decode_attn(layer, W.N, L.q, L.q_sid, L.q_pos, W.scale, o=o, ws=ws)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, eager)
        assert torch.equal(layer.len, len_after)
    assert m.device_status(layer) == 0
    del g


def test_empty_calls():
    m = gu.pp()
    layer = m.KVLayer(2, 64, 16, 4, 8, DEV)
    e = torch.empty((0, 2, 64), dtype=torch.bfloat16, device=DEV)
    m.kv_append(layer, e, e, torch.empty((0,), dtype=torch.int16, device=DEV),
                torch.empty((0,), dtype=torch.int32, device=DEV))
    o = m.decode_attn(layer, 16, e, torch.empty((0,), dtype=torch.int16, device=DEV),
                      torch.empty((0,), dtype=torch.int32, device=DEV), 0.125)
    torch.cuda.synchronize()
    assert o.shape == (0, 2, 64)
    assert int(layer.len.sum()) == 0 and m.device_status(layer) == 0


def test_bad_query_stream_flagged():
    m = gu.pp()
    W = wl.make_decode(layers=1, H=2, d=64, N=64, P=3, q=(1, 2), a=(0, 1), seed=12, device=DEV)
    L = W.layer(0)
    layer = gu.load_decode(W, L, DEV)
    q_sid = L.q_sid.clone()
    q_sid[1] = 0          # a document query: not served by the decode call
    o = m.decode_attn(layer, W.N, L.q, q_sid, L.q_pos, W.scale)
    torch.cuda.synchronize()
    assert m.device_status(layer) & m.PP_DEV_BAD_STREAM
    assert torch.all(o[1] == 0)
