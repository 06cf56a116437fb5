"""pp_decode_attn_noalloc: decode attention for callers that cannot allocate
device memory (for example a plugin inside a host application that owns all
device memory and offers it no allocator, or a serving loop that forbids
cudaMalloc after start-up because it can synchronise the device).

It runs the same kernels on the same split as pp_decode_attn with a
caller-allocated workspace, so it must give the same bits, call after call
(its built-in scratch is reused); it must refuse work that needs more
scratch than it has, and report argument errors as pp_decode_attn does.  This file is collected
last, so a run that stops at the first failure has run everything else."""
import numpy as np
import pytest
import torch

from shared_context_decode_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _compare_to_workspace_call(W, l=0):
    m = gu.pp()
    L = W.layer(l)
    layer = gu.load_decode(W, L, DEV)
    lse_ref = torch.empty((W.P, W.H), dtype=torch.float32, device=DEV)
    o_ref = m.decode_attn(layer, W.N, L.q, L.q_sid, L.q_pos, W.scale, lse=lse_ref)
    o = torch.empty_like(L.q)
    lse = torch.empty((W.P, W.H), dtype=torch.float32, device=DEV)
    m.decode_attn_noalloc(layer, W.N, L.q, L.q_sid, L.q_pos, W.scale, o=o, lse=lse)
    torch.cuda.synchronize()
    assert m.device_status(layer) == 0
    assert torch.isfinite(o.float()).all()
    assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(lse, lse_ref)


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row():
    # first call: two M tiles, ragged document tail; second call: a different
    # shape right after, reusing the same built-in scratch
    _compare_to_workspace_call(
        wl.make_decode(layers=1, H=4, d=128, N=1000, P=200, q=(1, 20), a=(0, 10), seed=21,
                       device=DEV))
    _compare_to_workspace_call(
        wl.make_decode(layers=1, H=8, d=128, N=3000, P=64, q=(4, 30), a=(0, 20), seed=22,
                       device=DEV))


def test_noalloc_rejects_work_beyond_its_scratch():
    m = gu.pp()
    H, d, N, P = 32, 128, 16384, 2048       # 8 row groups x 32 heads of partials
    need = m.decode_workspace_bytes(P, H, d, N)
    assert need > m.NOALLOC_SCRATCH_BYTES
    layer = m.KVLayer(H, d, N, P, 8, DEV)
    q = torch.zeros((P, H, d), dtype=torch.bfloat16, device=DEV)
    sid = torch.arange(1, P + 1, dtype=torch.int16, device=DEV)
    pos = torch.full((P,), N, dtype=torch.int32, device=DEV)
    o = torch.full_like(q, 7.0)
    with pytest.raises(m.PPError) as e:
        m.decode_attn_noalloc(layer, N, q, sid, pos, 0.1, o=o)
    assert e.value.status == m.PP_ERR_CAPACITY
    torch.cuda.synchronize()
    assert torch.all(o == 7.0)               # nothing was launched
    # more rows than the layer has streams: the argument error comes first,
    # with pp_decode_attn's code, although the size is also too large
    small = m.KVLayer(H, d, N, 8, 8, DEV)
    with pytest.raises(m.PPError) as e:
        m.decode_attn_noalloc(small, N, q, sid, pos, 0.1, o=o)
    assert e.value.status == m.PP_ERR_UNSUPPORTED
