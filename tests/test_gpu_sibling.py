"""The sibling-scan comparison mode (pp_options.sibling_scan): every query
scans all streams' answer tokens and the stream mask rejects the siblings',
as the pages' kernel does.  Same result as the per-stream segments."""
import numpy as np
import pytest
import torch

from shared_context_decode_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0) if torch.cuda.is_available() else None


@pytest.mark.parametrize("H,d,N,P,seed", [(4, 128, 1000, 40, 0), (3, 64, 300, 130, 1),
                                         (2, 128, 0, 7, 2)])
def test_sibling_scan_decode_matches_oracle(H, d, N, P, seed):
    m = gu.pp()
    W = wl.make_decode(layers=1, H=H, d=d, N=N, P=P, q=(1, 12), a=(0, 6), seed=seed, device=DEV)
    L = W.layer(0)
    layer = gu.load_decode(W, L, DEV)
    lse = torch.empty((W.P, W.H), dtype=torch.float32, device=DEV)
    o = m.decode_attn(layer, W.N, L.q, L.q_sid, L.q_pos, W.scale, lse=lse,
                      opt=m.Options(sibling_scan=1))
    torch.cuda.synchronize()
    assert m.device_status(layer) == 0
    o_ref, lse_ref, _ = gu.oracle_decode(W, L)
    gu.compare(o, lse, o_ref, lse_ref, "sibling scan decode")
    # and the segment path gives the same answer within the same bar
    o2 = m.decode_attn(layer, W.N, L.q, L.q_sid, L.q_pos, W.scale)
    torch.cuda.synchronize()
    assert (o.float() - o2.float()).abs().max().item() <= 2 * gu.O_MAX


def test_sibling_scan_prefill_matches_oracle():
    m = gu.pp()
    W = wl.make_prefill(layers=1, H=2, d=128, N=200, P=9, q=(3, 17), seed=3, device=DEV)
    L = W.layer(0)
    layer = gu.load_prefill(W, L, DEV)
    lse = torch.empty((W.R, W.H), dtype=torch.float32, device=DEV)
    o = m.prefill_attn(layer, W.N, L.q, L.sid, L.pos, W.scale, lse=lse,
                       opt=m.Options(sibling_scan=1))
    torch.cuda.synchronize()
    assert m.device_status(layer) == 0
    o_ref, lse_ref, _ = gu.oracle_prefill(W, L)
    gu.compare(o, lse, o_ref, lse_ref, "sibling scan prefill")
