"""GPU parity: the C-ABI path against the fp64 oracle, element by element.

Small cases are compared in full and span several document tiles, both M
tiles of a row group, two row groups, ragged tails and forced split counts
that make CTAs cross head boundaries; the named full-size workloads are
compared on whole layers (every row, head and dimension) in the launch
configuration the bench uses.
"""
import numpy as np
import pytest
import torch

import oracle
from shared_context_decode_b200 import workloads as wl
from tests import flat
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
DEV = "cuda"


def decode_case(W, l=0, opt=None, rows=None, with_lse=True):
    m = gu.pp()
    L = W.layer(l)
    layer = gu.load_decode(W, L, DEV)
    lse = torch.empty((W.P, W.H), dtype=torch.float32, device=DEV) if with_lse else None
    o = m.decode_attn(layer, W.N, L.q, L.q_sid, L.q_pos, W.scale, lse=lse, opt=opt)
    torch.cuda.synchronize()
    assert m.device_status(layer) == 0
    o_ref, lse_ref, _ = gu.oracle_decode(W, L, rows)
    sel = slice(None) if rows is None else rows
    return gu.compare(o[sel], None if lse is None else lse[sel], o_ref, lse_ref, W.name)


def test_tiny_config_full():
    decode_case(wl.make_decode("tiny", device=DEV))


@pytest.mark.parametrize("splits", [0, 1, 3, 5, 7, 16])
def test_ragged_two_mtiles_split_variants(splits):
    # 8 key tiles with a 104-key tail, 200 rows = 128 + 72, 4 heads
    W = wl.make_decode(layers=1, H=4, d=128, N=1000, P=200, q=(1, 20), a=(0, 10), seed=1,
                       device=DEV)
    opt = gu.pp().Options(splits=splits) if splits else None
    decode_case(W, opt=opt)


@pytest.mark.parametrize("P", [64, 128])
@pytest.mark.parametrize("splits", [1, 3, 7, 20, 32])
def test_single_mtile_many_splits(P, splits):
    """Row groups of at most 128 rows (one M tile, one CTA per slot) under
    split counts from one slot to one key tile per slot, so segments of one
    tile and of odd length occur; 8 key tiles with a 104-key tail, 4 heads."""
    W = wl.make_decode(layers=1, H=4, d=128, N=1000, P=P, q=(1, 20), a=(0, 10), seed=31,
                       device=DEV)
    decode_case(W, opt=gu.pp().Options(splits=splits))


@pytest.mark.parametrize("splits", [1, 4, 9, 25, 33])
def test_mixed_row_group_sizes_across_segments(splits):
    """P = 300: the first row group has two M tiles, the second one (44 rows)
    only one, so a slot's CTA pair crosses from a full group into one whose
    second M tile is empty."""
    W = wl.make_decode(layers=1, H=3, d=128, N=1000, P=300, q=(1, 9), a=(0, 4), seed=32,
                       device=DEV)
    decode_case(W, opt=gu.pp().Options(splits=splits))


def test_two_row_groups():
    W = wl.make_decode(layers=1, H=2, d=128, N=300, P=300, q=(1, 9), a=(0, 4), seed=2,
                       device=DEV)
    decode_case(W, opt=gu.pp().Options(splits=5))


def test_d64_two_mtiles():
    W = wl.make_decode(layers=1, H=3, d=64, N=777, P=130, q=(2, 12), a=(0, 7), seed=3, device=DEV)
    decode_case(W)


def test_small_p_single_row():
    W = wl.make_decode(layers=1, H=2, d=128, N=129, P=1, q=(3, 3), a=(1, 1), seed=4, device=DEV)
    decode_case(W)


def test_no_document():
    W = wl.make_decode(layers=1, H=2, d=128, N=0, P=5, q=(1, 6), a=(0, 3), seed=5, device=DEV)
    decode_case(W)


def test_ablation_doc_per_stream_matches():
    W = wl.make_decode(layers=1, H=4, d=128, N=1000, P=40, q=(1, 20), a=(0, 10), seed=6,
                       device=DEV)
    decode_case(W, opt=gu.pp().Options(ablation_doc_per_stream=1))


def test_inactive_rows_are_zero():
    m = gu.pp()
    W = wl.make_decode(layers=1, H=2, d=128, N=260, P=20, q=(1, 5), a=(0, 3), seed=7, device=DEV)
    active = np.arange(W.P) % 3 != 1
    L = W.layer(0, active=active)
    layer = gu.load_decode(W, L, DEV)
    lse = torch.empty((W.P, W.H), dtype=torch.float32, device=DEV)
    o = m.decode_attn(layer, W.N, L.q, L.q_sid, L.q_pos, W.scale, lse=lse)
    torch.cuda.synchronize()
    o_ref, lse_ref, _ = gu.oracle_decode(W, L)
    gu.compare(o, lse, o_ref, lse_ref, "inactive")
    assert torch.all(o[torch.from_numpy(~active).to(DEV)] == 0)
    assert torch.all(torch.isinf(lse[torch.from_numpy(~active).to(DEV)]))


@pytest.mark.parametrize("P,H,d,a,active_every", [(300, 16, 128, (0, 40), 3), (5000, 1, 64, (0, 20), 0),
                                                  (257, 14, 128, (0, 63), 0)])
def test_equal_item_counts_per_warp(P, H, d, a, active_every):
    """The suffix pass with equal item counts per warp on inactive rows
    mixed with active ones, more rows than the balanced mode takes, and a
    head count that leaves a ragged last warp."""
    m = gu.pp()
    W = wl.make_decode(layers=1, H=H, d=d, N=300, P=P, q=(1, 20), a=a, seed=33, device=DEV)
    active = (np.arange(P) % active_every != 1) if active_every else None
    L = W.layer(0, active=active)
    layer = gu.load_decode(W, L, DEV)
    lse = torch.empty((W.P, W.H), dtype=torch.float32, device=DEV)
    o = m.decode_attn(layer, W.N, L.q, L.q_sid, L.q_pos, W.scale, lse=lse,
                      opt=m.Options(suffix_slices=1))
    torch.cuda.synchronize()
    assert m.device_status(layer) == 0
    o_ref, lse_ref, _ = gu.oracle_decode(W, L)
    gu.compare(o, lse, o_ref, lse_ref, "equal item counts")


def test_doc_pass_stays_in_segment_when_other_streams_longer():
    # Streams with very different suffix lengths; the mask must not leak.
    W = wl.make_decode(layers=1, H=2, d=128, N=400, P=9, q=(1, 60), a=(0, 60), seed=8, device=DEV)
    decode_case(W)


@pytest.mark.parametrize("name", ["doc8k_p64", "doc16k_p256"])
def test_full_size_whole_layers(name):
    """Every row, head and output dimension of the first and the last layer
    of the full-size workloads, in the bench's launch configuration."""
    W = wl.make_decode(name, device=DEV)
    for l in (0, W.layers - 1):
        decode_case(W, l=l)


@pytest.mark.parametrize("P,H,q,a", [(3, 2, (10, 20), (1500, 2500)), (40, 2, (1, 30), (0, 600)),
                                     (7, 1, (1, 1), (0, 0))])
@pytest.mark.parametrize("slices", [0, 1, 2])
def test_segments_split_between_warps(P, H, q, a, slices):
    """Few streams with long segments: with work-balanced slices the suffix
    pass cuts long items between warps, and the last warp of each item merges
    the partials of the others; also one-key segments with more warps than
    work.  Each slicing of the work gives the oracle's result."""
    m = gu.pp()
    W = wl.make_decode(layers=1, H=H, d=128, N=700, P=P, q=q, a=a, seed=21, device=DEV)
    decode_case(W, opt=m.Options(suffix_slices=slices))


@pytest.mark.parametrize("slices", [1, 2])
def test_ragged_rows_both_slicings(slices):
    m = gu.pp()
    W = wl.make_decode(layers=1, H=4, d=64, N=1000, P=200, q=(1, 20), a=(0, 90), seed=23,
                       device=DEV)
    decode_case(W, opt=m.Options(suffix_slices=slices))


def test_split_items_replayed_in_a_graph_stay_exact():
    """The arrival counters are zeroed by the document pass of every call:
    repeated graph replays give identical outputs."""
    m = gu.pp()
    W = wl.make_decode(layers=1, H=2, d=128, N=500, P=5, q=(5, 9), a=(300, 700), seed=22,
                       device=DEV)
    L = W.layer(0)
    layer = gu.load_decode(W, L, DEV)
    o = torch.empty_like(L.q)
    ws = m.workspace(m.decode_workspace_bytes(W.P, W.H, W.d, W.N), DEV)
    opt = m.Options(suffix_slices=2)
    m.decode_attn(layer, W.N, L.q, L.q_sid, L.q_pos, W.scale, o=o, ws=ws, opt=opt)
    torch.cuda.synchronize()
    first = o.clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            m.decode_attn(layer, W.N, L.q, L.q_sid, L.q_pos, W.scale, o=o, ws=ws, opt=opt)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(5):
        o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), first.view(torch.int16))
    o_ref, lse_ref, _ = gu.oracle_decode(W, L)
    gu.compare(first, None, o_ref, None, "split items")


def test_prefill_small_full():
    m = gu.pp()
    W = wl.make_prefill(layers=1, H=2, d=128, N=700, P=12, q=(1, 40), seed=9, device=DEV)
    L = W.layer(0)
    layer = gu.load_prefill(W, L, DEV)
    lse = torch.empty((W.R, W.H), dtype=torch.float32, device=DEV)
    o = m.prefill_attn(layer, W.N, L.q, L.sid, L.pos, W.scale, lse=lse)
    torch.cuda.synchronize()
    assert m.device_status(layer) == 0
    o_ref, lse_ref, _ = gu.oracle_prefill(W, L)
    gu.compare(o, lse, o_ref, lse_ref, "prefill small")


def test_prefill_full_size():
    """Question prefill at full size (8260 rows, 33 row groups): every row of
    the first 256-row group, of a middle group and of the ragged last group
    on all heads, and every row of the call on the first and the last head."""
    m = gu.pp()
    W = wl.make_prefill("prefill_doc12k_p256", device=DEV)
    L = W.layer(0)
    layer = gu.load_prefill(W, L, DEV)
    lse = torch.empty((W.R, W.H), dtype=torch.float32, device=DEV)
    o = m.prefill_attn(layer, W.N, L.q, L.sid, L.pos, W.scale, lse=lse)
    torch.cuda.synchronize()
    assert m.device_status(layer) == 0
    G = -(-W.R // 256)
    rows = np.concatenate([np.arange(0, 256), np.arange(256 * (G // 2), 256 * (G // 2 + 1)),
                           np.arange(256 * (G - 1), W.R)])
    o_ref, lse_ref, _ = gu.oracle_prefill(W, L, rows)
    gu.compare(o[rows], lse[rows], o_ref, lse_ref, "prefill full, three row groups")
    heads = [0, W.H - 1]
    k, v, ks, kp = flat.prefill_slots(L, W.N)
    q, qs, qp = flat.prefill_queries(L)
    o_ref, lse_ref, _ = oracle.masked_attention(q[:, heads], qs, qp, k[:, heads], v[:, heads],
                                                ks, kp, W.scale)
    gu.compare(o[:, heads], lse[:, heads], o_ref, lse_ref, "prefill full, every row")
