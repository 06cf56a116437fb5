"""Prefill calls against the oracle on layouts the named workloads do not
reach: rows of many streams interleaved (runs of one or two rows, a stream
split into several runs), runs of many 16-row tiles over segments longer
than one 48-key chunk, follow-up questions behind cached answers (rows whose
segment holds earlier tokens), inactive and out-of-range rows inside runs,
d = 64, no document, runs that cross a 256-row group of document partials,
row counts that leave a ragged last tile, more (run, head) tasks than the
kernel has warps with one workspace reused across calls.

Visibility rule: project page "Read Once, Answer Many", section "How it
works", item 1 -- a row sees the document and the tokens of its own stream
that are not later than itself."""
import numpy as np
import pytest
import torch

import oracle
from shared_context_decode_b200 import workloads as wl
from shared_context_decode_b200.workloads import bf16_bits
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0) if torch.cuda.is_available() else None


def build(H, d, N, seg_len, S_cap, seed):
    """A layer with N document tokens and stream s holding seg_len[s-1]
    tokens at positions N .. N + seg_len[s-1] - 1."""
    m = gu.pp()
    P = len(seg_len)
    rnd = lambda shape, tag: wl.randn_bf16(shape, wl.seed_of("pfblock", tag, seed), DEV)
    layer = m.KVLayer(H, d, max(N, 1), P, S_cap, DEV)
    ks, vs, ss, ps = [], [], [], []
    if N:
        dk, dv = rnd((N, H, d), "dk"), rnd((N, H, d), "dv")
        sid, pos = gu.doc_tags(N, DEV)
        m.kv_append(layer, dk, dv, sid, pos)
        ks.append(dk), vs.append(dv), ss.append(sid), ps.append(pos)
    for s, n in enumerate(seg_len, start=1):
        if n == 0:
            continue
        k, v = rnd((n, H, d), f"k{s}"), rnd((n, H, d), f"v{s}")
        sid = torch.full((n,), s, dtype=torch.int16, device=DEV)
        pos = torch.arange(N, N + n, dtype=torch.int32, device=DEV)
        m.kv_append(layer, k, v, sid, pos)
        ks.append(k), vs.append(v), ss.append(sid), ps.append(pos)
    keys = (np.concatenate([bf16_bits(a) for a in ks]), np.concatenate([bf16_bits(a) for a in vs]),
            np.concatenate([a.cpu().numpy().astype(np.int32) for a in ss]),
            np.concatenate([a.cpu().numpy() for a in ps]))
    return layer, keys


def run(layer, keys, N, H, d, q_sid, q_pos, seed, scale=0.11, expect_status=0):
    m = gu.pp()
    R = len(q_sid)
    q = wl.randn_bf16((R, H, d), wl.seed_of("pfblock", "q", seed), DEV)
    sid_t = torch.from_numpy(np.asarray(q_sid, np.int16)).to(DEV)
    pos_t = torch.from_numpy(np.asarray(q_pos, np.int32)).to(DEV)
    lse = torch.empty((R, H), dtype=torch.float32, device=DEV)
    o = m.prefill_attn(layer, N, q, sid_t, pos_t, scale, lse=lse)
    torch.cuda.synchronize()
    assert m.device_status(layer) == expect_status
    served = np.array([1 <= s <= layer.P_max for s in q_sid])
    k, v, kks, kkp = keys
    ref_o, ref_lse, _ = oracle.masked_attention(bf16_bits(q)[served], np.asarray(q_sid)[served],
                                                np.asarray(q_pos)[served], k, v, kks, kkp, scale)
    idx = torch.from_numpy(np.nonzero(served)[0]).to(DEV)
    gu.compare(o[idx], lse[idx], ref_o, ref_lse, "prefill block")
    if (~served).any():
        rest = torch.from_numpy(np.nonzero(~served)[0]).to(DEV)
        assert torch.count_nonzero(o[rest]).item() == 0
        assert torch.isneginf(lse[rest]).all().item()


def question_rows(seg_len, N, last=None):
    """Rows of each stream's last `last[s]` tokens (all of them when None),
    grouped by stream: a question prefill, or a follow-up question behind
    cached answer tokens."""
    sid, pos = [], []
    for s, n in enumerate(seg_len, start=1):
        k = n if last is None else min(n, last[s - 1])
        sid += [s] * k
        pos += list(range(N + n - k, N + n))
    return sid, pos


@pytest.mark.parametrize("d", [128, 64])
def test_long_segments_several_chunks(d):
    # segments of 1 .. 150 keys: up to five 32-key chunks, ragged tails
    H, N = 3, 300
    seg = [150, 33, 32, 31, 1, 64, 97]
    layer, keys = build(H, d, N, seg, 160, seed=1)
    sid, pos = question_rows(seg, N)
    run(layer, keys, N, H, d, sid, pos, seed=1)


def test_follow_up_questions_behind_answers():
    # each stream holds question + answer tokens; the new rows are the last
    # few tokens only, so they see every earlier token of their stream
    H, d, N = 2, 128, 500
    seg = [40, 70, 12, 90]
    layer, keys = build(H, d, N, seg, 96, seed=2)
    sid, pos = question_rows(seg, N, last=[5, 17, 12, 3])
    run(layer, keys, N, H, d, sid, pos, seed=2)


def test_streams_interleaved_within_blocks():
    # row order shuffled: a 16-row block holds rows of up to 16 streams
    H, d, N = 2, 128, 260
    seg = [int(x) for x in np.random.default_rng(3).integers(1, 45, size=20)]
    layer, keys = build(H, d, N, seg, 48, seed=3)
    sid, pos = question_rows(seg, N)
    perm = np.random.default_rng(4).permutation(len(sid))
    run(layer, keys, N, H, d, np.asarray(sid)[perm], np.asarray(pos)[perm], seed=3)


def test_inactive_rows_and_ragged_last_block():
    m = gu.pp()
    H, d, N = 2, 64, 129
    seg = [20, 9, 35]
    layer, keys = build(H, d, N, seg, 40, seed=5)
    sid, pos = question_rows(seg, N)
    sid[3] = -1            # inactive rows: zero output, -inf lse, no error
    sid[40] = -1
    run(layer, keys, N, H, d, sid, pos, seed=5)       # 64 rows
    sid2, pos2 = sid[:51], pos[:51]                   # 3 blocks + 3 rows
    run(layer, keys, N, H, d, sid2, pos2, seed=6)
    bad = list(sid2)
    bad[7] = 9             # past P_max: flagged, served as inactive
    run(layer, keys, N, H, d, bad, pos2, seed=7, expect_status=m.PP_DEV_BAD_STREAM)


def test_no_document():
    H, d = 2, 128
    seg = [17, 48, 5]
    layer, keys = build(H, d, 0, seg, 48, seed=8)
    sid, pos = question_rows(seg, 0)
    run(layer, keys, 0, H, d, sid, pos, seed=8)


def test_rows_spanning_two_row_groups():
    # 300 rows: the document partials come from two row groups of 256
    H, d, N = 2, 128, 700
    seg = [30] * 10
    layer, keys = build(H, d, N, seg, 32, seed=9)
    sid, pos = question_rows(seg, N)
    run(layer, keys, N, H, d, sid, pos, seed=9)


def test_many_tasks_and_a_reused_workspace():
    # 48 questions x 32 heads = 1536 (run, head) tasks, more than the
    # question kernel's warps (8 per SM), so most warps draw further tasks
    # from the counter in the workspace.  One workspace, filled with 0xff
    # bytes first, serves two calls: each call starts its counter from zero,
    # so both give the same bits, and they match the oracle.
    m = gu.pp()
    H, d, N = 32, 64, 200
    seg = [int(x) for x in np.random.default_rng(11).integers(1, 40, size=48)]
    layer, keys = build(H, d, N, seg, 40, seed=11)
    sid, pos = question_rows(seg, N)
    R = len(sid)
    ws = m.workspace(m.prefill_workspace_bytes(R, H, d, N), DEV)
    ws.fill_(255)
    q = wl.randn_bf16((R, H, d), wl.seed_of("pfblock", "q", 11), DEV)
    sid_t = torch.from_numpy(np.asarray(sid, np.int16)).to(DEV)
    pos_t = torch.from_numpy(np.asarray(pos, np.int32)).to(DEV)
    outs = []
    for _ in range(2):
        lse = torch.empty((R, H), dtype=torch.float32, device=DEV)
        o = m.prefill_attn(layer, N, q, sid_t, pos_t, 0.11, lse=lse, ws=ws)
        torch.cuda.synchronize()
        assert m.device_status(layer) == 0
        outs.append((o, lse))
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])
    k, v, kks, kkp = keys
    ref_o, ref_lse, _ = oracle.masked_attention(bf16_bits(q), np.asarray(sid), np.asarray(pos),
                                                k, v, kks, kkp, 0.11)
    gu.compare(outs[1][0], outs[1][1], ref_o, ref_lse, "prefill, reused workspace")
