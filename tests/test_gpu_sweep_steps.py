"""The ragged answer-generation sweep against the oracle, step by step.

"Read Once, Answer Many" (project page, section "How it works"): every decode
step appends one token per stream and runs as one fixed-shape CUDA graph, and
each answer is the same as decoding its question alone.  Here one graph holds
the step of every layer (the append and the attention of all P rows); it is
captured once and replayed for all 32 steps while streams stop at their
seeded geometric lengths, L_s = min(32, Geometric(1/24)) -- a stopped
stream keeps its row with stream id -1 (no append, no suffix work).  Every
step has its own decode tokens, copied into the graph's input buffers before
the replay, as a generation loop does.

After every step the segment lengths and the slot each active stream just
gained (its stream id, position and K/V bits) must equal the append replay
bit for bit, and stopped rows must give exactly zero.  On a seeded set of
steps (the first, the first with a stopped stream, a middle one and the
last) the whole cache (every slot's tags and K/V bits) must equal the
replay, and o and lse of every row and head must match the oracle over the
replayed cache within the stated bar.
"""
import math

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


def expected_state(rep, H, d, S_cap):
    """Dense arrays of the replayed segments in the library's layout:
    len [P], sid/pos [P, S_cap], k/v bits [P, H, S_cap, d]; unused slots 0."""
    P = rep.P_max
    ln = np.zeros(P, np.int32)
    sid = np.zeros((P, S_cap), np.int16)
    pos = np.zeros((P, S_cap), np.int32)
    k = np.zeros((P, H, S_cap, d), np.uint16)
    v = np.zeros((P, H, S_cap, d), np.uint16)
    for s in range(1, P + 1):
        seg = rep.seg[s]
        ln[s - 1] = len(seg)
        for t, (kk, vv, ss, pp) in enumerate(seg):
            sid[s - 1, t], pos[s - 1, t] = ss, pp
            k[s - 1, :, t, :] = kk
            v[s - 1, :, t, :] = vv
    return ln, sid, pos, k, v


def check_state(layer, rep, what):
    ln, sid, pos, k, v = expected_state(rep, layer.H, layer.d, layer.S_cap)
    assert np.array_equal(layer.len.cpu().numpy(), ln), f"{what}: segment lengths"
    assert np.array_equal(layer.sid.cpu().numpy(), sid), f"{what}: slot stream ids"
    assert np.array_equal(layer.pos.cpu().numpy(), pos), f"{what}: slot positions"
    assert np.array_equal(bf16_bits(layer.k_suf), k), f"{what}: slot keys"
    assert np.array_equal(bf16_bits(layer.v_suf), v), f"{what}: slot values"


def check_new_slots(layer, rep, before, active, what):
    """Lengths of every stream, and the slot each active stream gained in
    this step, against the replay (its last slot)."""
    ln = layer.len.cpu().numpy()
    want = np.array([rep.length(s) for s in range(1, rep.P_max + 1)], np.int32)
    assert np.array_equal(ln, want), f"{what}: segment lengths"
    idx_s = np.nonzero(active)[0]
    if idx_s.size == 0:
        return
    idx_t = before[idx_s]
    dev = layer.len.device
    si, ti = torch.from_numpy(idx_s).to(dev), torch.from_numpy(idx_t.astype(np.int64)).to(dev)
    sid = layer.sid[si, ti].cpu().numpy()
    pos = layer.pos[si, ti].cpu().numpy()
    k = bf16_bits(layer.k_suf[si, :, ti, :])
    v = bf16_bits(layer.v_suf[si, :, ti, :])
    for n, s in enumerate(idx_s + 1):
        kk, vv, ss, pp = rep.seg[s][-1]
        assert sid[n] == ss and pos[n] == pp, f"{what}: tags of stream {s}'s new slot"
        assert np.array_equal(k[n], kk) and np.array_equal(v[n], vv), \
            f"{what}: K/V bits of stream {s}'s new slot"


def oracle_step(rep, doc_k, doc_v, N, q, q_sid, q_pos, scale):
    """fp64 attention of this step's rows over the document and the replayed
    segments."""
    ks, vs, ss, ps = [doc_k], [doc_v], [np.zeros(N, np.int32)], [np.arange(N, dtype=np.int32)]
    for s in range(1, rep.P_max + 1):
        seg = rep.seg[s]
        if seg:
            ks.append(np.stack([x[0] for x in seg]))
            vs.append(np.stack([x[1] for x in seg]))
            ss.append(np.array([x[2] for x in seg], np.int32))
            ps.append(np.array([x[3] for x in seg], np.int32))
    return oracle.masked_attention(q, q_sid, q_pos, np.concatenate(ks), np.concatenate(vs),
                                   np.concatenate(ss), np.concatenate(ps), scale)


@pytest.mark.parametrize("N,P,layers,fused", [(8192, 64, 2, True), (8192, 64, 2, False),
                                               (12288, 256, 1, True)])
def test_sweep_graph_steps_match_oracle(N, P, layers, fused):
    m = gu.pp()
    cfg = wl.sweep_config(N, P)
    name = f"sweep_N{N}_P{P}"
    steps = cfg["steps"]
    W = wl.make_decode(None, layers=layers, H=cfg["H"], d=cfg["d"], N=N, P=P, q=cfg["q"],
                       a=cfg["a"], device=DEV)
    H, d = W.H, W.d
    stops = wl.stop_lengths(P, name)
    S_cap = int(math.ceil((int(W.q_len.max()) + steps + 1) / 16) * 16)
    sids = np.arange(1, P + 1, dtype=np.int16)
    base_pos = (N + W.q_len).astype(np.int32)
    # steps whose outputs are compared with the oracle
    first_stop = int(stops.min())
    checked = sorted({0, min(first_stop, steps - 1), steps // 2, steps - 1})
    assert (stops < steps).any() and first_stop < steps, "the seeded stops must make the step ragged"

    caches, reps, docs, bufs = [], [], [], []
    for l in range(layers):
        L = W.layer(l)
        kv = m.KVLayer(H, d, N, P, S_cap, DEV)
        dsid, dpos = gu.doc_tags(N, DEV)
        m.kv_append(kv, L.doc_k, L.doc_v, dsid, dpos)
        m.kv_append(kv, L.suf_k, L.suf_v, L.suf_sid, L.suf_pos)
        rep = AppendReplay(P, S_cap, N)
        rep.append(bf16_bits(L.suf_k), bf16_bits(L.suf_v), L.suf_sid.cpu().numpy(),
                   L.suf_pos.cpu().numpy())
        caches.append(kv)
        reps.append(rep)
        docs.append((bf16_bits(L.doc_k), bf16_bits(L.doc_v)))
        bufs.append(dict(k=torch.empty((P, H, d), dtype=torch.bfloat16, device=DEV),
                         v=torch.empty((P, H, d), dtype=torch.bfloat16, device=DEV),
                         q=torch.empty((P, H, d), dtype=torch.bfloat16, device=DEV),
                         o=torch.empty((P, H, d), dtype=torch.bfloat16, device=DEV),
                         lse=torch.empty((P, H), dtype=torch.float32, device=DEV)))
        del L
    q_sid = torch.empty(P, dtype=torch.int16, device=DEV)
    q_pos = torch.empty(P, dtype=torch.int32, device=DEV)
    ws = m.workspace(m.decode_workspace_bytes(P, H, d, N), DEV)

    def body():
        for l in range(layers):
            x = bufs[l]
            if fused:
                m.decode_step(caches[l], N, x["k"], x["v"], x["q"], q_sid, q_pos, W.scale,
                              o=x["o"], lse=x["lse"], ws=ws)
            else:
                m.kv_append(caches[l], x["k"], x["v"], q_sid, q_pos)
                m.decode_attn(caches[l], N, x["q"], q_sid, q_pos, W.scale, o=x["o"],
                              lse=x["lse"], ws=ws)

    # Capture on a scratch copy of the lengths, so the capture-time warm-up
    # call leaves the real cache untouched: run once eagerly (per-device
    # setup outside the capture), then restore the cache lengths.
    len0 = [c.len.clone() for c in caches]
    q_sid.fill_(-1)
    q_pos.zero_()
    for x in bufs:
        for n in ("k", "v", "q"):
            x[n].zero_()
    body()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(DEV)
    s.wait_stream(torch.cuda.current_stream(DEV))
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            body()
    torch.cuda.current_stream(DEV).wait_stream(s)
    torch.cuda.synchronize()
    for c, l0 in zip(caches, len0):
        c.len.copy_(l0)
    for l in range(layers):
        check_state(caches[l], reps[l], f"layer {l} before the first step")

    for t in range(steps):
        active = t < stops
        sid_t = np.where(active, sids, -1).astype(np.int16)
        pos_t = (base_pos + t).astype(np.int32)
        q_sid.copy_(torch.from_numpy(sid_t))
        q_pos.copy_(torch.from_numpy(pos_t))
        host = []
        for l in range(layers):
            x = bufs[l]
            for n in ("k", "v", "q"):
                x[n].copy_(wl.randn_bf16((P, H, d), wl.seed_of(name, l, t, n), DEV))
            host.append({n: bf16_bits(x[n]) for n in ("k", "v", "q")})
        before = [c.len.cpu().numpy().copy() for c in caches]
        g.replay()
        torch.cuda.synchronize()
        for l in range(layers):
            kv, rep, hx = caches[l], reps[l], host[l]
            rep.append(hx["k"], hx["v"], sid_t, pos_t)
            assert m.device_status(kv) == 0, f"step {t} layer {l}: device status"
            check_new_slots(kv, rep, before[l], active, f"step {t} layer {l}")
            if t in checked:
                check_state(kv, rep, f"step {t} layer {l}")
            o = bufs[l]["o"]
            assert torch.count_nonzero(o[torch.from_numpy(~active).to(DEV)]) == 0, \
                f"step {t} layer {l}: stopped rows must give zero output"
            if t in checked:
                ref_o, ref_lse, _ = oracle_step(rep, docs[l][0], docs[l][1], N, hx["q"],
                                                sid_t.astype(np.int32), pos_t, W.scale)
                gu.compare(o, bufs[l]["lse"], ref_o, ref_lse, f"step {t} layer {l}")
    # every stream appended exactly min(stop, steps) tokens
    want = W.q_len + np.minimum(stops, steps)
    for l in range(layers):
        assert np.array_equal(caches[l].len.cpu().numpy(), want.astype(np.int32))
    del g
