"""Document prefill on the GPU (pp_doc_prefill_attn) against the oracle:
document token i attends to document tokens 0..i (project page "Read Once,
Answer Many", section "How it works": the document is encoded once and
shared; stream 0 is the document)."""
import numpy as np
import pytest
import torch

import oracle
from shared_context_decode_b200 import workloads as wl
from shared_context_decode_b200.workloads import bf16_bits
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0) if torch.cuda.is_available() else None


def make(N, H, d, seed):
    k = wl.randn_bf16((N, H, d), wl.seed_of("docpf", N, H, d, "k", seed), DEV)
    v = wl.randn_bf16((N, H, d), wl.seed_of("docpf", N, H, d, "v", seed), DEV)
    q = wl.randn_bf16((N, H, d), wl.seed_of("docpf", N, H, d, "q", seed), DEV)
    m = gu.pp()
    layer = m.KVLayer(H, d, N, 4, 8, DEV)
    sid, pos = gu.doc_tags(N, DEV)
    m.kv_append(layer, k, v, sid, pos)
    return layer, q, k, v


def oracle_rows(q, k, v, rows, scale):
    N = k.shape[0]
    idx = np.arange(N, dtype=np.int32)
    return oracle.masked_attention(bf16_bits(q)[rows], np.zeros(len(rows), np.int32), idx[rows],
                                   bf16_bits(k), bf16_bits(v), np.zeros(N, np.int32), idx, scale)


def check(o, lse, ref_o, ref_lse):
    err = np.abs(o.float().cpu().numpy() - ref_o)
    assert err.max() <= gu.O_MAX and err.mean() <= gu.O_MEAN, (err.max(), err.mean())
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=gu.LSE_MAX)


@pytest.mark.parametrize("N,H,d,splits", [
    (1000, 3, 128, 0), (1000, 3, 128, 1), (1000, 3, 128, 5), (513, 2, 128, 7),
    (300, 2, 64, 0), (300, 2, 64, 3), (129, 1, 128, 0), (256, 2, 64, 16), (1, 1, 64, 0)])
def test_doc_prefill_matches_oracle(N, H, d, splits):
    m = gu.pp()
    layer, q, k, v = make(N, H, d, seed=splits)
    scale = 1.0 / np.sqrt(d)
    lse = torch.empty((N, H), dtype=torch.float32, device=DEV)
    opt = m.Options(splits=splits) if splits else None
    o = m.doc_prefill_attn(layer, N, q, scale, lse=lse, opt=opt)
    torch.cuda.synchronize()
    assert m.device_status(layer) == 0
    ref_o, ref_lse, nvis = oracle_rows(q, k, v, np.arange(N), scale)
    assert nvis.tolist() == list(range(1, N + 1))
    check(o, lse, ref_o, ref_lse)
    # row 0 sees key 0 only: o = v_0 exactly, lse = q_0 . k_0 * scale
    assert torch.equal(o[0], v[0])


def test_doc_prefill_full_size():
    """16384 document tokens, 32 heads, d = 128 (the headline document): every
    row of the first and the last 256-row group on all heads, and every row
    of the document on the first and the last head."""
    m = gu.pp()
    N, H, d = 16384, 32, 128
    layer, q, k, v = make(N, H, d, seed=11)
    scale = 1.0 / np.sqrt(d)
    lse = torch.empty((N, H), dtype=torch.float32, device=DEV)
    o = m.doc_prefill_attn(layer, N, q, scale, lse=lse)
    torch.cuda.synchronize()
    assert m.device_status(layer) == 0
    rows = np.concatenate([np.arange(0, 256), np.arange(N - 256, N)])
    ref_o, ref_lse, _ = oracle_rows(q, k, v, rows, scale)
    sel = torch.from_numpy(rows).to(DEV)
    check(o[sel], lse[sel], ref_o, ref_lse)
    heads = [0, H - 1]
    idx = np.arange(N, dtype=np.int32)
    ref_o, ref_lse, _ = oracle.masked_attention(
        bf16_bits(q)[:, heads], np.zeros(N, np.int32), idx, bf16_bits(k)[:, heads],
        bf16_bits(v)[:, heads], np.zeros(N, np.int32), idx, scale)
    check(o[:, heads], lse[:, heads], ref_o, ref_lse)


def test_doc_prefill_then_decode_sees_the_same_document():
    """A decode step over the document the prefill used: the answer stream's
    first query sees all N document keys plus its own token."""
    m = gu.pp()
    N, H, d, P = 700, 2, 128, 3
    layer, q, k, v = make(N, H, d, seed=5)
    m.doc_prefill_attn(layer, N, q, 0.1)
    nk = wl.randn_bf16((P, H, d), 99, DEV)
    nv = wl.randn_bf16((P, H, d), 98, DEV)
    qd = wl.randn_bf16((P, H, d), 97, DEV)
    sid = torch.arange(1, P + 1, dtype=torch.int16, device=DEV)
    pos = torch.full((P,), N, dtype=torch.int32, device=DEV)
    m.kv_append(layer, nk, nv, sid, pos)
    lse = torch.empty((P, H), dtype=torch.float32, device=DEV)
    o = m.decode_attn(layer, N, qd, sid, pos, 0.1, lse=lse)
    torch.cuda.synchronize()
    kk = np.concatenate([bf16_bits(k), bf16_bits(nk)])
    vv = np.concatenate([bf16_bits(v), bf16_bits(nv)])
    ks = np.concatenate([np.zeros(N, np.int32), np.arange(1, P + 1, dtype=np.int32)])
    kp = np.concatenate([np.arange(N, dtype=np.int32), np.full(P, N, np.int32)])
    ref_o, ref_lse, nvis = oracle.masked_attention(bf16_bits(qd), np.arange(1, P + 1), np.full(P, N),
                                                   kk, vv, ks, kp, 0.1)
    assert nvis.tolist() == [N + 1] * P
    check(o, lse, ref_o, ref_lse)
