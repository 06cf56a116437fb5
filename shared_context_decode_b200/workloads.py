"""Seeded synthetic workloads for the Parallel Prompting attention path.

This module holds shapes, sizes and random draws only -- none of the
method's arithmetic.  It is the one module that both sides use: the CUDA path
(through the binding) and the oracle (through the tests) receive the same
generated bf16 bits.  It imports neither side.

Workload recipe (every size below is a named configuration):
  * q, k, v ~ N(0, 1) drawn in fp32 by a seeded torch generator on the chosen
    device, cast to bf16 with round-to-nearest-even; softmax scale 1/sqrt(d);
  * question lengths and cached-answer lengths are integer-uniform on the
    inclusive ranges of each configuration (numpy PCG64, seeded);
  * positions follow the shared-position rule of the project page "Read Once,
    Answer Many" (section "How it works", item 2): document token i has
    position i, token j of every stream (question, then answers) has position
    N + j, so the decode token of stream s sits at N + q_s + a_s;
  * stream ids: 0 = document, 1..P = answer streams, -1 = inactive row;
  * the ragged sweep stops stream s after L_s = min(32, G_s) tokens with
    G_s ~ Geometric(p = 1/24) on {1, 2, ...};
  * every layer draws its own tensors; the seed of each tensor is a CRC32 of
    (workload name, layer, tensor name, base seed).
"""
from __future__ import annotations

import dataclasses
import math
import zlib
from typing import Optional

import numpy as np
import torch


# name -> shape parameters.  q/a are inclusive integer ranges of question
# length and of answer tokens already cached before the step.
CONFIGS = {
    # 1 layer, H=4, d=64, doc 256, 4 streams, 8-token questions, 3 answers
    "tiny": dict(layers=1, H=4, d=64, N=256, P=4, q=(8, 8), a=(3, 3)),
    # CodeLlama-7B attention shapes, doc 8192, 64 streams
    "doc8k_p64": dict(layers=32, H=32, d=128, N=8192, P=64, q=(16, 48), a=(0, 31)),
    # same shapes, doc 16384, 256 streams: the memory-bound headline case
    "doc16k_p256": dict(layers=32, H=32, d=128, N=16384, P=256, q=(16, 48), a=(0, 63)),
    # long answers: doc 8192, 128 streams, 1024 answer tokens already cached
    # (the long-answer point of the pages' answer-length figure)
    "doc8k_p128_a1k": dict(layers=8, H=32, d=128, N=8192, P=128, q=(16, 48), a=(1024, 1024)),
    # question prefill: doc 12000 cached, 256 questions of 16..48 tokens
    "prefill_doc12k_p256": dict(layers=32, H=32, d=128, N=12000, P=256, q=(16, 48),
                                a=(0, 0)),
}

# answer-generation sweep: doc x streams, 32 decode steps x 32 layers
SWEEP_DOCS = (8192, 12288, 16384)
SWEEP_STREAMS = (64, 128, 256)
SWEEP_STEPS = 32
SWEEP_STOP_MEAN = 24
SWEEP_STOP_CAP = 32


def sweep_config(N: int, P: int) -> dict:
    return dict(layers=32, H=32, d=128, N=N, P=P, q=(16, 48), a=(0, 0),
                steps=SWEEP_STEPS)


def seed_of(*parts) -> int:
    return zlib.crc32("/".join(str(p) for p in parts).encode()) & 0x7FFFFFFF


def randn_bf16(shape, seed: int, device="cpu") -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return x.to(torch.bfloat16)


def lengths(cfg: dict, name: str, seed: int = 0):
    """Question lengths and cached-answer lengths per stream (int32 [P])."""
    rng = np.random.default_rng(seed_of(name, "lengths", seed))
    P = cfg["P"]
    q = rng.integers(cfg["q"][0], cfg["q"][1] + 1, size=P).astype(np.int32)
    a = rng.integers(cfg["a"][0], cfg["a"][1] + 1, size=P).astype(np.int32)
    return q, a


def stop_lengths(P: int, name: str, seed: int = 0):
    """Per-stream stop length L_s = min(cap, Geometric(1/mean)) (int32 [P])."""
    rng = np.random.default_rng(seed_of(name, "stops", seed))
    g = rng.geometric(1.0 / SWEEP_STOP_MEAN, size=P)
    return np.minimum(g, SWEEP_STOP_CAP).astype(np.int32)


@dataclasses.dataclass
class DecodeLayer:
    """One layer of one decode step.

    doc_k, doc_v [N,H,d]    document rows (stream 0, position = row index)
    suf_k, suf_v [T,H,d]    cached stream rows (questions and answers),
                            grouped by stream, in position order
    suf_sid [T] int16, suf_pos [T] int32
    new_k, new_v [P,H,d]    the decode token of every stream
    q [P,H,d]               its query
    q_sid [P] int16, q_pos [P] int32
    """
    doc_k: torch.Tensor
    doc_v: torch.Tensor
    suf_k: torch.Tensor
    suf_v: torch.Tensor
    suf_sid: torch.Tensor
    suf_pos: torch.Tensor
    new_k: torch.Tensor
    new_v: torch.Tensor
    q: torch.Tensor
    q_sid: torch.Tensor
    q_pos: torch.Tensor


@dataclasses.dataclass
class Decode:
    name: str
    layers: int
    H: int
    d: int
    N: int
    P: int
    q_len: np.ndarray
    a_len: np.ndarray
    scale: float
    seed: int
    device: str

    @property
    def S_need(self) -> int:
        """Slots a segment needs to hold the cache plus the decode token."""
        return int((self.q_len + self.a_len).max()) + 1

    def suffix_tokens(self) -> int:
        return int((self.q_len + self.a_len).sum())

    def layer(self, l: int, active: Optional[np.ndarray] = None) -> DecodeLayer:
        """Draw layer l.  `active` (bool [P]) marks streams with a decode token;
        inactive rows get stream id -1."""
        H, d, N, P, dev = self.H, self.d, self.N, self.P, self.device
        nm, sd = self.name, self.seed
        tot = self.q_len + self.a_len
        T = int(tot.sum())
        sid = np.repeat(np.arange(1, P + 1, dtype=np.int16), tot)
        pos = np.concatenate([N + np.arange(t, dtype=np.int32) for t in tot]) \
            if T else np.zeros(0, np.int32)
        q_sid = np.arange(1, P + 1, dtype=np.int16)
        if active is not None:
            q_sid = np.where(active, q_sid, -1).astype(np.int16)
        q_pos = (N + tot).astype(np.int32)
        return DecodeLayer(
            doc_k=randn_bf16((N, H, d), seed_of(nm, l, "doc_k", sd), dev),
            doc_v=randn_bf16((N, H, d), seed_of(nm, l, "doc_v", sd), dev),
            suf_k=randn_bf16((T, H, d), seed_of(nm, l, "suf_k", sd), dev),
            suf_v=randn_bf16((T, H, d), seed_of(nm, l, "suf_v", sd), dev),
            suf_sid=torch.from_numpy(sid).to(dev),
            suf_pos=torch.from_numpy(pos.astype(np.int32)).to(dev),
            new_k=randn_bf16((P, H, d), seed_of(nm, l, "new_k", sd), dev),
            new_v=randn_bf16((P, H, d), seed_of(nm, l, "new_v", sd), dev),
            q=randn_bf16((P, H, d), seed_of(nm, l, "q", sd), dev),
            q_sid=torch.from_numpy(q_sid).to(dev),
            q_pos=torch.from_numpy(q_pos).to(dev),
        )


def make_decode(name: str = None, *, seed: int = 0, device="cpu", **shape) -> Decode:
    """A decode workload from a named configuration, or from explicit
    shape keywords (layers, H, d, N, P, q=(lo,hi), a=(lo,hi))."""
    cfg = dict(CONFIGS[name]) if name is not None else {}
    cfg.update(shape)
    nm = name if name is not None else "custom:" + ",".join(
        f"{k}={cfg[k]}" for k in sorted(cfg))
    q, a = lengths(cfg, nm, seed)
    return Decode(name=nm, layers=cfg.get("layers", 1), H=cfg["H"], d=cfg["d"],
                  N=cfg["N"], P=cfg["P"], q_len=q, a_len=a,
                  scale=1.0 / math.sqrt(cfg["d"]), seed=seed, device=str(device))


@dataclasses.dataclass
class PrefillLayer:
    """One layer of a question prefill.

    doc_k, doc_v [N,H,d]; the question rows qk, qv [R,H,d] with sid [R]
    int16 and pos [R] int32, grouped by stream (row_off [P+1] int32 gives the
    first row of every stream); q [R,H,d] are the question queries.
    """
    doc_k: torch.Tensor
    doc_v: torch.Tensor
    qk: torch.Tensor
    qv: torch.Tensor
    sid: torch.Tensor
    pos: torch.Tensor
    q: torch.Tensor
    row_off: torch.Tensor


@dataclasses.dataclass
class Prefill:
    name: str
    layers: int
    H: int
    d: int
    N: int
    P: int
    q_len: np.ndarray
    scale: float
    seed: int
    device: str

    @property
    def R(self) -> int:
        return int(self.q_len.sum())

    def layer(self, l: int) -> PrefillLayer:
        H, d, N, P, dev = self.H, self.d, self.N, self.P, self.device
        nm, sd = self.name, self.seed
        R = self.R
        sid = np.repeat(np.arange(1, P + 1, dtype=np.int16), self.q_len)
        pos = np.concatenate([N + np.arange(t, dtype=np.int32) for t in self.q_len])
        off = np.concatenate([[0], np.cumsum(self.q_len)]).astype(np.int32)
        return PrefillLayer(
            doc_k=randn_bf16((N, H, d), seed_of(nm, l, "doc_k", sd), dev),
            doc_v=randn_bf16((N, H, d), seed_of(nm, l, "doc_v", sd), dev),
            qk=randn_bf16((R, H, d), seed_of(nm, l, "qk", sd), dev),
            qv=randn_bf16((R, H, d), seed_of(nm, l, "qv", sd), dev),
            sid=torch.from_numpy(sid).to(dev),
            pos=torch.from_numpy(pos.astype(np.int32)).to(dev),
            q=randn_bf16((R, H, d), seed_of(nm, l, "q", sd), dev),
            row_off=torch.from_numpy(off).to(dev),
        )


def make_prefill(name: str = None, *, seed: int = 0, device="cpu", **shape) -> Prefill:
    cfg = dict(CONFIGS[name]) if name is not None else {}
    cfg.update(shape)
    cfg.setdefault("a", (0, 0))
    nm = name if name is not None else "prefill:" + ",".join(
        f"{k}={cfg[k]}" for k in sorted(cfg))
    q, _ = lengths(cfg, nm, seed)
    return Prefill(name=nm, layers=cfg.get("layers", 1), H=cfg["H"], d=cfg["d"],
                   N=cfg["N"], P=cfg["P"], q_len=q, scale=1.0 / math.sqrt(cfg["d"]),
                   seed=seed, device=str(device))


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bf16 bit patterns of a tensor, as uint16 on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
