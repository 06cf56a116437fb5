"""Oracle for Parallel Prompting attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  It shares no
code with the CUDA path and never imports it.

Contents
--------
``masked_attention``  fp64 two-pass masked softmax attention over a flat list
                      of tagged KV slots (C, OpenMP; ``ppo.c``).  Follows the
                      project page "Read Once, Answer Many", section "How it
                      works", items 1 (stream mask) and 2 (shared positions).
``visibility``        the same mask rule as a dense 0/1 matrix (C).
``brute.per_stream_causal``  numpy fp64 brute force: ordinary causal attention
                      of each stream over document + own question + own
                      answers, with no stream ids at all (the independence
                      claim of the same section: each answer is the same as
                      decoding its question alone).
``append.AppendReplay``  plain replay of the KV-append rules on a logical
                      cache model (stream segments as Python lists).

Every function here is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_pins.py`` against closed forms, invariants, a library
routine or a hand example, never against itself.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i32, dbl = ctypes.c_int32, ctypes.c_double
        p = ctypes.c_void_p
        lib.ppo_attention.argtypes = [i32, i32, i32, i32, p, p, p, p, p, p, p,
                                      dbl, p, p, p]
        lib.ppo_attention.restype = ctypes.c_int
        lib.ppo_visibility.argtypes = [i32, i32, p, p, p, p, p]
        lib.ppo_visibility.restype = ctypes.c_int
        lib.ppo_num_threads.argtypes = []
        lib.ppo_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def masked_attention(q, q_sid, q_pos, k, v, k_sid, k_pos, scale):
    """fp64 masked attention.

    q: uint16 bf16 bits [nq, H, d]; k, v: uint16 bf16 bits [nk, H, d];
    *_sid, *_pos: integer [nq] / [nk].  Returns (o [nq,H,d] f64,
    lse [nq,H] f64, nvis [nq] int32).
    """
    q = np.asarray(q)
    nq, H, d = q.shape
    nk = int(np.asarray(k).shape[0])
    assert np.asarray(k).shape == (nk, H, d) and np.asarray(v).shape == (nk, H, d)
    qa, qp = _c(q, np.uint16)
    ka, kp = _c(k, np.uint16)
    va, vp = _c(v, np.uint16)
    qs, qsp = _c(q_sid, np.int32)
    qo, qop = _c(q_pos, np.int32)
    ks, ksp = _c(k_sid, np.int32)
    ko, kop = _c(k_pos, np.int32)
    o = np.zeros((nq, H, d), np.float64)
    lse = np.zeros((nq, H), np.float64)
    nvis = np.zeros((nq,), np.int32)
    rc = _load().ppo_attention(nq, nk, H, d, qp, qsp, qop, kp, vp, ksp, kop,
                               float(scale), o.ctypes.data_as(ctypes.c_void_p),
                               lse.ctypes.data_as(ctypes.c_void_p),
                               nvis.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError("ppo_attention rejected its arguments")
    return o, lse, nvis


def visibility(q_sid, q_pos, k_sid, k_pos):
    """Dense 0/1 visibility matrix [nq, nk] (uint8) of the stream-mask rule."""
    qs, qsp = _c(q_sid, np.int32)
    qo, qop = _c(q_pos, np.int32)
    ks, ksp = _c(k_sid, np.int32)
    ko, kop = _c(k_pos, np.int32)
    m = np.zeros((qs.shape[0], ks.shape[0]), np.uint8)
    rc = _load().ppo_visibility(qs.shape[0], ks.shape[0], qsp, qop, ksp, kop,
                                m.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError("ppo_visibility rejected its arguments")
    return m


def num_threads():
    """Host threads the C oracle runs on (OpenMP)."""
    return int(_load().ppo_num_threads())
