"""C-ABI checks that need no GPU: the library loads, exports every entry
point include/ppattn.h declares, rejects bad arguments on the host before
any launch, and plans the document split correctly."""
import ctypes
import os
import re

import pytest

from shared_context_decode_b200 import build as ppbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pp():
    ppbuild.build()
    from shared_context_decode_b200 import ppattn
    return ppattn


def declared_functions():
    src = open(os.path.join(ROOT, "include", "ppattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pp_[a-z_0-9]+)\s*\(", src)))


def header_struct_fields(name):
    """Field names, in order, of `typedef struct name {...} name;` in the header."""
    src = open(os.path.join(ROOT, "include", "ppattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    body = re.search(r"typedef struct " + name + r"\s*\{(.*?)\}\s*" + name + ";", src, re.S).group(1)
    fields = []
    for decl in body.split(";"):
        if decl.strip():
            _type, names = decl.strip().split(None, 1)
            fields += [x.strip().lstrip("*").strip() for x in names.split(",")]
    return fields


def test_ctypes_structs_match_the_header(pp):
    """The binding's layer descriptor and options mirror the C structs field by
    field (a reordered or missing field would silently shift every later one)."""
    assert [f for f, _ in pp.LayerStruct._fields_] == header_struct_fields("pp_kv_layer")
    assert [f for f, _ in pp.Options._fields_] == header_struct_fields("pp_options")


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("pp_kv_append", "pp_decode_attn", "pp_prefill_attn"):
        assert n in names


def test_every_declared_symbol_is_exported(pp):
    lib = ctypes.CDLL(pp.LIB_PATH)
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ppattn.h but not exported"
    assert set(names) == set(pp.EXPORTED)


def test_status_strings_and_version(pp):
    assert pp.abi_version() == 1
    assert pp.status_str(0) == "PP_OK"
    assert pp.status_str(3) == "PP_ERR_CAPACITY"
    assert pp.status_str(99) == "PP_ERR_UNKNOWN"


def fake_layer(pp, **kw):
    """A descriptor with plausible aligned (never dereferenced) addresses."""
    base = dict(H=4, d=128, doc_cap=1024, P_max=8, S_cap=64, reserved=0,
                k_doc=0x10000, v_doc=0x20000, k_suf=0x30000, v_suf=0x40000,
                sid=0x50000, pos=0x60000, len=0x70000, status=0x80000)
    base.update(kw)
    return pp.LayerStruct(**base)


def call_decode(pp, L, doc_len=10, P=4, ws_bytes=1 << 30, opt=None, q=0x90000):
    return pp._decode(ctypes.byref(L), doc_len, q, 0xA0000, 0xB0000, P, 0.1, 0xC0000, None,
                      0xD0000, ws_bytes, None if opt is None else ctypes.byref(opt), None)


def test_host_validation_codes(pp):
    L = fake_layer(pp)
    # layer checks
    assert pp._kv_reset(None, None) == pp.PP_ERR_INVALID_ARG
    assert call_decode(pp, fake_layer(pp, d=96)) == pp.PP_ERR_UNSUPPORTED
    assert call_decode(pp, fake_layer(pp, P_max=0)) == pp.PP_ERR_UNSUPPORTED
    assert call_decode(pp, fake_layer(pp, P_max=40000)) == pp.PP_ERR_UNSUPPORTED
    assert call_decode(pp, fake_layer(pp, k_suf=0x30008)) == pp.PP_ERR_INVALID_ARG
    assert call_decode(pp, fake_layer(pp, len=0)) == pp.PP_ERR_INVALID_ARG
    # call checks
    assert call_decode(pp, L, P=9) == pp.PP_ERR_UNSUPPORTED           # P > P_max
    assert call_decode(pp, L, doc_len=1025) == pp.PP_ERR_CAPACITY     # doc_len > doc_cap
    assert call_decode(pp, L, doc_len=-1) == pp.PP_ERR_INVALID_ARG
    assert call_decode(pp, L, q=0x90004) == pp.PP_ERR_INVALID_ARG     # misaligned q
    assert call_decode(pp, L, P=0) == pp.PP_OK                        # empty: nothing launched
    opt = pp.Options(splits=4)
    assert call_decode(pp, L, ws_bytes=16, opt=opt) == pp.PP_ERR_CAPACITY
    assert call_decode(pp, L, opt=pp.Options(suffix_slices=3)) == pp.PP_ERR_INVALID_ARG
    assert call_decode(pp, L, opt=pp.Options(suffix_slices=-1)) == pp.PP_ERR_INVALID_ARG
    # append
    assert pp._kv_append(ctypes.byref(L), 0x1000, 0x2000, 0x3000, 0x4000, -1, None) == \
        pp.PP_ERR_INVALID_ARG
    assert pp._kv_append(ctypes.byref(L), 0x1000, 0x2000, 0x3000, 0x4000, 0, None) == pp.PP_OK
    assert pp._kv_append(ctypes.byref(L), 0x1008, 0x2000, 0x3000, 0x4000, 3, None) == \
        pp.PP_ERR_INVALID_ARG
    # prefill
    assert pp._prefill(ctypes.byref(L), 2000, 0x90000, 0xA0000, 0xB0000, 5, 0.1, 0xC0000, None,
                       0xD0000, 1 << 30, None, None) == pp.PP_ERR_CAPACITY
    # fused decode step: the attention checks, plus k and v
    def step(k=0xE0000, v=0xF0000, **kw):
        a = dict(doc_len=10, P=4, q=0x90000, ws=1 << 30)
        a.update(kw)
        return pp._decode_step(ctypes.byref(a.pop("L", L)), a["doc_len"], k, v, a["q"], 0xA0000,
                               0xB0000, a["P"], 0.1, 0xC0000, None, 0xD0000, a["ws"], None, None)
    assert step(P=9) == pp.PP_ERR_UNSUPPORTED                          # P > P_max
    assert step(k=0) == pp.PP_ERR_INVALID_ARG
    assert step(v=0xF0008) == pp.PP_ERR_INVALID_ARG                    # misaligned v
    assert step(q=0x90004) == pp.PP_ERR_INVALID_ARG
    assert step(doc_len=1025) == pp.PP_ERR_CAPACITY
    assert step(ws=16) == pp.PP_ERR_CAPACITY
    assert step(P=0) == pp.PP_OK
    assert step(L=fake_layer(pp, d=96)) == pp.PP_ERR_UNSUPPORTED
    # visibility
    assert pp._visibility(ctypes.byref(L), 5, 0x1000, 0x2000, -1, 0x3000, None, None) == \
        pp.PP_ERR_INVALID_ARG
    # no-alloc decode: argument errors come first, with pp_decode_attn's codes
    # (a P far above the layer's streams is not reported as a size problem)
    def noalloc(lay, P=4):
        return pp._decode_noalloc(ctypes.byref(lay), 10, 0x90000, 0xA0000, 0xB0000, P, 0.1,
                                  0xC0000, None, None, None)
    assert noalloc(L, P=100000) == pp.PP_ERR_UNSUPPORTED
    assert noalloc(fake_layer(pp, d=96)) == pp.PP_ERR_UNSUPPORTED
    assert noalloc(fake_layer(pp, len=0)) == pp.PP_ERR_INVALID_ARG


def test_workspace_sizes_with_explicit_split(pp):
    opt = pp.Options(splits=148)
    ws = pp.decode_workspace_bytes(256, 32, 128, 16384, opt)
    plan = pp.split_plan(256, 32, 16384, 148)
    slots = plan["units"] * plan["max_chunks"] * 256
    groups = plan["units"] // 32
    # document partials (O; max and sum), then one stream length per row
    # (rounded up to whole row groups) for a step whose append the pass carries
    expect = slots * 128 * 4 + slots * 2 * 4 + groups * 256 * 4
    assert ws == expect
    # a question prefill adds its question runs: 16 bytes a row (whole row
    # groups) and their count in one 256-byte-aligned word, with a document
    # or without one
    assert pp.prefill_workspace_bytes(256, 32, 128, 16384, opt) == expect + groups * 256 * 16 + 256
    assert pp.prefill_workspace_bytes(300, 2, 64, 0, opt) == 2 * 256 * 16 + 256
    assert pp.decode_workspace_bytes(4, 4, 96, 10, opt) == 0
    # no document: nothing to carry between kernels
    assert pp.decode_workspace_bytes(8, 2, 64, 0, opt) == 0


@pytest.mark.parametrize("rows,H,doc_len,ctas", [
    (256, 32, 16384, 148), (64, 32, 8192, 148), (8192, 32, 12000, 148), (4, 4, 256, 148),
    (200, 4, 1000, 3), (300, 2, 300, 7), (1, 1, 1, 148), (256, 32, 16384, 1), (130, 3, 129, 5)])
def test_split_plan_invariants(pp, rows, H, doc_len, ctas):
    p = pp.split_plan(rows, H, doc_len, ctas)
    T = -(-doc_len // 128)       # document tile: 128 keys
    units = -(-rows // 256) * H
    assert p["T"] == T and p["units"] == units and p["W"] == units * T
    assert p["C"] == min(ctas, units * T)
    W, C = p["W"], p["C"]
    begin = [c * W // C for c in range(C + 1)]
    sizes = [begin[c + 1] - begin[c] for c in range(C)]
    assert min(sizes) >= W // C and max(sizes) <= -(-W // C)    # balanced to one tile
    for u, (c0, c1) in enumerate(p["chunks"]):
        # the CTAs listed are exactly those whose range meets the unit's tiles
        meets = [c for c in range(C) if begin[c] < (u + 1) * T and begin[c + 1] > u * T]
        assert (c0, c1) == (meets[0], meets[-1])
        assert c1 - c0 + 1 <= p["max_chunks"]
    assert p["max_chunks"] == max(c1 - c0 + 1 for c0, c1 in p["chunks"])


@pytest.mark.parametrize("doc_len,H,ctas", [
    (16384, 32, 74), (12000, 4, 148), (1000, 3, 7), (300, 2, 5), (129, 1, 3), (1, 1, 148),
    (256, 2, 1), (257, 5, 16), (2049, 1, 9)])
def test_causal_split_plan_invariants(pp, doc_len, H, ctas):
    """Document prefill split: unit (head, group g) holds key tiles
    0 .. min(T, 2g+2)-1 (rows 256g..256g+255 see keys up to their own
    position), units laid out head-major, ranges balanced over the slots."""
    p = pp.split_plan(doc_len, H, doc_len, ctas, causal=True)
    T = -(-doc_len // 128)
    G = -(-doc_len // 256)
    tiles = [min(T, 2 * g + 2) for g in range(G)]
    # every key tile a group's rows can see is in its unit, and no more
    for g in range(G):
        last_row = min(doc_len, 256 * (g + 1)) - 1
        assert tiles[g] == last_row // 128 + 1
    W = H * sum(tiles)
    assert p["T"] == T and p["units"] == G * H and p["W"] == W
    C = p["C"]
    assert C == min(ctas, W)
    begin = [c * W // C for c in range(C + 1)]
    ub = 0
    for u, (c0, c1) in enumerate(p["chunks"]):
        n = tiles[u % G]
        meets = [c for c in range(C) if begin[c] < ub + n and begin[c + 1] > ub]
        assert (c0, c1) == (meets[0], meets[-1])
        ub += n
    assert ub == W
    assert p["max_chunks"] == max(c1 - c0 + 1 for c0, c1 in p["chunks"])


def test_doc_prefill_host_validation(pp):
    L = fake_layer(pp)

    def call(doc_len=10, q=0x90000, ws_bytes=1 << 30, opt=None, o=0xC0000):
        return pp._doc_prefill(ctypes.byref(L), doc_len, q, 0.1, o, None, 0xD0000, ws_bytes,
                               None if opt is None else ctypes.byref(opt), None)

    assert call(doc_len=0) == pp.PP_OK                              # nothing to do
    assert call(doc_len=-1) == pp.PP_ERR_INVALID_ARG
    assert call(doc_len=1025) == pp.PP_ERR_CAPACITY                # above doc_cap
    assert call(q=0x90004) == pp.PP_ERR_INVALID_ARG                # misaligned q
    assert call(o=0) == pp.PP_ERR_INVALID_ARG
    assert call(opt=pp.Options(ablation_doc_per_stream=1)) == pp.PP_ERR_UNSUPPORTED
    assert call(opt=pp.Options(sibling_scan=1)) == pp.PP_ERR_UNSUPPORTED
    assert call(ws_bytes=16, opt=pp.Options(splits=4)) == pp.PP_ERR_CAPACITY
    opt = pp.Options(splits=148)
    plan = pp.split_plan(5000, 32, 5000, 148, causal=True)
    slots = plan["units"] * plan["max_chunks"] * 256
    assert pp.doc_prefill_workspace_bytes(32, 128, 5000, opt) == slots * 128 * 4 + slots * 2 * 4


def test_reset_streams_host_validation(pp):
    L = fake_layer(pp)
    assert pp._reset_streams(ctypes.byref(L), 0x1000, 0, None) == pp.PP_OK    # nothing to do
    assert pp._reset_streams(ctypes.byref(L), 0x1000, -1, None) == pp.PP_ERR_INVALID_ARG
    assert pp._reset_streams(ctypes.byref(L), None, 3, None) == pp.PP_ERR_INVALID_ARG
    assert pp._reset_streams(ctypes.byref(L), 0x1001, 3, None) == pp.PP_ERR_INVALID_ARG
    assert pp._reset_streams(None, 0x1000, 3, None) == pp.PP_ERR_INVALID_ARG
