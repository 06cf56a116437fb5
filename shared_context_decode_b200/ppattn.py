"""ctypes binding of libppattn (include/ppattn.h): argument marshalling only.

Every step of the attention path runs in the library's sm_100a kernels; this
module checks tensor types, passes ``data_ptr()`` values and the current
CUDA stream, and turns error codes into exceptions.  Importing it loads
``libppattn.so`` and raises if the library is missing -- there is no
fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libppattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is not built; run shared_context_decode_b200.build.build() "
        "(or __graft_entry__.build()) first")

_lib = ctypes.CDLL(LIB_PATH)

# ---------------------------------------------------------------- ABI -----
PP_OK, PP_ERR_INVALID_ARG, PP_ERR_UNSUPPORTED, PP_ERR_CAPACITY, PP_ERR_CUDA, \
    PP_ERR_DEVICE_TIMEOUT = range(6)
PP_DEV_SEGMENT_OVERFLOW = 0x1
PP_DEV_DOC_OUT_OF_RANGE = 0x2
PP_DEV_BAD_STREAM = 0x4
PP_DEV_TIMEOUT = 0x8

_i32, _vp, _sz = ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t


class LayerStruct(ctypes.Structure):
    _fields_ = [("H", _i32), ("d", _i32), ("doc_cap", _i32), ("P_max", _i32), ("S_cap", _i32),
                ("reserved", _i32), ("k_doc", _vp), ("v_doc", _vp), ("k_suf", _vp),
                ("v_suf", _vp), ("sid", _vp), ("pos", _vp), ("len", _vp), ("status", _vp)]


class Options(ctypes.Structure):
    _fields_ = [("splits", _i32), ("ablation_doc_per_stream", _i32),
                ("debug_inject_timeout", _i32), ("wait_limit_log2", _i32),
                ("events", ctypes.POINTER(_vp)), ("sibling_scan", _i32),
                ("suffix_slices", _i32)]

    def set_events(self, events):
        """Record 3 CUDA events (torch.cuda.Event, enable_timing=True) around
        the kernels of each decode/prefill call -- before the document pass,
        after it, after the suffix pass with its merge; None clears them."""
        if events is None:
            self.events = None
            self._ev = None
            return
        for e in events:
            if e.cuda_event == 0:   # torch creates the event on first record
                e.record()
        if len(events) != 3:
            raise ValueError("set_events takes 3 events")
        self._ev = (_vp * 3)(*[e.cuda_event for e in events])
        self.events = ctypes.cast(self._ev, ctypes.POINTER(_vp))


_LP = ctypes.POINTER(LayerStruct)
_OP = ctypes.POINTER(Options)


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_status_str = _sig("pp_status_str", ctypes.c_char_p, _i32)
_abi_version = _sig("pp_abi_version", _i32)
_kv_reset = _sig("pp_kv_reset", _i32, _LP, _vp)
_kv_append = _sig("pp_kv_append", _i32, _LP, _vp, _vp, _vp, _vp, _i32, _vp)
_dec_ws = _sig("pp_decode_workspace_bytes", _sz, _i32, _i32, _i32, _i32, _OP)
_pre_ws = _sig("pp_prefill_workspace_bytes", _sz, _i32, _i32, _i32, _i32, _OP)
_decode = _sig("pp_decode_attn", _i32, _LP, _i32, _vp, _vp, _vp, _i32, ctypes.c_float, _vp, _vp,
               _vp, _sz, _OP, _vp)
_decode_step = _sig("pp_decode_step", _i32, _LP, _i32, _vp, _vp, _vp, _vp, _vp, _i32,
                    ctypes.c_float, _vp, _vp, _vp, _sz, _OP, _vp)
_decode_noalloc = _sig("pp_decode_attn_noalloc", _i32, _LP, _i32, _vp, _vp, _vp, _i32,
                      ctypes.c_float, _vp, _vp, _OP, _vp)
_prefill = _sig("pp_prefill_attn", _i32, _LP, _i32, _vp, _vp, _vp, _i32, ctypes.c_float, _vp,
                _vp, _vp, _sz, _OP, _vp)
_visibility = _sig("pp_debug_visibility", _i32, _LP, _i32, _vp, _vp, _i32, _vp, _vp, _vp)
_exp2 = _sig("pp_debug_exp2", _i32, _vp, _vp, _vp, _i32, _vp)
_dev_status = _sig("pp_get_device_status", _i32, _LP, ctypes.POINTER(_i32), _vp)
_split_plan = _sig("pp_debug_split_plan", _i32, _i32, _i32, _i32, _i32,
                   ctypes.POINTER(ctypes.c_int64), _i32)
_split_plan_causal = _sig("pp_debug_split_plan_causal", _i32, _i32, _i32, _i32,
                          ctypes.POINTER(ctypes.c_int64), _i32)
_reset_streams = _sig("pp_kv_reset_streams", _i32, _LP, _vp, _i32, _vp)
_doc_ws = _sig("pp_doc_prefill_workspace_bytes", _sz, _i32, _i32, _i32, _OP)
_doc_prefill = _sig("pp_doc_prefill_attn", _i32, _LP, _i32, _vp, ctypes.c_float, _vp, _vp, _vp,
                    _sz, _OP, _vp)

EXPORTED = ("pp_status_str", "pp_abi_version", "pp_kv_reset", "pp_kv_append",
            "pp_decode_workspace_bytes", "pp_prefill_workspace_bytes", "pp_decode_attn",
            "pp_prefill_attn", "pp_debug_visibility", "pp_get_device_status",
            "pp_debug_split_plan", "pp_debug_exp2", "pp_decode_attn_noalloc",
            "pp_doc_prefill_workspace_bytes", "pp_doc_prefill_attn", "pp_debug_split_plan_causal",
            "pp_kv_reset_streams", "pp_decode_step")

# Size of the scratch array built into the library for pp_decode_attn_noalloc.
NOALLOC_SCRATCH_BYTES = 32 << 20


class PPError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)}")


def status_str(status: int) -> str:
    return _status_str(int(status)).decode()


def abi_version() -> int:
    return int(_abi_version())


def _check(status: int, what: str):
    if status != PP_OK:
        raise PPError(status, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _want(t: torch.Tensor, dtype, name: str, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _opts(opt: Optional[Options]):
    return None if opt is None else ctypes.byref(opt)


# ------------------------------------------------------------- KV cache ---
class KVLayer:
    """One layer's KV cache in the library's layout, allocated with torch.

    k_doc, v_doc [H, doc_cap, d] bf16; k_suf, v_suf [P_max, H, S_cap, d] bf16;
    sid [P_max, S_cap] int16; pos [P_max, S_cap] int32; len [P_max] int32;
    status [1] int32.
    """

    def __init__(self, H: int, d: int, doc_cap: int, P_max: int, S_cap: int, device="cuda",
                 len_buf: Optional[torch.Tensor] = None):
        dev = torch.device(device)
        if dev.type == "cuda" and dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        self.H, self.d, self.doc_cap, self.P_max, self.S_cap = H, d, doc_cap, P_max, S_cap
        bf = torch.bfloat16
        self.k_doc = torch.zeros((H, doc_cap, d), dtype=bf, device=dev)
        self.v_doc = torch.zeros((H, doc_cap, d), dtype=bf, device=dev)
        self.k_suf = torch.zeros((P_max, H, S_cap, d), dtype=bf, device=dev)
        self.v_suf = torch.zeros((P_max, H, S_cap, d), dtype=bf, device=dev)
        self.sid = torch.zeros((P_max, S_cap), dtype=torch.int16, device=dev)
        self.pos = torch.zeros((P_max, S_cap), dtype=torch.int32, device=dev)
        if len_buf is not None:      # caller-provided view, e.g. one row of [layers, P_max]
            _want(len_buf, torch.int32, "len_buf", dev)
            if len_buf.shape != (P_max,):
                raise ValueError("len_buf must be [P_max] int32")
            len_buf.zero_()
            self.len = len_buf
        else:
            self.len = torch.zeros((P_max,), dtype=torch.int32, device=dev)
        self.status = torch.zeros((1,), dtype=torch.int32, device=dev)
        self.struct = LayerStruct(H, d, doc_cap, P_max, S_cap, 0,
                                  self.k_doc.data_ptr(), self.v_doc.data_ptr(),
                                  self.k_suf.data_ptr(), self.v_suf.data_ptr(),
                                  self.sid.data_ptr(), self.pos.data_ptr(),
                                  self.len.data_ptr(), self.status.data_ptr())

    @property
    def ref(self):
        return ctypes.byref(self.struct)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.k_doc, self.v_doc, self.k_suf, self.v_suf, self.sid, self.pos,
                    self.len, self.status))


def kv_reset(layer: KVLayer):
    _check(_kv_reset(layer.ref, _stream(layer.device)), "pp_kv_reset")


def kv_reset_streams(layer: KVLayer, sid: torch.Tensor):
    """Free the segments of the streams listed in sid [n] int16 (ids 1..P_max,
    -1 = unused place) for new questions: their len becomes 0."""
    _want(sid, torch.int16, "sid", layer.device)
    _check(_reset_streams(layer.ref, _ptr(sid), sid.numel(), _stream(layer.device)),
           "pp_kv_reset_streams")


def kv_append(layer: KVLayer, k: torch.Tensor, v: torch.Tensor, sid: torch.Tensor,
              pos: torch.Tensor):
    """Append rows k, v [n, H, d] bf16 with stream ids sid [n] int16 and
    positions pos [n] int32."""
    dev = layer.device
    _want(k, torch.bfloat16, "k", dev)
    _want(v, torch.bfloat16, "v", dev)
    _want(sid, torch.int16, "sid", dev)
    _want(pos, torch.int32, "pos", dev)
    n = sid.shape[0]
    if k.shape != (n, layer.H, layer.d) or v.shape != k.shape or pos.shape != (n,):
        raise ValueError("kv_append: shapes must be k, v [n, H, d], sid, pos [n]")
    _check(_kv_append(layer.ref, _ptr(k), _ptr(v), _ptr(sid), _ptr(pos), n, _stream(dev)),
           "pp_kv_append")


def decode_workspace_bytes(P: int, H: int, d: int, doc_len: int, opt: Optional[Options] = None):
    return int(_dec_ws(P, H, d, doc_len, _opts(opt)))


def prefill_workspace_bytes(R: int, H: int, d: int, doc_len: int,
                            opt: Optional[Options] = None):
    return int(_pre_ws(R, H, d, doc_len, _opts(opt)))


def workspace(nbytes: int, device) -> torch.Tensor:
    """A caller-owned workspace buffer (256-byte aligned by the allocator)."""
    return torch.empty((max(nbytes, 256),), dtype=torch.uint8, device=device)


def _attn(fn, name, layer, doc_len, q, q_sid, q_pos, scale, o, lse, ws, opt, ws_fn):
    dev = layer.device
    rows = q_sid.shape[0]
    _want(q, torch.bfloat16, "q", dev)
    _want(q_sid, torch.int16, "q_sid", dev)
    _want(q_pos, torch.int32, "q_pos", dev)
    if q.shape != (rows, layer.H, layer.d) or q_pos.shape != (rows,):
        raise ValueError(f"{name}: q must be [rows, H, d], q_sid and q_pos [rows]")
    if o is None:
        o = torch.empty_like(q)
    _want(o, torch.bfloat16, "o", dev)
    if lse is not None:
        _want(lse, torch.float32, "lse", dev)
    if ws is None:
        ws = workspace(ws_fn(rows, layer.H, layer.d, doc_len, opt), dev)
    _want(ws, torch.uint8, "ws", dev)
    _check(fn(layer.ref, doc_len, _ptr(q), _ptr(q_sid), _ptr(q_pos), rows, float(scale), _ptr(o),
              _ptr(lse), _ptr(ws), ws.numel(), _opts(opt), _stream(dev)), name)
    return o


def doc_prefill_workspace_bytes(H: int, d: int, doc_len: int, opt: Optional[Options] = None):
    return int(_doc_ws(H, d, doc_len, _opts(opt)))


def doc_prefill_attn(layer: KVLayer, doc_len: int, q: torch.Tensor, scale: float,
                     o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                     ws: Optional[torch.Tensor] = None,
                     opt: Optional[Options] = None) -> torch.Tensor:
    """Causal attention of the document's own tokens: q [doc_len, H, d] bf16,
    row i = document token i; its K/V must already be appended (stream 0)."""
    dev = layer.device
    _want(q, torch.bfloat16, "q", dev)
    if q.shape != (doc_len, layer.H, layer.d):
        raise ValueError("pp_doc_prefill_attn: q must be [doc_len, H, d]")
    if o is None:
        o = torch.empty_like(q)
    _want(o, torch.bfloat16, "o", dev)
    if lse is not None:
        _want(lse, torch.float32, "lse", dev)
    if ws is None:
        ws = workspace(doc_prefill_workspace_bytes(layer.H, layer.d, doc_len, opt), dev)
    _want(ws, torch.uint8, "ws", dev)
    _check(_doc_prefill(layer.ref, doc_len, _ptr(q), float(scale), _ptr(o), _ptr(lse), _ptr(ws),
                        ws.numel(), _opts(opt), _stream(dev)), "pp_doc_prefill_attn")
    return o


def decode_attn(layer: KVLayer, doc_len: int, q: torch.Tensor, q_sid: torch.Tensor,
                q_pos: torch.Tensor, scale: float, o: Optional[torch.Tensor] = None,
                lse: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                opt: Optional[Options] = None) -> torch.Tensor:
    """Decode-step attention of P query rows; returns o [P, H, d] bf16."""
    return _attn(_decode, "pp_decode_attn", layer, doc_len, q, q_sid, q_pos, scale, o, lse, ws,
                 opt, decode_workspace_bytes)


def decode_step(layer: KVLayer, doc_len: int, k: torch.Tensor, v: torch.Tensor, q: torch.Tensor,
                q_sid: torch.Tensor, q_pos: torch.Tensor, scale: float,
                o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                ws: Optional[torch.Tensor] = None, opt: Optional[Options] = None) -> torch.Tensor:
    """One decode step of a layer: append row i's k/v to stream q_sid[i] at
    q_pos[i], then attend; returns o [P, H, d] bf16."""
    dev = layer.device
    rows = q_sid.shape[0]
    for t, nm in ((k, "k"), (v, "v")):
        _want(t, torch.bfloat16, nm, dev)
        if t.shape != (rows, layer.H, layer.d):
            raise ValueError(f"pp_decode_step: {nm} must be [rows, H, d]")

    def fn(ref, doc_len_, qp, sp, pp_, n, sc, op, lp, wp, wn, optp, st):
        return _decode_step(ref, doc_len_, _ptr(k), _ptr(v), qp, sp, pp_, n, sc, op, lp, wp, wn,
                            optp, st)

    return _attn(fn, "pp_decode_step", layer, doc_len, q, q_sid, q_pos, scale, o, lse, ws, opt,
                 decode_workspace_bytes)


def decode_attn_noalloc(layer: KVLayer, doc_len: int, q: torch.Tensor, q_sid: torch.Tensor,
                        q_pos: torch.Tensor, scale: float, o: Optional[torch.Tensor] = None,
                        lse: Optional[torch.Tensor] = None,
                        opt: Optional[Options] = None) -> torch.Tensor:
    """decode_attn without a workspace, for callers that cannot allocate
    device memory (the library's built-in scratch holds the partials).  Pass
    `o` to avoid the one torch allocation this wrapper would otherwise make.
    Calls must not overlap on the GPU: they share the scratch."""
    dev = layer.device
    rows = q_sid.shape[0]
    _want(q, torch.bfloat16, "q", dev)
    _want(q_sid, torch.int16, "q_sid", dev)
    _want(q_pos, torch.int32, "q_pos", dev)
    if q.shape != (rows, layer.H, layer.d) or q_pos.shape != (rows,):
        raise ValueError("pp_decode_attn_noalloc: q must be [rows, H, d], q_sid and q_pos [rows]")
    if o is None:
        o = torch.empty_like(q)
    _want(o, torch.bfloat16, "o", dev)
    if lse is not None:
        _want(lse, torch.float32, "lse", dev)
    _check(_decode_noalloc(layer.ref, doc_len, _ptr(q), _ptr(q_sid), _ptr(q_pos), rows,
                           float(scale), _ptr(o), _ptr(lse), _opts(opt), _stream(dev)),
           "pp_decode_attn_noalloc")
    return o


def prefill_attn(layer: KVLayer, doc_len: int, q: torch.Tensor, q_sid: torch.Tensor,
                 q_pos: torch.Tensor, scale: float, o: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                 opt: Optional[Options] = None) -> torch.Tensor:
    """Question-prefill attention of R rows; returns o [R, H, d] bf16."""
    return _attn(_prefill, "pp_prefill_attn", layer, doc_len, q, q_sid, q_pos, scale, o, lse, ws,
                 opt, prefill_workspace_bytes)


def debug_visibility(layer: KVLayer, doc_len: int, q_sid: torch.Tensor, q_pos: torch.Tensor,
                     with_mask: bool = True):
    """(count [nq] int32, mask [nq, P_max*S_cap] uint8 or None) from the
    kernels' own mask predicate."""
    dev = layer.device
    _want(q_sid, torch.int16, "q_sid", dev)
    _want(q_pos, torch.int32, "q_pos", dev)
    nq = q_sid.shape[0]
    count = torch.empty((nq,), dtype=torch.int32, device=dev)
    mask = torch.empty((nq, layer.P_max * layer.S_cap), dtype=torch.uint8, device=dev) \
        if with_mask else None
    _check(_visibility(layer.ref, doc_len, _ptr(q_sid), _ptr(q_pos), nq, _ptr(count), _ptr(mask),
                       _stream(dev)), "pp_debug_visibility")
    return count, mask


def debug_exp2(x: torch.Tensor):
    """(polynomial 2^x, hardware 2^x) for a float32 CUDA tensor x."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise TypeError("x must be a contiguous float32 CUDA tensor")
    yp, yh = torch.empty_like(x), torch.empty_like(x)
    _check(_exp2(_ptr(x), _ptr(yp), _ptr(yh), x.numel(), _stream(x.device)), "pp_debug_exp2")
    return yp, yh


def device_status(layer: KVLayer) -> int:
    """The layer's device status word (PP_DEV_* bits).  A word with
    PP_DEV_TIMEOUT set is returned too (the call reports it as
    PP_ERR_DEVICE_TIMEOUT; device_status_code gives that code)."""
    return device_status_code(layer)[1]


def device_status_code(layer: KVLayer):
    """(pp_status of pp_get_device_status, status word)."""
    out = _i32(0)
    rc = int(_dev_status(layer.ref, ctypes.byref(out), _stream(layer.device)))
    if rc not in (PP_OK, PP_ERR_DEVICE_TIMEOUT):
        _check(rc, "pp_get_device_status")
    return rc, int(out.value)


def split_plan(rows: int, H: int, doc_len: int, ctas: int, causal: bool = False):
    """The document split the library would use: dict with T, units, W, C,
    max_chunks and, per unit, its (first CTA, last CTA).  causal: the split
    of a document prefill (rows = doc_len)."""
    units = -(-(doc_len if causal else rows) // 256) * H
    buf = (ctypes.c_int64 * (5 + 2 * units))()
    if causal:
        _check(_split_plan_causal(doc_len, H, ctas, buf, len(buf)), "pp_debug_split_plan_causal")
    else:
        _check(_split_plan(rows, H, doc_len, ctas, buf, len(buf)), "pp_debug_split_plan")
    vals = list(buf)
    return dict(T=vals[0], units=vals[1], W=vals[2], C=vals[3], max_chunks=vals[4],
                chunks=[(vals[5 + 2 * u], vals[6 + 2 * u]) for u in range(units)])
