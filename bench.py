"""Benchmark of the Parallel Prompting decode step on B200.

A step is one decode step of a request with P answer streams over all L
layers: per layer, append every stream's new K/V (pp_kv_append), then the
decode attention (pp_decode_attn: document pass on the tensor cores, suffix
pass, log-sum-exp merge).  The step is captured once as a CUDA graph and
replayed; the KV cache is restored to its pre-step lengths at the start of
every step, so each step does identical work on identical inputs.

Default workload: doc 16384 tokens, P = 256 streams, H = 32, d = 128,
32 layers, question lengths U[16,48], cached answers U[0,63] (bf16, seeded
synthetic data).  The document KV one step reads (8.6 GB) is far larger than
the 126 MB L2, so no flush is needed between steps.

The end-to-end figure (e2e) replays the same step with every layer's inputs
copied from pinned host memory and its output copied back, as one CUDA graph
on three streams so that the copies overlap the kernels.

Output: one JSON line on rank 0 (see the keys in main()).  Multi-GPU
(torchrun): every rank runs an independent replica (weak scaling, no data
collective); time is the max over ranks.

Secondary measurements (--mode, one GPU, one JSON line each):
  prefill   question prefill of the prefill_doc12k_p256 workload: per layer,
            append the R question rows, then pp_prefill_attn; rows/s and the
            document part's TFLOP/s
  ablation  the decode step with the per-stream document pass (every stream
            reads the whole document) instead of the shared one
  siblingscan  the decode step with the suffix part done as the pages' kernel
            does it (every query scans all streams' answer tokens, masked)
  docprefill  causal attention of a 16384-token document over its own
            tokens (pp_doc_prefill_attn), 32 heads, d = 128; tokens/s and TFLOP/s
  sweep     answer generation over doc x streams: 32 decode steps x 32
            layers per combination, streams stopping after geometric lengths
            (inactive rows keep their place in the fixed-shape graph)
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn stream-tokens/s"
UNIT = "stream-tokens/s"


# ------------------------------------------------------------ distributed --
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(x: float, world: int, device) -> float:
    """Max over ranks of a per-rank float (a timing)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def aggregate(units_per_rank: float, ms_per_step_rank: float, world: int, device):
    """Whole-job throughput: units of all ranks / the slowest rank's time."""
    ms = reduce_max(ms_per_step_rank, world, device)
    units = reduce_sum(units_per_rank, world, device)
    return units / (ms / 1e3), ms


# ---------------------------------------------------------------- clocks ---
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms; summary()
    keeps the samples taken inside [t_start, t_end] (host clock)."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        # raw samples: $PP_CLOCKS_DIR if set, else the system temporary directory
        import tempfile
        d = os.environ.get("PP_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(d, f"pp_clocks_rank{gpu_index}.csv")
        self.t_start = self.t_end = None

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv",
                 "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.5)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def mark(self, which: str):
        setattr(self, "t_" + which, time.time())

    def summary(self):
        import datetime
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        mhz, mx, reasons, seen = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path).read().splitlines()[1:]:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, mxv = float(f[2].split()[0]), float(f[3].split()[0])
            except ValueError:
                continue
            seen += 1
            if self.t_start is not None and not (self.t_start - 0.25 <= ts <= self.t_end + 0.25):
                continue
            mhz.append(sm)
            mx = mxv
            for n, v in zip(names, f[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(mhz)) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz), "samples_total": seen}


# --------------------------------------------------------------- workload --
class DecodeStep:
    """Device-resident cache of all layers, the step's inputs, and the
    captured CUDA graph of one decode step."""

    def __init__(self, name: str, layers: int, device, seed: int = 0):
        from shared_context_decode_b200 import ppattn as pp
        from shared_context_decode_b200 import workloads as wl
        self.pp = pp
        self.W = W = wl.make_decode(name, seed=seed, device=device)
        self.layers = layers
        self.device = device
        self.S_cap = int(math.ceil(W.S_need / 16) * 16)
        self.len_all = torch.zeros((layers, W.P), dtype=torch.int32, device=device)
        self.cache, self.inp = [], []
        for l in range(layers):
            L = W.layer(l)
            kv = pp.KVLayer(W.H, W.d, W.N, W.P, self.S_cap, device, len_buf=self.len_all[l])
            pp.kv_append(kv, L.doc_k, L.doc_v, torch.zeros(W.N, dtype=torch.int16, device=device),
                         torch.arange(W.N, dtype=torch.int32, device=device))
            pp.kv_append(kv, L.suf_k, L.suf_v, L.suf_sid, L.suf_pos)
            self.cache.append(kv)
            self.inp.append(dict(k=L.new_k, v=L.new_v, q=L.q, sid=L.q_sid, pos=L.q_pos,
                                 o=torch.empty_like(L.q)))
            del L
        torch.cuda.synchronize()
        self.len0 = self.len_all.clone()
        self.opts = None   # per-layer pp_options of the captured step (None = default)
        # one pp_decode_step per layer (the append inside the document pass);
        # False: pp_kv_append then pp_decode_attn, for comparison
        self.fused = True
        self.ws = pp.workspace(pp.decode_workspace_bytes(W.P, W.H, W.d, W.N), device)
        self.graph = None

    def layer_call(self, l, opt):
        """Append layer l's decode tokens and attend."""
        pp, x = self.pp, self.inp[l]
        if self.fused:
            pp.decode_step(self.cache[l], self.W.N, x["k"], x["v"], x["q"], x["sid"], x["pos"],
                           self.W.scale, o=x["o"], ws=self.ws, opt=opt)
        else:
            pp.kv_append(self.cache[l], x["k"], x["v"], x["sid"], x["pos"])
            pp.decode_attn(self.cache[l], self.W.N, x["q"], x["sid"], x["pos"], self.W.scale,
                           o=x["o"], ws=self.ws, opt=opt)

    def run_eager(self, opts=None):
        """One decode step, launched eagerly (also the body that is captured);
        opts: per-layer pp_options or None."""
        opts = opts if opts is not None else self.opts
        self.len_all.copy_(self.len0)
        for l in range(self.layers):
            self.layer_call(l, None if opts is None else opts[l])

    def capture(self):
        self.run_eager()           # warm: per-device setup happens outside the capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                self.run_eager()
        torch.cuda.current_stream(self.device).wait_stream(s)
        torch.cuda.synchronize()
        self.graph = g

    def replay(self):
        self.graph.replay()

    def capture_e2e(self, host_in, host_out, names):
        """The step end to end as one CUDA graph on three streams: every
        layer's inputs are copied from pinned host memory on an input stream
        (all issued up front, so the copies run ahead of the kernels), each
        layer's kernels wait only for that layer's inputs, and each layer's
        output is copied back to pinned host memory on an output stream as
        soon as the layer ends."""
        pp, dev = self.pp, self.device
        comp, cin, cout = (torch.cuda.Stream(dev) for _ in range(3))
        g = torch.cuda.CUDAGraph()
        comp.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(comp):
            with torch.cuda.graph(g, stream=comp):
                self.len_all.copy_(self.len0)
                cin.wait_stream(comp)
                cout.wait_stream(comp)
                ev_in = []
                with torch.cuda.stream(cin):
                    for l in range(self.layers):
                        for n in names:
                            self.inp[l][n].copy_(host_in[l][n], non_blocking=True)
                        e = torch.cuda.Event()
                        e.record(cin)
                        ev_in.append(e)
                for l in range(self.layers):
                    x = self.inp[l]
                    comp.wait_event(ev_in[l])
                    self.layer_call(l, None if self.opts is None else self.opts[l])
                    e = torch.cuda.Event()
                    e.record(comp)
                    cout.wait_event(e)
                    with torch.cuda.stream(cout):
                        host_out[l].copy_(x["o"], non_blocking=True)
                comp.wait_stream(cin)
                comp.wait_stream(cout)
        torch.cuda.current_stream(dev).wait_stream(comp)
        torch.cuda.synchronize()
        self.graph_e2e = g

    def kernels_per_step(self) -> int:
        # per layer: the document pass (carrying the append) and the suffix
        # pass + merge; the append's own two kernels when it runs separately
        # (unfused, or beside the ablation and sibling-scan modes)
        n = 0
        for l in range(self.layers):
            o = None if self.opts is None else self.opts[l]
            other = o is not None and (o.ablation_doc_per_stream or o.sibling_scan)
            n += 4 if (not self.fused or other or self.W.N == 0) else 2
        return n

    def check_status(self):
        for kv in self.cache:
            st = self.pp.device_status(kv)
            if st:
                raise RuntimeError(f"device status {st:#x}")


class PrefillStep:
    """Question prefill of all layers as one CUDA graph: per layer, append the
    R question rows to their stream segments (emptied at the start of every
    step), then pp_prefill_attn (document pass with M = 128-row tiles of all
    R rows, the causal question part, merge)."""

    def __init__(self, name: str, layers: int, device, seed: int = 0):
        from shared_context_decode_b200 import ppattn as pp
        from shared_context_decode_b200 import workloads as wl
        self.pp = pp
        self.W = W = wl.make_prefill(name, seed=seed, device=device)
        self.layers = layers
        self.device = device
        S_cap = int(math.ceil(int(W.q_len.max()) / 16) * 16)
        self.len_all = torch.zeros((layers, W.P), dtype=torch.int32, device=device)
        self.cache, self.inp = [], []
        for l in range(layers):
            L = W.layer(l)
            kv = pp.KVLayer(W.H, W.d, W.N, W.P, S_cap, device, len_buf=self.len_all[l])
            pp.kv_append(kv, L.doc_k, L.doc_v, torch.zeros(W.N, dtype=torch.int16, device=device),
                         torch.arange(W.N, dtype=torch.int32, device=device))
            self.cache.append(kv)
            self.inp.append(dict(k=L.qk, v=L.qv, q=L.q, sid=L.sid, pos=L.pos,
                                 o=torch.empty_like(L.q)))
            del L
        torch.cuda.synchronize()
        self.ws = pp.workspace(pp.prefill_workspace_bytes(W.R, W.H, W.d, W.N), device)
        self.graph = None

    def run_eager(self, opts=None):
        pp = self.pp
        self.len_all.zero_()
        for l in range(self.layers):
            x = self.inp[l]
            pp.kv_append(self.cache[l], x["k"], x["v"], x["sid"], x["pos"])
            pp.prefill_attn(self.cache[l], self.W.N, x["q"], x["sid"], x["pos"], self.W.scale,
                            o=x["o"], ws=self.ws, opt=None if opts is None else opts[l])

    capture = DecodeStep.capture
    replay = DecodeStep.replay
    check_status = DecodeStep.check_status

    def kernels_per_step(self) -> int:
        return self.layers * 4


def eager_e2e(step, host_in, host_out, names, steps: int, world: int, dev):
    """The decode step end to end with no graph: for each layer, copy its
    inputs from pinned host memory, call the C ABI (pp_decode_step, or the
    step's configured calls), copy o back, all on the current stream.
    Returns the throughput, the device time per step and the host time spent
    issuing one layer (copies + C-ABI call), the per-call host cost a caller
    that does not capture a graph pays."""
    cur = torch.cuda.current_stream(dev)

    def one():
        step.len_all.copy_(step.len0)
        for l in range(step.layers):
            x = step.inp[l]
            for n in names:
                x[n].copy_(host_in[l][n], non_blocking=True)
            step.layer_call(l, None if step.opts is None else step.opts[l])
            host_out[l].copy_(x["o"], non_blocking=True)

    one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for _ in range(steps):
        one()
    e1.record(cur)
    torch.cuda.synchronize()
    value, ms = aggregate(step.W.P, e0.elapsed_time(e1) / steps, world, dev)
    # host cost of issuing a step, one step at a time from an idle stream (a
    # long run of eager steps fills the launch queue and the issuing thread
    # then waits for the GPU, which is not the cost of the call)
    host_s = []
    for _ in range(3):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        one()
        host_s.append(time.perf_counter() - t0)
    torch.cuda.synchronize()
    return {"value": value, "unit": UNIT, "ms_per_step": ms,
            "host_us_per_layer_call": min(host_s) / step.layers * 1e6,
            "form": "eager: per layer copies in, one C-ABI call, o copied out"}


def timed_replays(step, steps: int, warmup: int, world: int, local: int):
    for _ in range(warmup):
        step.replay()
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        torch.cuda.synchronize()
        clocks.mark("start")
        t0.record()
        for _ in range(steps):
            step.replay()
        t1.record()
        torch.cuda.synchronize()
        clocks.mark("end")
    barrier(world)
    return t0.elapsed_time(t1) / steps, clocks.summary()


def mode_prefill(args, world, rank, local, dev):
    name = "prefill_doc12k_p256"
    from shared_context_decode_b200 import workloads as wl
    nl = args.layers or wl.CONFIGS[name]["layers"]
    step = PrefillStep(name, nl, dev)
    step.capture()
    W = step.W
    ms, clocks = timed_replays(step, args.steps, args.warmup, world, local)
    step.check_status()
    value, ms = aggregate(W.R, ms, world, dev)
    flops = 4.0 * W.R * W.N * W.d * W.H * nl
    tfs = flops / (ms / 1e3) / 1e12 * world
    peaks = load_peaks()
    durs = measure_doc_pass(step, 2)          # per-layer document pass / question part times
    doc_tfs = 4.0 * W.R * W.N * W.d * W.H / (durs["doc"] * 1e-3) / 1e12
    # question part + merge: segments read once, q read, o written, the
    # document partials (one chunk per row) read
    q_bytes = W.R * W.H * W.d * 2 * 2 + 2 * W.R * W.H * W.d * 2 + W.R * W.H * (W.d + 2) * 4
    q_gbs = q_bytes / (durs["suffix"] * 1e-3) / 1e9
    line = {"mode": "prefill", "metric": "prefill rows/s", "value": value, "unit": "rows/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": name, "layers": nl, "H": W.H, "d": W.d, "doc_tokens": W.N,
                       "streams": W.P, "rows": W.R,
                       "l2": "per-layer document KV and question rows exceed L2"},
            "doc_tflops": tfs, "doc_frac_of_sustained_bf16": tfs / world / peaks["bf16_sustained"],
            "per_layer_us": {"doc_pass": durs["doc"] * 1e3, "question_part": durs["suffix"] * 1e3,
                             "doc_pass_tflops": doc_tfs,
                             "doc_pass_frac_burst_bf16": doc_tfs / peaks["bf16"],
                             "doc_pass_frac_sustained_bf16": doc_tfs / peaks["bf16_sustained"],
                             "doc_pass_frac_spec_bf16": doc_tfs / SPEC_BF16_TFLOPS,
                             "question_part_bytes": q_bytes, "question_part_gbs": q_gbs,
                             "question_part_frac_hbm": q_gbs / peaks["hbm"]},
            "gpu_launches": step.kernels_per_step() * args.steps, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del step.graph


def mode_ablation(args, world, rank, local, dev, sibling=False):
    from shared_context_decode_b200 import workloads as wl
    nl = args.layers or 4
    step = DecodeStep(args.workload, nl, dev)
    pp = step.pp
    step.opts = [pp.Options(sibling_scan=1) if sibling else pp.Options(ablation_doc_per_stream=1)
                 for _ in range(nl)]
    step.capture()
    W = step.W
    ms, clocks = timed_replays(step, args.steps, args.warmup, world, local)
    step.check_status()
    value, ms = aggregate(W.P, ms, world, dev)
    shared_b, _ = doc_pass_algorithmic(W)
    line = {"mode": "siblingscan" if sibling else "ablation", "metric": METRIC, "value": value,
            "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": args.workload, "layers": nl, "H": W.H, "d": W.d,
                       "doc_tokens": W.N, "streams": W.P,
                       "ablation": "sibling_scan" if sibling else "doc_per_stream"},
            **({"suffix_keys_per_query_scanned": W.suffix_tokens() + W.P,
                "suffix_keys_per_query_own_segment": (W.suffix_tokens() + W.P) / W.P}
               if sibling else
               {"doc_bytes_per_layer_shared": shared_b,
                "doc_bytes_per_layer_ablation": shared_b * W.P}),
            "gpu_launches": step.kernels_per_step() * args.steps, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del step.graph


def mode_longanswer(args, world, rank, local, dev):
    """Decode step with long answers (1024 cached answer tokens per stream):
    the suffix pass dominates.  Timed with the automatic slicing of the
    suffix work (the value) and with each slicing forced."""
    from shared_context_decode_b200 import workloads as wl
    name = "doc8k_p128_a1k"
    nl = args.layers or wl.CONFIGS[name]["layers"]
    step = DecodeStep(name, nl, dev)
    pp, W = step.pp, step.W
    runs = {}
    for mode, sl in (("automatic", 0), ("equal_items", 1), ("balanced", 2)):
        step.opts = [pp.Options(suffix_slices=sl) for _ in range(nl)]
        step.capture()
        ms, clocks = timed_replays(step, args.steps, args.warmup, world, local)
        step.check_status()
        per = measure_doc_pass(step, args.roofline_reps)
        # measure_doc_pass gives milliseconds
        runs[mode] = {"ms_per_step": ms, "doc_us": per["doc"] * 1e3,
                      "suffix_merge_us": per["suffix"] * 1e3,
                      "clocks": clocks}
        del step.graph
    ms = runs["automatic"]["ms_per_step"]
    value, ms = aggregate(W.P, ms, world, dev)
    suf_bytes = W.suffix_tokens() * W.H * W.d * 2 * 2 + W.P * W.H * W.d * 2 * 2
    line = {"mode": "longanswer", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": name, "layers": nl, "H": W.H, "d": W.d, "doc_tokens": W.N,
                       "streams": W.P, "suffix_tokens": W.suffix_tokens()},
            "suffix_bytes_per_layer": suf_bytes,
            "suffix_hbm_gbs": {k: suf_bytes / (v["suffix_merge_us"] * 1e3) for k, v in runs.items()},  # B/us / 1e3 = GB/s
            "runs": runs, "gpu_launches": step.kernels_per_step() * args.steps * 3,
            "clocks": runs["automatic"]["clocks"]}
    if rank == 0:
        print(json.dumps(line), flush=True)


def mode_docprefill(args, world, rank, local, dev):
    """Document prefill: per layer, causal attention of the document's own
    tokens with the document K/V already cached (written once, outside the
    timed region, as the append of the document would)."""
    from shared_context_decode_b200 import ppattn as pp
    from shared_context_decode_b200 import workloads as wl
    N, H, d = 16384, 32, 128
    nl = args.layers or 8
    layers, inp = [], []
    for l in range(nl):
        k = wl.randn_bf16((N, H, d), wl.seed_of("docprefill", l, "k"), dev)
        v = wl.randn_bf16((N, H, d), wl.seed_of("docprefill", l, "v"), dev)
        kv = pp.KVLayer(H, d, N, 1, 16, dev)
        pp.kv_append(kv, k, v, torch.zeros(N, dtype=torch.int16, device=dev),
                     torch.arange(N, dtype=torch.int32, device=dev))
        del k, v
        q = wl.randn_bf16((N, H, d), wl.seed_of("docprefill", l, "q"), dev)
        layers.append(kv)
        inp.append((q, torch.empty_like(q)))
    ws = pp.workspace(pp.doc_prefill_workspace_bytes(H, d, N), dev)
    scale = 1.0 / math.sqrt(d)

    class Step:
        def run_eager(self):
            for l in range(nl):
                pp.doc_prefill_attn(layers[l], N, inp[l][0], scale, o=inp[l][1], ws=ws)

    step = Step()
    step.device, step.cache, step.pp = dev, layers, pp
    DecodeStep.capture(step)
    step.replay = lambda: step.graph.replay()
    ms, clocks = timed_replays(step, args.steps, args.warmup, world, local)
    DecodeStep.check_status(step)
    value, ms = aggregate(N * nl, ms, world, dev)
    flops = 4.0 * d * H * (N * (N + 1) / 2) * nl   # the causal half of S = QK^T and O = PV
    tfs = flops / (ms / 1e3) / 1e12 * world
    peaks = load_peaks()
    line = {"mode": "docprefill", "metric": "document-prefill tokens/s", "value": value,
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "document prefill", "layers": nl, "H": H, "d": d,
                       "doc_tokens": N},
            "tflops": tfs, "frac_of_sustained_bf16": tfs / world / peaks["bf16_sustained"],
            "frac_of_burst_bf16": tfs / world / peaks["bf16"],
            "gpu_launches": 2 * nl * args.steps, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del step.graph


def sweep_roof_ms(W, stops, steps: int, layers: int, peaks) -> float:
    """Roof time of one sweep combination: per step, the slower of its
    algorithmic bytes at the HBM copy rate and its FLOPs at the burst bf16
    rate, summed over the steps.  Bytes per layer: the document K/V once,
    every active stream's segment once (question, answers so far, the new
    token), the new tokens' K/V read and written, q read and o written;
    FLOPs: S = QK^T and O = PV of the active rows over the document and
    their segments.  A stream is active at step t iff t < its stop length."""
    N, P = W.N, W.P
    kvb = W.H * W.d * 2 * 2
    roof_ms = 0.0
    for t in range(steps):
        act = t < stops
        seg_tok = float(((W.q_len + t + 1) * act).sum())
        byt = layers * (N * kvb + seg_tok * kvb + 2 * int(act.sum()) * kvb + P * kvb)
        fl = layers * 4.0 * W.d * W.H * (int(act.sum()) * N + seg_tok)
        roof_ms += max(byt / (peaks["hbm"] * 1e9), fl / (peaks["bf16"] * 1e12)) * 1e3
    return roof_ms


def sweep_combo(N: int, P: int, layers: int, dev, warm: bool = True):
    """One doc x streams combination of the answer-generation sweep: returns
    (active stream-tokens, device ms) over its decode steps.  The graph holds
    all P rows; a stream past its stop length keeps its row with stream id -1
    (no append, no suffix work, zero output)."""
    from shared_context_decode_b200 import ppattn as pp
    from shared_context_decode_b200 import workloads as wl
    cfg = wl.sweep_config(N, P)
    name = f"sweep_N{N}_P{P}"
    W = wl.make_decode(None, layers=layers, H=cfg["H"], d=cfg["d"], N=N, P=P, q=cfg["q"],
                       a=cfg["a"], device=dev)
    stops = wl.stop_lengths(P, name)
    steps = cfg["steps"]
    S_cap = int(math.ceil((int(W.q_len.max()) + steps + 1) / 16) * 16)
    len_all = torch.zeros((layers, P), dtype=torch.int32, device=dev)
    cache, inp = [], []
    for l in range(layers):
        L = W.layer(l)
        kv = pp.KVLayer(W.H, W.d, N, P, S_cap, dev, len_buf=len_all[l])
        pp.kv_append(kv, L.doc_k, L.doc_v, torch.zeros(N, dtype=torch.int16, device=dev),
                     torch.arange(N, dtype=torch.int32, device=dev))
        pp.kv_append(kv, L.suf_k, L.suf_v, L.suf_sid, L.suf_pos)
        cache.append(kv)
        inp.append(dict(k=L.new_k, v=L.new_v, q=L.q, o=torch.empty_like(L.q)))
        del L
    torch.cuda.synchronize()
    len0 = len_all.clone()
    q_sid = torch.empty(P, dtype=torch.int16, device=dev)
    q_pos = torch.empty(P, dtype=torch.int32, device=dev)
    ws = pp.workspace(pp.decode_workspace_bytes(P, W.H, W.d, N), dev)
    base_pos = (N + W.q_len).astype(np.int32)
    sids = np.arange(1, P + 1, dtype=np.int16)
    host = [(torch.from_numpy(np.where(t < stops, sids, -1).astype(np.int16)).pin_memory(),
             torch.from_numpy(base_pos + t).pin_memory(), int((t < stops).sum()))
            for t in range(steps)]
    roof_ms = sweep_roof_ms(W, stops, steps, layers, load_peaks())

    def body():
        for l in range(layers):
            x = inp[l]
            pp.kv_append(cache[l], x["k"], x["v"], q_sid, q_pos)
            pp.decode_attn(cache[l], N, x["q"], q_sid, q_pos, W.scale, o=x["o"], ws=ws)

    q_sid.copy_(host[0][0])
    q_pos.copy_(host[0][1])
    body()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            body()
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize()
    tokens, ms = 0, 0.0
    for rep in range(2 if warm else 1):
        len_all.copy_(len0)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for t in range(steps):
            q_sid.copy_(host[t][0], non_blocking=True)
            q_pos.copy_(host[t][1], non_blocking=True)
            ev[t][0].record()
            g.replay()
            ev[t][1].record()
        torch.cuda.synchronize()
        tokens = sum(h[2] for h in host)
        ms = sum(a.elapsed_time(b) for a, b in ev)
    for kv in cache:
        st = pp.device_status(kv)
        if st:
            raise RuntimeError(f"device status {st:#x} in sweep N={N} P={P}")
    # every stream appended exactly min(stop, steps) tokens
    want = len0.cpu() + torch.from_numpy(np.minimum(stops, steps).astype(np.int32))
    if not torch.equal(len_all.cpu(), want):
        raise RuntimeError(f"segment lengths after the sweep differ (N={N} P={P})")
    del g
    return tokens, ms, float(np.mean(stops)), roof_ms


def mode_sweep(args, world, rank, local, dev):
    from shared_context_decode_b200 import workloads as wl
    nl = args.layers or 32
    peaks = load_peaks()
    rows, tot_tok, tot_ms, tot_roof = [], 0, 0.0, 0.0
    with ClockSampler(local) as clocks:
        clocks.mark("start")
        for N in wl.SWEEP_DOCS:
            for P in wl.SWEEP_STREAMS:
                tok, ms, mean_stop, roof_ms = sweep_combo(N, P, nl, dev)
                torch.cuda.empty_cache()
                rows.append({"N": N, "P": P, "stream_tokens": tok, "ms": ms,
                             "value": tok / (ms / 1e3), "mean_stop": mean_stop,
                             "roof_ms": roof_ms, "frac_of_roofline": roof_ms / ms})
                tot_tok += tok
                tot_ms += ms
                tot_roof += roof_ms
        clocks.mark("end")
    value, ms = aggregate(tot_tok, tot_ms, world, dev)
    line = {"mode": "sweep", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": wl.SWEEP_STEPS, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "sweep", "layers": nl, "docs": list(wl.SWEEP_DOCS),
                       "streams": list(wl.SWEEP_STREAMS),
                       "stops": f"min({wl.SWEEP_STOP_CAP}, Geometric(1/{wl.SWEEP_STOP_MEAN}))"},
            "roofline": {"roof_ms": tot_roof, "ms": tot_ms, "frac": tot_roof / tot_ms,
                         "peaks": f"HBM copy and burst bf16, {peaks['source']}"},
            "combos": rows, "clocks": clocks.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)


def doc_pass_algorithmic(W):
    """Algorithmic bytes and FLOPs of one document-pass launch (one layer):
    every document K and V byte read once; S = Q K^T and O = P V over all
    P rows."""
    bytes_ = 2 * W.N * W.H * W.d * 2
    flops = 4 * W.P * W.N * W.d * W.H
    return bytes_, flops


# Nominal B200 figures (dense bf16, HBM3e), the stricter denominators.
SPEC_HBM_GBS, SPEC_BF16_TFLOPS = 8000.0, 2250.0


def doc_roofline(W, durs, peaks, traffic, sustained: bool = False):
    """Roofline record of the document pass.  The roof time is the slower of
    the algorithmic bytes at the measured HBM copy rate and the FLOPs at the
    bf16 tensor peak, and frac is roof time / measured time.  The tensor
    peak is the burst one when the run was short and cool (timed region
    under a second, no power cap in the clock samples), else the sustained
    one (the rate a seconds-long loop under the power cap settles at):
    sustained=True.  The fractions against both peaks and against the
    nominal figures (8 TB/s, 2.25 PFLOP/s: the stricter gate) are reported
    beside it."""
    b, f = doc_pass_algorithmic(W)
    t_doc = durs["doc"] * 1e-3
    gbs, tfs = b / t_doc / 1e9, f / t_doc / 1e12
    bf16 = peaks["bf16_sustained"] if sustained else peaks["bf16"]
    t_hbm, t_tc = b / (peaks["hbm"] * 1e9), f / (bf16 * 1e12)
    if t_tc > t_hbm:
        roof = {"bound": "tensor", "achieved": tfs, "peak": bf16, "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s"}
    roof["frac"] = max(t_hbm, t_tc) / t_doc
    t_burst = f / (peaks["bf16"] * 1e12)
    t_sus = f / (peaks["bf16_sustained"] * 1e12)
    t_spec = max(b / (SPEC_HBM_GBS * 1e9), f / (SPEC_BF16_TFLOPS * 1e12))
    tensor_peak = "sustained bf16" if sustained else "burst bf16"
    roof.update({"traffic": traffic, "kernel": f"pp::doc_pass_tc<{W.d}>",
                 "peak_source": peaks["source"] + (" " + tensor_peak if roof["bound"] == "tensor"
                                                   else " copy"),
                 "tensor_peak": tensor_peak,
                 "peak_rule": "burst bf16 when the timed region is under 1 s and the clock "
                              "samples show no power cap, else sustained bf16",
                 "roof_us": max(t_hbm, t_tc) * 1e6,
                 "doc_us": durs["doc"] * 1e3, "suffix_merge_us": durs["suffix"] * 1e3,
                 "doc_hbm_gbs": gbs, "doc_tflops": tfs,
                 "frac_hbm": gbs / peaks["hbm"], "frac_tensor_burst": tfs / peaks["bf16"],
                 "frac_burst": max(t_hbm, t_burst) / t_doc,
                 "frac_sustained": max(t_hbm, t_sus) / t_doc,
                 "frac_spec": t_spec / t_doc,
                 "frac_gate": min(max(t_hbm, t_tc), t_spec) / t_doc})
    return roof


def doc_profile(workload: str) -> str:
    """The committed ncu summary of the document pass on this workload."""
    return os.path.join(ROOT, "profiles", f"doc_pass_tc_{workload}.md")
DOC_SOURCES = ("doc_tc.cu", "append_warp.cuh", "common.cuh")


def kernel_source_hash(files=DOC_SOURCES) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "shared_context_decode_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profile_traffic(path: str, files=DOC_SOURCES):
    """DRAM bytes (read + write) per launch from a committed ncu summary, or
    None when the summary is absent or the kernel's sources changed since
    the capture (the summary records their sha256)."""
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path).read().splitlines():
        if ":" in line and line.startswith("- "):
            k, v = line[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    try:
        if fields.get("sources sha256") != kernel_source_hash(files):
            return None
        return float(fields["dram bytes per launch (read + write)"])
    except (KeyError, ValueError):
        return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def measure_doc_pass(step: DecodeStep, reps: int):
    """Average device duration of the document-pass kernel and of what follows
    it (the suffix kernel of a decode step; the run finding and question
    kernel of a prefill), from CUDA events the library records around them on the
    launching stream.  The step with the events is captured as its own CUDA
    graph (event-record nodes), so host launch overhead cannot leak into the
    intervals; each replay re-records all 3 events of every layer."""
    pp = step.pp
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(step.layers)]
    opts = []
    for l in range(step.layers):
        o = pp.Options()
        if getattr(step, "opts", None) is not None:   # same kernels as the timed step, plus the events
            for f, _ in pp.Options._fields_:
                if f != "events":
                    setattr(o, f, getattr(step.opts[l], f))
        o.set_events(evs[l])
        opts.append(o)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(step.device)
    s.wait_stream(torch.cuda.current_stream(step.device))
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step.run_eager(opts=opts)
    torch.cuda.current_stream(step.device).wait_stream(s)
    durs = {"doc": [], "suffix": []}
    for _ in range(reps + 1):
        g.replay()
        torch.cuda.synchronize()
        for e in evs:
            durs["doc"].append(e[0].elapsed_time(e[1]))
            durs["suffix"].append(e[1].elapsed_time(e[2]))
    n = step.layers
    del g
    return {k: float(np.mean(v[n:])) for k, v in durs.items()}   # first replay = warm-up


# ------------------------------------------------------------ CPU oracle ---
def oracle_sample(W, target_s: float, layer: int = 0):
    """Time the fp64 oracle on a bounded sample of the workload: all heads
    of the first n stream rows of one layer, n grown until the sample takes
    about target_s seconds.  The metric's unit is a stream token through all
    W.layers layers, so the sample's throughput is n / (W.layers * seconds):
    one layer is timed and the per-layer cost is taken as the same for the
    others (the layers differ only in their random draws).  Returns a dict
    with the throughput, the threads, and what was timed."""
    import oracle
    from shared_context_decode_b200.workloads import bf16_bits
    L = W.layer(layer)
    k = np.concatenate([bf16_bits(L.doc_k), bf16_bits(L.suf_k), bf16_bits(L.new_k)])
    v = np.concatenate([bf16_bits(L.doc_v), bf16_bits(L.suf_v), bf16_bits(L.new_v)])
    ks = np.concatenate([np.zeros(W.N, np.int32), L.suf_sid.cpu().numpy().astype(np.int32),
                         L.q_sid.cpu().numpy().astype(np.int32)])
    kp = np.concatenate([np.arange(W.N, dtype=np.int32), L.suf_pos.cpu().numpy(),
                         L.q_pos.cpu().numpy()])
    q, qs, qp = bf16_bits(L.q), L.q_sid.cpu().numpy(), L.q_pos.cpu().numpy()
    n, spent = 1, 0.0
    while True:
        t0 = time.perf_counter()
        oracle.masked_attention(q[:n], qs[:n], qp[:n], k, v, ks, kp, W.scale)
        spent = time.perf_counter() - t0
        if spent >= target_s or n >= W.P:
            break
        n = min(W.P, max(n + 1, int(n * min(4.0, 1.2 * target_s / max(spent, 1e-3)))))
    value = n / (spent * W.layers)
    desc = (f"layer {layer}: {n} of {W.P} stream rows x all {W.H} heads in {spent:.1f} s; "
            f"1 of {W.layers} layers timed, throughput = rows / ({W.layers} x seconds)")
    return {"value": value, "threads": oracle.num_threads(), "sample": desc, "rows_timed": n,
            "layers_timed": 1, "extrapolated_to_layers": W.layers, "seconds": spent,
            "ms_per_layer_of_rows": spent * 1e3}


def reference_arm(args, world, rank):
    """--impl reference: the oracle as it stands, on the host cores.  Each
    step is one bounded sample (oracle_sample) of the same workload; its
    inputs are drawn on the GPU when there is one, so they are the same bits
    the CUDA arm uses (the generators are device-specific)."""
    if rank != 0:
        return
    from shared_context_decode_b200 import workloads as wl
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    W = wl.make_decode(args.workload, device=gen_dev)
    vals, secs, units, samples = [], [], [], []
    for i in range(args.warmup + args.steps):
        r = oracle_sample(W, args.ref_seconds, layer=i % W.layers)
        if i >= args.warmup:
            vals.append(r["value"])
            secs.append(r["seconds"])
            units.append(r["rows_timed"] / W.layers)
            samples.append(r["sample"])
    value = float(np.sum(units) / np.sum(secs))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": float(np.mean(secs)) * 1e3,
            "units_per_step": float(np.mean(units)),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": args.workload, "layers": W.layers, "H": W.H, "d": W.d,
                       "doc_tokens": W.N, "streams": W.P},
            "step_definition": "one bounded oracle sample: the first rows of one layer, all "
                               "heads; stream tokens = rows / layers",
            "inputs": "same bits as the CUDA arm (drawn on the GPU)" if gen_dev == "cuda"
                      else "drawn on the CPU: the bits differ from the CUDA arm's",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": r["threads"],
                             "kind": "oracle", "sample": samples[-1],
                             "layers_timed": 1, "extrapolated_to_layers": W.layers},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main ---
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="doc16k_p256")
    ap.add_argument("--layers", type=int, default=0, help="0 = the workload's layer count")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU-baseline sample budget (0 = skip)")
    ap.add_argument("--ref-seconds", type=float, default=10.0)
    ap.add_argument("--roofline-reps", type=int, default=3)
    ap.add_argument("--separate-append", action="store_true",
                    help="decode: pp_kv_append + pp_decode_attn per layer instead of "
                         "pp_decode_step (append inside the document pass), for comparison")
    ap.add_argument("--suffix-slices", type=int, default=0, choices=[0, 1, 2],
                    help="decode: how the suffix pass's warps share the work "
                         "(pp_options.suffix_slices; 0 = automatic)")
    ap.add_argument("--mode", default="decode",
                    choices=["decode", "prefill", "ablation", "siblingscan", "sweep", "docprefill",
                             "longanswer"],
                    help="decode: the headline step (default); others: secondary measurements")
    args = ap.parse_args()
    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl" if torch.cuda.is_available() else "gloo",
                                timeout=datetime.timedelta(seconds=300))
    if args.impl == "reference":
        reference_arm(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    assert args.warmup >= 3, "at least 3 warm-up steps"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.mode != "decode":
        {"prefill": mode_prefill, "ablation": mode_ablation, "sweep": mode_sweep,
         "docprefill": mode_docprefill, "longanswer": mode_longanswer,
         "siblingscan": lambda *a: mode_ablation(*a, sibling=True)}[args.mode](
            args, world, rank, local, dev)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    from shared_context_decode_b200 import workloads as wl
    nl = args.layers or wl.CONFIGS[args.workload]["layers"]
    step = DecodeStep(args.workload, nl, dev)
    step.fused = not args.separate_append
    if args.suffix_slices:
        step.opts = [step.pp.Options(suffix_slices=args.suffix_slices) for _ in range(nl)]
    W = step.W
    step.capture()

    # ---- device-resident throughput: graph replays
    for _ in range(args.warmup):
        step.replay()
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        torch.cuda.synchronize()
        clocks.mark("start")
        t0.record()
        for _ in range(args.steps):
            step.replay()
        t1.record()
        torch.cuda.synchronize()
        clocks.mark("end")
    barrier(world)
    ms_rank = t0.elapsed_time(t1) / args.steps
    step.check_status()
    value, ms = aggregate(W.P, ms_rank, world, dev)

    # ---- end to end through the C ABI with host buffers
    names = ("k", "v", "q", "sid", "pos")
    host_in = [{n: step.inp[l][n].cpu().pin_memory() for n in names} for l in range(nl)]
    host_out = [torch.empty_like(step.inp[l]["o"], device="cpu").pin_memory() for l in range(nl)]
    h2d = sum(t.numel() * t.element_size() for d in host_in for t in d.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out)

    step.capture_e2e(host_in, host_out, names)

    def e2e_step():
        step.graph_e2e.replay()

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ek = max(3, args.steps // 2)
    e0.record()
    for _ in range(ek):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_value, e2e_ms = aggregate(W.P, e0.elapsed_time(e1) / ek, world, dev)
    # the overlapped copies must deliver the same output as the device step
    step.replay()
    torch.cuda.synchronize()
    for l in (0, nl - 1):
        if not torch.equal(host_out[l], step.inp[l]["o"].cpu()):
            raise RuntimeError(f"end-to-end output of layer {l} differs from the device step")

    # ---- end to end without a graph: per layer, the host->device copies of
    # its inputs, the C-ABI call and the copy of o back, issued eagerly on
    # one stream; the wall time of the issuing loop alone gives the host
    # cost per C-ABI call
    eager = eager_e2e(step, host_in, host_out, names, max(3, args.steps // 10), world, dev)

    # ---- roofline of the dominant kernel (document pass), live CUDA events
    durs = measure_doc_pass(step, args.roofline_reps)
    # the tensor peak the document pass is held to: burst for a short, cool
    # run, sustained when the timed region lasted a second or more or the
    # clocks were held down by the power cap
    clk = clocks.summary()
    sustained = args.steps * ms_rank >= 1000.0 or "sw_power_cap" in clk.get("reasons", [])
    roof = doc_roofline(W, durs, load_peaks(), profile_traffic(doc_profile(args.workload)),
                        sustained=sustained)

    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        r = oracle_sample(W, args.cpu_seconds)
        cpu = {"value": r["value"], "unit": UNIT, "cores": r["threads"], "kind": "oracle",
               "sample": r["sample"], "rows_timed": r["rows_timed"], "layers_timed": 1,
               "extrapolated_to_layers": r["extrapolated_to_layers"],
               "inputs": "same bits as the GPU run"}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": args.workload, "layers": nl, "H": W.H, "d": W.d,
                       "doc_tokens": W.N, "streams": W.P,
                       "suffix_tokens": W.suffix_tokens(),
                       "l2": "inputs larger than L2 (8.6 GB of document KV per step)"
                             if nl == 32 else "per-layer document KV exceeds L2",
                       "append": "inside the document pass (pp_decode_step)" if step.fused
                                 else "separate kernels (pp_kv_append)",
                       "suffix_slices": {0: "automatic", 1: "equal item counts",
                                         2: "balanced by work"}[args.suffix_slices],
                       "parallelism": f"replicas x{world}"},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "form": "one CUDA graph per step (copies overlapped on three streams)",
                    "eager": eager},
            "gpu_launches": step.kernels_per_step() * args.steps,
            "roofline": roof,
            "cpu_baseline": cpu,
            "clocks": clocks.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del step.graph, step.graph_e2e
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
