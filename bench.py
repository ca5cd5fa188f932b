#!/usr/bin/env python
"""Benchmark of the residual KV-cache compression hot path (librkv) on B200.

Headline workload (default): the Llama-3-8B-shaped 32-layer stack, 131072 tokens,
32 q / 8 kv heads, D=128, bf16, stride 16, k=4, int4 residuals.  One step is the
whole path over the stack: every layer's reference store, reference search and
residual encoding (the prefill cache compressed), then 64 decode steps, each a
decode-attention call on every one of the 32 layers.  All inputs (17 GB of K and V,
the queries of every step and layer) are resident in HBM when the timed region
starts; each layer's K and V (537 MB) and each layer's compressed cache (183 MB)
are larger than L2, and 31 other layers run between two visits of a layer, so L2 is
never warm for the data a stage reads.

Reported: `value` = compression Mtok/s (positions x layers of the stack over the
compression time of the step), `decode_us_per_step` = one decode step over all 32
layers, its achieved HBM GB/s and roofline fraction, and the per-stage times.  The
other workloads (tiny, Llama-shaped layer, Qwen2.5-7B-shaped ragged batch of 28
layers, 1M-token layer with the dynamic stride) are measured the same way and
reported under `configs`; the next rows (selective decode, incremental append,
int4 reference store, learned-coder shapes) under `next_rows`.  With N GPUs
(torchrun) every rank compresses its own independent stack; times are the maximum
over ranks.  `--impl reference` times the CPU oracle on a bounded row sample of the
headline workload.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "decode-attn µs/step & HBM GB/s vs roofline; compress Mtok/s; 1 B200"
HEADLINE = "llama3_8b_stack"
OTHER_WORKLOADS = ("tiny", "llama3_8b_layer", "qwen2_5_7b_batch", "ultra_long_1m")
NEXT_ROWS_WORKLOAD = "llama3_8b_layer"
SPARSE_SEL = 2048          # positions per unit of the selective-decode measurement
APPEND_TOKENS = 64         # tokens appended one at a time in the incremental-compression measurement
L2_BYTES = 126 << 20


def replica_layer(rank: int, layers: int = 1) -> int:
    """First layer index (generator seed) of a rank's replica: every rank works on its own
    independent layers."""
    return rank * layers


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Maximum of a per-rank time over all ranks (the job's time); identity on one rank."""
    if world <= 1:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, ms: float) -> float:
    """Whole-job Mtok/s: all ranks' tokens over the max-over-ranks time."""
    return world * tokens_per_rank / (ms * 1e-3) / 1e6


def _load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# fp32 FMA issue peak of the CUDA cores: 148 SMs x 128 lanes x 2 flop x 1.965 GHz
ALU_FP32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def host_cores() -> dict:
    """The host's core counts: os.cpu_count() and the cores this process may run on."""
    try:
        aff = len(os.sched_getaffinity(0))
    except AttributeError:
        aff = os.cpu_count() or 1
    return {"cpu_count": os.cpu_count() or 1, "affinity": aff}


def workload_quantities(wl, lengths):
    """Algorithmic work of one layer (sums over its units); the reference positions come
    from the library's host-side schedule."""
    import long_context_attention_rkv_b200 as rkv

    D = wl.head_dim
    per_tok = 2 * D * wl.bits // 8 + 2 * (D // 32) * 2 + 2 * wl.k
    flops = dec_bytes = dec_bytes4 = cmp_tokens = enc_bytes = refs_bytes = 0
    for n in lengths:
        cfg = rkv.make_config(head_dim=D, n_kv_heads=wl.n_kv_heads, n_q_heads=wl.n_q_heads, k=wl.k, bits=wl.bits,
                              stride0=wl.stride0, batch=1, max_len=max(n, 1), refs_per_phase=wl.refs_per_phase)
        ref_pos = rkv.rkv_schedule(cfg, n)
        R = len(ref_pos)
        C = n - R
        # search: every compressed token against its earlier references, 2*D flops each
        is_ref = np.zeros(n, dtype=bool)
        is_ref[ref_pos] = True
        cpos = np.nonzero(~is_ref)[0]
        ncand = np.searchsorted(ref_pos, cpos, side="right").astype(np.int64)
        flops += wl.n_kv_heads * int(ncand.sum()) * 2 * D
        cmp_tokens += wl.n_kv_heads * C
        dec_bytes += wl.n_kv_heads * (C * per_tok + R * 4 * D)
        # int4 reference store: codes (D/2 bytes) and binary16 scales (D/32) per row and side
        dec_bytes4 += wl.n_kv_heads * (C * per_tok + R * 2 * (D // 2 + 2 * (D // 32)))
        enc_bytes += wl.n_kv_heads * C * (2 * D * wl.elem_bytes + per_tok)
        refs_bytes += wl.n_kv_heads * R * (2 * D * wl.elem_bytes + 4 * D + 8)
    return dict(tokens=sum(lengths), tokens_cmp=cmp_tokens, search_flops=flops, decode_bytes=dec_bytes,
                decode_bytes_int4_refs=dec_bytes4, encode_bytes=enc_bytes, refs_bytes=refs_bytes,
                bytes_per_token=per_tok)


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML in a thread."""

    def __init__(self, index: int, period_s: float = 0.002):
        self.index = index
        self.period = period_s
        self.samples = []
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def start(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((mhz, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self._stop.set()
        if self._t:
            self._t.join()
        if not self.ok:
            return None
        names = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                 0x80: "hw_power_brake_slowdown"}
        seen = set()
        for _, r in self.samples:
            for bit, nm in names.items():
                if r & bit:
                    seen.add(nm)
        mhz = [m for m, _ in self.samples]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(seen), "samples": len(mhz)}


DECODE_SRC = ["long_context_attention_rkv_b200/csrc/kernels_decode_mma.cu",
              "long_context_attention_rkv_b200/csrc/kernels_decode_tc.cu",
              "long_context_attention_rkv_b200/csrc/decode_mma.h"]
ENCODE_SRC = ["long_context_attention_rkv_b200/csrc/kernels_encode.cu"]


def _src_sha(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(kernel: str, src: list[str], workload: str):
    """Per-launch DRAM bytes of a kernel on a workload from the committed ncu summary, if
    they were captured (or scaled from a capture) on the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(kernel, {}).get(workload)
    if not e or e.get("src_sha") != _src_sha(src):
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------------------
# the GPU path

def _cfg(rkv, wl, max_len, **kw):
    return rkv.make_config(head_dim=wl.head_dim, n_kv_heads=wl.n_kv_heads, n_q_heads=wl.n_q_heads, k=wl.k,
                           bits=wl.bits, stride0=wl.stride0, batch=wl.batch, max_len=max_len,
                           refs_per_phase=wl.refs_per_phase, in_dtype=wl.dtype_code, out_dtype=wl.dtype_code, **kw)


def pinned_layer(wl, layer: int, lengths, max_len: int):
    """One layer's K, V generated straight into pinned host tensors (bf16 as raw int16)."""
    import torch

    import synth

    shape = (wl.batch, wl.n_kv_heads, max_len, wl.head_dim)
    tdt = torch.int16 if wl.dtype == "bf16" else torch.float32
    Kp = torch.empty(shape, dtype=tdt, pin_memory=True)
    Vp = torch.empty(shape, dtype=tdt, pin_memory=True)
    view = (lambda t: t.numpy().view(np.uint16)) if wl.dtype == "bf16" else (lambda t: t.numpy())
    synth.fill_layer(wl, layer, view(Kp), view(Vp), lengths)
    return Kp, Vp


class Stack:
    """n_layers layers of one workload on one device: per-layer caches sharing one workspace,
    the layers' K and V and every (step, layer) query resident in HBM, one CUDA graph per
    (layer, compression stage) and one per decode step (all layers)."""

    STAGES = ("build_refs", "search", "encode")

    def __init__(self, wl, dev, layer0: int, n_layers: int, decode_steps: int, keep_host_layers: int = 0):
        import torch

        import long_context_attention_rkv_b200 as rkv
        import synth

        self.wl, self.dev, self.n_layers, self.decode_steps = wl, dev, n_layers, decode_steps
        self.lengths = wl.lengths()
        self.max_len = max(self.lengths)
        self.cfg = _cfg(rkv, wl, self.max_len)
        self.K, self.V, self.host = [], [], []
        for li in range(n_layers):
            Kp, Vp = pinned_layer(wl, layer0 + li, self.lengths, self.max_len)
            self.K.append(Kp.to(dev, non_blocking=False))
            self.V.append(Vp.to(dev, non_blocking=False))
            if li < keep_host_layers:
                self.host.append((Kp, Vp))
            else:
                del Kp, Vp
        tdt = torch.int16 if wl.dtype == "bf16" else torch.float32
        qshape = (wl.batch, wl.n_q_heads, wl.head_dim)
        qh = np.empty((decode_steps, n_layers) + qshape, dtype=synth.np_dtype(wl))
        for t in range(decode_steps):
            for li in range(n_layers):
                synth.gen_query(wl, layer0 + li, t, out=qh[t, li])
        self.q_host = torch.from_numpy(qh.view(np.int16) if wl.dtype == "bf16" else qh).pin_memory()
        self.q = self.q_host.to(dev)
        self.out = torch.empty((decode_steps, n_layers) + qshape, dtype=tdt, device=dev)
        _, ws = rkv.rkv_cache_size(self.cfg, self.lengths)
        self.workspace = torch.empty(max(256, ws), dtype=torch.uint8, device=dev)
        self.layers = [rkv.Layer(self.cfg, self.lengths, device=dev, workspace=self.workspace)
                       for _ in range(n_layers)]
        self.Q = workload_quantities(wl, self.lengths)
        self.graphs = None

    def _stage(self, li, nm):
        L, K, V = self.layers[li], self.K[li], self.V[li]
        if nm == "build_refs":
            L.build_refs(K, V)
        elif nm == "search":
            L.search(K)
        else:
            L.encode(K, V)

    def _decode_step(self, t):
        for li, L in enumerate(self.layers):
            L.decode(self.q[t, li], self.out[t, li])

    def capture(self, stream):
        import torch

        with torch.cuda.stream(stream):
            for li in range(self.n_layers):                 # eager pass first (also a warm-up)
                for nm in self.STAGES:
                    self._stage(li, nm)
            for t in range(self.decode_steps):
                self._decode_step(t)
            torch.cuda.synchronize(self.dev)
            self.g_stage = {}
            for li in range(self.n_layers):
                for nm in self.STAGES:
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=stream):
                        self._stage(li, nm)
                    self.g_stage[li, nm] = g
            self.g_dec = []
            for t in range(self.decode_steps):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    self._decode_step(t)
                self.g_dec.append(g)
        torch.cuda.synchronize(self.dev)
        self.check()

    def check(self):
        for L in self.layers:
            err = L.device_error()
            assert err == 0, f"device error {err}"

    def step(self, stream, record=False, flush=None):
        """Compression of every layer, then the decode steps.  record: a (start, end) event pair
        around every stage graph and every decode-step graph (none inside a graph); flush: an L2
        flush before every span, outside it (for workloads whose data would stay in L2)."""
        import torch

        def ev():
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            return e

        spans = {"stage": [], "decode": []}
        for li in range(self.n_layers):
            for nm in self.STAGES:
                if flush is not None:
                    flush.zero_()
                s = ev() if record else None
                self.g_stage[li, nm].replay()
                if record:
                    spans["stage"].append((li, nm, s, ev()))
        for t in range(self.decode_steps):
            if flush is not None:
                flush.zero_()
            s = ev() if record else None
            self.g_dec[t].replay()
            if record:
                spans["decode"].append((t, s, ev()))
        return spans

    def release(self):
        self.g_stage = None
        self.g_dec = None
        self.layers = None
        self.K = self.V = self.host = None


def summarise_steps(stack, all_spans, flushed: bool):
    """Per-step compression time (first stage start to last stage end; with flushes, the sum of
    the stage spans), per-stage means, and every decode step's time, in ms."""
    comp, stage, dec = [], {nm: [] for nm in Stack.STAGES}, []
    for spans in all_spans:
        st = spans["stage"]
        per = [s.elapsed_time(e) for _, _, s, e in st]
        for (_, nm, _, _), ms in zip(st, per):
            stage[nm].append(ms)
        comp.append(sum(per) if flushed else st[0][2].elapsed_time(st[-1][3]))
        dec.extend(s.elapsed_time(e) for _, s, e in spans["decode"])
    return comp, {nm: statistics.mean(v) for nm, v in stage.items()}, dec


def measure(wl, dev, stream, args, rank, world, n_layers, decode_steps, steps, warmup, keep_host_layers=0,
            clocks=False):
    """Times `steps` steps of a Stack (after `warmup` untimed ones); returns the stack (still
    alive, for the e2e and oracle legs) and a result dict (times max over ranks)."""
    import torch

    stack = Stack(wl, dev, replica_layer(rank, n_layers), n_layers, decode_steps, keep_host_layers)
    stack.capture(stream)
    # single-layer workloads: flush L2 (256 MiB write) before every timed span, outside it
    per_layer_bytes = 2 * wl.batch * wl.n_kv_heads * stack.max_len * wl.head_dim * wl.elem_bytes
    flushed = n_layers == 1 or per_layer_bytes < 2 * L2_BYTES
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flushed else None
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            stack.step(stream, flush=flush)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev.index if dev.index is not None else 0) if clocks else None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
    t0 = time.perf_counter()
    all_spans = []
    with torch.cuda.stream(stream):
        for _ in range(steps):
            all_spans.append(stack.step(stream, record=True, flush=flush))
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - t0
    if world > 1:
        torch.distributed.barrier()
    clk = sampler.stop() if sampler else None
    stack.check()
    comp, stage, dec = summarise_steps(stack, all_spans, flushed)
    Q = stack.Q
    comp_ms = max_over_ranks(statistics.mean(comp), world, dev)
    dec_ms = max_over_ranks(statistics.mean(dec), world, dev) if dec else 0.0
    stage = {nm: max_over_ranks(v, world, dev) for nm, v in stage.items()}
    peaks = _load_peaks()
    tokens = Q["tokens"] * n_layers
    dec_bytes = Q["decode_bytes"] * n_layers
    res = {
        "layers": n_layers, "decode_steps": decode_steps, "steps": steps, "warmup": warmup,
        "l2": ("flushed before every timed span (256 MiB write, outside the span)" if flushed else
               "not flushed: every layer's K, V (%.0f MB) and compressed cache exceed L2, and the other "
               "layers run between two visits of a layer" % (per_layer_bytes / 1e6)),
        "compress_ms": comp_ms,
        "compress_mtok_s": job_throughput(world, tokens, comp_ms),
        "decode_us_per_step": 1e3 * dec_ms,
        "decode_bytes_per_step": dec_bytes,
        "decode_hbm_gbs": dec_bytes / (dec_ms * 1e-3) / 1e9 if dec_ms else None,
        "decode_roofline_frac": (dec_bytes / (dec_ms * 1e-3) / 1e9) / peaks["hbm"] if dec_ms else None,
        "stage_us_per_layer": {nm: 1e3 * v for nm, v in stage.items()},
        "search_tflops": Q["search_flops"] / (stage["search"] * 1e-3) / 1e12,
        "search_flops_per_layer": Q["search_flops"],
        "encode_gbs": Q["encode_bytes"] / (stage["encode"] * 1e-3) / 1e9,
        "encode_bytes_per_layer": Q["encode_bytes"],
        "ms_per_step": max_over_ranks(statistics.mean(
            [c + sum(dec[i * decode_steps:(i + 1) * decode_steps]) for i, c in enumerate(comp)]), world, dev),
        "wall_s": wall,
    }
    if clk is not None:
        res["clocks"] = clk
    return stack, res


def e2e_leg(stack, dev, stream, steps, world):
    """The same step through the public API with host buffers: every layer's K and V copied in
    from pinned host memory (a copy stream, two device buffers, so layer l+1's copies overlap
    layer l's compression), then every decode call with its query copied in and its output
    copied out.  Returns compression Mtok/s and decode us/step measured over those spans."""
    import torch

    wl = stack.wl
    n_host = len(stack.host)
    Kb = [torch.empty_like(stack.K[0]) for _ in range(2)]
    Vb = [torch.empty_like(stack.V[0]) for _ in range(2)]
    cstream = torch.cuda.Stream(device=dev)
    out_h = torch.empty(stack.out.shape, dtype=stack.out.dtype, pin_memory=True)
    comp_ms, dec_ms = [], []
    h2d = d2h = 0
    for rep in range(steps + 1):                         # the first pass warms up
        copied = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        torch.cuda.synchronize(dev)
        h2d = d2h = 0
        e0.record(stream)
        cstream.wait_stream(stream)
        for li in range(stack.n_layers):
            b = li % 2
            Kp, Vp = stack.host[li % n_host]
            with torch.cuda.stream(cstream):
                if li >= 2:
                    cstream.wait_event(done[b])          # layer li-2 is done with this buffer
                Kb[b].copy_(Kp, non_blocking=True)
                Vb[b].copy_(Vp, non_blocking=True)
                copied[b].record(cstream)
            h2d += Kp.numel() * Kp.element_size() + Vp.numel() * Vp.element_size()
            with torch.cuda.stream(stream):
                stream.wait_event(copied[b])
                L = stack.layers[li]
                L.build_refs(Kb[b], Vb[b])
                L.compress(Kb[b], Vb[b])
                done[b].record(stream)
        e1.record(stream)
        with torch.cuda.stream(stream):
            for t in range(stack.decode_steps):
                for li, L in enumerate(stack.layers):
                    stack.q[t, li].copy_(stack.q_host[t, li], non_blocking=True)
                    L.decode(stack.q[t, li], stack.out[t, li])
                    out_h[t, li].copy_(stack.out[t, li], non_blocking=True)
        h2d += stack.q_host.numel() * stack.q_host.element_size()
        d2h += out_h.numel() * out_h.element_size()
        e2.record(stream)
        e2.synchronize()
        if rep > 0:
            comp_ms.append(e0.elapsed_time(e1))
            dec_ms.append(e1.elapsed_time(e2) / max(1, stack.decode_steps))
    stack.check()
    cm = max_over_ranks(statistics.mean(comp_ms), world, dev)
    dm = max_over_ranks(statistics.mean(dec_ms), world, dev)
    return {"value": job_throughput(world, stack.Q["tokens"] * stack.n_layers, cm), "unit": "Mtok/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "decode_us_per_step": 1e3 * dm, "compress_ms": cm,
            "host_layers": n_host,
            "note": ("every layer's K and V copied from its own pinned host buffer" if n_host == stack.n_layers else
                     "K and V copied from a ring of %d pinned host layers (host memory bound per rank)" % n_host)}


def next_rows(dev, stream, args):
    """The next rows on the Llama-shaped layer, each timed alone with L2 flushed before every
    call: selective decode, incremental append, the int4 reference store and the learned-coder
    shapes (seeded random weights)."""
    import torch

    import long_context_attention_rkv_b200 as rkv
    import synth

    wl = synth.WORKLOADS[NEXT_ROWS_WORKLOAD]
    lengths = wl.lengths()
    max_len = max(lengths)
    Kp, Vp = pinned_layer(wl, 0, lengths, max_len)
    K, V = Kp.to(dev), Vp.to(dev)
    q = torch.from_numpy(synth.gen_query(wl, 0, 0).view(np.int16)).to(dev)
    out = torch.empty((wl.batch, wl.n_q_heads, wl.head_dim), dtype=torch.int16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    Q = workload_quantities(wl, lengths)
    reps = max(3, min(args.steps, 20))

    def timed(fn, n=reps):
        ms = []
        with torch.cuda.stream(stream):
            for i in range(n + 2):
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                e1.synchronize()
                if i >= 2:
                    ms.append(e0.elapsed_time(e1))
        return statistics.mean(ms)

    def graphs_of(stages):
        g = {}
        with torch.cuda.stream(stream):
            for nm in stages:
                stages[nm]()
            torch.cuda.synchronize(dev)
            for nm in stages:
                gg = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gg, stream=stream):
                    stages[nm]()
                g[nm] = gg
        torch.cuda.synchronize(dev)
        return g

    res = {"workload": wl.name}
    L = rkv.Layer(_cfg(rkv, wl, max_len), lengths, device=dev)
    L.build_refs(K, V)
    L.compress(K, V)
    # selective decode: SPARSE_SEL seeded uniform positions per unit
    rng = np.random.default_rng(0x5E1)
    n_units = wl.batch * wl.n_kv_heads
    sel = np.zeros((n_units, SPARSE_SEL), dtype=np.int32)
    cnt = np.zeros(n_units, dtype=np.int32)
    for u in range(n_units):
        n = lengths[u // wl.n_kv_heads]
        m = min(n, SPARSE_SEL)
        sel[u, :m] = np.sort(rng.choice(n, m, replace=False))
        cnt[u] = m
    sel_d, cnt_d = torch.from_numpy(sel).to(dev), torch.from_numpy(cnt).to(dev)
    res["sparse_decode_us"] = 1e3 * timed(lambda: L.decode_sparse(q, sel_d, cnt_d, out, stream=stream))
    res["sparse_decode_positions_per_unit"] = SPARSE_SEL
    assert L.device_error() == 0
    del L

    # incremental compression: the last APPEND_TOKENS positions appended one at a time
    La = rkv.Layer(_cfg(rkv, wl, max_len), lengths, device=dev)
    start = [max(0, n - APPEND_TOKENS) for n in lengths]
    La.set_lengths(start)
    La.build_refs(K, V)
    La.compress(K, V)
    Hkv = wl.n_kv_heads
    bi = torch.arange(wl.batch, device=dev).repeat_interleave(Hkv)
    hi = torch.arange(Hkv, device=dev).repeat(wl.batch)
    rows = []
    for t in range(APPEND_TOKENS):
        pos = torch.tensor([min(s0 + t, max_len - 1) for s0 in start], device=dev).repeat_interleave(Hkv)
        rows.append((K[bi, hi, pos].contiguous(), V[bi, hi, pos].contiguous()))
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        # a busy-wait ahead of the span keeps the device behind the host while the appends are
        # issued, so the span holds the appends' device time, not Python's
        torch.cuda._sleep(20_000_000)
        e0.record(stream)
        for Kn, Vn in rows:
            La.append(Kn, Vn, stream=stream)
        e1.record(stream)
        e1.synchronize()
    assert La.device_error() == 0
    res["append_us_per_token"] = 1e3 * e0.elapsed_time(e1) / APPEND_TOKENS
    del La

    # int4 reference store
    L4 = rkv.Layer(_cfg(rkv, wl, max_len, ref_bits=4), lengths, device=dev)
    g4 = graphs_of({"build_refs": lambda: L4.build_refs(K, V), "search": lambda: L4.search(K),
                    "encode": lambda: L4.encode(K, V), "decode": lambda: L4.decode(q, out)})
    t4 = {nm: timed(g.replay) for nm, g in g4.items()}
    assert L4.device_error() == 0
    del g4, L4
    res["int4_refs"] = {
        "build_refs_us": 1e3 * t4["build_refs"], "search_us": 1e3 * t4["search"], "encode_us": 1e3 * t4["encode"],
        "decode_us_per_step": 1e3 * t4["decode"], "decode_bytes_per_step": Q["decode_bytes_int4_refs"],
        "decode_hbm_gbs": Q["decode_bytes_int4_refs"] / (t4["decode"] * 1e-3) / 1e9,
        "compress_mtok_s": Q["tokens"] / ((t4["build_refs"] + t4["search"] + t4["encode"]) * 1e-3) / 1e6}

    # learned-coder shapes: seeded random bf16 weights (scale 1/sqrt(D))
    wrng = np.random.default_rng(0xC0DE)
    cw = [torch.from_numpy((wrng.standard_normal((wl.head_dim, wl.head_dim)) / np.sqrt(wl.head_dim))
                           .astype(np.float32)).to(torch.bfloat16).to(dev) for _ in range(8)]
    Lc = rkv.Layer(_cfg(rkv, wl, max_len, coder=1), lengths, device=dev)
    Lc.set_coder(cw)
    gc = graphs_of({"build_refs": lambda: Lc.build_refs(K, V), "search": lambda: Lc.search(K),
                    "encode": lambda: Lc.encode(K, V), "decode": lambda: Lc.decode(q, out)})
    tc = {nm: timed(g.replay, n=max(3, min(args.steps, 10))) for nm, g in gc.items()}
    assert Lc.device_error() == 0
    del gc, Lc
    res["learned_coder"] = {
        "encode_us": 1e3 * tc["encode"], "decode_us_per_step": 1e3 * tc["decode"],
        "encode_latent_gflop": 2 * 2 * Q["tokens_cmp"] * 5 * wl.head_dim * wl.head_dim / 1e9,
        "compress_mtok_s": Q["tokens"] / ((tc["build_refs"] + tc["search"] + tc["encode"]) * 1e-3) / 1e6}
    return res


# ---------------------------------------------------------------------------------------
# the CPU oracle (a deliberately plain, slow program: the baseline, not the target)

def _row_sample(oracle, wl, n, seed, uniform=2048):
    """Deterministic compressed-position sample of one unit: the first k*s rows, the rows within
    2 of every dynamic-stride phase boundary, and `uniform` uniformly drawn rows."""
    ref_pos = oracle.schedule(n, wl.stride0, wl.refs_per_phase)
    cpos, is_ref = oracle.positions_split(n, ref_pos)
    pick = set(int(p) for p in cpos[:wl.k * wl.stride0])
    if wl.refs_per_phase:
        s, start = wl.stride0, 0
        while start < n:
            for d in range(-2, 3):
                p = start + d
                if 0 <= p < n and not is_ref[p]:
                    pick.add(p)
            start += wl.refs_per_phase * s
            s *= 2
    rng = np.random.default_rng(seed)
    pick.update(int(p) for p in rng.choice(cpos, min(uniform, len(cpos)), replace=False))
    return np.array(sorted(pick), dtype=np.int32), ref_pos


def _unit_rows(wl, layer, b, h, n):
    import synth

    K, V = synth.gen_unit(wl, layer, b, h, 0, n)
    return synth.as_f32(wl, K), synth.as_f32(wl, V)


def layer_rows(wl, layer):
    """Every unit's K, V rows of one layer as float arrays (the oracle's inputs)."""
    lengths = wl.lengths()
    return {(b, h): _unit_rows(wl, layer, b, h, lengths[b]) for b in range(wl.batch) for h in range(wl.n_kv_heads)}


def oracle_compress_sample(wl, layer, threads, uniform=2048, seed=7, data=None):
    """Oracle compression of the row sample of every unit of one layer, threads across units.
    Returns (positions of the layer compressed (each with all its kv heads), seconds, description)."""
    import oracle

    lengths = wl.lengths()
    units = [(b, h) for b in range(wl.batch) for h in range(wl.n_kv_heads)]
    data = layer_rows(wl, layer) if data is None else data
    samples = {u: _row_sample(oracle, wl, lengths[u[0]], seed + 97 * u[0] + u[1], uniform)[0] for u in units}

    def work(u):
        Xk, Xv = data[u]
        oracle.compress_unit(Xk, Xv, wl.stride0, wl.refs_per_phase, wl.k, wl.bits, positions=samples[u])

    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, units))
    dt = time.perf_counter() - t0
    rows = sum(len(s) for s in samples.values())
    desc = (f"{rows} compressed positions over the {len(units)} units of layer {layer} (per unit: the first k*s "
            f"rows, dynamic-phase boundary rows +-2, {uniform} uniform rows): oracle reference store, top-{wl.k} "
            f"brute-force search, encode; {threads} threads across units")
    # Mtok/s counts a position of the layer with all its kv heads, as the GPU figure does
    return rows / len(units) * wl.batch, dt, desc


def oracle_full_unit(wl, layer, threads):
    """Oracle compression of one whole unit (sequence 0, kv head 0), its positions split into
    `threads` row ranges (every position's selection is independent)."""
    import oracle

    n = wl.lengths()[0]
    Xk, Xv = _unit_rows(wl, layer, 0, 0, n)
    ref_pos = oracle.schedule(n, wl.stride0, wl.refs_per_phase)
    cpos, _ = oracle.positions_split(n, ref_pos)
    chunks = np.array_split(cpos, max(1, threads))

    def work(ch):
        if len(ch):
            oracle.compress_unit(Xk, Xv, wl.stride0, wl.refs_per_phase, wl.k, wl.bits, positions=ch)

    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, chunks))
    return n, time.perf_counter() - t0


def oracle_decode_layer(wl, stack_layer, q_f32, threads):
    """Oracle decode of one layer over the GPU's compressed cache (read back): per unit the
    reconstruction of every position and double-precision attention of its query heads."""
    import oracle

    G = wl.n_q_heads // wl.n_kv_heads
    units = [(b, h) for b in range(wl.batch) for h in range(wl.n_kv_heads)]
    arrays = {u: unit_arrays(stack_layer, wl, *u) for u in units}

    def work(u):
        b, h = u
        A = arrays[u]
        Kh, Vh = oracle.unit_cache_rows(A["n"], A["ref_pos"], A["refK"], A["refV"], A["idx"], A["codesK"],
                                        A["scalesK"], A["codesV"], A["scalesV"], wl.bits)
        return oracle.attention(q_f32[b, h * G:(h + 1) * G], Kh, Vh)

    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, units))
    return time.perf_counter() - t0


def unit_arrays(layer, wl, b, h):
    """One unit's compressed cache copied to host numpy arrays (bf16 reference rows as uint16)."""
    v = layer.unit(b, h)
    base = layer.cache.data_ptr()

    def grab(ptr, nbytes):
        off = ptr - base
        return layer.cache[off:off + nbytes].cpu().numpy()

    D = wl.head_dim
    out = {"n": v.n,
           "ref_pos": grab(v.ref_pos, 4 * v.n_ref).view(np.int32).copy(),
           "refK": grab(v.ref_K, 2 * v.n_ref * D).view(np.uint16).reshape(v.n_ref, D).copy(),
           "refV": grab(v.ref_V, 2 * v.n_ref * D).view(np.uint16).reshape(v.n_ref, D).copy(),
           "idx": grab(v.idx, 2 * v.n_cmp * v.k).view(np.uint16).reshape(v.n_cmp, v.k).copy(),
           "codesK": grab(v.codes_K, v.n_cmp * v.code_bytes).reshape(v.n_cmp, v.code_bytes).copy(),
           "codesV": grab(v.codes_V, v.n_cmp * v.code_bytes).reshape(v.n_cmp, v.code_bytes).copy(),
           "scalesK": grab(v.scale_K, 2 * v.n_cmp * v.n_groups).view(np.uint16).reshape(v.n_cmp, v.n_groups).copy(),
           "scalesV": grab(v.scale_V, 2 * v.n_cmp * v.n_groups).view(np.uint16).reshape(v.n_cmp, v.n_groups).copy()}
    return out


def cpu_baseline(wl, stack, threads_max):
    """The oracle as it stands on the host cores, beside the GPU numbers: the headline
    workload's row sample (compression Mtok/s), one whole unit, and one layer's decode over the
    GPU-produced cache; then the small workloads in full (the tiny one also single-threaded)."""
    import synth

    cores = host_cores()
    thr_units = min(threads_max, wl.batch * wl.n_kv_heads)
    tok, dt, desc = oracle_compress_sample(wl, 0, thr_units)
    n_full, dt_full = oracle_full_unit(wl, 0, threads_max)
    q0 = synth.as_f32(wl, stack.q_host[0, 0].numpy().view(np.uint16) if wl.dtype == "bf16"
                      else stack.q_host[0, 0].numpy())
    dt_dec = oracle_decode_layer(wl, stack.layers[0], q0, thr_units)
    res = {"value": tok / dt / 1e6, "unit": "Mtok/s", "cores": cores["affinity"], "cpu_count": cores["cpu_count"],
           "threads": thr_units, "kind": "oracle", "sample": desc, "seconds": dt,
           "full_unit": {"unit": "sequence 0, kv head 0 of layer 0", "positions": n_full, "seconds": dt_full,
                         "threads": threads_max,
                         "mtok_s_one_head": n_full / dt_full / 1e6},
           "decode_one_layer": {"ms": 1e3 * dt_dec, "threads": thr_units,
                                "what": "reconstruction of every position of the 8 units (GPU-produced "
                                        "cache) and attention of the 32 query heads, one step"}}
    per = {}
    for name in ("tiny", "llama3_8b_layer"):
        w = synth.WORKLOADS[name]
        n = w.lengths()[0]
        units = [(b, h) for b in range(w.batch) for h in range(w.n_kv_heads)]
        data = {u: _unit_rows(w, 0, u[0], u[1], n) for u in units}
        thr = [1, min(threads_max, len(units))] if name == "tiny" else [min(threads_max, len(units))]
        for t in thr:
            import oracle

            def comp(u):
                Xk, Xv = data[u]
                return oracle.compress_unit(Xk, Xv, w.stride0, w.refs_per_phase, w.k, w.bits)

            t0 = time.perf_counter()
            with ThreadPoolExecutor(t) as ex:
                outs = list(ex.map(comp, units))
            tc = time.perf_counter() - t0
            qf = synth.as_f32(w, synth.gen_query(w, 0, 0))
            G = w.n_q_heads // w.n_kv_heads

            def dec(i):
                b, h = units[i]
                r = outs[i]
                Kh, Vh = oracle.unit_cache_rows(n, r["ref_pos"], r["refK"], r["refV"], r["idx"], r["codesK"],
                                                r["scalesK"], r["codesV"], r["scalesV"], w.bits)
                return oracle.attention(qf[b, h * G:(h + 1) * G], Kh, Vh)

            t0 = time.perf_counter()
            with ThreadPoolExecutor(t) as ex:
                list(ex.map(dec, range(len(units))))
            td = time.perf_counter() - t0
            per[f"{name}_threads{t}"] = {"compress_mtok_s": n * w.batch / tc / 1e6, "compress_s": tc,
                                         "decode_us_per_step": 1e6 * td, "threads": t,
                                         "what": "full oracle compression and decode (all units)"}
    res["per_config"] = per
    return res


def run_reference(args, rank, world):
    """The oracle on the host cores, on the headline workload: every step compresses a bounded
    row sample of layer 0 (all units); value = positions per second."""
    import synth

    if rank != 0:
        return
    wl = synth.WORKLOADS[args.workload]
    cores = host_cores()
    threads = min(cores["affinity"], wl.batch * wl.n_kv_heads)
    uniform = args.ref_rows
    times, toks = [], []
    desc = ""
    data = layer_rows(wl, 0)
    for i in range(args.warmup + args.steps):
        tok, dt, desc = oracle_compress_sample(wl, 0, threads, uniform=uniform, seed=11 + i, data=data)
        if i >= args.warmup:
            times.append(dt)
            toks.append(tok)
    v = sum(toks) / sum(times) / 1e6
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "Mtok/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded prototype-cluster caches)", "config": _config(wl),
            "cpu_baseline": {"value": v, "unit": "Mtok/s", "cores": cores["affinity"],
                             "cpu_count": cores["cpu_count"], "threads": threads, "kind": "oracle",
                             "sample": desc + " (one such sample per step)"},
            "e2e": {"value": v, "unit": "Mtok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _config(wl):
    return {"workload": wl.name, "layers": wl.layers, "batch": wl.batch, "seq_len": wl.seq_len,
            "n_kv_heads": wl.n_kv_heads, "n_q_heads": wl.n_q_heads, "head_dim": wl.head_dim,
            "stride": wl.stride0, "refs_per_phase": wl.refs_per_phase, "k": wl.k, "bits": wl.bits,
            "group": wl.group, "decode_steps": wl.steps, "global_batch": wl.batch,
            "parallelism": "replicas (one independent stack per GPU)"}


def run_ours(args, rank, world, local_rank):
    import torch

    import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    wl = synth.WORKLOADS[args.workload]
    cores = host_cores()
    # pinned host copies for the e2e leg: every layer when it fits in a quarter of the host's
    # memory shared by the ranks, else a ring of two layers
    layer_bytes = 2 * wl.batch * wl.n_kv_heads * max(wl.lengths()) * wl.head_dim * wl.elem_bytes
    try:
        import psutil

        host_mem = psutil.virtual_memory().total
    except Exception:
        host_mem = 64 << 30
    keep = wl.layers if wl.layers * layer_bytes * world <= host_mem // 4 else 2
    steps, warmup = args.steps, args.warmup
    stack, head = measure(wl, dev, stream, args, rank, world, wl.layers, max(1, wl.steps), steps, warmup,
                          keep_host_layers=keep, clocks=True)
    e2e = e2e_leg(stack, dev, stream, max(2, min(steps, 3)), world)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, stack, cores["affinity"])
    stack.release()
    del stack
    torch.cuda.empty_cache()

    configs = {}
    if not args.headline_only:
        for name in OTHER_WORKLOADS:
            if name == wl.name:
                continue
            w = synth.WORKLOADS[name]
            st, r = measure(w, dev, stream, args, rank, world, w.layers, max(1, w.steps), max(3, min(steps, 5)), 3)
            st.release()
            del st
            torch.cuda.empty_cache()
            r.pop("wall_s", None)
            configs[name] = r
    nxt = None if args.headline_only else next_rows(dev, stream, args)

    peaks = _load_peaks()
    Q = workload_quantities(wl, wl.lengths())
    search_us = head["stage_us_per_layer"]["search"]
    encode_us = head["stage_us_per_layer"]["encode"]
    dec_layer_us = head["decode_us_per_step"] / wl.layers
    kernels = {"search": search_us, "encode": encode_us, "decode": dec_layer_us}
    dominant = max(kernels, key=lambda s: kernels[s] * (wl.layers * max(1, wl.steps) if s == "decode" else wl.layers))
    tensor = wl.dtype == "bf16"
    if dominant == "search":
        # the search runs back to back over the stack's layers (seconds of tensor work per
        # step): the sustained (power-capped) bf16 peak is its denominator
        if tensor:
            peak, bound, unit = peaks["bf16_sustained"], "tensor", "TFLOP/s"
        else:
            peak, bound, unit = ALU_FP32_TFLOPS, "alu", "TFLOP/s"
        ach = head["search_tflops"]
        kern = "select_tc" if tensor else "select_simt"
        traffic = _traffic(kern, ["long_context_attention_rkv_b200/csrc/kernels_%s.cu" % kern], wl.name)
    elif dominant == "encode":
        peak, bound, unit, ach = peaks["hbm"], "hbm", "GB/s", head["encode_gbs"]
        traffic = _traffic("encode", ENCODE_SRC, wl.name)
    else:
        peak, bound, unit, ach = peaks["hbm"], "hbm", "GB/s", head["decode_hbm_gbs"]
        traffic = _traffic("decode", DECODE_SRC, wl.name)
    roofline = {"kernel": dominant, "bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
                "traffic": traffic, "peak_source": peaks["source"] + (" sustained" if bound == "tensor" else ""),
                "frac_of_burst_peak": (ach / peaks["bf16"]) if bound == "tensor" else None,
                "decode": {"achieved_gbs": head["decode_hbm_gbs"], "peak_gbs": peaks["hbm"],
                           "frac": head["decode_roofline_frac"]},
                "encode": {"achieved_gbs": head["encode_gbs"], "peak_gbs": peaks["hbm"],
                           "frac": head["encode_gbs"] / peaks["hbm"]},
                "search": {"achieved_tflops": head["search_tflops"], "peak_tflops_sustained": peaks["bf16_sustained"],
                           "frac": head["search_tflops"] / peaks["bf16_sustained"],
                           "frac_of_burst_peak": head["search_tflops"] / peaks["bf16"]}}
    # kernels of this library launched per step: per layer the reference store (1), the search
    # (1, +1 bf16 key copy with the int4 store), the encoder's two passes; three per decode call
    per_step = wl.layers * 4 + wl.layers * max(1, wl.steps) * 3
    if rank == 0:
        line = {
            "metric": METRIC, "value": head["compress_mtok_s"], "unit": "Mtok/s", "n_gpus": world,
            "steps": steps, "warmup": warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if tensor else "f32",
            "data": "synthetic (seeded prototype-cluster caches)", "config": _config(wl),
            "decode_us_per_step": head["decode_us_per_step"],
            "decode_hbm_gbs": head["decode_hbm_gbs"], "decode_roofline_frac": head["decode_roofline_frac"],
            "parts": head,
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": per_step * steps,
            "clocks": head.get("clocks"),
            "configs": configs,
            "next_rows": nxt,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split(chr(10))[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true", help="skip the other workloads and the next rows")
    ap.add_argument("--ref-rows", type=int, default=1024,
                    help="uniform rows per unit of each reference-arm step (plus the first k*s rows)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch

            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
