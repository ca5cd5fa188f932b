#!/usr/bin/env python
"""Benchmark of the residual KV-cache compression hot path (librkv) on B200.

One step = the whole path over one layer of the Llama-3-8B-shaped workload
(32 q / 8 kv heads, D=128, bf16, 32768 tokens, stride 16, k=4, int4 residuals):
reference store, reference search, residual encoding, one decode-attention
step, and a 256-row reconstruction.  Inputs are resident in HBM when the timed
region starts; L2 is flushed (256 MiB write) before every timed step, outside
the timed spans.  With N GPUs (torchrun) every rank runs its own replica on an
independent layer; value is the whole-job throughput over the max-over-ranks
step time.  Outside the step, a selective decode (2048 seeded positions per unit),
incremental compression (the last 64 tokens appended one at a time), the same layer
with the int4 reference store (reference store, search, encode, decode) and with the
learned-coder shapes (random weights) are timed as well.  `--impl reference` times the CPU oracle on a bounded sample of
the same workload on the host cores.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
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
WORKLOAD = "llama3_8b_layer"
# kernels launched per step, by stage
LAUNCHES = {"build_refs": 1, "search": 1, "encode": 1, "decode": 3, "reconstruct": 1}
RECON_ROWS = 256
SPARSE_SEL = 2048          # positions per unit of the selective-decode measurement
APPEND_TOKENS = 64         # tokens appended one at a time in the incremental-compression measurement


def replica_layer(rank: int) -> int:
    """Layer index a rank compresses: every replica works on its own independent layer."""
    return rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Maximum of a per-rank time over all ranks (the job's time); identity on one rank."""
    if world <= 1:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job Mtok/s: all ranks' tokens over the max-over-ranks step time."""
    return world * tokens_per_rank / (ms_per_step * 1e-3) / 1e6


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


def workload_quantities(wl, lengths):
    """Algorithmic work of one step over one layer (per-unit sums); the reference positions
    come from the library's host-side schedule."""
    import long_context_attention_rkv_b200 as rkv

    D = wl.head_dim
    per_tok = 2 * D * wl.bits // 8 + 2 * (D // 32) * 2 + 2 * wl.k
    flops = 0
    dec_bytes = 0
    dec_bytes4 = 0
    cmp_tokens = 0
    enc_bytes = 0
    refs_bytes = 0
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
                decode_bytes_int4_refs=dec_bytes4,
                encode_bytes=enc_bytes, refs_bytes=refs_bytes, bytes_per_token=per_tok)


class ClockSampler:
    """Samples SM clock, power and clock-event reasons with NVML in a thread."""

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


def _src_sha(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(kernel: str, src: list[str]):
    """Per-launch DRAM bytes of a kernel from a committed ncu summary, if its source is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(kernel)
    if not e or e.get("src_sha") != _src_sha(src):
        return None
    return e.get("dram_bytes_per_launch")


class OracleSample:
    """Times the CPU oracle on a bounded sample of one step: S uniformly drawn compressed positions
    of every kv head are searched, encoded, reconstructed and attended over."""

    def __init__(self, wl, lengths, layer: int, threads: int):
        self.wl, self.lengths, self.layer, self.threads = wl, lengths, layer, threads
        self.S = 64
        self.reps = 1
        self._prep()

    def _prep(self):
        import oracle
        import synth

        wl, lengths, layer = self.wl, self.lengths, self.layer
        self._setup(oracle, synth, wl, lengths, layer)

    def _setup(self, oracle, synth, wl, lengths, layer):
        self.oracle = oracle
        n = lengths[0]
        K, V = synth.gen_layer(wl, layer, [n])
        self.G = wl.n_q_heads // wl.n_kv_heads
        self.qf = synth.as_f32(wl, synth.gen_query(wl, layer, 0))
        self.ref_pos = oracle.schedule(n, wl.stride0, wl.refs_per_phase)
        self.cpos, _ = oracle.positions_split(n, self.ref_pos)
        self.units = [(0, h) for h in range(wl.n_kv_heads)]
        self.Xs = {u: (synth.as_f32(wl, K[u[0], u[1], :n]), synth.as_f32(wl, V[u[0], u[1], :n])) for u in self.units}

    def _work(self, u, pos):
        oracle, wl, ref_pos, G = self.oracle, self.wl, self.ref_pos, self.G
        Xk, Xv = self.Xs[u]
        refK = oracle.build_refs(Xk, ref_pos)
        refV = oracle.build_refs(Xv, ref_pos)
        idx, _, _ = oracle.select(Xk[pos], pos, refK, ref_pos, wl.k)
        ek = oracle.encode(Xk[pos], refK, idx, wl.bits)
        ev = oracle.encode(Xv[pos], refV, idx, wl.bits)
        Kh = oracle.reconstruct(refK, idx, ek["codes"], ek["scales"], wl.bits)
        Vh = oracle.reconstruct(refV, idx, ev["codes"], ev["scales"], wl.bits)
        h = u[1]
        oracle.attention(self.qf[0, h * G:(h + 1) * G], Kh, Vh)

    def timed(self, S, seed, reps=1):
        rng = np.random.default_rng(seed)
        pos = np.sort(rng.choice(self.cpos, S, replace=False)).astype(np.int32)
        t0 = time.perf_counter()
        with ThreadPoolExecutor(self.threads) as ex:
            for _ in range(reps):
                list(ex.map(lambda u: self._work(u, pos), self.units))
        return time.perf_counter() - t0

    def calibrate(self, target_s: float):
        t = self.timed(self.S, 1)
        want = self.S * target_s / max(t, 1e-3)
        self.S = int(min(len(self.cpos), max(64, want)))
        self.reps = max(1, int(round(want / self.S)))   # whole sets repeated when all positions are too few
        return self

    def run(self, seed=2):
        """(positions per second, sample description, seconds)."""
        t = self.timed(self.S, seed, self.reps)
        reps = f" (the set processed {self.reps} times)" if self.reps > 1 else ""
        desc = (f"{self.S} uniformly drawn compressed positions{reps} x {len(self.units)} kv heads of one layer: "
                f"oracle reference store, top-{self.wl.k} search, encode, reconstruct and {self.G}-head "
                f"attention over the sampled rows; {self.threads} threads across kv heads")
        return self.S * self.reps / t, desc, t


def run_reference(args, rank, world):
    import synth

    if rank != 0:
        return
    wl = synth.WORKLOADS[args.workload]
    lengths = wl.lengths()
    threads = min(os.cpu_count() or 1, wl.n_kv_heads)
    per_step = max(0.5, min(4.0, 150.0 / max(1, args.steps + args.warmup)))
    sampler = OracleSample(wl, lengths, 0, threads).calibrate(per_step)
    rates = []
    for i in range(args.warmup + args.steps):
        rate, desc, t = sampler.run(seed=10 + i)
        if i >= args.warmup:
            rates.append(rate)
    v = statistics.mean(rates) / 1e6
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "Mtok/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * wl.seq_len / (v * 1e6),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _config(wl, lengths),
            "cpu_baseline": {"value": v, "unit": "Mtok/s", "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": "Mtok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _config(wl, lengths):
    return {"workload": wl.name, "layers": 1, "batch": wl.batch, "seq_len": wl.seq_len,
            "n_kv_heads": wl.n_kv_heads, "n_q_heads": wl.n_q_heads, "head_dim": wl.head_dim,
            "stride": wl.stride0, "k": wl.k, "bits": wl.bits, "group": wl.group, "global_batch": wl.batch,
            "l2": "flushed before every timed step (256 MiB write, outside the timed spans)",
            "parallelism": "replicas (one independent layer per GPU)"}


def run_ours(args, rank, world, local_rank):
    import torch

    import long_context_attention_rkv_b200 as rkv
    import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[args.workload]
    lengths = wl.lengths()
    layer_id = replica_layer(rank)
    Kh, Vh = synth.gen_layer(wl, layer_id, lengths)
    q_h = synth.gen_query(wl, layer_id, 0)
    tdt = torch.int16 if wl.dtype == "bf16" else torch.float32

    def pinned(a):
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).pin_memory()
        return t

    Kp, Vp, qp = pinned(Kh), pinned(Vh), pinned(q_h)
    K = Kp.to(dev)
    V = Vp.to(dev)
    q = qp.to(dev)
    cfg = rkv.make_config(head_dim=wl.head_dim, n_kv_heads=wl.n_kv_heads, n_q_heads=wl.n_q_heads, k=wl.k,
                          bits=wl.bits, stride0=wl.stride0, batch=wl.batch, max_len=K.shape[2],
                          refs_per_phase=wl.refs_per_phase, in_dtype=wl.dtype_code, out_dtype=wl.dtype_code)
    L = rkv.Layer(cfg, lengths, device=dev)
    out = torch.empty((wl.batch, wl.n_q_heads, wl.head_dim), dtype=tdt, device=dev)
    out_h = torch.empty_like(out, device="cpu").pin_memory()
    rpos = torch.arange(0, lengths[0], max(1, lengths[0] // RECON_ROWS), dtype=torch.int32,
                        device=dev)[:RECON_ROWS].contiguous()
    Kr = torch.empty((RECON_ROWS, wl.head_dim), dtype=torch.float32, device=dev)
    Vr = torch.empty_like(Kr)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    stages = {
        "build_refs": lambda: L.build_refs(K, V),
        "search": lambda: L.search(K),
        "encode": lambda: L.encode(K, V),
        "decode": lambda: L.decode(q, out),
        "reconstruct": lambda: L.reconstruct(0, 0, rpos, RECON_ROWS, Kr, Vr, rkv.RKV_DTYPE_F32),
    }
    names = list(stages)
    # one CUDA graph per stage (launch gaps removed; each stage timed by events around its replay)
    graphs = {}
    with torch.cuda.stream(stream):
        for nm in names:                               # eager run first (also a warm-up)
            stages[nm]()
        torch.cuda.synchronize(dev)
        for nm in names:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                stages[nm]()
            graphs[nm] = g
    torch.cuda.synchronize(dev)
    assert L.device_error() == 0

    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        for i, nm in enumerate(names):
            graphs[nm].replay()
            if evs is not None:
                evs[i + 1].record(stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.zero_()
            step()
    torch.cuda.synchronize(dev)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush.zero_()
            step(evs[i])
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    stage_ms = {nm: [] for nm in names}
    step_ms = []
    for e in evs:
        for i, nm in enumerate(names):
            stage_ms[nm].append(e[i].elapsed_time(e[i + 1]))
        step_ms.append(e[0].elapsed_time(e[-1]))
    mean_step = max_over_ranks(statistics.mean(step_ms), world, dev)
    assert L.device_error() == 0

    # encode and decode alone with a cold L2 (flushed before every replay): inside the step the
    # encoder reads K right after the search streamed it, and the decode reads the codes the
    # encoder just wrote, so part of their traffic can hit L2; their HBM rates are taken here
    def cold(nm, before=None):
        ms = []
        with torch.cuda.stream(stream):
            for i in range(max(3, min(args.steps, 30)) + 2):
                if before is not None:
                    graphs[before].replay()     # untimed: the stage the timed one consumes
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                graphs[nm].replay()
                e1.record(stream)
                e1.synchronize()
                if i >= 2:
                    ms.append(e0.elapsed_time(e1))
        return max_over_ranks(statistics.mean(ms), world, dev)

    encode_cold = cold("encode", before="search")    # the encoder reads the search's candidates
    decode_cold = cold("decode")
    assert L.device_error() == 0

    # end to end through the public API: every step copies its inputs in from pinned host memory
    # and its output back out.  Two input buffers let step i+1's copies (copy stream) run while
    # step i computes (compute stream); the time is the span of all steps over their number.
    h2d = Kp.numel() * Kp.element_size() + Vp.numel() * Vp.element_size() + qp.numel() * qp.element_size()
    d2h = out.numel() * out.element_size()
    bufs = [(K, V, q), (torch.empty_like(K), torch.empty_like(V), torch.empty_like(q))]
    cstream = torch.cuda.Stream(device=dev)

    def e2e_step(Kb, Vb, qb):
        L.build_refs(Kb, Vb)
        L.search(Kb)
        L.encode(Kb, Vb)
        L.decode(qb, out)
        L.reconstruct(0, 0, rpos, RECON_ROWS, Kr, Vr, rkv.RKV_DTYPE_F32)
        out_h.copy_(out, non_blocking=True)

    e2e_ms = []
    n_e2e = max(3, min(args.steps, 50))
    for rep in range(2):                                  # the first pass warms up
        copied = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        cstream.wait_stream(stream)
        for i in range(n_e2e):
            b = i % 2
            Kb, Vb, qb = bufs[b]
            with torch.cuda.stream(cstream):
                if i >= 2:
                    cstream.wait_event(done[b])              # step i-2 is done with this buffer
                Kb.copy_(Kp, non_blocking=True)
                Vb.copy_(Vp, non_blocking=True)
                qb.copy_(qp, non_blocking=True)
                copied[b].record(cstream)
            with torch.cuda.stream(stream):
                stream.wait_event(copied[b])
                e2e_step(Kb, Vb, qb)
                done[b].record(stream)
        e1.record(stream)
        e1.synchronize()
        if rep == 1:
            e2e_ms.append(e0.elapsed_time(e1) / n_e2e)
    assert L.device_error() == 0
    e2e_step = max_over_ranks(statistics.mean(e2e_ms), world, dev)

    # selective decode (outside the step): SPARSE_SEL seeded uniform positions per unit
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
    sp_ms = []
    with torch.cuda.stream(stream):
        for i in range(max(3, min(args.steps, 20)) + 2):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            L.decode_sparse(q, sel_d, cnt_d, out)
            e1.record(stream)
            e1.synchronize()
            if i >= 2:
                sp_ms.append(e0.elapsed_time(e1))
    assert L.device_error() == 0
    sparse_us = 1e3 * statistics.mean(sp_ms)

    # incremental compression (outside the step): the last APPEND_TOKENS positions of every
    # sequence appended one at a time to a layer compressed up to them
    La = rkv.Layer(cfg, lengths, device=dev)
    start = [max(0, n - APPEND_TOKENS) for n in lengths]
    La.set_lengths(start)
    La.build_refs(K, V)
    La.compress(K, V)
    Hkv = wl.n_kv_heads
    bi = torch.arange(wl.batch, device=dev).repeat_interleave(Hkv)
    hi = torch.arange(Hkv, device=dev).repeat(wl.batch)
    rows = []
    for t in range(APPEND_TOKENS):
        pos = torch.tensor([min(s0 + t, K.shape[2] - 1) for s0 in start], device=dev).repeat_interleave(Hkv)
        rows.append((K[bi, hi, pos].contiguous(), V[bi, hi, pos].contiguous()))
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        # a busy-wait ahead of the timed span keeps the device behind the host while the
        # appends are issued, so the span holds the appends' device time, not Python's
        torch.cuda._sleep(20_000_000)
        e0.record(stream)
        for Kn, Vn in rows:
            La.append(Kn, Vn, stream=stream)
        e1.record(stream)
        e1.synchronize()
    assert La.device_error() == 0
    append_us = 1e3 * e0.elapsed_time(e1) / APPEND_TOKENS
    del La

    # int4 reference store (outside the step): the same layer with references stored as
    # int4 codes + binary16 scales; each stage a CUDA graph, L2 flushed before each replay
    cfg4 = rkv.make_config(head_dim=wl.head_dim, n_kv_heads=wl.n_kv_heads, n_q_heads=wl.n_q_heads, k=wl.k,
                           bits=wl.bits, stride0=wl.stride0, batch=wl.batch, max_len=K.shape[2],
                           refs_per_phase=wl.refs_per_phase, in_dtype=wl.dtype_code, out_dtype=wl.dtype_code,
                           ref_bits=4)
    L4 = rkv.Layer(cfg4, lengths, device=dev)
    st4 = {"build_refs": lambda: L4.build_refs(K, V), "search": lambda: L4.search(K),
           "encode": lambda: L4.encode(K, V), "decode": lambda: L4.decode(q, out)}
    g4 = {}
    with torch.cuda.stream(stream):
        for nm in st4:
            st4[nm]()
        torch.cuda.synchronize(dev)
        for nm in st4:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                st4[nm]()
            g4[nm] = g
    torch.cuda.synchronize(dev)
    ms4 = {nm: [] for nm in st4}
    with torch.cuda.stream(stream):
        for i in range(max(3, min(args.steps, 20)) + 2):
            for nm in st4:
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g4[nm].replay()
                e1.record(stream)
                e1.synchronize()
                if i >= 2:
                    ms4[nm].append(e0.elapsed_time(e1))
    assert L4.device_error() == 0
    del g4, L4
    avg4 = {nm: statistics.mean(v) for nm, v in ms4.items()}

    # learned-coder shapes (outside the step): seeded random bf16 weights (scale 1/sqrt(D));
    # encode adds the latent pass (SwiGLU fc of every token and of its mean), decode folds fd
    wrng = np.random.default_rng(0xC0DE)
    cw = [torch.from_numpy((wrng.standard_normal((wl.head_dim, wl.head_dim)) / np.sqrt(wl.head_dim))
                           .astype(np.float32)).to(torch.bfloat16).to(dev) for _ in range(8)]
    cfgc = rkv.make_config(head_dim=wl.head_dim, n_kv_heads=wl.n_kv_heads, n_q_heads=wl.n_q_heads, k=wl.k,
                           bits=wl.bits, stride0=wl.stride0, batch=wl.batch, max_len=K.shape[2],
                           refs_per_phase=wl.refs_per_phase, in_dtype=wl.dtype_code, out_dtype=wl.dtype_code,
                           coder=1)
    Lc = rkv.Layer(cfgc, lengths, device=dev)
    Lc.set_coder(cw)
    stc = {"build_refs": lambda: Lc.build_refs(K, V), "search": lambda: Lc.search(K),
           "encode": lambda: Lc.encode(K, V), "decode": lambda: Lc.decode(q, out)}
    gc = {}
    with torch.cuda.stream(stream):
        for nm in stc:
            stc[nm]()
        torch.cuda.synchronize(dev)
        for nm in stc:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                stc[nm]()
            gc[nm] = g
    torch.cuda.synchronize(dev)
    msc = {nm: [] for nm in stc}
    with torch.cuda.stream(stream):
        for i in range(max(3, min(args.steps, 10)) + 2):
            for nm in stc:
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                gc[nm].replay()
                e1.record(stream)
                e1.synchronize()
                if i >= 2:
                    msc[nm].append(e0.elapsed_time(e1))
    assert Lc.device_error() == 0
    del gc, Lc
    avgc = {nm: statistics.mean(v) for nm, v in msc.items()}

    Q = workload_quantities(wl, lengths)
    tokens = Q["tokens"]
    value = job_throughput(world, tokens, mean_step)
    avg = {nm: statistics.mean(v) for nm, v in stage_ms.items()}
    peaks = _load_peaks()
    decode_gbs = Q["decode_bytes"] / (decode_cold * 1e-3) / 1e9
    encode_gbs = Q["encode_bytes"] / (encode_cold * 1e-3) / 1e9
    search_tflops = Q["search_flops"] / (avg["search"] * 1e-3) / 1e12
    search_tensor = wl.dtype == "bf16"
    search_kernel = "select_tc" if search_tensor else "select_simt"
    search_src = ["long_context_attention_rkv_b200/csrc/kernels_%s.cu" % search_kernel]
    dominant = max(("search", "encode", "decode"), key=lambda s: avg[s])
    if dominant == "search":
        if search_tensor:
            peak, bound, ach, unit = peaks["bf16"], "tensor", search_tflops, "TFLOP/s"
        else:
            peak, bound, ach, unit = ALU_FP32_TFLOPS, "alu", search_tflops, "TFLOP/s"
        traffic = _traffic(search_kernel, search_src)
    elif dominant == "encode":
        peak, bound, ach, unit = peaks["hbm"], "hbm", encode_gbs, "GB/s"
        traffic = _traffic("encode", ["long_context_attention_rkv_b200/csrc/kernels_encode.cu"])
    else:
        peak, bound, ach, unit = peaks["hbm"], "hbm", decode_gbs, "GB/s"
        traffic = _traffic("decode", ["long_context_attention_rkv_b200/csrc/kernels_decode_mma.cu"])
    roofline = {"kernel": dominant, "bound": bound, "achieved": ach, "peak": peak, "unit": unit,
                "frac": ach / peak, "traffic": traffic, "peak_source": peaks["source"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = min(os.cpu_count() or 1, wl.n_kv_heads)
        rate, desc, t = OracleSample(wl, lengths, 0, threads).calibrate(args.cpu_seconds).run()
        cpu = {"value": rate / 1e6, "unit": "Mtok/s", "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": t}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "Mtok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": mean_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded prototype-cluster caches)",
            "config": _config(wl, lengths),
            "parts": {
                "build_refs_us": 1e3 * avg["build_refs"], "search_us": 1e3 * avg["search"],
                "encode_us": 1e3 * avg["encode"], "encode_cold_us": 1e3 * encode_cold,
                "decode_us_per_step": 1e3 * decode_cold,
                "decode_in_step_us": 1e3 * avg["decode"],
                "reconstruct_us": 1e3 * avg["reconstruct"],
                "decode_hbm_gbs": decode_gbs, "decode_roofline_frac": decode_gbs / peaks["hbm"],
                "decode_bytes_per_step": Q["decode_bytes"],
                "search_tflops": search_tflops, "search_flops": Q["search_flops"],
                "encode_gbs": encode_gbs, "compress_mtok_s": tokens / ((avg["search"] + avg["encode"] +
                                                                        avg["build_refs"]) * 1e-3) / 1e6,
                "sparse_decode_us": sparse_us, "sparse_decode_positions_per_unit": SPARSE_SEL,
                "append_us_per_token": append_us,
                "int4_refs": {
                    "build_refs_us": 1e3 * avg4["build_refs"], "search_us": 1e3 * avg4["search"],
                    "encode_us": 1e3 * avg4["encode"], "decode_us_per_step": 1e3 * avg4["decode"],
                    "decode_bytes_per_step": Q["decode_bytes_int4_refs"],
                    "decode_hbm_gbs": Q["decode_bytes_int4_refs"] / (avg4["decode"] * 1e-3) / 1e9,
                    "compress_mtok_s": tokens / ((avg4["build_refs"] + avg4["search"] + avg4["encode"]) * 1e-3)
                    / 1e6,
                },
                "learned_coder": {
                    "encode_us": 1e3 * avgc["encode"], "decode_us_per_step": 1e3 * avgc["decode"],
                    "encode_latent_gflop": 2 * 2 * Q["tokens_cmp"] * 5 * wl.head_dim * wl.head_dim / 1e9,
                    "compress_mtok_s": tokens / ((avgc["build_refs"] + avgc["search"] + avgc["encode"]) * 1e-3)
                    / 1e6,
                },
            },
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": job_throughput(world, tokens, e2e_step), "unit": "Mtok/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": sum(LAUNCHES.values()) * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    for g in graphs.values():
        g.reset()


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
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
