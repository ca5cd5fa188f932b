"""Seeded synthetic KV caches and queries (inputs only).

Both the CUDA path (tests, ``bench.py``) and the CPU oracle read the bits this
module writes; it holds none of the compression arithmetic.  The generator
itself is plain C (``rkv_synth.c``): counter-based splitmix64 draws and
Box-Muller Gaussians, so any row of any unit can be regenerated on its own.

Workloads are the five named shapes used by the tests and the bench.  Each
follows the ResidualKV / DeltaKV pages' description of KV caches with
long-range similarity (p1 "Key Empirical Observations": similar tokens are
spread over the whole context): per unit, P prototypes ~N(0,1)^D, every token
a uniformly drawn prototype plus sigma * N(0,1) noise.
"""
from __future__ import annotations

import ctypes
import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "librkv_synth.so")

BASE_SEED = 0x524B56
DTYPE_BF16 = 0
DTYPE_F32 = 1


class _Params(ctypes.Structure):
    _fields_ = [
        ("seed", ctypes.c_uint64),
        ("workload", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("n_proto", ctypes.c_int32),
        ("n_outlier", ctypes.c_int32),
        ("sigma", ctypes.c_double),
        ("outlier_scale", ctypes.c_double),
        ("dtype", ctypes.c_int32),
        ("pad_", ctypes.c_int32),
    ]


def build(force: bool = False) -> str:
    """Compile the generator into ``synth/librkv_synth.so`` (gcc, -O2)."""
    src = os.path.join(_HERE, "rkv_synth.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        import subprocess

        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", tmp, src, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.POINTER(_Params)
        L.rkv_synth_kv.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.rkv_synth_kv.restype = ctypes.c_int
        L.rkv_synth_query.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                      ctypes.c_void_p]
        L.rkv_synth_query.restype = ctypes.c_int
        L.rkv_synth_length.argtypes = [P, ctypes.c_int, ctypes.c_int32, ctypes.c_int32]
        L.rkv_synth_length.restype = ctypes.c_int32
        L.rkv_synth_outlier_channels.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
        L.rkv_synth_outlier_channels.restype = ctypes.c_int
        L.rkv_synth_proto_id.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64]
        L.rkv_synth_proto_id.restype = ctypes.c_int32
        L.rkv_synth_checksum.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64]
        L.rkv_synth_checksum.restype = ctypes.c_uint64
        _lib = L
    return _lib


@dataclass(frozen=True)
class Workload:
    """One named synthetic workload: model shape, cache generator and coder settings."""

    name: str
    wid: int
    layers: int
    batch: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    seq_len: int            # maximum (and, unless ragged, every) sequence length
    dtype: str              # "bf16" or "f32" for K, V and q
    n_proto: int
    sigma: float
    n_outlier: int = 0
    outlier_scale: float = 8.0
    ragged: tuple | None = None   # (lo, hi): lengths uniform in [lo, hi]
    stride0: int = 16
    refs_per_phase: int = 0       # 0: fixed stride; else stride doubles after every this many refs
    k: int = 4
    bits: int = 4
    group: int = 32
    steps: int = 1                # decode steps
    q_scale: float = 1.0 / 8.0

    @property
    def dtype_code(self) -> int:
        return DTYPE_BF16 if self.dtype == "bf16" else DTYPE_F32

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    def params(self) -> _Params:
        return _Params(BASE_SEED, self.wid, self.head_dim, self.n_proto, self.n_outlier, self.sigma,
                       self.outlier_scale, self.dtype_code, 0)

    def lengths(self) -> list[int]:
        if self.ragged is None:
            return [self.seq_len] * self.batch
        lo, hi = self.ragged
        p = self.params()
        return [int(lib().rkv_synth_length(ctypes.byref(p), b, lo, hi)) for b in range(self.batch)]


WORKLOADS = {
    # 1 layer, 1 kv-head, D=64, fp32, 2048 tokens, 32 prototypes, s=16, k=4, int8
    "tiny": Workload("tiny", 1, layers=1, batch=1, n_kv_heads=1, n_q_heads=1, head_dim=64, seq_len=2048,
                     dtype="f32", n_proto=32, sigma=0.15, stride0=16, k=4, bits=8),
    # Llama-3-8B-shaped layer: 32 q / 8 kv heads, D=128, bf16, 32K tokens, 4 outlier key channels x8
    "llama3_8b_layer": Workload("llama3_8b_layer", 2, layers=1, batch=1, n_kv_heads=8, n_q_heads=32,
                                head_dim=128, seq_len=32768, dtype="bf16", n_proto=256, sigma=0.15,
                                n_outlier=4, stride0=16, k=4, bits=4),
    # the same shape, 32 layers x 128K tokens, 64 decode steps
    "llama3_8b_stack": Workload("llama3_8b_stack", 3, layers=32, batch=1, n_kv_heads=8, n_q_heads=32,
                                head_dim=128, seq_len=131072, dtype="bf16", n_proto=256, sigma=0.15,
                                n_outlier=4, stride0=16, k=4, bits=4, steps=64),
    # Qwen2.5-7B-shaped batch: 28 q / 4 kv heads, 28 layers, 8 ragged sequences in [16K, 32K]
    "qwen2_5_7b_batch": Workload("qwen2_5_7b_batch", 4, layers=28, batch=8, n_kv_heads=4, n_q_heads=28,
                                 head_dim=128, seq_len=32768, dtype="bf16", n_proto=512, sigma=0.2,
                                 ragged=(16384, 32768), stride0=32, k=8, bits=4),
    # 1M tokens, stride 16 doubling after every 1024 references
    "ultra_long_1m": Workload("ultra_long_1m", 5, layers=1, batch=1, n_kv_heads=8, n_q_heads=32, head_dim=128,
                              seq_len=1048576, dtype="bf16", n_proto=1024, sigma=0.15, stride0=16,
                              refs_per_phase=1024, k=4, bits=4, steps=16),
}


def np_dtype(wl: Workload):
    return np.uint16 if wl.dtype == "bf16" else np.float32


def gen_unit(wl: Workload, layer: int, seq: int, head: int, t0: int, t1: int, k_out=None, v_out=None):
    """Rows [t0, t1) of one unit as numpy arrays [t1-t0][D] (bf16 as raw uint16)."""
    D = wl.head_dim
    if k_out is None:
        k_out = np.empty((t1 - t0, D), dtype=np_dtype(wl))
    if v_out is None:
        v_out = np.empty((t1 - t0, D), dtype=np_dtype(wl))
    scratch = np.empty(2 * wl.n_proto * D, dtype=np.float64)
    p = wl.params()
    rc = lib().rkv_synth_kv(ctypes.byref(p), layer, seq, head, t0, t1, k_out.ctypes.data, v_out.ctypes.data,
                            scratch.ctypes.data)
    if rc != 0:
        raise ValueError("rkv_synth_kv failed")
    return k_out, v_out


def fill_layer(wl: Workload, layer: int, K: np.ndarray, V: np.ndarray, lengths=None, threads=None):
    """Fill K, V [B][Hkv][max_len][D] with one layer's cache (rows past a length are zeroed)."""
    lengths = wl.lengths() if lengths is None else lengths
    B, H, Nmax, D = K.shape
    assert V.shape == K.shape and B == len(lengths) and H == wl.n_kv_heads and D == wl.head_dim
    chunk = 8192
    jobs = []
    for b in range(B):
        for h in range(H):
            n = lengths[b]
            if n < Nmax:
                K[b, h, n:] = 0
                V[b, h, n:] = 0
            for t0 in range(0, n, chunk):
                jobs.append((b, h, t0, min(n, t0 + chunk)))

    def run(job):
        b, h, t0, t1 = job
        gen_unit(wl, layer, b, h, t0, t1, K[b, h, t0:t1], V[b, h, t0:t1])

    threads = threads or max(1, os.cpu_count() or 1)
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(run, jobs))
    return K, V


def gen_layer(wl: Workload, layer: int, lengths=None, max_len=None, threads=None):
    lengths = wl.lengths() if lengths is None else lengths
    max_len = max(lengths) if max_len is None else max_len
    shape = (wl.batch, wl.n_kv_heads, max_len, wl.head_dim)
    K = np.empty(shape, dtype=np_dtype(wl))
    V = np.empty(shape, dtype=np_dtype(wl))
    return fill_layer(wl, layer, K, V, lengths, threads)


def gen_query(wl: Workload, layer: int, step: int, out=None):
    """Decode queries [B][Hq][D] = q_scale * N(0,1) for one (layer, step)."""
    if out is None:
        out = np.empty((wl.batch, wl.n_q_heads, wl.head_dim), dtype=np_dtype(wl))
    p = wl.params()
    lib().rkv_synth_query(ctypes.byref(p), layer, step, wl.batch, wl.n_q_heads, wl.q_scale, out.ctypes.data)
    return out


def outlier_channels(wl: Workload, layer: int, seq: int, head: int) -> list[int]:
    p = wl.params()
    out = (ctypes.c_int32 * max(1, wl.n_outlier))()
    n = lib().rkv_synth_outlier_channels(ctypes.byref(p), layer, seq, head, out)
    return [int(out[i]) for i in range(max(0, n))]


def proto_id(wl: Workload, layer: int, seq: int, head: int, t: int) -> int:
    p = wl.params()
    return int(lib().rkv_synth_proto_id(ctypes.byref(p), layer, seq, head, t))


def checksum(arr: np.ndarray, h: int = 0) -> int:
    a = np.ascontiguousarray(arr)
    return int(lib().rkv_synth_checksum(a.ctypes.data, a.nbytes, h))


# --- bf16 helpers (bit-level; generator side) ------------------------------------------

def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    """Exact widening of raw bf16 bits to float32."""
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def as_f32(wl: Workload, arr: np.ndarray) -> np.ndarray:
    return bf16_to_f32(arr) if wl.dtype == "bf16" else np.asarray(arr, dtype=np.float32)


def sharp_query(wl: Workload, K_unit_f32: np.ndarray, t: int, n_q: int) -> np.ndarray:
    """A query aligned with key t: q = 4*sqrt(D)*K_t/|K_t| (for sensitivity tests)."""
    kt = K_unit_f32[t].astype(np.float64)
    q = 4.0 * math.sqrt(wl.head_dim) * kt / np.linalg.norm(kt)
    return np.tile(q, (n_q, 1))
