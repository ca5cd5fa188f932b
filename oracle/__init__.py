"""CPU oracle for residual KV-cache compression — TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct statement of what the CUDA path computes
(``rkv_oracle.cpp``, plain C++ built with ``-ffp-contract=off``), plus numpy
glue that composes its steps per (layer, sequence, kv-head) unit.  Only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the library path never does, and this
package never imports the library.

Steps and the page sections they follow (pages on ResidualKV / DeltaKV):
  schedule, build_refs   p1 "DeltaKV Framework Architecture" (strided reference
                         set T); p3 "How ResidualKV Works" (dynamic stride)
  select                 p1 "DeltaKV Framework Architecture" (top-k nearest
                         references by L2 distance)
  encode                 p1 "DeltaKV Framework Architecture" (residual against
                         the mean reference); p3 "How ResidualKV Works"
                         (quantized residual codes)
  reconstruct            p1 "DeltaKV Framework Architecture" (KV = KV_delta + KV_R)
  attention              softmax(q.K/sqrt(D)) V in double (decode step)

Pins: every function is checked in ``tests/test_oracle_pins.py`` against
closed forms, brute force, library routines and invariants.  Parity with the
pages' own numbers is unpinned: the pages print no worked example.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "librkv_oracle.so")
_SRC = os.path.join(_HERE, "rkv_oracle.cpp")

SENTINEL = 0xFFFF


def build(force: bool = False) -> str:
    """Compile the oracle (g++ -O2 -ffp-contract=off, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                               "-shared", "-o", tmp, _SRC])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None
_vp = ctypes.c_void_p


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        L.orc_schedule.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _vp, ctypes.c_int64]
        L.orc_schedule.restype = ctypes.c_int64
        L.orc_build_refs.argtypes = [ctypes.c_int, _vp, _vp, ctypes.c_int64, _vp]
        L.orc_bf16_round.argtypes = [_vp, ctypes.c_int64, _vp]
        L.orc_l2.argtypes = [ctypes.c_int, _vp, _vp]
        L.orc_l2.restype = ctypes.c_double
        sel = [ctypes.c_int, ctypes.c_int64, _vp, _vp, ctypes.c_int64, _vp, _vp, ctypes.c_int, _vp, _vp, _vp]
        L.orc_select.argtypes = sel
        L.orc_select_f.argtypes = sel
        L.orc_encode.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, _vp, _vp, ctypes.c_int64,
                                 _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp]
        L.orc_encode.restype = ctypes.c_int
        L.orc_encode_f.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, _vp, _vp, _vp,
                                   ctypes.c_int, _vp, _vp, _vp, _vp, _vp]
        L.orc_encode_f.restype = ctypes.c_int
        L.orc_quantize_rows.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, _vp,
                                        _vp, _vp]
        L.orc_quantize_rows.restype = ctypes.c_int
        L.orc_dequantize_rows.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, _vp, _vp, _vp]
        L.orc_unpack_codes.argtypes = [ctypes.c_int, ctypes.c_int, _vp, _vp]
        L.orc_coder_fc.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp]
        L.orc_encode_latent.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int64, _vp, _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp]
        L.orc_encode_latent.restype = ctypes.c_int
        L.orc_reconstruct_latent.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                             _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp]
        L.orc_reconstruct.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, _vp,
                                      ctypes.c_int64, _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp]
        L.orc_reconstruct_f.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, _vp, _vp,
                                        ctypes.c_int, _vp, _vp, _vp, _vp, _vp]
        L.orc_attention.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp]
        L.orc_fp16_round_up.argtypes = [ctypes.c_float, _vp]
        L.orc_fp16_round_up.restype = ctypes.c_uint16
        L.orc_fp16_value.argtypes = [ctypes.c_uint16]
        L.orc_fp16_value.restype = ctypes.c_float
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --- steps ---------------------------------------------------------------------------

def schedule(n: int, stride0: int, refs_per_phase: int = 0) -> np.ndarray:
    """Reference positions (ascending int32)."""
    R = lib().orc_schedule(n, stride0, refs_per_phase, None, 0)
    pos = np.empty(R, dtype=np.int32)
    lib().orc_schedule(n, stride0, refs_per_phase, pos.ctypes.data, R)
    return pos


def bf16_round(x) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().orc_bf16_round(x.ctypes.data, x.size, out.ctypes.data)
    return out


def bf16_value(u16) -> np.ndarray:
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def build_refs(X: np.ndarray, ref_pos: np.ndarray) -> np.ndarray:
    """Reference store [R][D] (bf16 bits) from float rows X[n][D]."""
    X = _c(X, np.float32)
    ref_pos = _c(ref_pos, np.int32)
    out = np.empty((len(ref_pos), X.shape[1]), dtype=np.uint16)
    lib().orc_build_refs(X.shape[1], X.ctypes.data, ref_pos.ctypes.data, len(ref_pos), out.ctypes.data)
    return out


def l2(a, b) -> float:
    a = _c(a, np.float32)
    b = _c(b, np.float32)
    return lib().orc_l2(a.size, a.ctypes.data, b.ctypes.data)


def _refs(refs):
    """(array, is_values): bf16 reference rows (uint16 bits) or stored values (float32)."""
    if np.asarray(refs).dtype == np.float32:
        return _c(refs, np.float32), True
    return _c(refs, np.uint16), False


def select(x: np.ndarray, tok_pos: np.ndarray, refK: np.ndarray, ref_pos: np.ndarray, k: int):
    """Top-k references per token: (idx [n][k] uint16 ascending, k_eff [n], dist [n][k+1]).

    refK: bf16 rows (uint16 bits) or stored values (float32, e.g. the int4 reference store)."""
    x = _c(x, np.float32)
    tok_pos = _c(tok_pos, np.int32)
    refK, values = _refs(refK)
    ref_pos = _c(ref_pos, np.int32)
    n, D = x.shape
    idx = np.empty((n, k), dtype=np.uint16)
    keff = np.empty(n, dtype=np.int32)
    dist = np.empty((n, k + 1), dtype=np.float64)
    fn = lib().orc_select_f if values else lib().orc_select
    fn(D, n, x.ctypes.data, tok_pos.ctypes.data, len(ref_pos), refK.ctypes.data, ref_pos.ctypes.data,
       k, idx.ctypes.data, keff.ctypes.data, dist.ctypes.data)
    return idx, keff, dist


def encode(x: np.ndarray, refs: np.ndarray, idx: np.ndarray, bits: int, group: int = 32, want_detail=False):
    """Residual codes for rows x[n][D] against refs[R][D] (bf16 bits, or float32 stored values)
    and idx[n][k].

    Returns dict(codes [n][D*bits/8] uint8, scales [n][D/group] uint16 fp16 bits, overflow,
    and with want_detail: mean, delta (fp32), delta_exact (bits=0, double)).
    """
    x = _c(x, np.float32)
    refs, values = _refs(refs)
    idx = _c(idx, np.uint16)
    n, D = x.shape
    k = idx.shape[1]
    codes = np.zeros((n, max(1, D * bits // 8)), dtype=np.uint8)
    scales = np.zeros((n, D // group), dtype=np.uint16)
    mean = np.empty((n, D), dtype=np.float32) if (want_detail or bits == 0) else None
    delta = np.empty((n, D), dtype=np.float32) if (want_detail or bits == 0) else None
    dex = np.empty((n, D), dtype=np.float64) if bits == 0 else None
    if values:
        ov = lib().orc_encode_f(D, bits, group, n, x.ctypes.data, refs.ctypes.data, idx.ctypes.data, k,
                                codes.ctypes.data, scales.ctypes.data, _p(mean), _p(delta), _p(dex))
    else:
        ov = lib().orc_encode(D, bits, group, n, x.ctypes.data, refs.ctypes.data, refs.shape[0], idx.ctypes.data,
                              k, codes.ctypes.data, scales.ctypes.data, _p(mean), _p(delta), _p(dex))
    out = dict(codes=codes, scales=scales, overflow=int(ov))
    if mean is not None:
        out.update(mean=mean, delta=delta)
    if dex is not None:
        out["delta_exact"] = dex
    return out


def unpack_codes(codes_row: np.ndarray, D: int, bits: int) -> np.ndarray:
    codes_row = _c(codes_row, np.uint8)
    out = np.empty(D, dtype=np.int32)
    lib().orc_unpack_codes(D, bits, codes_row.ctypes.data, out.ctypes.data)
    return out


def reconstruct(refs, idx, codes, scales, bits: int, group: int = 32, D: int | None = None, delta_exact=None):
    """Reconstructed rows: float32 [n][D] (or float64 when bits == 0)."""
    refs, values = _refs(refs)
    idx = _c(idx, np.uint16)
    n, k = idx.shape
    D = refs.shape[1] if D is None else D

    def call(b, cp, sp, dp, op, oxp):
        if values:
            lib().orc_reconstruct_f(D, b, group, n, refs.ctypes.data, idx.ctypes.data, k, cp, sp, dp, op, oxp)
        else:
            lib().orc_reconstruct(D, b, group, n, refs.ctypes.data, refs.shape[0], idx.ctypes.data, k, cp, sp, dp,
                                  op, oxp)

    if bits == 0:
        dex = _c(delta_exact, np.float64)
        out = np.empty((n, D), dtype=np.float64)
        call(0, None, None, dex.ctypes.data, None, out.ctypes.data)
        return out
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint16)
    out = np.empty((n, D), dtype=np.float32)
    call(bits, codes.ctypes.data, scales.ctypes.data, None, out.ctypes.data, None)
    return out


def quantize_rows(X: np.ndarray, bits: int = 4, group: int = 32, pow2: bool = True):
    """Group quantiser applied to each row of X[n][D] by itself: (codes, scales, overflow).
    pow2: scales rounded up to a power of two (the int4 reference store) instead of to the
    next binary16 value (the residuals' quantiser)."""
    X = _c(X, np.float32)
    n, D = X.shape
    codes = np.zeros((n, D * bits // 8), dtype=np.uint8)
    scales = np.zeros((n, D // group), dtype=np.uint16)
    ov = lib().orc_quantize_rows(D, bits, group, int(pow2), n, X.ctypes.data, codes.ctypes.data,
                                 scales.ctypes.data)
    return codes, scales, int(ov)


def dequantize_rows(codes: np.ndarray, scales: np.ndarray, D: int, bits: int = 4, group: int = 32) -> np.ndarray:
    """Stored values code * scale (float32 [n][D])."""
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint16)
    n = codes.shape[0]
    out = np.empty((n, D), dtype=np.float32)
    lib().orc_dequantize_rows(D, bits, group, n, codes.ctypes.data, scales.ctypes.data, out.ctypes.data)
    return out


def build_refs_quantized(X: np.ndarray, ref_pos: np.ndarray, bits: int = 4, group: int = 32):
    """int4 reference store of float rows X at ref_pos: (codes, scales, stored values, overflow)."""
    X = _c(X, np.float32)
    rows = X[np.asarray(ref_pos, dtype=np.int64)]
    codes, scales, ov = quantize_rows(rows, bits, group)
    return codes, scales, dequantize_rows(codes, scales, X.shape[1], bits, group), ov


# --- learned-coder shapes (fc SwiGLU into a latent, fd linear back) ----------------------

class Coder:
    """Weights of one side's coder (float32 holding bf16 values, row-major [out][in]):
    fc(x) = Wo (silu(Wg x) * (Wu x)), fd(z) = Wd z."""

    def __init__(self, Wg, Wu, Wo, Wd):
        self.Wg, self.Wu, self.Wo, self.Wd = (_c(w, np.float32) for w in (Wg, Wu, Wo, Wd))
        self.H, self.D = self.Wg.shape
        self.L = self.Wo.shape[0]


def coder_fc(X: np.ndarray, w: Coder) -> np.ndarray:
    X = _c(X, np.float32)
    n = X.shape[0]
    out = np.empty((n, w.L), dtype=np.float64)
    lib().orc_coder_fc(w.D, w.H, w.L, n, X.ctypes.data, w.Wg.ctypes.data, w.Wu.ctypes.data, w.Wo.ctypes.data,
                       out.ctypes.data)
    return out


def encode_latent(x: np.ndarray, refs: np.ndarray, idx: np.ndarray, bits: int, w: Coder, group: int = 32):
    """Latent residual codes z = fc(x) - fc(mean of refs): dict(codes, scales, overflow, z)."""
    x = _c(x, np.float32)
    refs = _c(refs if np.asarray(refs).dtype == np.float32 else bf16_value(refs), np.float32)
    idx = _c(idx, np.uint16)
    n = x.shape[0]
    k = idx.shape[1]
    codes = np.zeros((n, max(1, w.L * bits // 8)), dtype=np.uint8)
    scales = np.zeros((n, w.L // group), dtype=np.uint16)
    z = np.empty((n, w.L), dtype=np.float64)
    ov = lib().orc_encode_latent(w.D, w.H, w.L, bits, group, n, x.ctypes.data, refs.ctypes.data, idx.ctypes.data, k,
                                 w.Wg.ctypes.data, w.Wu.ctypes.data, w.Wo.ctypes.data, codes.ctypes.data,
                                 scales.ctypes.data, z.ctypes.data)
    return dict(codes=codes, scales=scales, overflow=int(ov), z=z)


def reconstruct_latent(refs, idx, codes, scales, bits: int, w: Coder, group: int = 32, z_exact=None) -> np.ndarray:
    """Rebuilt rows m + fd(z_hat) (double [n][D])."""
    refs = _c(refs if np.asarray(refs).dtype == np.float32 else bf16_value(refs), np.float32)
    idx = _c(idx, np.uint16)
    n, k = idx.shape
    out = np.empty((n, w.D), dtype=np.float64)
    if bits == 0:
        zx = _c(z_exact, np.float64)
        lib().orc_reconstruct_latent(w.D, w.L, 0, group, n, refs.ctypes.data, idx.ctypes.data, k, None, None,
                                     zx.ctypes.data, w.Wd.ctypes.data, out.ctypes.data)
        return out
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint16)
    lib().orc_reconstruct_latent(w.D, w.L, bits, group, n, refs.ctypes.data, idx.ctypes.data, k, codes.ctypes.data,
                                 scales.ctypes.data, None, w.Wd.ctypes.data, out.ctypes.data)
    return out


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """softmax(q K^T / sqrt(D)) V for q [G][D], K, V [n][D]; double."""
    q = _c(q, np.float64)
    K = _c(K, np.float64)
    V = _c(V, np.float64)
    G, D = q.shape
    n = K.shape[0]
    out = np.empty((G, D), dtype=np.float64)
    lib().orc_attention(n, D, G, q.ctypes.data, K.ctypes.data if n else None, V.ctypes.data if n else None,
                        out.ctypes.data)
    return out


def fp16_round_up(f: float):
    ov = ctypes.c_int32(0)
    bits = lib().orc_fp16_round_up(ctypes.c_float(f), ctypes.byref(ov))
    return int(bits), int(ov.value)


def fp16_value(bits: int) -> float:
    return float(lib().orc_fp16_value(bits))


# --- per-unit compositions -------------------------------------------------------------

def positions_split(n: int, ref_pos: np.ndarray):
    """(compressed positions ascending, boolean is_ref[n])."""
    is_ref = np.zeros(n, dtype=bool)
    is_ref[ref_pos] = True
    return np.nonzero(~is_ref)[0].astype(np.int32), is_ref


def compress_unit(Xk: np.ndarray, Xv: np.ndarray, stride0: int, refs_per_phase: int, k: int, bits: int,
                  group: int = 32, positions=None, ref_bits: int = 16, coder=None):
    """Compress one unit given float rows Xk, Xv [n][D] (exact input values).

    positions: compressed positions to encode (default: all).  ref_bits 16: bf16 reference
    rows (refK, refV uint16 bits); 4: the int4 reference store (refK, refV are the stored
    values, float32, and ref_codesK/ref_scalesK/ref_codesV/ref_scalesV are added).  Returns a
    dict with ref_pos, refK, refV, pos (encoded positions), idx, keff, dist, codesK, scalesK,
    codesV, scalesV, overflow.  coder: (Coder K, Coder V) for latent residuals (learned-coder
    shapes) instead of the identity coder.
    """
    n = Xk.shape[0]
    ref_pos = schedule(n, stride0, refs_per_phase)
    extra = {}
    if ref_bits == 4:
        rcK, rsK, refK, ovk = build_refs_quantized(Xk, ref_pos, 4, group)
        rcV, rsV, refV, ovv = build_refs_quantized(Xv, ref_pos, 4, group)
        extra = dict(ref_codesK=rcK, ref_scalesK=rsK, ref_codesV=rcV, ref_scalesV=rsV, ref_overflow=ovk | ovv)
    else:
        refK = build_refs(Xk, ref_pos)
        refV = build_refs(Xv, ref_pos)
    if positions is None:
        positions, _ = positions_split(n, ref_pos)
    positions = np.asarray(positions, dtype=np.int32)
    idx, keff, dist = select(Xk[positions], positions, refK, ref_pos, k)
    if coder is not None:                       # (Coder for K, Coder for V): latent residuals
        ek = encode_latent(Xk[positions], refK, idx, bits, coder[0], group)
        ev = encode_latent(Xv[positions], refV, idx, bits, coder[1], group)
    else:
        ek = encode(Xk[positions], refK, idx, bits, group)
        ev = encode(Xv[positions], refV, idx, bits, group)
    return dict(ref_pos=ref_pos, refK=refK, refV=refV, pos=positions, idx=idx, keff=keff, dist=dist,
                codesK=ek["codes"], scalesK=ek["scales"], codesV=ev["codes"], scalesV=ev["scales"],
                overflow=ek["overflow"] | ev["overflow"], **extra)


def unit_cache_rows(n: int, ref_pos, refK, refV, idx, codesK, scalesK, codesV, scalesV, bits: int,
                    group: int = 32, coder=None):
    """Reconstructed K, V [n][D] (float64) of a whole unit (reference rows are the stored
    values: bf16 rows given as uint16 bits, or float32 values of the int4 reference store;
    coder: latent residuals rebuilt through fd)."""
    D = refK.shape[1]
    cpos, is_ref = positions_split(n, np.asarray(ref_pos))
    Kh = np.empty((n, D), dtype=np.float64)
    Vh = np.empty((n, D), dtype=np.float64)
    stored = (lambda r: r) if np.asarray(refK).dtype == np.float32 else bf16_value
    Kh[ref_pos] = stored(refK)
    Vh[ref_pos] = stored(refV)
    if len(cpos) and coder is not None:
        Kh[cpos] = reconstruct_latent(refK, idx, codesK, scalesK, bits, coder[0], group)
        Vh[cpos] = reconstruct_latent(refV, idx, codesV, scalesV, bits, coder[1], group)
    elif len(cpos):
        Kh[cpos] = reconstruct(refK, idx, codesK, scalesK, bits, group)
        Vh[cpos] = reconstruct(refV, idx, codesV, scalesV, bits, group)
    return Kh, Vh


def decode_unit(q_group: np.ndarray, Kh: np.ndarray, Vh: np.ndarray) -> np.ndarray:
    """Attention of the unit's G query heads over its reconstructed cache (double)."""
    return attention(q_group, Kh, Vh)
