"""Python binding of librkv, the residual KV-cache compression library for B200.

Argument marshalling only: every function here forwards to the C ABI declared
in ``include/rkv.h`` (same names), and every step of the path runs in the
library's CUDA kernels.  PyTorch is used for device memory and streams.  If
``librkv.so`` has not been built the import of the library fails loudly; there
is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librkv.so")

RKV_DTYPE_BF16 = 0
RKV_DTYPE_F32 = 1
RKV_FLAG_SELECT_SIMT = 0x1
RKV_FLAG_DECODE_DIRECT = 0x2
RKV_FLAG_DECODE_SIMT = 0x4
RKV_IDX_UNUSED = 0xFFFF
RKV_CACHE_DESC_BYTES = 32768

STATUS = {0: "RKV_OK", 1: "RKV_ERR_INVALID_ARG", 2: "RKV_ERR_UNSUPPORTED", 3: "RKV_ERR_WORKSPACE",
          4: "RKV_ERR_CUDA", 5: "RKV_ERR_CORRUPT", 6: "RKV_ERR_TIMEOUT"}
STATUS_CODE = {v: k for k, v in STATUS.items()}

EXPORTED = ["rkv_abi_version", "rkv_status_string", "rkv_schedule", "rkv_cache_size", "rkv_cache_bind",
            "rkv_unit_view_get", "rkv_build_refs", "rkv_search", "rkv_encode", "rkv_compress", "rkv_decode_attn", "rkv_reconstruct",
            "rkv_read_device_error", "rkv_compress_noalloc", "rkv_decode_attn_sparse", "rkv_cache_set_lengths",
            "rkv_append", "rkv_set_coder", "rkv_selftest_wait_timeout"]


class RkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class rkv_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("head_dim", "n_kv_heads", "n_q_heads", "k", "bits", "group",
                                              "stride0", "refs_per_phase", "in_dtype", "out_dtype", "batch",
                                              "max_len")] + [("flags", ctypes.c_uint32), ("ref_bits", ctypes.c_int32),
                                                             ("coder", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class rkv_unit_view(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("n", "n_ref", "n_cmp", "k", "code_bytes", "n_groups", "ref_bits",
                                              "reserved")] + \
               [(n, ctypes.c_void_p) for n in ("ref_K", "ref_V", "ref_half_norm", "ref_pos", "codes_K", "codes_V",
                                               "scale_K", "scale_V", "idx", "ref_scale_K", "ref_scale_V")]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded librkv.so (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"librkv.so is not built ({LIB_PATH}); run long_context_attention_rkv_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
        cfgp = ctypes.POINTER(rkv_config)
        L.rkv_abi_version.restype = i32
        L.rkv_status_string.argtypes = [ctypes.c_int]
        L.rkv_status_string.restype = ctypes.c_char_p
        L.rkv_schedule.argtypes = [cfgp, i32, vp, i64, ctypes.POINTER(i32)]
        L.rkv_cache_size.argtypes = [cfgp, vp, ctypes.POINTER(u64), ctypes.POINTER(u64)]
        L.rkv_cache_bind.argtypes = [cfgp, vp, vp, u64, vp]
        L.rkv_unit_view_get.argtypes = [vp, i32, i32, ctypes.POINTER(rkv_unit_view)]
        L.rkv_build_refs.argtypes = [vp, vp, vp, vp]
        L.rkv_search.argtypes = [vp, vp, vp, u64, vp]
        L.rkv_encode.argtypes = [vp, vp, vp, vp, u64, vp]
        L.rkv_compress.argtypes = [vp, vp, vp, vp, u64, vp]
        L.rkv_decode_attn.argtypes = [vp, vp, vp, vp, u64, vp]
        L.rkv_reconstruct.argtypes = [vp, i32, i32, vp, i64, vp, vp, i32, vp]
        L.rkv_read_device_error.argtypes = [vp, vp, ctypes.POINTER(i32)]
        L.rkv_compress_noalloc.argtypes = [vp, vp, vp, vp]
        L.rkv_decode_attn_sparse.argtypes = [vp, vp, vp, vp, i32, vp, vp, u64, vp]
        L.rkv_cache_set_lengths.argtypes = [vp, vp, vp]
        L.rkv_append.argtypes = [vp, vp, vp, vp, vp]
        L.rkv_set_coder.argtypes = [vp, vp]
        L.rkv_selftest_wait_timeout.argtypes = [vp, vp]
        for name in EXPORTED[2:]:
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise RkvError(status, where)


def _ptr(x):
    if x is None:
        return None
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    return int(x)


def _stream(stream):
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if hasattr(stream, "cuda_stream"):
        return stream.cuda_stream
    return int(stream)


def _lengths(lengths):
    arr = np.ascontiguousarray(np.asarray(lengths, dtype=np.int32))
    return arr, arr.ctypes.data


class CacheDesc:
    """Host-side handle of a bound cache (the opaque rkv_cache_desc blob)."""

    def __init__(self):
        self.buf = ctypes.create_string_buffer(RKV_CACHE_DESC_BYTES)

    @property
    def ptr(self):
        return ctypes.addressof(self.buf)


def make_config(head_dim, n_kv_heads, n_q_heads, k, bits, stride0, batch, max_len, refs_per_phase=0,
                in_dtype=RKV_DTYPE_BF16, out_dtype=None, group=32, flags=0, ref_bits=0, coder=0) -> rkv_config:
    """ref_bits: 0 (or 16) bf16 reference rows; 4 the int4 reference store.  coder: 0 identity,
    1 the learned-coder shapes (weights bound with rkv_set_coder)."""
    return rkv_config(head_dim, n_kv_heads, n_q_heads, k, bits, group, stride0, refs_per_phase, in_dtype,
                      in_dtype if out_dtype is None else out_dtype, batch, max_len, flags, ref_bits, coder, 0)


# --- the C ABI, one function each ------------------------------------------------------

def rkv_abi_version() -> int:
    return lib().rkv_abi_version()


def rkv_status_string(status: int) -> str:
    return lib().rkv_status_string(status).decode()


def rkv_schedule(cfg: rkv_config, n: int) -> np.ndarray:
    cnt = ctypes.c_int32(0)
    _check(lib().rkv_schedule(ctypes.byref(cfg), n, None, 0, ctypes.byref(cnt)), "rkv_schedule")
    pos = np.empty(cnt.value, dtype=np.int32)
    _check(lib().rkv_schedule(ctypes.byref(cfg), n, pos.ctypes.data, cnt.value, ctypes.byref(cnt)), "rkv_schedule")
    return pos


def rkv_cache_size(cfg: rkv_config, lengths) -> tuple[int, int]:
    arr, p = _lengths(lengths)
    cb, wb = ctypes.c_uint64(0), ctypes.c_uint64(0)
    _check(lib().rkv_cache_size(ctypes.byref(cfg), p, ctypes.byref(cb), ctypes.byref(wb)), "rkv_cache_size")
    return cb.value, wb.value


def rkv_cache_bind(cfg: rkv_config, lengths, dev_buf, nbytes: int) -> CacheDesc:
    arr, p = _lengths(lengths)
    d = CacheDesc()
    _check(lib().rkv_cache_bind(ctypes.byref(cfg), p, _ptr(dev_buf), nbytes, d.ptr), "rkv_cache_bind")
    return d


def rkv_unit_view_get(desc: CacheDesc, seq: int, kv_head: int) -> rkv_unit_view:
    v = rkv_unit_view()
    _check(lib().rkv_unit_view_get(desc.ptr, seq, kv_head, ctypes.byref(v)), "rkv_unit_view_get")
    return v


def rkv_build_refs(desc: CacheDesc, K, V, stream=None):
    _check(lib().rkv_build_refs(desc.ptr, _ptr(K), _ptr(V), _stream(stream)), "rkv_build_refs")


def rkv_search(desc: CacheDesc, K, workspace, workspace_bytes: int, stream=None):
    _check(lib().rkv_search(desc.ptr, _ptr(K), _ptr(workspace), workspace_bytes, _stream(stream)), "rkv_search")


def rkv_encode(desc: CacheDesc, K, V, workspace, workspace_bytes: int, stream=None):
    _check(lib().rkv_encode(desc.ptr, _ptr(K), _ptr(V), _ptr(workspace), workspace_bytes, _stream(stream)),
           "rkv_encode")


def rkv_compress(desc: CacheDesc, K, V, workspace, workspace_bytes: int, stream=None):
    _check(lib().rkv_compress(desc.ptr, _ptr(K), _ptr(V), _ptr(workspace), workspace_bytes, _stream(stream)),
           "rkv_compress")


def rkv_compress_noalloc(desc: CacheDesc, K, V, stream=None):
    """rkv_compress with the library's own fixed scratch array instead of a workspace (for callers
    that cannot allocate); see include/rkv.h for its limit and sharing rules."""
    _check(lib().rkv_compress_noalloc(desc.ptr, _ptr(K), _ptr(V), _stream(stream)), "rkv_compress_noalloc")


def rkv_decode_attn(desc: CacheDesc, q, out, workspace, workspace_bytes: int, stream=None):
    _check(lib().rkv_decode_attn(desc.ptr, _ptr(q), _ptr(out), _ptr(workspace), workspace_bytes, _stream(stream)),
           "rkv_decode_attn")


def rkv_cache_set_lengths(desc: CacheDesc, lengths, stream=None):
    arr, p = _lengths(lengths)
    _check(lib().rkv_cache_set_lengths(desc.ptr, p, _stream(stream)), "rkv_cache_set_lengths")


def rkv_append(desc: CacheDesc, K_new, V_new, active=None, stream=None):
    act = None if active is None else (ctypes.c_uint8 * len(active))(*[1 if x else 0 for x in active])
    _check(lib().rkv_append(desc.ptr, _ptr(K_new), _ptr(V_new), act, _stream(stream)), "rkv_append")


def rkv_set_coder(desc: CacheDesc, weights):
    """weights: eight device bf16 tensors [D][D]: Wg, Wu, Wo, Wd of K, then of V."""
    assert len(weights) == 8
    arr = (ctypes.c_void_p * 8)(*[_ptr(w) for w in weights])
    _check(lib().rkv_set_coder(desc.ptr, arr), "rkv_set_coder")


def rkv_decode_attn_sparse(desc: CacheDesc, q, positions, counts, max_sel: int, out, workspace, workspace_bytes: int,
                           stream=None):
    _check(lib().rkv_decode_attn_sparse(desc.ptr, _ptr(q), _ptr(positions), _ptr(counts), max_sel, _ptr(out),
                                        _ptr(workspace), workspace_bytes, _stream(stream)), "rkv_decode_attn_sparse")


def rkv_reconstruct(desc: CacheDesc, seq: int, kv_head: int, positions, n_pos: int, K_out, V_out,
                    out_dtype: int, stream=None):
    _check(lib().rkv_reconstruct(desc.ptr, seq, kv_head, _ptr(positions), n_pos, _ptr(K_out), _ptr(V_out),
                                 out_dtype, _stream(stream)), "rkv_reconstruct")


def rkv_read_device_error(desc: CacheDesc, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(lib().rkv_read_device_error(desc.ptr, _stream(stream), ctypes.byref(v)), "rkv_read_device_error")
    return v.value


def rkv_selftest_wait_timeout(err_dev, stream=None):
    """Queues the bounded-wait self-test; after a stream synchronisation err_dev (a device int32
    tensor) holds RKV_ERR_TIMEOUT (about 2 s later)."""
    _check(lib().rkv_selftest_wait_timeout(_ptr(err_dev), _stream(stream)), "rkv_selftest_wait_timeout")


# --- buffers ---------------------------------------------------------------------------

class Layer:
    """One layer's compressed cache: torch-allocated cache and workspace buffers plus the bound handle."""

    def __init__(self, cfg: rkv_config, lengths, device="cuda", workspace=None):
        import torch

        self.cfg = cfg
        self.lengths = [int(x) for x in lengths]
        self.cache_bytes, self.ws_bytes = rkv_cache_size(cfg, self.lengths)
        self.cache = torch.empty(self.cache_bytes, dtype=torch.uint8, device=device)
        if workspace is None:
            workspace = torch.empty(max(256, self.ws_bytes), dtype=torch.uint8, device=device)
        if workspace is not False:           # False: no workspace (calls that need none)
            assert workspace.numel() >= self.ws_bytes
        self.workspace = workspace if workspace is not False else None
        self.desc = rkv_cache_bind(cfg, self.lengths, self.cache, self.cache_bytes)

    def build_refs(self, K, V, stream=None):
        rkv_build_refs(self.desc, K, V, stream)

    def search(self, K, stream=None):
        rkv_search(self.desc, K, self.workspace, self.workspace.numel(), stream)

    def encode(self, K, V, stream=None):
        rkv_encode(self.desc, K, V, self.workspace, self.workspace.numel(), stream)

    def compress(self, K, V, stream=None):
        rkv_compress(self.desc, K, V, self.workspace, self.workspace.numel(), stream)

    def decode(self, q, out, stream=None):
        rkv_decode_attn(self.desc, q, out, self.workspace, self.workspace.numel(), stream)

    def set_coder(self, weights):
        """Learned-coder weights (kept referenced here so they outlive the handle's use)."""
        self._coder_weights = list(weights)
        rkv_set_coder(self.desc, self._coder_weights)

    def set_lengths(self, lengths, stream=None):
        """Current lengths (<= the bound ones, which are the capacity)."""
        rkv_cache_set_lengths(self.desc, lengths, stream)

    def append(self, K_new, V_new, active=None, stream=None):
        """One new token per active sequence: K_new, V_new [batch, kv_heads, head_dim] on the device."""
        rkv_append(self.desc, K_new, V_new, active, stream)

    def decode_sparse(self, q, positions, counts, out, stream=None):
        """positions: int32 [n_units, max_sel] on the device, counts: int32 [n_units] on the device."""
        rkv_decode_attn_sparse(self.desc, q, positions, counts, positions.shape[-1], out, self.workspace,
                               self.workspace.numel(), stream)

    def reconstruct(self, seq, kv_head, positions, n_pos, K_out, V_out, out_dtype, stream=None):
        rkv_reconstruct(self.desc, seq, kv_head, positions, n_pos, K_out, V_out, out_dtype, stream)

    def device_error(self, stream=None) -> int:
        return rkv_read_device_error(self.desc, stream)

    def unit(self, seq: int, kv_head: int) -> rkv_unit_view:
        return rkv_unit_view_get(self.desc, seq, kv_head)
