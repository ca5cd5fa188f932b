"""rkv_compress_noalloc: compression for callers that cannot allocate device memory.

Such callers (an engine whose whole device memory is a fixed pool, say) get the
search -> encoder scratch from a fixed array inside the library instead of a
workspace.  Its result must equal rkv_compress's on the same inputs, on two calls in
a row (the array keeps the previous call's contents), and a cache whose scratch
would not fit must be refused before any work is queued.
"""
import numpy as np
import pytest
import torch

import long_context_attention_rkv_b200 as rkv
import synth
from gpu_harness import config, to_dev

pytestmark = pytest.mark.gpu

NOALLOC_SCRATCH_BYTES = 16 << 20     # RKV_NOALLOC_SCRATCH_BYTES in rkv.h


def _compressed(layer, wl):
    out = {}
    for h in range(wl.n_kv_heads):
        v = layer.unit(0, h)
        for name, ptr, nbytes in (("idx", v.idx, 2 * v.n_cmp * v.k), ("codesK", v.codes_K, v.n_cmp * v.code_bytes),
                                  ("codesV", v.codes_V, v.n_cmp * v.code_bytes),
                                  ("scaleK", v.scale_K, 2 * v.n_cmp * v.n_groups),
                                  ("scaleV", v.scale_V, 2 * v.n_cmp * v.n_groups)):
            off = ptr - layer.cache.data_ptr()
            out[(name, h)] = layer.cache[off:off + nbytes].cpu().numpy().copy()
    return out


def test_noalloc_compress_matches_workspace_compress_twice():
    wl = synth.WORKLOADS["llama3_8b_layer"]
    lengths = wl.lengths()
    cfg = config(wl, lengths, out_dtype=rkv.RKV_DTYPE_BF16)
    ref_layer = rkv.Layer(cfg, lengths)
    nta_layer = rkv.Layer(cfg, lengths, workspace=False)
    for layer_id in (0, 1):                      # two calls in a row, different inputs
        K, V = synth.gen_layer(wl, layer_id, lengths)
        Kd, Vd = to_dev(K), to_dev(V)
        ref_layer.build_refs(Kd, Vd)
        ref_layer.compress(Kd, Vd)
        nta_layer.build_refs(Kd, Vd)
        rkv.rkv_compress_noalloc(nta_layer.desc, Kd, Vd)
        torch.cuda.synchronize()
        assert ref_layer.device_error() == 0 and nta_layer.device_error() == 0
        want = _compressed(ref_layer, wl)
        got = _compressed(nta_layer, wl)
        for key in want:
            assert np.array_equal(want[key], got[key]), f"call {layer_id}: {key} differs"


def test_noalloc_refuses_oversized_cache():
    wl = synth.WORKLOADS["llama3_8b_stack"]          # 8 x 122880 rows x 8 candidates: ~47 MB of lists
    lengths = wl.lengths()
    layer = rkv.Layer(config(wl, lengths), lengths, workspace=False)
    st = rkv.lib().rkv_compress_noalloc(layer.desc.ptr, 256, 256, None)
    assert st == rkv.STATUS_CODE["RKV_ERR_WORKSPACE"]


def test_noalloc_limit_counts_the_int4_key_copy():
    # the 32768-token Llama-shaped layer fits the array with bf16 references (13.8 MB of
    # search workspace) but not with the int4 reference store, whose search also keeps the
    # stored keys as bf16 rows (4.2 MB more): the header's formula, checked both ways
    wl = synth.WORKLOADS["llama3_8b_layer"]
    lengths = wl.lengths()
    rows, ref_rows, kc, D = 8 * 30720, 8 * 2048, 8, wl.head_dim

    def a256(x):
        return (x + 255) // 256 * 256

    search16 = a256(2 * rows * kc) + a256(4 * rows * kc) + a256(8 + 8 * rows)
    assert search16 <= NOALLOC_SCRATCH_BYTES < search16 + a256(2 * ref_rows * D)
    layer = rkv.Layer(config(wl, lengths, ref_bits=4), lengths, workspace=False)
    st = rkv.lib().rkv_compress_noalloc(layer.desc.ptr, 256, 256, None)
    assert st == rkv.STATUS_CODE["RKV_ERR_WORKSPACE"]
