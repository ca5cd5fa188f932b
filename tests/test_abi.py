"""The C-ABI library: it loads, exports every declared symbol, and its host-side logic
(schedule, sizing, validation) is right.  No device calls."""
import ctypes
import os
import re

import numpy as np
import pytest

import long_context_attention_rkv_b200 as rkv
import oracle


def _declared_symbols(repo_root):
    with open(os.path.join(repo_root, "include", "rkv.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^RKV_API[^(]*?\b(rkv_\w+)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol(repo_root):
    declared = _declared_symbols(repo_root)
    assert len(declared) >= 11
    L = rkv.lib()
    for name in declared:
        assert hasattr(L, name), name
    assert sorted(rkv.EXPORTED) == declared
    assert rkv.rkv_abi_version() == 1
    assert rkv.rkv_status_string(5) == "corrupted cache contents"


def _cfg(**kw):
    base = dict(head_dim=128, n_kv_heads=8, n_q_heads=32, k=4, bits=4, stride0=16, batch=1, max_len=32768)
    base.update(kw)
    return rkv.make_config(**base)


@pytest.mark.parametrize("n,s,rpp", [(2048, 16, 0), (32768, 16, 0), (131072, 16, 0), (1048576, 16, 1024),
                                     (1, 16, 0), (0, 16, 0), (3000, 2, 64), (30000, 32, 0), (5000, 4, 100)])
def test_schedule_matches_oracle(n, s, rpp):
    cfg = _cfg(stride0=s, refs_per_phase=rpp, max_len=max(n, 1))
    assert np.array_equal(rkv.rkv_schedule(cfg, n), oracle.schedule(n, s, rpp))


def test_cache_size_accounts_every_array():
    lengths = [32768]
    cb, wb = rkv.rkv_cache_size(_cfg(), lengths)
    R, C, H, D = 2048, 30720, 8, 128
    # reference rows (K, V bf16), half norm + position, augmented search column (16 bf16),
    # then per compressed token: codes K/V, scales K/V, 4 ordinals; per unit the append
    # search's candidate lists (32 chunks x 16 (distance f64, ordinal i32))
    payload = H * (2 * R * D * 2 + R * 8 + R * 32 + C * (2 * 64 + 2 * 8 + 4 * 2) + 32 * 16 * 12)
    assert payload <= cb <= payload + 64 * 1024
    assert wb >= H * C * 8 * 6            # search candidates: kc = 8 ordinals + scores per token


def test_int4_reference_store_sizes():
    """int4 reference rows: D/2 code bytes and D/32 binary16 scales per row and side, and the
    search workspace carries a bf16 copy of the stored keys."""
    lengths = [32768]
    c16, w16 = rkv.rkv_cache_size(_cfg(), lengths)
    c4, w4 = rkv.rkv_cache_size(_cfg(ref_bits=4), lengths)
    R, H, D = 2048, 8, 128
    assert c16 - c4 == pytest.approx(H * R * 2 * (2 * D - (D // 2 + 2 * D // 32)), abs=8 * 1024)
    assert w4 >= w16 + H * R * D * 2                       # plus the stored keys as bf16 rows
    for bad in (8, 2, 5):
        with pytest.raises(rkv.RkvError) as ei:
            rkv.rkv_cache_size(_cfg(ref_bits=bad), lengths)
        assert rkv.STATUS[ei.value.status] == "RKV_ERR_UNSUPPORTED"


def test_learned_coder_validation():
    assert rkv.rkv_cache_size(_cfg(coder=1), [4096])[0] > 0
    for bad in (dict(coder=2), dict(coder=1, head_dim=64), dict(coder=1, bits=8), dict(coder=1, ref_bits=4),
                dict(coder=1, k=9), dict(coder=1, n_q_heads=8 * 9)):
        with pytest.raises(rkv.RkvError) as ei:
            rkv.rkv_cache_size(_cfg(**bad), [4096])
        assert rkv.STATUS[ei.value.status] == "RKV_ERR_UNSUPPORTED", bad
    d = rkv.CacheDesc()
    arr = (ctypes.c_void_p * 8)(*([16] * 8))
    assert rkv.lib().rkv_set_coder(d.ptr, arr) == rkv.STATUS_CODE["RKV_ERR_INVALID_ARG"]


def test_ragged_sizes_and_validation():
    cfg = _cfg(n_kv_heads=4, n_q_heads=28, k=8, stride0=32, batch=3)
    cb, _ = rkv.rkv_cache_size(cfg, [16384, 0, 20000])
    assert cb > 0
    for bad, code in [(dict(head_dim=96), "RKV_ERR_UNSUPPORTED"), (dict(bits=2), "RKV_ERR_UNSUPPORTED"),
                      (dict(k=17), "RKV_ERR_UNSUPPORTED"), (dict(n_q_heads=30), "RKV_ERR_INVALID_ARG"),
                      (dict(stride0=1), "RKV_ERR_INVALID_ARG"), (dict(group=16), "RKV_ERR_UNSUPPORTED")]:
        with pytest.raises(rkv.RkvError) as ei:
            rkv.rkv_cache_size(_cfg(**bad), [1024])
        assert rkv.STATUS[ei.value.status] == code
    with pytest.raises(rkv.RkvError) as ei:
        rkv.rkv_cache_size(_cfg(max_len=100), [101])          # length beyond the row pitch
    assert ei.value.status == rkv.STATUS_CODE["RKV_ERR_INVALID_ARG"]
    with pytest.raises(rkv.RkvError) as ei:                  # > 65535 references per unit
        rkv.rkv_cache_size(_cfg(stride0=2, max_len=200000), [200000])
    assert ei.value.status == rkv.STATUS_CODE["RKV_ERR_UNSUPPORTED"]


def test_calls_reject_unbound_handles():
    d = rkv.CacheDesc()                                       # never bound: zero magic
    for fn, args in [(rkv.lib().rkv_build_refs, (d.ptr, 16, 16, None)),
                     (rkv.lib().rkv_compress, (d.ptr, 16, 16, 256, 0, None)),
                     (rkv.lib().rkv_decode_attn, (d.ptr, 16, 16, 256, 0, None)),
                     (rkv.lib().rkv_reconstruct, (d.ptr, 0, 0, None, 0, 16, 16, 0, None)),
                     (rkv.lib().rkv_decode_attn_sparse, (d.ptr, 16, 16, 16, 1, 16, 256, 0, None))]:
        assert fn(*args) == rkv.STATUS_CODE["RKV_ERR_INVALID_ARG"]


def test_wait_selftest_rejects_bad_status_pointers():
    for ptr in (None, 2):                                     # null, and not 4-byte aligned
        assert rkv.lib().rkv_selftest_wait_timeout(ptr, None) == rkv.STATUS_CODE["RKV_ERR_INVALID_ARG"]


def test_bind_without_usable_device_fails_cleanly():
    import torch

    if torch.cuda.is_available():
        pytest.skip("a device is present")
    cfg = _cfg(max_len=4096)
    with pytest.raises(rkv.RkvError) as ei:
        rkv.rkv_cache_bind(cfg, [4096], 256, 1 << 30)
    assert ei.value.status in (rkv.STATUS_CODE["RKV_ERR_CUDA"], rkv.STATUS_CODE["RKV_ERR_UNSUPPORTED"])
