"""GPU parity: the CUDA path through the C ABI against the CPU oracle, element by element.

Small cases run every stage on every token (several tiles, ragged tails, short
and empty sequences, dynamic stride); the named workloads run at full size in
the bench's launch configuration, checking sampled compressed rows exactly and
decode over every unit.
"""
import numpy as np
import pytest
import torch

import long_context_attention_rkv_b200 as rkv
import oracle
import synth
from gpu_harness import (DeviceRun, check_compress, check_decode, check_reconstruct, check_refs, config, sample_positions,
                         to_dev, unit_rows)

pytestmark = pytest.mark.gpu


def _small(name, **kw):
    return synth.WORKLOADS[name].with_(**kw)


def _full_unit_checks(run, wl, K, V, lengths, recon=True):
    stats = {}
    for b, n in enumerate(lengths):
        for h in range(wl.n_kv_heads):
            g = run.unit(b, h)
            Xk, Xv = unit_rows(wl, K, V, b, h, n)
            if n:
                check_refs(wl, g, Xk, Xv)
                check_compress(wl, g, Xk, Xv, stats=stats)
                if recon:
                    check_reconstruct(run, g, b, h)
    return stats


def test_tiny_workload_every_stage():
    wl = synth.WORKLOADS["tiny"]
    lengths = wl.lengths()
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths)
    stats = _full_unit_checks(run, wl, K, V, lengths)
    assert stats["tokens"] == 1920
    check_decode(run, synth.gen_query(wl, 0, 0))


@pytest.mark.parametrize("bits", [4, 8])
def test_bf16_ragged_batch_every_stage(bits):
    wl = _small("llama3_8b_layer", n_kv_heads=2, n_q_heads=8, bits=bits, batch=4, seq_len=5000)
    lengths = [5000, 777, 1, 0]
    K, V = synth.gen_layer(wl, 0, lengths, max_len=5003)
    run = DeviceRun(wl, K, V, lengths)
    _full_unit_checks(run, wl, K, V, lengths)
    check_decode(run, synth.gen_query(wl, 0, 0))


def test_near_duplicate_references_every_stage():
    # four prototypes and almost no noise: most tokens have many references within the
    # search's error band of their k-th nearest (2354 of 2812 tokens per unit need the
    # exhaustive exact rescan, 284 the exact re-rank), so both deferred passes of the encoder
    # carry most of the layer
    wl = _small("llama3_8b_layer", n_kv_heads=2, n_q_heads=8, seq_len=3000, n_proto=4, sigma=0.001, n_outlier=0)
    lengths = [3000]
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths)
    _full_unit_checks(run, wl, K, V, lengths)
    check_decode(run, synth.gen_query(wl, 0, 0))


def test_dynamic_stride_every_stage():
    wl = _small("ultra_long_1m", n_kv_heads=1, n_q_heads=4, head_dim=64, stride0=4, refs_per_phase=64, k=3,
                bits=8, seq_len=6000, n_proto=64)
    lengths = [6000]
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths)
    stats = _full_unit_checks(run, wl, K, V, lengths)
    assert stats["tokens"] == 6000 - len(oracle.schedule(6000, 4, 64))
    check_decode(run, synth.gen_query(wl, 0, 0))


def test_k8_stride32_group7_every_stage():
    wl = _small("qwen2_5_7b_batch", n_kv_heads=2, n_q_heads=14, batch=2, seq_len=3000, ragged=None)
    lengths = [3000, 2500]
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths)
    _full_unit_checks(run, wl, K, V, lengths)
    check_decode(run, synth.gen_query(wl, 0, 0))


def test_simt_search_matches_default_search():
    wl = _small("llama3_8b_layer", n_kv_heads=2, n_q_heads=8, seq_len=4100)
    lengths = [4100]
    K, V = synth.gen_layer(wl, 0, lengths)
    a = DeviceRun(wl, K, V, lengths)
    b = DeviceRun(wl, K, V, lengths, flags=rkv.RKV_FLAG_SELECT_SIMT)
    for h in range(2):
        ga, gb = a.unit(0, h), b.unit(0, h)
        Xk, Xv = unit_rows(wl, K, V, 0, h, 4100)
        check_compress(wl, gb, Xk, Xv)
        same = np.all(ga["idx"] == gb["idx"], axis=1).mean()
        assert same > 0.995


def test_decode_sharp_query_and_bf16_output():
    wl = _small("llama3_8b_layer", n_kv_heads=2, n_q_heads=8, seq_len=3000)
    lengths = [3000]
    K, V = synth.gen_layer(wl, 0, lengths)
    Kf = synth.as_f32(wl, K)
    q = np.zeros((1, 8, 128), dtype=np.float32)
    for h in range(2):
        q[0, h * 4:(h + 1) * 4] = synth.sharp_query(wl, Kf[0, h], 1234 + 77 * h, 4)
    qb = oracle.bf16_round(q)                                  # the query is a bf16 input
    run = DeviceRun(wl, K, V, lengths)
    check_decode(run, qb)
    run16 = DeviceRun(wl, K, V, lengths, out_dtype=rkv.RKV_DTYPE_BF16)
    check_decode(run16, qb)


def test_reconstruct_position_list():
    wl = _small("llama3_8b_layer", n_kv_heads=1, n_q_heads=4, seq_len=2500)
    lengths = [2500]
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths)
    g = run.unit(0, 0)
    pos = np.array([0, 1, 15, 16, 17, 2499, 1024, 3, 3], dtype=np.int32)
    check_reconstruct(run, g, 0, 0, pos)


def test_corrupted_cache_is_reported_not_faulted():
    wl = _small("llama3_8b_layer", n_kv_heads=1, n_q_heads=4, seq_len=1000)
    lengths = [1000]
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths)
    v = run.layer.unit(0, 0)
    off = v.idx - run.layer.cache.data_ptr()
    saved = run.layer.cache[off:off + 2].clone()
    run.layer.cache[off:off + 2] = torch.tensor([0xF0, 0x7F], dtype=torch.uint8, device="cuda")  # ordinal 0x7FF0
    q = to_dev(synth.gen_query(wl, 0, 0))
    out = torch.empty((1, 4, 128), dtype=torch.float32, device="cuda")
    run.layer.decode(q, out)
    assert run.layer.device_error() == rkv.STATUS_CODE["RKV_ERR_CORRUPT"]
    assert run.layer.device_error() == 0                       # read clears it
    Kout = torch.empty((4, 128), dtype=torch.float32, device="cuda")
    run.layer.reconstruct(0, 0, to_dev(np.array([1, 2, 3, 5000], dtype=np.int32)), 4, Kout, None,
                          rkv.RKV_DTYPE_F32)
    st = run.layer.device_error()
    assert st in (rkv.STATUS_CODE["RKV_ERR_CORRUPT"], rkv.STATUS_CODE["RKV_ERR_INVALID_ARG"])
    run.layer.cache[off:off + 2] = saved
    run.layer.decode(q, out)
    assert run.layer.device_error() == 0


# --- named workloads at full size (sampled rows for the search, full decode) ----------------

def _named(name, layers, steps, n_uniform=2048):
    wl = synth.WORKLOADS[name]
    lengths = wl.lengths()
    worst = 0.0
    for layer in layers:
        K, V = synth.gen_layer(wl, layer, lengths)
        run = DeviceRun(wl, K, V, lengths, out_dtype=rkv.RKV_DTYPE_BF16)
        stats = {}
        for b, n in enumerate(lengths):
            for h in range(wl.n_kv_heads):
                g = run.unit(b, h)
                Xk, Xv = unit_rows(wl, K, V, b, h, n)
                check_refs(wl, g, Xk, Xv)
                check_compress(wl, g, Xk, Xv, sample_positions(wl, n, n_uniform, seed=b * 97 + h), stats)
        for step in steps:
            worst = max(worst, check_decode(run, synth.gen_query(wl, layer, step)))
        del run
        torch.cuda.empty_cache()
    return worst


def test_llama3_8b_layer_full_size():
    _named("llama3_8b_layer", layers=[0], steps=[0])


def test_llama3_8b_stack_full_size_two_layers():
    _named("llama3_8b_stack", layers=[0, 31], steps=[0, 63], n_uniform=512)


def test_qwen2_5_7b_batch_full_size_two_layers():
    _named("qwen2_5_7b_batch", layers=[0, 27], steps=[0], n_uniform=512)


def test_ultra_long_full_size():
    _named("ultra_long_1m", layers=[0], steps=[0, 15], n_uniform=512)


def test_direct_decode_flag_matches_oracle():
    wl = _small("qwen2_5_7b_batch", n_kv_heads=2, n_q_heads=14, batch=2, seq_len=2100, ragged=None)
    lengths = [2100, 900]
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths, flags=rkv.RKV_FLAG_DECODE_DIRECT)
    check_decode(run, synth.gen_query(wl, 0, 0))


def test_simt_decode_flag_matches_oracle():
    wl = _small("llama3_8b_layer", n_kv_heads=2, n_q_heads=8, batch=2, seq_len=3100, ragged=None)
    lengths = [3100, 1500]
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths, flags=rkv.RKV_FLAG_DECODE_SIMT)
    check_decode(run, synth.gen_query(wl, 0, 0))


@pytest.mark.parametrize("n_q_heads", [6, 16])
def test_decode_many_short_units(n_q_heads):
    """More 128-token tiles than SMs, so one CTA of the tensor-core decode crosses unit
    boundaries; group sizes 3 (heads padded to 4) and 8."""
    wl = _small("llama3_8b_layer", n_kv_heads=2, n_q_heads=n_q_heads, batch=16, seq_len=1700, ragged=None)
    lengths = [1700 - 97 * i for i in range(16)]
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths)
    check_decode(run, synth.gen_query(wl, 0, 0))
    simt = DeviceRun(wl, K, V, lengths, flags=rkv.RKV_FLAG_DECODE_SIMT)
    q = synth.gen_query(wl, 0, 0)
    a, b = run.decode(q), simt.decode(q)
    assert np.abs(a - b).max() <= 2e-3


def _sparse_check(run, wl, lengths, sel, q):
    """Sparse decode on the GPU against the oracle's attention over the listed rows."""
    n_units = len(lengths) * wl.n_kv_heads
    max_sel = max(1, max(len(x) for x in sel))
    pos = np.zeros((n_units, max_sel), dtype=np.int32)
    cnt = np.zeros(n_units, dtype=np.int32)
    for u, x in enumerate(sel):
        pos[u, :len(x)] = x
        cnt[u] = len(x)
    out = torch.empty((len(lengths), wl.n_q_heads, wl.head_dim), dtype=torch.float32, device="cuda")
    run.layer.decode_sparse(to_dev(q), torch.from_numpy(pos).cuda(), torch.from_numpy(cnt).cuda(), out)
    torch.cuda.synchronize()
    assert run.layer.device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    qf = synth.as_f32(wl, q)
    G = wl.n_q_heads // wl.n_kv_heads
    for b, n in enumerate(lengths):
        for h in range(wl.n_kv_heads):
            u = b * wl.n_kv_heads + h
            g = run.unit(b, h)
            if len(sel[u]) == 0:
                assert np.all(got[b, h * G:(h + 1) * G] == 0.0)
                continue
            Kh, Vh = oracle.unit_cache_rows(n, g["pos"], g["refK"], g["refV"], g["idx"], g["codesK"], g["scalesK"],
                                            g["codesV"], g["scalesV"], wl.bits, wl.group)
            ref = oracle.attention(qf[b, h * G:(h + 1) * G].astype(np.float64), Kh[sel[u]], Vh[sel[u]])
            err = np.abs(got[b, h * G:(h + 1) * G] - ref)
            assert err.max() <= 2e-3, f"sparse decode unit {(b, h)}: max err {err.max()}"


@pytest.mark.parametrize("name", ["llama3_8b_layer", "qwen2_5_7b_batch"])
def test_sparse_decode_matches_oracle_on_listed_rows(name):
    """Selective decompression: random position lists per unit (references and compressed
    tokens mixed, any order), a unit with an empty list, and one that lists every position."""
    wl = _small(name, n_kv_heads=2, n_q_heads=2 * (synth.WORKLOADS[name].n_q_heads // synth.WORKLOADS[name].n_kv_heads),
                batch=2, seq_len=3000, ragged=None)
    lengths = [3000, 1700]
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths)
    rng = np.random.default_rng(7)
    sel = []
    for b, n in enumerate(lengths):
        for h in range(wl.n_kv_heads):
            u = b * wl.n_kv_heads + h
            if u == 1:
                sel.append(np.zeros(0, dtype=np.int64))                # nothing selected
            elif u == 2:
                sel.append(rng.permutation(n))                         # everything, shuffled
            else:
                sel.append(rng.choice(n, size=min(n, 257), replace=False))
    _sparse_check(run, wl, lengths, sel, synth.gen_query(wl, 0, 0))


def test_sparse_decode_full_list_equals_dense_decode():
    wl = _small("llama3_8b_layer", n_kv_heads=2, n_q_heads=8, seq_len=2500)
    lengths = [2500]
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths)
    q = synth.gen_query(wl, 0, 0)
    dense = run.decode(q)
    sel = [np.arange(2500) for _ in range(2)]
    _sparse_check(run, wl, lengths, sel, q)
    pos = torch.from_numpy(np.stack(sel).astype(np.int32)).cuda()
    cnt = torch.full((2,), 2500, dtype=torch.int32, device="cuda")
    out = torch.empty((1, 8, 128), dtype=torch.float32, device="cuda")
    run.layer.decode_sparse(to_dev(q), pos, cnt, out)
    torch.cuda.synchronize()
    assert np.abs(out.cpu().numpy() - dense).max() <= 2e-3


def test_sparse_decode_reports_out_of_range_positions():
    wl = _small("llama3_8b_layer", n_kv_heads=1, n_q_heads=4, seq_len=1000)
    lengths = [1000]
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths)
    pos = torch.tensor([[5, 999, 1000, -1]], dtype=torch.int32, device="cuda")   # two outside [0, 1000)
    cnt = torch.tensor([4], dtype=torch.int32, device="cuda")
    out = torch.empty((1, 4, 128), dtype=torch.float32, device="cuda")
    run.layer.decode_sparse(to_dev(synth.gen_query(wl, 0, 0)), pos, cnt, out)
    torch.cuda.synchronize()
    assert run.layer.device_error() == rkv.STATUS_CODE["RKV_ERR_INVALID_ARG"]


@pytest.mark.parametrize("case", ["llama_int4", "dynamic_int8_d64"])
def test_append_equals_compressing_the_whole_sequence(case):
    """Incremental compression: a prefix compressed, then one token appended at a time (to
    both sequences, then to one of them), checked against the oracle's compression of the
    full sequences and decode over the grown cache."""
    if case == "llama_int4":
        wl = _small("llama3_8b_layer", n_kv_heads=2, n_q_heads=8, batch=2, seq_len=2600, ragged=None)
        cap, start = [2600, 2100], [1700, 900]
    else:
        wl = _small("ultra_long_1m", n_kv_heads=1, n_q_heads=4, head_dim=64, stride0=4, refs_per_phase=64, k=3,
                    bits=8, seq_len=1500, n_proto=64)
        cap, start = [1500], [200]
    K, V = synth.gen_layer(wl, 0, cap)
    run = DeviceRun(wl, K, V, cap, start_lengths=start)
    mid = [min(c, s + 300) for c, s in zip(cap, start)]
    run.append_until(mid)                        # every sequence
    run.append_until(cap)                        # then each up to its own capacity
    for b, n in enumerate(cap):
        for h in range(wl.n_kv_heads):
            g = run.unit(b, h)
            assert g["n"] == n
            Xk, Xv = unit_rows(wl, K, V, b, h, n)
            check_refs(wl, g, Xk, Xv)
            check_compress(wl, g, Xk, Xv)
    check_decode(run, synth.gen_query(wl, 0, 0))
    with pytest.raises(rkv.RkvError) as ei:      # at capacity: refused, nothing launched
        run.layer.append(run.Kd[:, :, 0].contiguous(), run.Vd[:, :, 0].contiguous())
    assert ei.value.status == rkv.STATUS_CODE["RKV_ERR_INVALID_ARG"]


# --- int4 reference store (paper summary page, "Improvements for AI systems": full-pipeline
#     4-bit quantisation of the uncompressed components too) -------------------------------

@pytest.mark.parametrize("case", ["llama", "qwen", "dynamic_d64_int8", "tiny_fp32"])
def test_int4_reference_store_every_stage(case):
    """Reference codes and scales bit-exact; selection over the stored values (exact outside
    the tie band); residual codes against the GPU's index sets; reconstruction; decode through
    the tensor-core, CUDA-core and gather forms; selective decode."""
    if case == "llama":
        wl = _small("llama3_8b_layer", n_kv_heads=2, n_q_heads=8, batch=2, seq_len=4100, ragged=None)
        lengths = [4100, 1333]
    elif case == "qwen":
        wl = _small("qwen2_5_7b_batch", n_kv_heads=2, n_q_heads=14, batch=2, seq_len=3000, ragged=None)
        lengths = [3000, 2100]
    elif case == "dynamic_d64_int8":
        wl = _small("ultra_long_1m", n_kv_heads=1, n_q_heads=4, head_dim=64, stride0=4, refs_per_phase=64, k=3,
                    bits=8, seq_len=3000, n_proto=64)
        lengths = [3000]
    else:
        wl = synth.WORKLOADS["tiny"]
        lengths = wl.lengths()
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths, ref_bits=4)
    assert run.unit(0, 0)["ref_bits"] == 4
    stats = _full_unit_checks(run, wl, K, V, lengths)
    assert stats["tokens"] > 0
    q = synth.gen_query(wl, 0, 0)
    check_decode(run, q)
    # a sharp query (logits of order 4 |k|): the stored reference keys must enter exactly
    G = wl.n_q_heads // wl.n_kv_heads
    sharp = np.zeros((len(lengths), wl.n_q_heads, wl.head_dim), dtype=np.float32)
    for b, n in enumerate(lengths):
        for h in range(wl.n_kv_heads):
            sharp[b, h * G:(h + 1) * G] = synth.sharp_query(wl, synth.as_f32(wl, K[b, h, :n]), n // 2, G)
    check_decode(run, sharp if q.dtype == np.float32 else oracle.bf16_round(sharp))
    rng = np.random.default_rng(3)
    sel = [rng.choice(n, size=min(n, 300), replace=False) for n in lengths for _ in range(wl.n_kv_heads)]
    _sparse_check(run, wl, lengths, sel, q)


@pytest.mark.parametrize("flags", ["simt", "direct"])
def test_int4_reference_store_decode_flags(flags):
    wl = _small("llama3_8b_layer", n_kv_heads=2, n_q_heads=8, batch=2, seq_len=2600, ragged=None)
    lengths = [2600, 1000]
    K, V = synth.gen_layer(wl, 0, lengths)
    f = rkv.RKV_FLAG_DECODE_SIMT if flags == "simt" else rkv.RKV_FLAG_DECODE_DIRECT
    run = DeviceRun(wl, K, V, lengths, ref_bits=4, flags=f)
    assert run.unit(0, 0)["ref_bits"] == 4
    check_decode(run, synth.gen_query(wl, 0, 0))


def test_int4_reference_store_append():
    wl = _small("llama3_8b_layer", n_kv_heads=2, n_q_heads=8, batch=2, seq_len=2200, ragged=None)
    cap, start = [2200, 1900], [1500, 700]
    K, V = synth.gen_layer(wl, 0, cap)
    run = DeviceRun(wl, K, V, cap, start_lengths=start, ref_bits=4)
    run.append_until(cap)
    for b, n in enumerate(cap):
        for h in range(wl.n_kv_heads):
            g = run.unit(b, h)
            assert g["n"] == n
            Xk, Xv = unit_rows(wl, K, V, b, h, n)
            check_refs(wl, g, Xk, Xv)
            check_compress(wl, g, Xk, Xv)
    check_decode(run, synth.gen_query(wl, 0, 0))



# --- learned-coder shapes (paper summary page, "DeltaKV Framework Architecture": z = fc(KV) -
#     fc(KV_R), KV = fd(z) + KV_R; "Improvements for AI systems": SwiGLU fc, linear fd) -------

def _random_coders(D, seed):
    rng = np.random.default_rng(seed)

    def w():
        return oracle.bf16_value(oracle.bf16_round(rng.standard_normal((D, D)) / np.sqrt(D)))
    return tuple(oracle.Coder(w(), w(), w(), w()) for _ in range(2))


@pytest.mark.parametrize("case", ["llama", "qwen"])
def test_learned_coder_shapes_every_stage(case):
    """Latent residual codes against the oracle's fc on the GPU's index sets; reconstruction
    through fd; decode with fd folded into the query and the latent output sum."""
    if case == "llama":
        wl = _small("llama3_8b_layer", n_kv_heads=2, n_q_heads=8, batch=2, seq_len=3000, ragged=None)
        lengths = [3000, 1200]
    else:
        wl = _small("qwen2_5_7b_batch", n_kv_heads=2, n_q_heads=14, batch=2, seq_len=2600, ragged=None)
        lengths = [2600, 2000]
    K, V = synth.gen_layer(wl, 0, lengths)
    coder = _random_coders(wl.head_dim, 11)
    run = DeviceRun(wl, K, V, lengths, coder=coder)
    stats = {}
    for b, n in enumerate(lengths):
        for h in range(wl.n_kv_heads):
            g = run.unit(b, h)
            Xk, Xv = unit_rows(wl, K, V, b, h, n)
            check_refs(wl, g, Xk, Xv)
            pos = sample_positions(wl, n, n_uniform=400, seed=b * 7 + h)
            check_compress(wl, g, Xk, Xv, positions=pos, stats=stats, coder=coder)
            check_reconstruct(run, g, b, h, positions=pos)
    assert stats["tokens"] > 0
    check_decode(run, synth.gen_query(wl, 0, 0))


def test_learned_coder_ragged_batch():
    """Learned-coder shapes over a ragged batch: one sequence spanning many 128-token tiles, one
    a tile and a ragged tail, one shorter than a tile, and an empty one (units without tiles
    between units with tiles); every compressed token checked."""
    wl = _small("llama3_8b_layer", n_kv_heads=2, n_q_heads=8, batch=4, seq_len=2100)
    lengths = [2100, 150, 17, 0]
    K, V = synth.gen_layer(wl, 0, lengths, max_len=2103)
    coder = _random_coders(wl.head_dim, 13)
    run = DeviceRun(wl, K, V, lengths, coder=coder)
    stats = {}
    for b, n in enumerate(lengths):
        if n == 0:
            continue
        for h in range(wl.n_kv_heads):
            g = run.unit(b, h)
            Xk, Xv = unit_rows(wl, K, V, b, h, n)
            check_refs(wl, g, Xk, Xv)
            check_compress(wl, g, Xk, Xv, stats=stats, coder=coder)
            check_reconstruct(run, g, b, h)
    n_cmp = sum(n - len(oracle.schedule(n, wl.stride0, wl.refs_per_phase)) for n in lengths if n)
    assert stats["tokens"] == wl.n_kv_heads * n_cmp
    check_decode(run, synth.gen_query(wl, 0, 0))


def test_learned_coder_refuses_what_it_does_not_cover():
    wl = _small("llama3_8b_layer", n_kv_heads=1, n_q_heads=4, seq_len=600)
    lengths = [600]
    K, V = synth.gen_layer(wl, 0, lengths)
    coder = _random_coders(wl.head_dim, 12)
    run = DeviceRun(wl, K, V, lengths, coder=coder)
    q = to_dev(synth.gen_query(wl, 0, 0))
    out = torch.empty((1, 4, 128), dtype=torch.float32, device="cuda")
    pos = torch.zeros((1, 4), dtype=torch.int32, device="cuda")
    cnt = torch.ones(1, dtype=torch.int32, device="cuda")
    for call in (lambda: run.layer.decode_sparse(q, pos, cnt, out),
                 lambda: run.layer.append(run.Kd[:, :, 0].contiguous(), run.Vd[:, :, 0].contiguous())):
        with pytest.raises(rkv.RkvError) as ei:
            call()
        assert ei.value.status == rkv.STATUS_CODE["RKV_ERR_UNSUPPORTED"]
    # a coder-1 cache without weights refuses to compress
    bare = rkv.Layer(config(wl, lengths, max_len=K.shape[2], coder=1), lengths)
    with pytest.raises(rkv.RkvError) as ei:
        bare.compress(run.Kd, run.Vd)
    assert ei.value.status == rkv.STATUS_CODE["RKV_ERR_INVALID_ARG"]
