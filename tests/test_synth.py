"""The synthetic input generator: determinism, random access and the workload shapes."""
import numpy as np

import synth


def test_rows_regenerate_independently():
    wl = synth.WORKLOADS["llama3_8b_layer"]
    k_all, v_all = synth.gen_unit(wl, 0, 0, 3, 0, 4096)
    k_mid, v_mid = synth.gen_unit(wl, 0, 0, 3, 1000, 1100)
    assert np.array_equal(k_all[1000:1100], k_mid) and np.array_equal(v_all[1000:1100], v_mid)
    k2, _ = synth.gen_unit(wl, 0, 0, 4, 0, 4096)
    assert not np.array_equal(k_all, k2)                     # units draw from different streams


def test_prototype_structure_and_outliers():
    wl = synth.WORKLOADS["llama3_8b_layer"]
    K, V = synth.gen_unit(wl, 1, 0, 0, 0, 8192)
    Kf, Vf = synth.bf16_to_f32(K), synth.bf16_to_f32(V)
    oc = synth.outlier_channels(wl, 1, 0, 0)
    assert len(set(oc)) == 4
    normal_ch = [c for c in range(128) if c not in oc]
    assert 5 < np.abs(Kf[:, oc]).mean() / np.abs(Kf[:, normal_ch]).mean() < 12
    # tokens that share a prototype differ by noise only: |K_i - K_j| ~ sigma*sqrt(2D) outside outliers
    ids = np.array([synth.proto_id(wl, 1, 0, 0, t) for t in range(8192)])
    a, b = np.nonzero(ids == ids[0])[0][:2]
    d = np.linalg.norm(Vf[a] - Vf[b])
    assert 0.5 * 0.15 * np.sqrt(256) < d < 2 * 0.15 * np.sqrt(256)
    assert abs(Vf.std() - 1.0) < 0.1


def test_lengths_and_queries():
    wl = synth.WORKLOADS["qwen2_5_7b_batch"]
    L = wl.lengths()
    assert len(L) == 8 and all(16384 <= n <= 32768 for n in L) and len(set(L)) > 1
    assert L == wl.lengths()
    q = synth.bf16_to_f32(synth.gen_query(wl, 0, 0))
    assert q.shape == (8, 28, 128) and abs(q.std() - 0.125) < 0.01
    q1 = synth.bf16_to_f32(synth.gen_query(wl, 0, 1))
    assert not np.array_equal(q, q1)


def test_fp32_workload():
    wl = synth.WORKLOADS["tiny"]
    K, V = synth.gen_layer(wl, 0)
    assert K.dtype == np.float32 and K.shape == (1, 1, 2048, 64)
    assert synth.checksum(K) == synth.checksum(synth.gen_layer(wl, 0)[0])
