"""Host-side logic of bench.py on CPU: the algorithmic work it divides by (closed forms of the
fixed-stride schedule) and the guard on the committed DRAM-traffic figures."""
import json

import pytest

import bench
import synth


@pytest.mark.parametrize("name", ["llama3_8b_layer", "llama3_8b_stack"])
def test_workload_quantities_match_the_closed_forms(name):
    """Fixed stride s, no dynamic phases: references at positions 0, s, 2s, ... (R = n / s per
    unit), and the compressed position p has floor(p / s) + 1 earlier references, so a block of
    s - 1 compressed positions after reference b contributes (s - 1)(b + 1) candidates."""
    wl = synth.WORKLOADS[name]
    assert wl.refs_per_phase == 0 and wl.batch == 1
    n, s, D, H = wl.seq_len, wl.stride0, wl.head_dim, wl.n_kv_heads
    R = n // s
    C = n - R
    per_tok = 2 * D * wl.bits // 8 + 2 * (D // 32) * 2 + 2 * wl.k      # codes, fp16 scales, u16 ordinals
    q = bench.workload_quantities(wl, wl.lengths())
    assert q["tokens_cmp"] == H * C
    assert q["bytes_per_token"] == per_tok == 152
    assert q["search_flops"] == H * (s - 1) * R * (R + 1) // 2 * 2 * D
    assert q["decode_bytes"] == H * (C * per_tok + R * 4 * D)
    assert q["encode_bytes"] == H * C * (2 * D * 2 + per_tok)


def _fake_tree(tmp_path, src_text):
    src = tmp_path / "kern.cu"
    src.write_text(src_text)
    (tmp_path / "profiles").mkdir()
    return ["kern.cu"]


def test_traffic_is_used_only_for_its_workload_and_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    srcs = _fake_tree(tmp_path, "kernel source v1")
    sha = bench._src_sha(srcs)
    entry = {"decode": {"wl_a": {"dram_bytes_per_launch": 1234, "src_sha": sha}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(entry))
    assert bench._traffic("decode", srcs, "wl_a") == 1234
    assert bench._traffic("decode", srcs, "wl_b") is None          # another workload
    assert bench._traffic("encode", srcs, "wl_a") is None          # another kernel
    (tmp_path / "kern.cu").write_text("kernel source v2")          # the kernel changed since
    assert bench._traffic("decode", srcs, "wl_a") is None


def test_traffic_without_a_summary_is_none(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    srcs = _fake_tree(tmp_path, "x")
    assert bench._traffic("decode", srcs, "wl_a") is None
