"""Pins of the CPU oracle against things other than itself (CPU only).

Each test ties one oracle step to a closed form, a library routine, brute
force, a hand-derived example or an invariant of the method, so that a
plausible mistake (a dropped term, a wrong sign or index, a transposed
operand, an off-by-one in the schedule) fails at least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch
from scipy.spatial.distance import cdist

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_vals(rng, shape, scale=1.0):
    """Random values that are exactly representable in bf16 (as float32)."""
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    return torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()


# --- reference schedule (paper summary page, "DeltaKV Framework Architecture";
#     news page, "How ResidualKV Works": dynamic-stride scheduling) -------------------

@pytest.mark.parametrize("n,s,R", [(2048, 16, 128), (32768, 16, 2048), (131072, 16, 8192), (1, 16, 1),
                                   (16, 16, 1), (17, 16, 2)])
def test_schedule_fixed_counts(n, s, R):
    pos = oracle.schedule(n, s)
    assert len(pos) == R
    assert np.array_equal(pos, np.arange(R, dtype=np.int32) * s)


def test_schedule_fixed_ceil_for_ragged_lengths():
    rng = np.random.default_rng(1)
    for n in list(rng.integers(16384, 32769, 50)) + [16384, 32768, 31, 32, 33]:
        assert len(oracle.schedule(int(n), 32)) == math.ceil(n / 32)


def test_schedule_dynamic_one_million():
    # stride 16 doubling after every 1024 references: phase p starts at
    # 1024*16*(2^p - 1) with stride 16*2^p; 6 full phases below 2^20 and 16 refs of the 7th
    pos = oracle.schedule(1 << 20, 16, 1024)
    assert len(pos) == 6 * 1024 + 16 == 6160
    for p in range(7):
        start = 1024 * 16 * (2 ** p - 1)
        assert pos[1024 * p] == start
        seg = pos[1024 * p: 1024 * (p + 1)]
        assert np.all(np.diff(seg) == 16 * 2 ** p)
    assert pos[-1] == 1032192 + 15 * 1024


def test_schedule_dynamic_count_closed_form():
    rng = np.random.default_rng(2)
    for n in list(rng.integers(1, 3_000_000, 40)) + [16384, 16385, 49152, 49153]:
        n = int(n)
        want, start, p = 0, 0, 0
        while start < n:
            stride = 16 * 2 ** p
            want += min(1024, -(-(n - start) // stride))
            start += 1024 * stride
            p += 1
        assert len(oracle.schedule(n, 16, 1024)) == want


# --- rounding helpers: against torch's bf16 and numpy's binary16 -----------------------

def test_bf16_round_matches_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 3,
                        # exact ties: bf16 value + half an ulp
                        (_bf16_vals(rng, 1000) * np.float32(1 + 2 ** -8)).astype(np.float32)])
    ours = oracle.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_fp16_round_up_is_smallest_binary16_above():
    rng = np.random.default_rng(4)
    vals = np.concatenate([np.exp(rng.uniform(math.log(1e-9), math.log(6.5e4), 4000)),
                           np.float16(rng.uniform(0, 100, 500)).astype(np.float64),  # exactly representable
                           [2.0 ** -24, 2.0 ** -25, 2.0 ** -14, 65504.0, 1e-45]]).astype(np.float32)
    for f in vals:
        bits, ov = oracle.fp16_round_up(float(f))
        assert ov == 0
        h = np.array([bits], dtype=np.uint16).view(np.float16)[0]
        assert float(h) == oracle.fp16_value(bits)
        assert float(h) >= float(f)
        below = np.nextafter(h, np.float16(0))
        assert float(below) < float(f)
    bits, ov = oracle.fp16_round_up(65505.0)
    assert ov == 1 and bits == 0x7C00
    assert oracle.fp16_round_up(0.0) == (0, 0)


# --- L2 distance: the expanded form in long double -----------------------------------

def test_l2_matches_expanded_form():
    rng = np.random.default_rng(5)
    for D in (4, 64, 128):
        for _ in range(200):
            a = (rng.standard_normal(D) * rng.uniform(0.1, 8)).astype(np.float32)
            b = (a + rng.standard_normal(D) * rng.uniform(1e-3, 1)).astype(np.float32)
            al = a.astype(np.longdouble)
            bl = b.astype(np.longdouble)
            exp = float(np.dot(al, al) - 2 * np.dot(al, bl) + np.dot(bl, bl))
            got = oracle.l2(a, b)
            assert abs(got - exp) <= 1e-12 * float(np.dot(al, al) + np.dot(bl, bl))


# --- top-k selection ------------------------------------------------------------------

def test_select_top_k_is_the_minimum_k_subset():
    """Exhaustive: the chosen set minimises the summed distance over all k-subsets."""
    rng = np.random.default_rng(6)
    n, D, s = 64, 4, 4
    for trial in range(6):
        X = rng.standard_normal((n, D)).astype(np.float32)
        ref_pos = oracle.schedule(n, s)
        refK = oracle.build_refs(X, ref_pos)
        rv = oracle.bf16_value(refK)
        for k in (1, 2, 3, 4):
            tok = np.arange(n, dtype=np.int32)
            idx, keff, _ = oracle.select(X, tok, refK, ref_pos, k)
            d = cdist(X.astype(np.float64), rv.astype(np.float64), "sqeuclidean")
            for t in range(n):
                cands = [j for j in range(len(ref_pos)) if ref_pos[j] <= t]
                kk = min(k, len(cands))
                assert keff[t] == kk
                best = min(itertools.combinations(cands, kk), key=lambda S: sum(d[t, j] for j in S))
                sums = sorted(sum(d[t, j] for j in S) for S in itertools.combinations(cands, kk))
                if len(sums) > 1:
                    assert sums[1] - sums[0] > 1e-9  # unique minimum on random data
                assert list(idx[t, :kk]) == sorted(best)
                assert all(v == oracle.SENTINEL for v in idx[t, kk:])


def test_select_planted_copies_and_causality():
    rng = np.random.default_rng(7)
    n, D, s, k = 512, 16, 16, 4
    X = _bf16_vals(rng, (n, D))
    ref_pos = oracle.schedule(n, s)
    # plant: token 300 is an exact copy of reference ordinal 5 (position 80),
    # token 301 of reference 18 (position 288)
    X[300] = X[80]
    X[301] = X[288]
    refK = oracle.build_refs(X, ref_pos)
    tok = np.arange(n, dtype=np.int32)
    idx, keff, dist = oracle.select(X, tok, refK, ref_pos, k)
    assert 5 in idx[300] and dist[300, 0] == 0.0
    assert 18 in idx[301] and dist[301, 0] == 0.0
    for t in range(n):
        ch = idx[t, :keff[t]]
        assert np.all(np.diff(ch.astype(int)) > 0)           # ascending ordinals
        assert np.all(ref_pos[ch] <= t)                      # only earlier (or same) positions
        assert np.all(np.diff(dist[t][~np.isnan(dist[t])]) >= 0)


def test_select_tie_break_lowest_ordinal():
    D = 8
    X = np.zeros((64, D), dtype=np.float32)
    X[:, 0] = 1.0                                            # every token identical
    ref_pos = oracle.schedule(64, 8)
    refK = oracle.build_refs(X, ref_pos)
    idx, keff, _ = oracle.select(X, np.array([63], dtype=np.int32), refK, ref_pos, 3)
    assert list(idx[0]) == [0, 1, 2]


# --- residual encoding ----------------------------------------------------------------

def _load_golden():
    vals = {}
    with open(os.path.join(GOLDEN, "quantiser_worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = rest
    return vals


def test_encode_matches_hand_derived_example():
    g = _load_golden()
    x = np.array([float(v) for v in g["x"]], dtype=np.float32)[None, :]
    refs = np.array([[0x3F80] * 32, [0x3F00] * 32], dtype=np.uint16)
    idx = np.array([[0, 1]], dtype=np.uint16)
    e4 = oracle.encode(x, refs, idx, 4, want_detail=True)
    assert np.array_equal(e4["mean"][0], np.full(32, 0.75, dtype=np.float32))
    assert np.array_equal(e4["delta"][0], np.array([float(v) for v in g["delta"]], dtype=np.float32))
    assert e4["scales"][0, 0] == int(g["int4_scale_bits"][0], 16)
    assert list(e4["codes"][0]) == [int(b, 16) for b in g["int4_bytes"]]
    assert list(oracle.unpack_codes(e4["codes"][0], 32, 4)) == [int(v) for v in g["int4_codes"]]
    e8 = oracle.encode(x, refs, idx, 8)
    assert e8["scales"][0, 0] == int(g["int8_scale_bits"][0], 16)
    assert list(e8["codes"][0].view(np.int8)) == [int(v) for v in g["int8_codes"]]


def _numpy_unpack(codes, D, bits):
    """Independent unpacking: two's complement bytes / nibbles, even channel low."""
    if bits == 8:
        return codes.view(np.int8).astype(np.int64)
    lo = (codes & 0xF).astype(np.int64)
    hi = (codes >> 4).astype(np.int64)
    out = np.empty(codes.shape[:-1] + (D,), dtype=np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return np.where(out >= 8, out - 16, out)


@pytest.mark.parametrize("bits", [4, 8])
def test_quantiser_invariants(bits):
    rng = np.random.default_rng(8 + bits)
    n, D, R, k = 400, 128, 40, 4
    qmax = 127 if bits == 8 else 7
    refs = oracle.bf16_round(rng.standard_normal((R, D)))
    idx = np.sort(np.stack([rng.choice(R, k, replace=False) for _ in range(n)]), axis=1).astype(np.uint16)
    idx[:50, 2:] = oracle.SENTINEL                           # k_eff = 2 rows
    idx[50:60, 1:] = oracle.SENTINEL                         # k_eff = 1 rows
    x = (oracle.bf16_value(refs)[idx[:, 0]] + rng.standard_normal((n, D)) * 0.2).astype(np.float32)
    x[60, :32] = 0.0                                         # (a group stays nonzero through the mean)
    e = oracle.encode(x, refs, idx, bits, want_detail=True)
    codes = _numpy_unpack(e["codes"], D, bits)
    scales = e["scales"].view(np.float16).astype(np.float64)
    delta = e["delta"].astype(np.float64)
    # mean = plain mean of the selected reference rows
    rv = oracle.bf16_value(refs).astype(np.float64)
    for t in range(n):
        sel = [j for j in idx[t] if j != oracle.SENTINEL]
        np.testing.assert_allclose(e["mean"][t], rv[sel].mean(axis=0), rtol=4 * 2 ** -24, atol=1e-30)
    np.testing.assert_array_equal(e["delta"], (x - e["mean"]).astype(np.float32))
    for t in range(n):
        for gi in range(D // 32):
            sl = slice(32 * gi, 32 * gi + 32)
            a = np.max(np.abs(delta[t, sl]))
            s = scales[t, gi]
            if a == 0:
                assert s == 0 and np.all(codes[t, sl] == 0)
                continue
            assert s >= np.float32(np.float32(a) / np.float32(qmax))
            assert float(np.nextafter(np.float16(s), np.float16(0))) < np.float32(np.float32(a) / np.float32(qmax))
            assert np.max(np.abs(codes[t, sl])) == qmax
            assert np.all(np.abs(delta[t, sl] - codes[t, sl] * s) <= s / 2 + 1e-12 * s)


def test_quantiser_grid_roundtrip():
    rng = np.random.default_rng(9)
    D = 64
    refs = oracle.bf16_round(np.zeros((1, D)))
    for bits, qmax in ((4, 7), (8, 127)):
        s = np.float32(0.125)                                # binary16-exact scale
        codes = rng.integers(-qmax, qmax + 1, (50, D))
        codes[:, ::32] = qmax                                # max|code| = qmax in every group
        x = (codes * s).astype(np.float32)
        e = oracle.encode(x, refs, np.zeros((50, 1), dtype=np.uint16), bits)
        assert np.all(e["scales"].view(np.float16) == np.float16(s))
        assert np.array_equal(_numpy_unpack(e["codes"], D, bits), codes)


def test_k1_at_reference_position_gives_zero_residual():
    rng = np.random.default_rng(10)
    n, D = 256, 64
    X = _bf16_vals(rng, (n, D))
    ref_pos = oracle.schedule(n, 16)
    refK = oracle.build_refs(X, ref_pos)
    idx, keff, dist = oracle.select(X[ref_pos], ref_pos, refK, ref_pos, 1)
    assert np.array_equal(idx[:, 0], np.arange(len(ref_pos)))
    assert np.all(dist[:, 0] == 0)
    for bits in (4, 8):
        e = oracle.encode(X[ref_pos], refK, idx, bits)
        assert np.all(e["codes"] == 0) and np.all(e["scales"] == 0)


# --- reconstruction and attention -----------------------------------------------------

def test_unquantised_reconstruction_is_exact():
    rng = np.random.default_rng(11)
    n, D = 1024, 64
    X = (rng.standard_normal((n, D)) * 2).astype(np.float32)   # fp32 inputs: refs get rounded
    c = oracle.compress_unit(X, X, 16, 0, 4, 4)
    e = oracle.encode(X[c["pos"]], c["refK"], c["idx"], 0)
    xh = oracle.reconstruct(c["refK"], c["idx"], None, None, 0, delta_exact=e["delta_exact"])
    assert np.array_equal(xh, X[c["pos"]].astype(np.float64))


def test_quantised_reconstruction_error_bound():
    rng = np.random.default_rng(12)
    n, D = 1024, 128
    X = _bf16_vals(rng, (n, D))
    for bits in (4, 8):
        c = oracle.compress_unit(X, X, 16, 0, 4, bits)
        xh = oracle.reconstruct(c["refK"], c["idx"], c["codesK"], c["scalesK"], bits)
        s = np.repeat(c["scalesK"].view(np.float16).astype(np.float64), 32, axis=1)
        err = np.abs(xh.astype(np.float64) - X[c["pos"]])
        assert np.all(err <= s / 2 + 4 * 2 ** -24 * np.abs(X[c["pos"]]) + 1e-30)


def _plain_attention(q, K, V):
    q = torch.from_numpy(np.asarray(q, np.float64))
    K = torch.from_numpy(np.asarray(K, np.float64))
    V = torch.from_numpy(np.asarray(V, np.float64))
    w = torch.softmax(q @ K.T / math.sqrt(K.shape[1]), dim=-1)
    return (w @ V).numpy()


def test_attention_matches_torch():
    rng = np.random.default_rng(13)
    for n in (1, 7, 300):
        q = rng.standard_normal((4, 32))
        K = rng.standard_normal((n, 32))
        V = rng.standard_normal((n, 32))
        np.testing.assert_allclose(oracle.attention(q, K, V), _plain_attention(q, K, V), rtol=1e-12, atol=1e-13)


def test_attention_special_cases():
    rng = np.random.default_rng(14)
    V = rng.standard_normal((5, 16))
    q = rng.standard_normal((2, 16))
    np.testing.assert_array_equal(oracle.attention(q, rng.standard_normal((1, 16)), V[:1]), np.tile(V[0], (2, 1)))
    K = np.tile(rng.standard_normal(16), (5, 1))
    np.testing.assert_allclose(oracle.attention(q, K, V), np.tile(V.mean(axis=0), (2, 1)), rtol=1e-13)
    assert np.all(oracle.attention(q, np.zeros((0, 16)), np.zeros((0, 16))) == 0)


def test_unquantised_cache_attention_equals_uncompressed_attention():
    rng = np.random.default_rng(15)
    n, D, G = 700, 64, 3
    Xk = _bf16_vals(rng, (n, D))
    Xv = _bf16_vals(rng, (n, D))
    c = oracle.compress_unit(Xk, Xv, 16, 0, 4, 4)
    ek = oracle.encode(Xk[c["pos"]], c["refK"], c["idx"], 0)
    ev = oracle.encode(Xv[c["pos"]], c["refV"], c["idx"], 0)
    Kh = np.empty((n, D))
    Vh = np.empty((n, D))
    Kh[c["ref_pos"]] = oracle.bf16_value(c["refK"])
    Vh[c["ref_pos"]] = oracle.bf16_value(c["refV"])
    Kh[c["pos"]] = oracle.reconstruct(c["refK"], c["idx"], None, None, 0, delta_exact=ek["delta_exact"])
    Vh[c["pos"]] = oracle.reconstruct(c["refV"], c["idx"], None, None, 0, delta_exact=ev["delta_exact"])
    q = rng.standard_normal((G, D))
    np.testing.assert_allclose(oracle.attention(q, Kh, Vh), _plain_attention(q, Xk, Xv), rtol=1e-12, atol=1e-13)


def test_compress_unit_dynamic_stride_smoke():
    rng = np.random.default_rng(16)
    n, D = 3000, 16
    X = _bf16_vals(rng, (n, D))
    c = oracle.compress_unit(X, X, 2, 64, 2, 4)
    assert len(c["ref_pos"]) == len(oracle.schedule(n, 2, 64))
    assert len(c["pos"]) == n - len(c["ref_pos"])
    assert c["overflow"] == 0


# --- int4 reference store (paper summary page, "Improvements for AI systems" and "Impact
#     and Future Directions": full-pipeline 4-bit quantisation of the uncompressed
#     components as well) -------------------------------------------------------------------

def test_reference_quantiser_invariants():
    """Each reference row quantised by itself: scale = the smallest power of two >= a / 7
    (so every stored value is an exact bf16 number), |x - code*scale| <= scale/2."""
    rng = np.random.default_rng(21)
    n, D, qmax = 300, 128, 7
    X = (rng.standard_normal((n, D)) * rng.uniform(0.01, 8, (n, 1))).astype(np.float32)
    X[5, 32:64] = 0.0                                        # an all-zero group
    X[6] = 0.0                                               # an all-zero row
    X[7, :32] = 1e-9                                         # below the smallest binary16 power of two x 7
    X[8, 32:64] = 3.5                                        # a / 7 exactly a power of two
    codes, scales, ov = oracle.quantize_rows(X, 4, 32)
    assert ov == 0 and codes.shape == (n, D // 2) and scales.shape == (n, D // 32)
    q = _numpy_unpack(codes, D, 4)
    s = scales.view(np.float16).astype(np.float64)
    for i in range(n):
        for g in range(D // 32):
            sl = slice(32 * g, 32 * g + 32)
            a = float(np.max(np.abs(X[i, sl])))
            if a == 0:
                assert s[i, g] == 0 and np.all(q[i, sl] == 0)
                continue
            v = float(np.float32(np.float32(a) / np.float32(qmax)))
            expect = max(2.0 ** int(np.ceil(np.log2(v))), 2.0 ** -24)
            assert s[i, g] == expect, (i, g, s[i, g], v)
            assert 4 <= np.max(np.abs(q[i, sl])) <= qmax or s[i, g] == 2.0 ** -24
            assert np.all(np.abs(X[i, sl] - q[i, sl] * s[i, g]) <= s[i, g] / 2 * (1 + 1e-12))
    assert s[8, 1] == 0.5 and np.max(np.abs(q[8, 32:64])) == 7
    # stored values: code * scale, decoded independently (numpy nibbles x numpy binary16);
    # every one is an exact bf16 value
    vals = oracle.dequantize_rows(codes, scales, D, 4, 32)
    np.testing.assert_array_equal(vals, (q * np.repeat(s, 32, axis=1)).astype(np.float32))
    assert np.array_equal(vals.astype(np.float64), q * np.repeat(s, 32, axis=1))   # exact in fp32
    assert np.array_equal(oracle.bf16_value(oracle.bf16_round(vals)), vals)
    # the residuals' rounding (next binary16 instead of the next power of two) on the same rows
    _, s16, _ = oracle.quantize_rows(X, 4, 32, pow2=False)
    e = oracle.encode(X, oracle.bf16_round(np.zeros((1, D))), np.zeros((n, 1), dtype=np.uint16), 4)
    assert np.array_equal(s16, e["scales"])


def test_reference_quantiser_grid_roundtrip():
    rng = np.random.default_rng(22)
    D = 64
    q = rng.integers(-7, 8, (40, D))
    q[:, ::32] = 7
    X = (q * np.float32(0.25)).astype(np.float32)
    codes, scales, _ = oracle.quantize_rows(X, 4, 32)
    assert np.all(scales.view(np.float16) == np.float16(0.25))
    assert np.array_equal(_numpy_unpack(codes, D, 4), q)
    assert np.array_equal(oracle.dequantize_rows(codes, scales, D), X)


def test_value_references_match_bf16_references_on_bf16_values():
    """The stored-value entry points equal the bf16 ones when the values are bf16 rows."""
    rng = np.random.default_rng(23)
    n, D, s, k = 600, 32, 8, 4
    X = _bf16_vals(rng, (n, D))
    ref_pos = oracle.schedule(n, s)
    refK = oracle.build_refs(X, ref_pos)
    vals = oracle.bf16_value(refK).astype(np.float32)
    tok = np.arange(n, dtype=np.int32)
    a = oracle.select(X, tok, refK, ref_pos, k)
    b = oracle.select(X, tok, vals, ref_pos, k)
    for u, v in zip(a, b):
        assert np.array_equal(u, v, equal_nan=True)
    e1 = oracle.encode(X, refK, a[0], 4, want_detail=True)
    e2 = oracle.encode(X, vals, a[0], 4, want_detail=True)
    for key in ("codes", "scales", "mean"):
        assert np.array_equal(e1[key], e2[key])
    r1 = oracle.reconstruct(refK, a[0], e1["codes"], e1["scales"], 4)
    r2 = oracle.reconstruct(vals, a[0], e1["codes"], e1["scales"], 4)
    assert np.array_equal(r1, r2)


def test_int4_reference_select_is_the_minimum_k_subset():
    """Exhaustive on tiny inputs: selection ranks the stored (dequantised) references."""
    rng = np.random.default_rng(24)
    n, D, s = 48, 32, 4
    X = rng.standard_normal((n, D)).astype(np.float32)
    ref_pos = oracle.schedule(n, s)
    _, _, vals, _ = oracle.build_refs_quantized(X, ref_pos)
    d = cdist(X.astype(np.float64), vals.astype(np.float64), "sqeuclidean")
    for k in (1, 2, 3):
        idx, keff, _ = oracle.select(X, np.arange(n, dtype=np.int32), vals, ref_pos, k)
        for t in range(n):
            cands = [j for j in range(len(ref_pos)) if ref_pos[j] <= t]
            kk = min(k, len(cands))
            best = min(itertools.combinations(cands, kk), key=lambda S: sum(d[t, j] for j in S))
            assert list(idx[t, :kk]) == sorted(best)


def test_int4_reference_store_unquantised_residuals_rebuild_the_input():
    """With int4 references and exact residuals, compressed positions rebuild the input
    exactly, reference positions give the stored value, and attention over that cache equals
    attention over [stored references, inputs]."""
    rng = np.random.default_rng(25)
    n, D, G = 600, 64, 2
    Xk = _bf16_vals(rng, (n, D))
    Xv = _bf16_vals(rng, (n, D))
    c = oracle.compress_unit(Xk, Xv, 16, 0, 4, 4, ref_bits=4)
    assert c["refK"].dtype == np.float32 and c["ref_overflow"] == 0
    # a copy of a stored reference selects that reference at distance 0
    idx, _, dist = oracle.select(c["refK"][3:4], np.array([n - 1], np.int32), c["refK"], c["ref_pos"], 1)
    assert idx[0, 0] == 3 and dist[0, 0] == 0
    ek = oracle.encode(Xk[c["pos"]], c["refK"], c["idx"], 0)
    ev = oracle.encode(Xv[c["pos"]], c["refV"], c["idx"], 0)
    Kh = np.empty((n, D))
    Vh = np.empty((n, D))
    Kh[c["ref_pos"]] = c["refK"]
    Vh[c["ref_pos"]] = c["refV"]
    Kh[c["pos"]] = oracle.reconstruct(c["refK"], c["idx"], None, None, 0, delta_exact=ek["delta_exact"])
    Vh[c["pos"]] = oracle.reconstruct(c["refV"], c["idx"], None, None, 0, delta_exact=ev["delta_exact"])
    assert np.array_equal(Kh[c["pos"]], Xk[c["pos"]].astype(np.float64))
    K2, V2 = Xk.astype(np.float64), Xv.astype(np.float64)
    K2[c["ref_pos"]] = c["refK"]
    V2[c["ref_pos"]] = c["refV"]
    q = rng.standard_normal((G, D))
    np.testing.assert_allclose(oracle.attention(q, Kh, Vh), _plain_attention(q, K2, V2), rtol=1e-12, atol=1e-13)
    # and the quantised cache's reconstruction rows sit within scale/2 of the input
    xh = oracle.reconstruct(c["refK"], c["idx"], c["codesK"], c["scalesK"], 4)
    sc = np.repeat(c["scalesK"].view(np.float16).astype(np.float64), 32, axis=1)
    assert np.all(np.abs(xh - Xk[c["pos"]]) <= sc / 2 + 4 * 2 ** -24 * np.abs(Xk[c["pos"]]) + 1e-30)


# --- learned-coder shapes (paper summary page, "DeltaKV Framework Architecture": z = fc(KV)
#     - fc(KV_R), KV = fd(z) + KV_R; "Improvements for AI systems": SwiGLU fc, linear fd) ------

def _coder(rng, D, H=None, L=None, scale=None):
    H = D if H is None else H
    L = D if L is None else L
    def w(o, i):
        return oracle.bf16_value(oracle.bf16_round(rng.standard_normal((o, i)) / np.sqrt(i)))
    return oracle.Coder(w(H, D), w(H, D), w(L, H), w(D, L))


def test_coder_fc_matches_torch_swiglu():
    rng = np.random.default_rng(31)
    D, H, L = 64, 96, 48
    c = _coder(rng, D, H, L)
    X = _bf16_vals(rng, (50, D), 2.0)
    x = torch.from_numpy(X.astype(np.float64))
    g = x @ torch.from_numpy(c.Wg.astype(np.float64)).T
    u = x @ torch.from_numpy(c.Wu.astype(np.float64)).T
    ref = (torch.nn.functional.silu(g) * u) @ torch.from_numpy(c.Wo.astype(np.float64)).T
    np.testing.assert_allclose(oracle.coder_fc(X, c), ref.numpy(), rtol=1e-12, atol=1e-12)


def test_latent_residual_is_fc_difference_and_zero_for_the_mean():
    rng = np.random.default_rng(32)
    n, D, R, k = 60, 64, 20, 2
    cK = _coder(rng, D)
    refs = oracle.bf16_round(rng.standard_normal((R, D)))
    idx = np.sort(np.stack([rng.choice(R, k, replace=False) for _ in range(n)]), axis=1).astype(np.uint16)
    x = _bf16_vals(rng, (n, D))
    rv = oracle.bf16_value(refs)
    mean = ((rv[idx[:, 0]] + rv[idx[:, 1]]) / np.float32(2)).astype(np.float32)
    x[:5] = mean[:5]                                          # tokens equal to their mean
    e = oracle.encode_latent(x, refs, idx, 4, cK)
    np.testing.assert_allclose(e["z"], oracle.coder_fc(x, cK) - oracle.coder_fc(mean, cK), rtol=1e-12, atol=1e-12)
    assert np.all(e["codes"][:5] == 0) and np.all(e["scales"][:5] == 0)
    # the codes are the residuals' group quantiser applied to z (rounded to fp32), with every
    # scale the smallest power of two >= fl32(a / 7) (numpy: a float32 division, then frexp)
    q = _numpy_unpack(e["codes"], D, 4)
    s = np.repeat(e["scales"].view(np.float16).astype(np.float64), 32, axis=1)
    z32 = e["z"].astype(np.float32)
    assert np.all(np.abs(z32.astype(np.float64) - q * s) <= s / 2 * (1 + 1e-12))
    a7 = (np.abs(z32).reshape(n, -1, 32).max(axis=2) / np.float32(7)).astype(np.float64)
    fr, ex = np.frexp(a7)
    want = np.where(a7 > 0, np.ldexp(1.0, np.where(fr == 0.5, ex - 1, ex)), 0.0)
    np.testing.assert_array_equal(e["scales"].view(np.float16).astype(np.float64), want)
    # a power-of-two scale divides exactly: every code is rint(z / s), ties to even
    np.testing.assert_array_equal(q, np.where(s > 0, np.rint(z32.astype(np.float64) / np.where(s > 0, s, 1)), 0))


def test_latent_decode_factorises_through_fd():
    """Attention over rows m + fd(z) equals the factorised form the decode uses:
    logits q.m + (Wd^T q).z, output sum p m + Wd (sum p z), over the softmax weights p."""
    rng = np.random.default_rng(33)
    n, D, G, R, k = 300, 64, 3, 30, 3
    cK, cV = _coder(rng, D), _coder(rng, D)
    refs = oracle.bf16_round(rng.standard_normal((R, D)))
    idx = np.sort(np.stack([rng.choice(R, k, replace=False) for _ in range(n)]), axis=1).astype(np.uint16)
    xk, xv = _bf16_vals(rng, (n, D)), _bf16_vals(rng, (n, D))
    ek = oracle.encode_latent(xk, refs, idx, 4, cK)
    ev = oracle.encode_latent(xv, refs, idx, 4, cV)
    Kh = oracle.reconstruct_latent(refs, idx, ek["codes"], ek["scales"], 4, cK)
    Vh = oracle.reconstruct_latent(refs, idx, ev["codes"], ev["scales"], 4, cV)
    q = rng.standard_normal((G, D))
    got = oracle.attention(q, Kh, Vh)
    # factorised, in numpy
    rv = oracle.bf16_value(refs).astype(np.float64)
    m = np.stack([rv[idx[t]].astype(np.float32).sum(axis=0, dtype=np.float32) / np.float32(k) for t in range(n)])
    zk = _numpy_unpack(ek["codes"], D, 4) * np.repeat(ek["scales"].view(np.float16).astype(np.float64), 32, axis=1)
    zv = _numpy_unpack(ev["codes"], D, 4) * np.repeat(ev["scales"].view(np.float16).astype(np.float64), 32, axis=1)
    qp = q @ cK.Wd.astype(np.float64)                         # Wd^T q per head
    logits = (q @ m.astype(np.float64).T + qp @ zk.T) / np.sqrt(D)
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    want = p @ m.astype(np.float64) + (p @ zv) @ cV.Wd.astype(np.float64).T
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_latent_reconstruction_error_bound():
    """m + fd(z_hat) is within |Wd| (scale/2) of m + fd(z): the quantiser's bound through fd."""
    rng = np.random.default_rng(34)
    n, D, R, k = 200, 64, 16, 4
    c = _coder(rng, D)
    refs = oracle.bf16_round(rng.standard_normal((R, D)))
    idx = np.sort(np.stack([rng.choice(R, k, replace=False) for _ in range(n)]), axis=1).astype(np.uint16)
    x = _bf16_vals(rng, (n, D))
    e = oracle.encode_latent(x, refs, idx, 4, c)
    exact = oracle.reconstruct_latent(refs, idx, None, None, 0, c, z_exact=e["z"])
    quant = oracle.reconstruct_latent(refs, idx, e["codes"], e["scales"], 4, c)
    s = np.repeat(e["scales"].view(np.float16).astype(np.float64), 32, axis=1)
    bound = (s / 2 + np.abs(e["z"]) * 2 ** -23) @ np.abs(c.Wd.astype(np.float64)).T
    assert np.all(np.abs(quant - exact) <= bound * (1 + 1e-9) + 1e-12)
