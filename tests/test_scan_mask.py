"""The search scan's compare: the sign bit of fl(thr - t), with thr first turned from -0 into +0
(thr + 0), is set exactly when t > thr.  Checked here in IEEE binary32 arithmetic (numpy,
round to nearest, subnormals kept, as the kernel is built without flush-to-zero) on random
values and on the edge cases: equal values, signed zeros, subnormals, huge magnitudes,
neighbours one ulp apart and the -FLT_MAX fill of the empty threshold."""
import numpy as np

F32_MAX = np.float32(np.finfo(np.float32).max)
TINY = np.float32(np.finfo(np.float32).smallest_subnormal)


def _mask_bit(thr, t):
    thr = np.float32(thr) + np.float32(0.0)          # -0 -> +0
    with np.errstate(over="ignore"):                  # an overflow to -inf keeps the sign
        d = np.float32(thr - np.float32(t))
    return bool(np.signbit(d))


def _cases():
    vals = [0.0, -0.0, 1.0, -1.0, TINY, -TINY, 2 * TINY, np.float32(1e-38), np.float32(-1e-38), 1e30, -1e30,
            F32_MAX, -F32_MAX, np.float32(300.25), np.float32(-300.25)]
    out = []
    np_err = np.seterr(over="ignore")                 # the neighbours of +-FLT_MAX are +-inf (skipped)
    for a in vals:
        a = np.float32(a)
        for b in vals:
            out.append((a, np.float32(b)))
        out.append((a, np.nextafter(a, np.float32(np.inf), dtype=np.float32)))
        out.append((a, np.nextafter(a, np.float32(-np.inf), dtype=np.float32)))
        out.append((np.nextafter(a, np.float32(np.inf), dtype=np.float32), a))
    np.seterr(**np_err)
    return out


def test_sign_of_difference_is_the_compare_on_edge_cases():
    for thr, t in _cases():
        if not (np.isfinite(thr) and np.isfinite(t)):
            continue
        assert _mask_bit(thr, t) == bool(t > thr), (thr, t)


def test_sign_of_difference_is_the_compare_on_random_values():
    rng = np.random.default_rng(7)
    thr = (rng.standard_normal(200000) * rng.choice([1e-30, 1e-3, 1.0, 300.0, 1e20], 200000)).astype(np.float32)
    t = (thr + rng.standard_normal(200000).astype(np.float32) * np.abs(thr) * np.float32(1e-6)).astype(np.float32)
    t[::7] = thr[::7]                                  # exact ties
    thr0 = (thr + np.float32(0.0)).astype(np.float32)
    d = (thr0 - t).astype(np.float32)
    assert np.array_equal(np.signbit(d), t > thr)


def test_empty_threshold_passes_every_finite_value_but_the_fill():
    thr = -F32_MAX
    for t in [np.float32(-3.0e38), np.float32(0.0), np.float32(-0.0), F32_MAX, np.float32(1e-40)]:
        assert _mask_bit(thr, t) == bool(t > thr)
    assert not _mask_bit(thr, -F32_MAX)                # the masked columns' fill never passes
