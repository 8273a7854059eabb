"""Pins for the oracle's AWQ clip search (CPU only), each against something other than the
oracle's own formula: exact rational arithmetic for the clipped scale and codes, pure-Python
brute force for the error, the unclipped quantiser as the one-ratio special case, and
invariances of the output error.

The pages name activation-guided clipping without giving its grid; the reading (shrink ratios
r_j = 1 - j/20 applied to both ends of the zero-inclusive range, per-group output error) is the
one stated in the oracle's docstring.
"""
import bisect
from fractions import Fraction

import numpy as np

from oracle import w4a16_oracle as O


def _fp16_grid():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16)
    return sorted({Fraction(float(v)) for v in vals[np.isfinite(vals)]})


_GRID = _fp16_grid()


def _fp16_ru(x: float) -> Fraction:
    i = bisect.bisect_left(_GRID, Fraction(x))
    return _GRID[i]


def _case(seed, T, N, K, outlier=True):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((T, K)).astype(np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    if outlier:  # a few large weights make clipping worthwhile
        W[rng.integers(0, N, 4), rng.integers(0, K, 4)] *= 12
    return X.astype(np.float16), W.astype(np.float16)


def test_ratio_grid_reading():
    r = O.clip_ratio_grid(10)
    assert r.dtype == np.float32 and r[0] == 1.0 and len(r) == 10
    assert np.array_equal(r, np.float32([1.0, 0.95, 0.9, 0.85, 0.8, 0.75, 0.7, 0.65, 0.6, 0.55]))


def test_one_ratio_is_plain_rtn():
    X, W = _case(1, 32, 8, 256)
    a = np.exp(np.random.default_rng(2).standard_normal(256) * 0.5).astype(np.float32)
    for act in (None, a):
        err, best, p, s, z = O.awq_clip_search(X, W, act, n_ratios=1)
        p0, s0, z0 = O.quantize_pack(W, act)
        assert (best == 0).all()
        assert np.array_equal(p, p0) and np.array_equal(s.view(np.uint16), s0.view(np.uint16))
        assert np.array_equal(z, z0)


def test_clipped_scale_and_codes_exact():
    """Clipped range: lo' = RN32(r lo), hi' = RN32(r hi); s16 = smallest fp16 >= RN32(RN32(hi'-lo')/15);
    every code is the nearest of the 16 levels (saturating beyond the shrunk range)."""
    _, W = _case(3, 4, 6, 256)
    r = np.float32(0.7)
    q, s, z = O.quantize_rtn(W, None, 128, np.full((6, 2), r, np.float32))
    v = W.astype(np.float32)
    for n in range(6):
        for g in range(2):
            blk = v[n, 128 * g:128 * g + 128]
            lo = np.float32(r * np.float32(min(0.0, float(blk.min()))))
            hi = np.float32(r * np.float32(max(0.0, float(blk.max()))))
            s32 = np.float32(np.float32(hi - lo) / np.float32(15))
            assert Fraction(float(s[n, g])) == _fp16_ru(float(s32))
            S, Z = Fraction(float(s[n, g])), int(z[n, g])
            assert abs(-Fraction(float(lo)) / S - Z) <= Fraction(1, 2) + Fraction(1, 1 << 18)
            for k in range(128 * g, 128 * g + 128):
                V = Fraction(float(v[n, k]))
                d = [abs(V - (lv - Z) * S) for lv in range(16)]
                assert d[int(q[n, k])] - min(d) <= S * Fraction(1, 1 << 20), (n, k)


def test_error_brute_force():
    """err[n, g, j] against explicit loops over t and k (pure Python floats)."""
    T, N, K, R = 5, 3, 256, 4
    X, W = _case(4, T, N, K)
    a = np.exp(np.random.default_rng(5).standard_normal(K) * 0.3).astype(np.float32)
    err, best, _, _, _ = O.awq_clip_search(X, W, a, n_ratios=R)
    v = W.astype(np.float32) * a[None, :]
    for j, r in enumerate(O.clip_ratio_grid(R)):
        q, s, z = O.quantize_rtn(W, a, 128, np.full((N, 2), r, np.float32))
        for n in range(N):
            for g in range(2):
                tot = 0.0
                for t in range(T):
                    acc = 0.0
                    for k in range(128 * g, 128 * g + 128):
                        w_hat = (int(q[n, k]) - int(z[n, g])) * float(s[n, g])
                        acc += float(X[t, k]) / float(a[k]) * (w_hat - float(v[n, k]))
                    tot += acc * acc
                assert abs(tot - err[n, g, j]) <= 1e-9 * max(tot, 1e-30), (n, g, j)
    for n in range(N):
        for g in range(2):
            e = err[n, g]
            assert best[n, g] == min(i for i in range(R) if e[i] == e.min())


def test_final_codes_use_each_groups_best_ratio():
    X, W = _case(6, 48, 8, 384)
    err, best, p, s, z = O.awq_clip_search(X, W, n_ratios=6)
    r = O.clip_ratio_grid(6)[best]
    q, s2, z2 = O.quantize_rtn(W, None, 128, r)
    assert np.array_equal(p, O.pack_nibbles(q)) and np.array_equal(z, z2)
    assert np.array_equal(s.view(np.uint16), s2.view(np.uint16))
    assert (best > 0).any()  # the outliers make clipping pay somewhere


def test_error_invariances():
    """Scaling X by 2 scales every error by 4 (a square); permuting the channels inside a group
    (X columns with W columns) changes nothing; both keep the choice."""
    X, W = _case(7, 24, 6, 256)
    err, best, p, _, _ = O.awq_clip_search(X, W, n_ratios=5)
    X2 = (X.astype(np.float32) * 2).astype(np.float16)
    err2, best2, p2, _, _ = O.awq_clip_search(X2, W, n_ratios=5)
    assert np.allclose(err2, 4 * err, rtol=1e-12, atol=0) and np.array_equal(best, best2)
    perm = np.concatenate([np.random.default_rng(8).permutation(128) + 128 * g for g in range(2)])
    err3, best3, _, _, _ = O.awq_clip_search(X[:, perm], W[:, perm], n_ratios=5)
    assert np.allclose(err3, err, rtol=1e-10, atol=1e-30) and np.array_equal(best, best3)


def test_zero_activation_channel_makes_its_weight_free():
    """A weight whose input channel is always zero contributes nothing to the error, so when a
    huge weight there alone sets the range, shrinking the range only refines the step for the
    other weights: the error falls by a large factor and the choice lies in the strongly
    clipped half of the grid (not necessarily its end: rounding makes the error ragged)."""
    T, K = 64, 128
    rng = np.random.default_rng(9)
    X = rng.standard_normal((T, K)).astype(np.float16)
    X[:, 5] = 0
    W = (rng.uniform(-1, 1, (1, K)) * 0.02).astype(np.float16)
    W[0, 5] = np.float16(0.5)
    err, best, _, _, _ = O.awq_clip_search(X, W, n_ratios=10)
    assert err[0, 0, -1] < 0.5 * err[0, 0, 0]
    assert best[0, 0] >= 5
