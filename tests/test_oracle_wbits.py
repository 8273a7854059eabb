"""Pins for the oracle of other widths and column orders (CPU only): the 4-bit case against the
INT4 oracle, the bit streams against a bit-string construction and a hand-worked 3-bit example,
the quantiser against brute force and its error bound, GPTQ against the INT4 GPTQ, the RTN
special case and permutation invariance, and the act-order matmul against the g_idx form.

Pages: "AutoGPTQ vs The Stack v2" (2/3/4/8-bit GPTQ, per-group quantisation, desc_act);
"GPTQ, AWQ and the rules of post-training quantization" (INT3 g128 and INT2 g64 results)."""
import numpy as np
import pytest

from oracle import w4a16_oracle as O
from oracle import wbits_oracle as B
from weight_only_int4_06_b200 import synth


def _w(N, K, seed):
    return (np.random.default_rng(seed).standard_normal((N, K)) * 0.02).astype(np.float16)


def test_four_bits_is_the_int4_quantiser():
    W = _w(16, 384, 1)
    a = np.random.default_rng(2).uniform(0.5, 2.0, 384).astype(np.float32)
    for act in (None, a):
        q, s, z = B.quantize_rtn_bits(W, 4, 128, act)
        q0, s0, z0 = O.quantize_rtn(W, act)
        assert np.array_equal(q, q0) and np.array_equal(z, z0)
        assert np.array_equal(s.view(np.uint16), s0.view(np.uint16))
        assert np.array_equal(B.pack_bits(q, 4), O.pack_nibbles(q))


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_bits_matches_a_bit_string(bits):
    rng = np.random.default_rng(bits)
    K = 64
    q = rng.integers(0, 1 << bits, size=(3, K), dtype=np.uint8)
    p = B.pack_bits(q, bits)
    for n in range(3):
        stream = "".join(format(int(c), f"0{bits}b")[::-1] for c in q[n])  # stream bit j = stream[j]
        want = [int(stream[32 * w:32 * w + 32][::-1], 2) for w in range(K * bits // 32)]
        assert [int(x) for x in p[n]] == want
    assert np.array_equal(B.unpack_bits(p, bits, K), q)


def test_int3_worked_example():
    """Codes 0..7 repeated: every 8 codes are the 24-bit pattern octal 76543210 = 0xFAC688, so
    the 96-bit stream is that pattern at bits 0, 24, 48, 72 (worked by hand)."""
    q = (np.arange(32) % 8).astype(np.uint8)[None, :]
    assert [hex(int(x)) for x in B.pack_bits(q, 3)[0]] == ["0x88fac688", "0xc688fac6", "0xfac688fa"]


@pytest.mark.parametrize("bits,group", [(2, 64), (3, 128), (8, 128), (2, 128)])
def test_quantiser_bound_and_ranges(bits, group):
    L = (1 << bits) - 1
    W = _w(32, 512, 10 + bits)
    q, s, z = B.quantize_rtn_bits(W, bits, group)
    assert q.max() <= L and z.max() <= L
    v = W.astype(np.float64)
    w_hat = B.dequantize_bits(B.pack_bits(q, bits), s, z, bits, group, 512)
    bound = np.repeat(s.astype(np.float64), group, axis=1) / 2
    assert np.all(np.abs(v - w_hat) <= bound * (1 + 1e-6))


@pytest.mark.parametrize("bits", [2, 3])
def test_codes_are_the_nearest_level(bits):
    L = (1 << bits) - 1
    W = _w(8, 128, 20 + bits)
    q, s, z = B.quantize_rtn_bits(W, bits, 64)
    v = W.astype(np.float64)
    sf = np.repeat(s.astype(np.float64), 64, axis=1)
    zf = np.repeat(z.astype(np.float64), 64, axis=1)
    cand = np.arange(L + 1, dtype=np.float64)[None, None, :]
    dist = np.abs(v[:, :, None] - (cand - zf[:, :, None]) * sf[:, :, None])
    chosen = np.abs(v - (q.astype(np.float64) - zf) * sf)
    assert np.allclose(chosen, dist.min(axis=2), rtol=0, atol=1e-12)


def test_values_on_the_grid_are_reproduced():
    """A 2-bit group whose values are (q - 1) * 2^-6 for q in 0..3 spans exactly 3 steps: the
    scale is 2^-6, the zero point 1 and every value comes back exactly."""
    levels = (np.arange(64) % 4 - 1) * 2.0 ** -6
    W = levels.astype(np.float16)[None, :]
    q, s, z = B.quantize_rtn_bits(W, 2, 64)
    assert float(s[0, 0]) == 2.0 ** -6 and int(z[0, 0]) == 1
    assert np.array_equal(B.dequantize_bits(B.pack_bits(q, 2), s, z, 2, 64, 64)[0], levels)


def test_gptq_four_bits_natural_order_is_the_int4_gptq():
    X, W = synth.awq_case(T=300, K=256, N=24, case_id=61)
    p, s, z, perm = B.gptq_quantize_bits(X, W, 4, 128)
    p0, s0, z0, _ = O.gptq_quantize(X, W)
    assert np.array_equal(perm, np.arange(256))
    assert np.array_equal(p, p0) and np.array_equal(z, z0)
    assert np.array_equal(s.view(np.uint16), s0.view(np.uint16))


@pytest.mark.parametrize("bits,group", [(2, 64), (3, 128)])
def test_gptq_diagonal_hessian_is_rtn(bits, group):
    K, N = 256, 16
    W = _w(N, K, 30 + bits)
    X = (np.eye(K) * 3.0).astype(np.float16)
    p, s, z, _ = B.gptq_quantize_bits(X, W, bits, group)
    p0, s0, z0 = B.quantize_pack_bits(W, bits, group)
    assert np.array_equal(p, p0) and np.array_equal(z, z0)
    assert np.array_equal(s.view(np.uint16), s0.view(np.uint16))


def test_act_order_with_sorted_diagonal_is_natural_order():
    X, W = synth.awq_case(T=400, K=256, N=16, case_id=62)
    d = np.einsum("tk,tk->k", X.astype(np.float64), X.astype(np.float64))
    order = np.argsort(-d, kind="stable")
    Xs, Ws = np.ascontiguousarray(X[:, order]), np.ascontiguousarray(W[:, order])  # diagonal now decreasing
    a = B.gptq_quantize_bits(Xs, Ws, 3, 128, act_order=True)
    b = B.gptq_quantize_bits(Xs, Ws, 3, 128, act_order=False)
    assert np.array_equal(a[3], np.arange(256))
    for u, v in zip(a[:3], b[:3]):
        assert np.array_equal(u.view(np.uint8), v.view(np.uint8))


def test_act_order_is_invariant_to_the_input_column_order():
    X, W = synth.awq_case(T=400, K=256, N=16, case_id=63)
    pi = np.random.default_rng(5).permutation(256)
    a = B.gptq_quantize_bits(X, W, 4, 128, act_order=True)
    b = B.gptq_quantize_bits(np.ascontiguousarray(X[:, pi]), np.ascontiguousarray(W[:, pi]), 4, 128, act_order=True)
    for u, v in zip(a[:3], b[:3]):
        assert np.array_equal(u.view(np.uint8), v.view(np.uint8))
    assert np.array_equal(pi[b[3]], a[3])  # the same original columns, processed in the same order


def test_act_order_matmul_equals_the_g_idx_form():
    X, W = synth.awq_case(T=200, K=384, N=24, case_id=64)
    p, s, z, perm = B.gptq_quantize_bits(X, W, 4, 128, act_order=True)
    Y = B.gemm_act_order(X[:8], p, s, z, perm, 4, 128)
    q_orig = np.empty((24, 384), dtype=np.uint8)
    q_orig[:, perm] = B.unpack_bits(p, 4, 384)
    Wd = B.dequantize_g_idx(q_orig, s, z, B.g_idx_from_perm(perm, 128))
    assert np.allclose(Y, X[:8].astype(np.float64) @ Wd.T, rtol=1e-12, atol=1e-12)
    assert not np.array_equal(perm, np.arange(384))  # the case really reorders


@pytest.mark.parametrize("bits,group", [(4, 128), (3, 128), (2, 64)])
def test_gptq_output_error_far_below_rtn_on_correlated_activations(bits, group):
    """With correlated channels the compensation pays: the output error on the calibration data
    drops several-fold against RTN at every width, in either column order (measured 0.05-0.10)."""
    X, W = synth.correlated_case(T=512, K=384, N=32, case_id=65)
    X64, W64 = X.astype(np.float64), W.astype(np.float64)
    pr, sr, zr = B.quantize_pack_bits(W, bits, group)
    e_r = np.sum((B.gemm_bits(X, pr, sr, zr, bits, group) - X64 @ W64.T) ** 2)
    for act_order in (False, True):
        p, s, z, perm = B.gptq_quantize_bits(X, W, bits, group, act_order=act_order)
        e_g = np.sum((B.gemm_act_order(X, p, s, z, perm, bits, group) - X64 @ W64.T) ** 2)
        assert e_g < 0.3 * e_r, (act_order, e_g, e_r)


def test_scaled_activations():
    X = (np.random.default_rng(3).standard_normal((4, 256))).astype(np.float16)
    assert np.array_equal(B.scale_activations(X, np.ones(256, np.float32)).view(np.uint16), X.view(np.uint16))
    s = np.float32(2.0) ** np.random.default_rng(4).integers(-3, 4, 256).astype(np.float32)
    want = (X.astype(np.float64) / s.astype(np.float64)).astype(np.float16)  # exact: powers of two
    assert np.array_equal(B.scale_activations(X, s).view(np.uint16), want.view(np.uint16))


def test_all_zero_group_any_width():
    for bits, group in ((2, 64), (3, 128), (8, 64)):
        q, s, z = B.quantize_rtn_bits(np.zeros((1, 2 * group), np.float16), bits, group)
        assert np.all(s == 1.0) and not z.any() and not q.any()


def test_act_order_ties_keep_index_order():
    """Channels in pairs of equal energy (exact copies): ties are broken by the lower index."""
    rng = np.random.default_rng(9)
    base = rng.standard_normal((40, 8)).astype(np.float16)
    X = np.ascontiguousarray(base[:, np.arange(256) % 8])  # column k copies column k % 8
    perm = B.act_order_perm(X)
    d = np.einsum("tk,tk->k", X.astype(np.float64), X.astype(np.float64))
    for i in range(255):
        a, b = perm[i], perm[i + 1]
        assert d[a] > d[b] or (d[a] == d[b] and a < b)


def _fp32_rn(f):
    """The fp32 value nearest to the rational f (ties to even), by exact comparison."""
    from fractions import Fraction
    c = np.float32(float(f))
    cands = [c, np.nextafter(c, np.float32(np.inf)), np.nextafter(c, np.float32(-np.inf))]
    best = min(cands, key=lambda v: (abs(Fraction(float(v)) - f), int(np.float32(v).view(np.uint32)) & 1))
    return np.float32(best)


def test_scaled_activations_are_one_division_then_fp16():
    """fp16(RN32(x / s)) with the quotient rounded once, checked with exact rationals on a random
    block and on elements chosen where multiplying by a rounded reciprocal would give another
    fp16 value (so a two-rounding implementation cannot pass)."""
    from fractions import Fraction
    rng = np.random.default_rng(12)
    X = (rng.standard_normal((40, 512)) * 3).astype(np.float16)
    s = rng.uniform(0.3, 7.0, 512).astype(np.float32)
    cases = [(X[m, k], s[k]) for m in range(0, 40, 4) for k in range(0, 512, 4)]
    xs = (rng.standard_normal(400000) * 3).astype(np.float16)
    ss = rng.uniform(0.3, 7.0, 400000).astype(np.float32)
    x32 = xs.astype(np.float32)
    hard = np.nonzero((x32 / ss).astype(np.float16) != (x32 * (np.float32(1) / ss)).astype(np.float16))[0][:64]
    assert len(hard) >= 8
    cases += [(xs[i], ss[i]) for i in hard]
    xa = np.array([c[0] for c in cases], np.float16)[None, :]
    sa = np.array([c[1] for c in cases], np.float32)
    got = B.scale_activations(xa, sa)[0]
    for i, (x, sv) in enumerate(cases):
        want = np.float16(_fp32_rn(Fraction(float(x)) / Fraction(float(sv))))
        assert got[i].view(np.uint16) == want.view(np.uint16), (float(x), float(sv))


def test_gptq_act_scale_of_ones_changes_nothing():
    X, W = synth.correlated_case(T=300, K=256, N=16, case_id=66)
    a = B.gptq_quantize_bits(X, W, 3, 128, act_order=True)
    b = B.gptq_quantize_bits(X, W, 3, 128, act_order=True, act_scale=np.ones(256, np.float32))
    for u, v in zip(a, b):
        assert np.array_equal(np.asarray(u).view(np.uint8), np.asarray(v).view(np.uint8))


def test_gptq_uniform_power_of_two_act_scale_scales_only_the_scales():
    """s = 4 everywhere: X / 4 and W * 4 are exact, every later step scales exactly by a power of two,
    so the codes, zero points and order are unchanged and each fp16 scale is exactly 4 times larger."""
    X, W = synth.correlated_case(T=300, K=256, N=16, case_id=67)
    p, s, z, perm = B.gptq_quantize_bits(X, W, 2, 64, act_order=True)
    p4, s4, z4, perm4 = B.gptq_quantize_bits(X, W, 2, 64, act_order=True, act_scale=np.full(256, 4.0, np.float32))
    assert np.array_equal(p, p4) and np.array_equal(z, z4) and np.array_equal(perm, perm4)
    assert np.array_equal(s4.astype(np.float64), 4.0 * s.astype(np.float64))
