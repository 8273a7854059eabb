"""Pins for the oracle's GPTQ quantiser (CPU only), each against something other than the
oracle's own update formula: a Hessian that is exactly diagonal makes GPTQ plain RTN bit for bit;
the correction after the first column equals the least-squares solution from numpy.linalg.solve;
the first group's parameters are RTN's on the untouched weights; the output error on the
calibration data is below RTN's.

Page: "GPTQ, AWQ and the rules of post-training quantization", section "GPTQ: pay for the error
with the other weights" (quantise one weight at a time and adjust the remaining ones to
compensate, using the second-order information of the calibration activations).
"""
import numpy as np

from oracle import w4a16_oracle as O
from weight_only_int4_06_b200 import synth


def test_diagonal_hessian_is_plain_rtn():
    K, N = 256, 24
    W = (np.random.default_rng(1).standard_normal((N, K)) * 0.02).astype(np.float16)
    X = (np.eye(K) * 3.0).astype(np.float16)  # X^T X = 9 I exactly: nothing to compensate
    p, s, z, Wc = O.gptq_quantize(X, W)
    p0, s0, z0 = O.quantize_pack(W)
    assert np.array_equal(p, p0) and np.array_equal(z, z0)
    assert np.array_equal(s.view(np.uint16), s0.view(np.uint16))
    assert np.array_equal(Wc, W.astype(np.float64))


def test_first_column_correction_is_least_squares():
    """After column 0: the other columns minimise (w - w_hat)^T H (w - w_hat) with column 0 fixed,
    i.e. v = w_r + H_rr^-1 H_r0 (w_0 - w_hat_0), solved here directly."""
    X, W = synth.awq_case(T=300, K=128, N=16, case_id=81)
    damp = 0.01
    _, s, z, Wc = O.gptq_quantize(X, W, damp=damp, stop_after=1)
    X64 = X.astype(np.float64)
    H = X64.T @ X64
    H[np.diag_indices(128)] += damp * np.mean(np.diag(H))
    w = W.astype(np.float64)
    v0 = W[:, 0].astype(np.float32)
    sf = s[:, 0].astype(np.float32)
    q0 = np.clip(np.rint(v0 / sf) + z[:, 0], 0, 15)
    d0 = w[:, 0] - (q0 - z[:, 0]) * sf.astype(np.float64)
    corr = np.linalg.solve(H[1:, 1:], H[1:, :1])[:, 0]  # H_rr^-1 H_r0
    expect = w[:, 1:] + np.outer(d0, corr)
    assert np.allclose(Wc[:, 1:], expect, rtol=1e-9, atol=1e-12)
    assert np.array_equal(Wc[:, 0], w[:, 0])


def test_first_group_parameters_are_rtn_of_the_untouched_weights():
    X, W = synth.awq_case(T=200, K=384, N=16, case_id=82)
    _, s, z, _ = O.gptq_quantize(X, W)
    _, s0, z0 = O.quantize_rtn(W)
    assert np.array_equal(s[:, 0].view(np.uint16), s0[:, 0].view(np.uint16))
    assert np.array_equal(z[:, 0], z0[:, 0])


def test_output_error_below_rtn():
    for case in (83, 84, 85):
        X, W = synth.awq_case(T=512, K=384, N=32, case_id=case)
        p, s, z, _ = O.gptq_quantize(X, W)
        X64, W64 = X.astype(np.float64), W.astype(np.float64)
        e_gptq = np.sum((X64 @ (O.dequantize(p, s, z) - W64).T) ** 2)
        e_rtn = np.sum((X64 @ (O.dequantize(*O.quantize_pack(W)) - W64).T) ** 2)
        assert e_gptq < 0.9 * e_rtn, (case, e_gptq, e_rtn)


def test_codes_in_range_and_format():
    X, W = synth.awq_case(T=64, K=256, N=8, case_id=86)
    p, s, z, _ = O.gptq_quantize(X, W)
    q = O.unpack_nibbles(p)
    assert q.min() >= 0 and q.max() <= 15 and p.dtype == np.uint32 and p.shape == (8, 32)
    assert s.dtype == np.float16 and z.dtype == np.uint8 and z.max() <= 15


def test_later_group_parameters_come_from_the_corrected_weights():
    """Reading: a group's scale and zero point are RTN's rule applied to the group's weights as
    corrected by all earlier columns (not to the original weights)."""
    X, W = synth.awq_case(T=400, K=256, N=32, case_id=87)
    _, s, z, _ = O.gptq_quantize(X, W)
    _, _, _, Wc = O.gptq_quantize(X, W, stop_after=128)
    v = Wc[:, 128:].astype(np.float32)
    lo = np.minimum(v.min(axis=1), 0).astype(np.float32)
    hi = np.maximum(v.max(axis=1), 0).astype(np.float32)
    s_exact = O.fp16_round_up((hi - lo) / np.float32(15))
    assert np.array_equal(s[:, 1].view(np.uint16), s_exact.view(np.uint16))
    _, s_orig, _ = O.quantize_rtn(W)
    assert not np.array_equal(s[:, 1].view(np.uint16), s_orig[:, 1].view(np.uint16))
