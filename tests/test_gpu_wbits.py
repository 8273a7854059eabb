"""GPU parity of the other widths and column orders against the oracle (oracle/wbits_oracle.py):
b-bit quantise-and-pack bit for bit, the b-bit matmul within the GEMM tolerance, activation
preparation (act-order gather, activation-side scale) bit for bit, GPTQ at other widths and in
act-order with the same near-tie rule as the INT4 GPTQ parity tests, and act-order weights served
end to end.

Pages: "AutoGPTQ vs The Stack v2" (2/3/4/8-bit GPTQ, per-group quantisation, desc_act); "GPTQ, AWQ
and the rules of post-training quantization" (INT3 g128, INT2 g64)."""
import numpy as np
import pytest
import torch

from oracle import w4a16_oracle as O
from oracle import wbits_oracle as OB
from weight_only_int4_06_b200 import synth
from weight_only_int4_06_b200 import w4a16 as B

pytestmark = pytest.mark.gpu

WIDTHS = [(2, 64), (2, 128), (3, 64), (3, 128), (4, 64), (4, 128), (8, 64), (8, 128)]


def _u32(t):
    return t.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("bits,group", WIDTHS)
@pytest.mark.parametrize("N,K", [(8, 128), (24, 384), (136, 1152)])
def test_quantize_pack_bits_bit_exact(bits, group, N, K):
    X, W = synth.layer_case(71, 1, K, N)
    a = np.random.default_rng(bits * 1000 + K).uniform(0.25, 4.0, K).astype(np.float32)
    for act in (None, a):
        p, s, z = B.w4_quantize_pack_bits(torch.from_numpy(W).cuda(), bits, group,
                                          torch.from_numpy(act).cuda() if act is not None else None)
        assert B.w4_check_device_status() == 0
        po, so, zo = OB.quantize_pack_bits(W, bits, group, act)
        assert np.array_equal(_u32(p), po)
        assert np.array_equal(s.cpu().numpy().view(np.uint16), so.view(np.uint16))
        assert np.array_equal(z.cpu().numpy(), zo)


def test_four_bit_group_128_is_w4_quantize_pack():
    _, W = synth.layer_case(72, 1, 1024, 264)
    Wd = torch.from_numpy(W).cuda()
    p, s, z = B.w4_quantize_pack_bits(Wd, 4, 128)
    p0, s0, z0 = B.w4_quantize_pack(Wd)
    assert torch.equal(p, p0) and torch.equal(s, s0) and torch.equal(z, z0)


def _check_gemm(Y, Yref):
    rms = np.sqrt(np.mean(Yref ** 2))
    err = np.abs(Y.astype(np.float64) - Yref)
    assert np.all(err <= 5e-3 * (np.abs(Yref) + rms)), float((err / (np.abs(Yref) + rms)).max())


@pytest.mark.parametrize("bits,group", [(2, 64), (3, 128), (8, 128), (4, 64)])
@pytest.mark.parametrize("M,K,N", [(1, 128, 8), (7, 384, 136), (130, 1152, 264)])
def test_wb_gemm_matches_oracle(bits, group, M, K, N):
    X, W = synth.layer_case(73, M, K, N)
    p, s, z = OB.quantize_pack_bits(W, bits, group)
    Y = B.wb_gemm(torch.from_numpy(X).cuda(), torch.from_numpy(p.view(np.int32)).cuda(), torch.from_numpy(s).cuda(),
                  torch.from_numpy(z).cuda(), bits, group)
    assert B.w4_check_device_status() == 0
    _check_gemm(Y.cpu().numpy(), OB.gemm_bits(X, p, s, z, bits, group))


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("M,K,N", [(130, 192, 136), (40, 320, 264)])
def test_wb_gemm_odd_multiple_of_64(bits, M, K, N):
    """Group 64 with K an odd multiple of 64: the tensor-core GEMM's last k-block is a half group."""
    test_wb_gemm_matches_oracle(bits, 64, M, K, N)


def test_act_prepare_bit_exact():
    X, _ = synth.layer_case(74, 5, 384, 8)
    rng = np.random.default_rng(74)
    perm = rng.permutation(384).astype(np.int32)
    s = rng.uniform(0.1, 10.0, 384).astype(np.float32)
    Xd = torch.from_numpy(X).cuda()
    pd, sd = torch.from_numpy(perm).cuda(), torch.from_numpy(s).cuda()
    g = B.w4_act_prepare(Xd, pd).cpu().numpy()
    assert np.array_equal(g.view(np.uint16), np.ascontiguousarray(X[:, perm]).view(np.uint16))
    g = B.w4_act_prepare(Xd, None, sd).cpu().numpy()
    assert np.array_equal(g.view(np.uint16), OB.scale_activations(X, s).view(np.uint16))
    g = B.w4_act_prepare(Xd, pd, sd).cpu().numpy()
    assert np.array_equal(g.view(np.uint16), np.ascontiguousarray(OB.scale_activations(X, s)[:, perm]).view(np.uint16))
    assert B.w4_check_device_status() == 0


def test_act_prepare_rejects_a_perm_entry_out_of_range():
    X, _ = synth.layer_case(75, 2, 128, 8)
    perm = np.arange(128, dtype=np.int32)
    perm[17] = 128 + 5  # outside [0, K): the kernel's own bounds check turns it into a status
    g = B.w4_act_prepare(torch.from_numpy(X).cuda(), torch.from_numpy(perm).cuda()).cpu().numpy()
    assert B.w4_check_device_status() == 8  # W4_ERR_RANGE
    assert np.all(g[:, 17] == 0) and np.array_equal(g[:, :17], X[:, :17])


def _margin(X, W_row, bits, group, damp, act_order, k_first, act_scale=None):
    """Distance of the oracle's decision at processing column k_first (or at its group's scale and
    zero point) from a rounding boundary, in units of a step."""
    L = (1 << bits) - 1
    g0 = (k_first // group) * group
    Wc, _ = OB.gptq_state_bits(X, W_row, bits, group, damp, act_order, g0, act_scale)
    v = Wc[0, g0:g0 + group].astype(np.float32)
    lo, hi = min(np.float32(0), v.min()), max(np.float32(0), v.max())
    s32 = (hi - lo) / np.float32(L)
    s16 = O.fp16_round_up(np.array([s32], np.float32))[0]
    below = np.nextafter(np.float16(s16), np.float16(0))
    m = [abs(float(s32) - float(below)) / float(s16), abs(abs(float(-lo / np.float32(s16)) % 1.0) - 0.5)]
    Wc, _ = OB.gptq_state_bits(X, W_row, bits, group, damp, act_order, k_first, act_scale)
    x = np.float32(Wc[0, k_first]) / np.float32(s16)
    m.append(abs(abs(float(x) % 1.0) - 0.5))
    return min(m)


def _check_gptq(X, W, bits, group, act_order, damp=0.01, act_scale=None):
    sd = torch.from_numpy(act_scale).cuda() if act_scale is not None else None
    p, s, z, perm = B.gptq_quantize_ex(torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda(), bits, group, damp,
                                       act_order, act_scale=sd)
    assert B.w4_check_device_status() == 0
    po, so, zo, permo = OB.gptq_quantize_bits(X, W, bits, group, damp, act_order, act_scale)
    K = W.shape[1]
    if act_order:
        assert np.array_equal(perm.cpu().numpy(), permo.astype(np.int32))
    q, qo = OB.unpack_bits(_u32(p), bits, K), OB.unpack_bits(po, bits, K)
    s_, z_ = s.cpu().numpy(), z.cpu().numpy()
    bad = np.nonzero(np.any(q != qo, axis=1) | np.any(s_.view(np.uint16) != so.view(np.uint16), axis=1)
                     | np.any(z_ != zo, axis=1))[0]
    assert len(bad) <= max(1, len(W) // 100), f"{len(bad)} of {len(W)} rows differ"
    for n in bad:
        cols = np.nonzero(q[n] != qo[n])[0]
        grp = np.nonzero((s_[n].view(np.uint16) != so[n].view(np.uint16)) | (z_[n] != zo[n]))[0]
        firsts = ([int(cols[0])] if len(cols) else []) + ([int(grp[0]) * group] if len(grp) else [])
        k_first = min(firsts)
        mg = _margin(X, W[n:n + 1], bits, group, damp, act_order, k_first, act_scale)
        assert mg < 1e-6, f"row {n} differs at processing column {k_first}, margin {mg:.3g}"
    return p, s, z, perm


@pytest.mark.parametrize("bits,group", [(2, 64), (3, 128), (4, 64), (8, 128)])
@pytest.mark.parametrize("act_order", [False, True])
def test_gptq_widths_and_orders_match_oracle(bits, group, act_order):
    X, W = synth.correlated_case(T=600, K=384, N=40, case_id=76)
    _check_gptq(X, W, bits, group, act_order)


def test_gptq_four_bit_natural_ex_equals_gptq_quantize():
    X, W = synth.correlated_case(T=300, K=256, N=16, case_id=77)
    Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda()
    a = B.gptq_quantize(Xd, Wd)
    b = B.gptq_quantize_ex(Xd, Wd, 4, 128, 0.01, False)
    for u, v in zip(a, b[:3]):
        assert torch.equal(u, v)


def test_act_order_weights_served_end_to_end():
    """4-bit group-128 act-order GPTQ output is w4_gemm's format: prepare the activations with perm,
    then the fused GEMM (decode and prefill shapes)."""
    X, W = synth.correlated_case(T=512, K=512, N=264, case_id=78)
    p, s, z, perm = _check_gptq(X, W, 4, 128, True)
    for M in (1, 8, 200):
        Xm = X[:M]
        Xp = B.w4_act_prepare(torch.from_numpy(Xm).cuda(), perm)
        Y = B.w4_gemm(Xp, p, s, z).cpu().numpy()
        Yref = OB.gemm_act_order(Xm, _u32(p), s.cpu().numpy(), z.cpu().numpy(), perm.cpu().numpy(), 4, 128)
        _check_gemm(Y, Yref)


def test_int3_gptq_served_by_wb_gemm():
    X, W = synth.correlated_case(T=512, K=384, N=64, case_id=79)
    p, s, z, _ = _check_gptq(X, W, 3, 128, False)
    Y = B.wb_gemm(torch.from_numpy(X[:16]).cuda(), p, s, z, 3, 128).cpu().numpy()
    _check_gemm(Y, OB.gemm_bits(X[:16], _u32(p), s.cpu().numpy(), z.cpu().numpy(), 3, 128))


@pytest.mark.parametrize("bits,group,act_order", [(2, 64, False), (4, 128, True)])
def test_gptq_after_awq_scaling_matches_oracle(bits, group, act_order):
    """AWQ's per-channel scale first, then GPTQ on X / s and W * s; served as (X / s) dequant(W)^T."""
    X, W = synth.correlated_case(T=600, K=384, N=40, case_id=80)
    a = np.random.default_rng(80).uniform(0.5, 2.0, 384).astype(np.float32)
    p, s, z, perm = _check_gptq(X, W, bits, group, act_order, act_scale=a)
    if bits == 4 and group == 128:
        Xp = B.w4_act_prepare(torch.from_numpy(X[:8]).cuda(), perm, torch.from_numpy(a).cuda())
        Y = B.w4_gemm(Xp, p, s, z).cpu().numpy()
        Xs = OB.scale_activations(X[:8], a)
        Yref = OB.gemm_act_order(Xs, _u32(p), s.cpu().numpy(), z.cpu().numpy(), perm.cpu().numpy(), 4, 128)
        _check_gemm(Y, Yref)


@pytest.mark.parametrize("bits,group", WIDTHS)
@pytest.mark.parametrize("M,K,N", [(1, 4096, 1032), (3, 11008, 264), (8, 1024, 136)])
def test_wb_gemm_decode_sizes_match_oracle(bits, group, M, K, N):
    """Decode-sized M takes the fused b-bit GEMV (bit stream read once, codes dequantised in
    registers, fp32 sums); same tolerance as every GEMM."""
    X, W = synth.layer_case(81, M, K, N)
    p, s, z = OB.quantize_pack_bits(W, bits, group)
    Y = B.wb_gemm(torch.from_numpy(X).cuda(), torch.from_numpy(p.view(np.int32)).cuda(), torch.from_numpy(s).cuda(),
                  torch.from_numpy(z).cuda(), bits, group)
    assert B.w4_check_device_status() == 0
    _check_gemm(Y.cpu().numpy(), OB.gemm_bits(X, p, s, z, bits, group))
