"""GPU parity: w4_quantize_pack bit-exact against the CPU oracle, w4_gemm within
|Y - Y_ref| <= 5e-3 (|Y_ref| + rms(Y_ref)) elementwise, on the workloads' seeded inputs.

Every input and expected value comes from the seeded generators and the oracle; the GEMM
tests feed the library the oracle's own packed weights."""
import hashlib

import numpy as np
import pytest
import torch

import oracle
from weight_only_int4_06_b200 import synth
from weight_only_int4_06_b200 import w4a16 as B

pytestmark = pytest.mark.gpu

TOL = 5e-3


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_quant(W, act=None):
    a = None if act is None else dev(np.asarray(act, np.float32))
    p, s, z = B.w4_quantize_pack(dev(W), a)
    st = B.w4_check_device_status()
    return p.cpu().numpy().view(np.uint32), s.cpu().numpy(), z.cpu().numpy(), st


def assert_quant_equal(W, act=None):
    p, s, z, st = gpu_quant(W, act)
    assert st == 0, B.STATUS_NAMES[st]
    po, so, zo = oracle.quantize_pack(W, act)
    assert np.array_equal(s.view(np.uint16), so.view(np.uint16)), "scales differ"
    assert np.array_equal(z, zo), "zeros differ"
    assert np.array_equal(p, po), "packed codes differ"
    return p, s, z


def gpu_gemm(X, packed, scales, zeros, variant=B.VARIANT_AUTO):
    Y = B.w4_gemm(dev(X), dev(packed.view(np.int32)), dev(scales), dev(zeros), variant=variant)
    assert B.w4_check_device_status() == 0
    return Y.cpu().numpy()


def assert_close(Y, Yref, what=""):
    Y = Y.astype(np.float64)
    rms = float(np.sqrt(np.mean(Yref ** 2))) if Yref.size else 0.0
    err = np.abs(Y - Yref)
    bound = TOL * (np.abs(Yref) + rms)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {err.size} outside tolerance; worst at {i}: "
                             f"got {Y[i]}, ref {Yref[i]}, bound {bound[i]}")
    assert np.isfinite(Y).all()


# ------------------------------------------------------------------ quantiser
def test_quant_single_layer_matches_oracle_and_golden():
    _, W = synth.single_layer_case()
    p, s, z = assert_quant_equal(W)
    golden = {}
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "single_layer_seed0.txt")
    for line in open(path):
        if "=" in line and not line.startswith("#"):
            k, v = line.split("=", 1)
            golden[k.strip()] = v.strip()
    assert hashlib.sha256(p.astype("<u4").tobytes()).hexdigest() == golden["packed_sha256"]
    assert hashlib.sha256(s.astype("<f2").tobytes()).hexdigest() == golden["scales_sha256"]
    assert hashlib.sha256(z.tobytes()).hexdigest() == golden["zeros_sha256"]


@pytest.mark.parametrize("N,K", [(8, 128), (24, 384), (40, 1152), (16, 11008), (264, 512)])
def test_quant_ragged_shapes(N, K):
    X, W = synth.layer_case(11, 1, K, N)
    assert_quant_equal(W)
    act = np.exp(np.random.default_rng([N, K]).standard_normal(K)).astype(np.float32)
    assert_quant_equal(W, act)


def test_quant_special_groups():
    K = 512
    W = np.zeros((16, K), np.float16)
    W[1, :] = 0.5                                   # constant group rows
    W[2, :] = np.abs(synth.layer_case(12, 1, K, 16)[1][2])    # all >= 0
    W[3, :] = -np.abs(synth.layer_case(12, 1, K, 16)[1][3])   # all <= 0
    W[4, 37] = 0.75                                 # single nonzero
    W[5, 300] = -0.75
    W[6, :] = ((np.arange(K) % 128 - 64) / 64.0).astype(np.float16)  # ramps
    W[7, :] = np.float16(1e-7)                      # subnormal-size values
    W[8, ::2] = np.float16(60000.0)                 # near the top of the fp16 range
    W[8, 1::2] = np.float16(-60000.0)
    assert_quant_equal(W)


def test_quant_range_overflow_is_reported():
    W = np.zeros((8, 128), np.float16)
    W[0, 0], W[0, 1] = 60000.0, -60000.0
    _, _, _, st = gpu_quant(W, np.full(128, 16.0, np.float32))
    assert st == 8  # W4_ERR_RANGE
    assert B.w4_check_device_status() == 0  # cleared by the read
    with pytest.raises(oracle.QuantRangeError):
        oracle.quantize_pack(W, np.full(128, 16.0, np.float32))


def test_quant_exact_midpoints():
    """Elements exactly at (n + 1/2) s16 (ties, rounded half to even) and one fp16 ulp either side."""
    rows = []
    for s in (0.0625, 0.046875, 0.001953125, 3.0, 0.75):
        for sign in (1.0, -1.0):
            base = np.array([15 * s] + [(n + 0.5) * s for n in range(15)] + [0.0], np.float64) * sign
            h = base.astype(np.float16)
            assert np.all(h.astype(np.float64) == base)   # exactly representable
            up = np.nextafter(h, np.float16(np.inf))
            dn = np.nextafter(h, np.float16(-np.inf))
            vals = np.concatenate([h, up[1:16], dn[1:16]])
            row = np.zeros(128, np.float16)
            row[:vals.size] = vals
            rows.append(row)
    W = np.stack(rows)
    W = np.concatenate([W, np.zeros(((-len(W)) % 8, 128), np.float16)])
    assert_quant_equal(W)


def test_quant_wide_act_scale_sweep():
    """16.7M quotients with fp32 activation scales spanning 2^-10 .. 2^10."""
    _, W = synth.layer_case(13, 1, 4096, 4096)
    act = np.exp2(np.random.default_rng(13).uniform(-10, 10, 4096)).astype(np.float32)
    assert_quant_equal(W, act)


@pytest.mark.parametrize("K,N", list(synth.DECODE_7B_SHAPES) + [(28672, 8192)])
def test_quant_full_size(K, N):
    _, W = synth.layer_case(2, 1, K, N)
    assert_quant_equal(W)


# ------------------------------------------------------------------ gemm
def oracle_case(case_id, M, K, N):
    X, W = synth.layer_case(case_id, M, K, N)
    p, s, z = oracle.quantize_pack(W)
    return X, p, s, z


def test_gemm_single_layer():
    X, W = synth.single_layer_case()
    p, s, z = oracle.quantize_pack(W)
    Y = gpu_gemm(X, p, s, z)
    assert_close(Y, oracle.gemm(X, p, s, z), "512x512")


@pytest.mark.parametrize("M", [1, 2, 3, 5, 7, 8, 9, 13, 16, 17, 24, 31, 32, 33, 40])
def test_gemm_m_sweep_ragged(M):
    X, p, s, z = oracle_case(21, M, 384, 136)
    assert_close(gpu_gemm(X, p, s, z), oracle.gemm(X, p, s, z), f"M={M}")


@pytest.mark.parametrize("K,N", [(128, 8), (128, 520), (1152, 264), (4096, 136), (11008, 40),
                                 (28672, 16), (2048, 4096)])
@pytest.mark.parametrize("M", [1, 4, 16, 32])
def test_gemm_split_shapes(M, K, N):
    X, p, s, z = oracle_case(22, M, K, N)
    assert_close(gpu_gemm(X, p, s, z, B.VARIANT_SKINNY), oracle.gemm(X, p, s, z), f"{M}x{K}x{N}")


@pytest.mark.parametrize("K,N", synth.DECODE_7B_SHAPES)
def test_gemm_decode_7b_full(K, N):
    X, p, s, z = oracle_case(2, 1, K, N)
    assert_close(gpu_gemm(X, p, s, z), oracle.gemm(X, p, s, z), f"decode {K}x{N}")


@pytest.mark.parametrize("K,N", synth.SMALL_BATCH_70B_SHAPES)
def test_gemm_small_batch_70b_full(K, N):
    for M in synth.SMALL_BATCH_MS:
        X, p, s, z = oracle_case(3, M, K, N)
        assert_close(gpu_gemm(X, p, s, z), oracle.gemm(X, p, s, z), f"M={M} {K}x{N}")


@pytest.mark.parametrize("M", synth.PREFILL_MS)
@pytest.mark.parametrize("K,N", synth.PREFILL_SHAPES)
def test_gemm_prefill_sampled(M, K, N):
    X, p, s, z = oracle_case(4, M, K, N)
    Y = gpu_gemm(X, p, s, z)
    r = np.random.default_rng([M, K, N])
    rows = np.concatenate([r.integers(0, M, 1500), [0, M - 1, M - 1]])
    cols = np.concatenate([r.integers(0, N, 1500), [0, N - 1, 0]])
    ref = oracle.gemm_entries(X, p, s, z, rows, cols)
    # tolerance uses the rms of the sampled reference values
    assert_close(Y[rows, cols], ref, f"prefill M={M} {K}x{N}")


def test_gemm_deterministic():
    X, p, s, z = oracle_case(23, 16, 8192, 1024)
    Y1 = gpu_gemm(X, p, s, z)
    Y2 = gpu_gemm(X, p, s, z)
    assert np.array_equal(Y1.view(np.uint16), Y2.view(np.uint16))


def test_gemm_empty_and_k0():
    Y = torch.full((3, 16), 7.0, dtype=torch.float16, device="cuda")
    X = torch.zeros((3, 0), dtype=torch.float16, device="cuda")
    p = torch.zeros((16, 0), dtype=torch.int32, device="cuda")
    s = torch.zeros((16, 0), dtype=torch.float16, device="cuda")
    z = torch.zeros((16, 0), dtype=torch.uint8, device="cuda")
    B.w4_gemm(X, p, s, z, out=Y)
    torch.cuda.synchronize()
    assert torch.all(Y == 0)
    X = torch.zeros((0, 128), dtype=torch.float16, device="cuda")
    p = torch.zeros((16, 16), dtype=torch.int32, device="cuda")
    s = torch.zeros((16, 1), dtype=torch.float16, device="cuda")
    z = torch.zeros((16, 1), dtype=torch.uint8, device="cuda")
    assert B.w4_gemm(X, p, s, z).shape == (0, 16)


def test_gemm_host_buffers_match_device():
    X, p, s, z = oracle_case(24, 1, 4096, 4096)
    Yd = gpu_gemm(X, p, s, z)
    Xh = torch.from_numpy(X).pin_memory()
    Yh = B.w4_gemm(Xh, dev(p.view(np.int32)), dev(s), dev(z))
    assert not Yh.is_cuda
    assert np.array_equal(Yh.numpy().view(np.uint16), Yd.view(np.uint16))


def test_gemm_async_pinned_host_out_on_a_side_stream():
    """Pinned host X and out: copies and kernel are enqueued on the given stream, no sync."""
    X, p, s, z = oracle_case(26, 3, 4096, 1032)
    Yd = gpu_gemm(X, p, s, z)
    Xh = torch.from_numpy(X).pin_memory()
    out = torch.full((3, 1032), 7.0, dtype=torch.float16).pin_memory()
    side = torch.cuda.Stream()
    r = B.w4_gemm(Xh, dev(p.view(np.int32)), dev(s), dev(z), out=out, stream=side)
    assert r is out
    side.synchronize()
    assert np.array_equal(out.numpy().view(np.uint16), Yd.view(np.uint16))
    with pytest.raises(ValueError):  # a pageable host out is refused
        B.w4_gemm(Xh, dev(p.view(np.int32)), dev(s), dev(z), out=torch.empty((3, 1032), dtype=torch.float16))


def test_gemm_host_entry_point_one_call():
    """w4_gemm_host: H2D of X, the GEMM and D2H of Y enqueued by one C call on a side stream."""
    X, p, s, z = oracle_case(28, 5, 1152, 520)
    Yd = gpu_gemm(X, p, s, z)
    Xh = torch.from_numpy(X).pin_memory()
    out = torch.zeros((5, 520), dtype=torch.float16).pin_memory()
    xs = torch.empty((5, 1152), dtype=torch.float16, device="cuda")
    ys = torch.empty((5, 520), dtype=torch.float16, device="cuda")
    side = torch.cuda.Stream()
    B.w4_gemm_host(Xh, dev(p.view(np.int32)), dev(s), dev(z), out, xs, ys, stream=side)
    side.synchronize()
    assert np.array_equal(out.numpy().view(np.uint16), Yd.view(np.uint16))
    assert_close(out.numpy(), oracle.gemm(X, p, s, z), "w4_gemm_host")


def test_gemm_misaligned_metadata_falls_back_or_reports():
    """The GEMV bulk-copies metadata and needs 16-byte aligned scales/zeros: w4_gemm falls back to
    the skinny kernel, the explicit GEMV family reports W4_ERR_ALIGN."""
    X, p, s, z = oracle_case(27, 1, 4096, 264)
    ref = oracle.gemm(X, p, s, z)
    sbuf = torch.zeros(s.size + 8, dtype=torch.float16, device="cuda")
    zbuf = torch.zeros(z.size + 16, dtype=torch.uint8, device="cuda")
    s_mis = sbuf[1:1 + s.size].view(s.shape)
    z_mis = zbuf[3:3 + z.size].view(z.shape)
    s_mis.copy_(dev(s))
    z_mis.copy_(dev(z))
    Xd, pd = dev(X), dev(p.view(np.int32))
    Y = B.w4_gemm(Xd, pd, s_mis, z_mis)
    assert_close(Y.cpu().numpy(), ref, "auto with misaligned metadata")
    with pytest.raises(B.W4Error) as e:
        B.w4_gemm(Xd, pd, s_mis, z_mis, variant=B.VARIANT_GEMV)
    assert e.value.status == 3  # W4_ERR_ALIGN


# ------------------------------------------------------------------ forced kernel families
@pytest.mark.parametrize("M,K,N", [(1, 128, 8), (7, 256, 136), (128, 384, 256), (129, 4096, 264),
                                   (300, 1152, 520), (512, 8192, 1024), (64, 11008, 4096)])
def test_gemm_tc_ragged(M, K, N):
    X, p, s, z = oracle_case(25, M, K, N)
    assert_close(gpu_gemm(X, p, s, z, B.VARIANT_TC), oracle.gemm(X, p, s, z), f"tc {M}x{K}x{N}")


@pytest.mark.parametrize("M,K,N", [(1, 128, 8), (1, 384, 24), (1, 1152, 136), (1, 4096, 4104),
                                   (1, 11008, 40), (1, 28672, 264), (3, 2048, 520), (1, 8192, 28672),
                                   # full-SM shapes with 3 and 2 ring stages (larger staged activations)
                                   (4, 8192, 264), (8, 4096, 1032), (3, 16384, 136), (5, 8192, 520),
                                   (2, 28672, 72), (8, 8192, 264), (7, 8192, 136),
                                   # K cut into slices: one stage each (the last one partial), two
                                   # stages each, seven; half tiles (N % 16 == 8)
                                   (8, 6144, 264), (8, 10240, 1032), (3, 16384, 136), (6, 28672, 520),
                                   (1, 28672, 4104),
                                   # 16-row launches: one slice (Y written directly), slices of 2048,
                                   # 3 slices with a ragged N, 14 slices; 16 + 8 and 16 + 16 rows
                                   (16, 2048, 520), (9, 4096, 264), (13, 6144, 1032), (16, 28672, 136),
                                   (24, 8192, 264), (32, 4096, 136), (12, 1536, 136)])
def test_gemm_gemv_ragged(M, K, N):
    X, p, s, z = oracle_case(28, M, K, N)
    assert_close(gpu_gemm(X, p, s, z, B.VARIANT_GEMV), oracle.gemm(X, p, s, z), f"gemv {M}x{K}x{N}")


@pytest.mark.parametrize("M,K,N", [(1, 128, 8), (1, 384, 24), (1, 1152, 136), (1, 4096, 4104),
                                   (1, 11008, 40), (2, 2048, 520), (5, 4096, 264), (8, 1536, 1032),
                                   (1, 4096, 12288), (1, 11008, 4096), (12, 512, 136)])
def test_gemm_gemv_tc_ragged(M, K, N):
    X, p, s, z = oracle_case(30, M, K, N)
    assert_close(gpu_gemm(X, p, s, z, B.VARIANT_GEMV_TC), oracle.gemm(X, p, s, z), f"gemv_tc {M}x{K}x{N}")


def test_gemm_gemv_tc_outlier_heavy_activations():
    X, p, s, z = oracle_case(31, 3, 4096, 1024)
    X = (X.astype(np.float32) * 40).astype(np.float16)
    assert_close(gpu_gemm(X, p, s, z, B.VARIANT_GEMV_TC), oracle.gemm(X, p, s, z), "gemv_tc x40")


def test_gemm_gemv_outlier_heavy_activations():
    """Large activations stress the offset removal (raw operands carry a 1024 offset)."""
    X, p, s, z = oracle_case(29, 1, 4096, 1024)
    X = (X.astype(np.float32) * 40).astype(np.float16)
    assert_close(gpu_gemm(X, p, s, z, B.VARIANT_GEMV), oracle.gemm(X, p, s, z), "gemv x40")


@pytest.mark.parametrize("M,K,N", [(1, 4096, 4096), (8, 8192, 1024), (32, 28672, 256)])
def test_gemm_weights_static_flag_same_bits(M, K, N):
    """The static-weights launch (programmatic dependent launch) computes the same bits."""
    X, p, s, z = oracle_case(26, M, K, N)
    Y0 = gpu_gemm(X, p, s, z, B.VARIANT_AUTO)
    Y1 = gpu_gemm(X, p, s, z, B.VARIANT_AUTO | B.FLAG_WEIGHTS_STATIC)
    assert np.array_equal(Y0.view(np.uint16), Y1.view(np.uint16))


def test_gemm_tc_tail_split_ragged():
    """Full waves of 256 x 256 tiles in one launch, the last partial wave's tiles cut along K (4
    slices here) with their partials summed per tile: ragged M and N tiles included."""
    M, K, N = 2000, 2048, 5000  # 8 x 20 = 160 tiles on 148 SMs: 12 tail tiles
    assert B.w4_gemm_plan(M, N, K) == (B.VARIANT_TC, 3)
    X, p, s, z = oracle_case(32, M, K, N)
    Y1 = gpu_gemm(X, p, s, z)
    assert_close(Y1, oracle.gemm(X, p, s, z), f"tail split {M}x{K}x{N}")
    assert np.array_equal(Y1.view(np.uint16), gpu_gemm(X, p, s, z).view(np.uint16))  # deterministic


def test_gemm_tc_deterministic():
    X, p, s, z = oracle_case(27, 1024, 4096, 2048)
    Y1 = gpu_gemm(X, p, s, z, B.VARIANT_TC)
    Y2 = gpu_gemm(X, p, s, z, B.VARIANT_TC)
    assert np.array_equal(Y1.view(np.uint16), Y2.view(np.uint16))
