"""More GPU parity cases for validated calls at shapes the other files do not reach, and the
prepared host call.

Pages: "GPTQ, AWQ and the rules of post-training quantization", section "AWQ: find the one percent
that matters" (the scale search); "AutoAWQ vs The Stack v2" (the W4A16 matmul)."""
import numpy as np
import pytest
import torch

import oracle
from weight_only_int4_06_b200 import synth
from weight_only_int4_06_b200 import w4a16 as B

pytestmark = pytest.mark.gpu


def test_gram_form_search_at_the_down_projection_width():
    """K = 11008 (86 groups; the Gram GEMMs' N = K is not a multiple of the 256-wide tile)."""
    X, W = synth.awq_case(T=2048, K=11008, N=264, case_id=44)
    mse, best, s = B.awq_scale_search_gram(torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda(), 5)
    assert B.w4_check_device_status() == 0
    mse_o, best_o, _, s_all = oracle.awq_scale_search(X, W, 5)
    mse = mse.cpu().numpy()
    assert np.all(np.abs(mse - mse_o) <= 1e-3 * mse_o)
    b = int(best.item())
    order = np.argsort(mse_o, kind="stable")
    if (mse_o[order[1]] - mse_o[order[0]]) <= 2e-3 * mse_o[order[0]]:
        assert b in (int(order[0]), int(order[1]))
    else:
        assert b == best_o
    assert np.array_equal(s.cpu().numpy(), s_all[b])


def test_prepared_host_call_matches_w4_gemm():
    X, W = synth.layer_case(45, 1, 4096, 11008)
    p, s, z = B.w4_quantize_pack(torch.from_numpy(W).cuda())
    Xh = torch.from_numpy(X).pin_memory()
    out = torch.empty((1, 11008), dtype=torch.float16).pin_memory()
    xd = torch.empty((1, 4096), dtype=torch.float16, device="cuda")
    yd = torch.empty((1, 11008), dtype=torch.float16, device="cuda")
    call = B.HostGemmCall(Xh, p, s, z, out, xd, yd)
    for _ in range(3):
        call.run()
    torch.cuda.current_stream().synchronize()
    ref = B.w4_gemm(torch.from_numpy(X).cuda(), p, s, z).cpu()
    assert torch.equal(out, ref)  # same kernel, same inputs: same bits
    Xh.copy_(torch.from_numpy(X[:, ::-1].copy()))  # new contents in the same buffer
    call.run()
    torch.cuda.current_stream().synchronize()
    ref2 = B.w4_gemm(torch.from_numpy(X[:, ::-1].copy()).cuda(), p, s, z).cpu()
    assert torch.equal(out, ref2)
    assert B.w4_check_device_status() == 0


def test_host_batch_matches_per_layer_gemm():
    """w4_gemm_host_batch (one copy in, the layers' GEMMs, one copy out) gives every layer the bits
    w4_gemm gives it, twice in a row with new inputs in the same buffers."""
    shapes = [(1, 4096, 4096), (1, 4096, 12288), (5, 1152, 520), (1, 11008, 4096), (40, 512, 264)]
    weights, Xs = [], []
    for i, (M, K, N) in enumerate(shapes):
        X, W = synth.layer_case(46 + i, M, K, N)
        weights.append(B.w4_quantize_pack(torch.from_numpy(W).cuda()))
        Xs.append(X)
    batch = B.HostGemmBatch(weights, shapes)
    for rep in range(2):
        for i, X in enumerate(Xs):
            batch.x(i).copy_(torch.from_numpy(X if rep == 0 else X[:, ::-1].copy()))
        batch.run()
        torch.cuda.current_stream().synchronize()
        for i, X in enumerate(Xs):
            Xi = X if rep == 0 else X[:, ::-1].copy()
            ref = B.w4_gemm(torch.from_numpy(Xi).cuda(), *weights[i]).cpu()
            assert torch.equal(batch.y(i), ref), (rep, shapes[i])
    assert B.w4_check_device_status() == 0


def test_host_batch_graph_replay_matches():
    """The batch call captured as a CUDA graph gives the same bits as the direct call, with new
    inputs written into the same host buffer between replays."""
    shapes = [(1, 4096, 4096), (3, 1152, 520)]
    weights, Xs = [], []
    for i, (M, K, N) in enumerate(shapes):
        X, W = synth.layer_case(52 + i, M, K, N)
        weights.append(B.w4_quantize_pack(torch.from_numpy(W).cuda()))
        Xs.append(X)
    batch = B.HostGemmBatch(weights, shapes)
    g = batch.capture()
    for rep in range(2):
        for i, X in enumerate(Xs):
            batch.x(i).copy_(torch.from_numpy(X if rep == 0 else -X))
        g.replay()
        torch.cuda.current_stream().synchronize()
        for i, X in enumerate(Xs):
            ref = B.w4_gemm(torch.from_numpy(X if rep == 0 else -X).cuda(), *weights[i]).cpu()
            assert torch.equal(batch.y(i), ref), (rep, shapes[i])
    assert B.w4_check_device_status() == 0


@pytest.mark.parametrize("pinned", [False, True])
def test_host_batch_pageable_and_ragged_buffers(pinned):
    """Host buffers the SMs cannot address (pageable), or whose sizes are not 16-byte multiples,
    go through the copy engines; pinned 16-byte multiples through the SM copies: same bits."""
    import ctypes
    shapes = [(1, 1152, 520), (3, 512, 136)]  # 2304 + 3072 bytes of X: y_bytes 1040 + 816 = 1856
    weights, Xs = [], []
    for i, (M, K, N) in enumerate(shapes):
        X, W = synth.layer_case(58 + i, M, K, N)
        weights.append(B.w4_quantize_pack(torch.from_numpy(W).cuda()))
        Xs.append(X)
    x_off = [0, 2304]
    y_off = [0, 1040]
    x_bytes, y_bytes = 2304 + 3072, 1040 + 816 + 8  # y_bytes not a multiple of 16
    xh = torch.zeros(x_bytes, dtype=torch.uint8)
    yh = torch.zeros(y_bytes, dtype=torch.uint8)
    if pinned:
        xh, yh = xh.pin_memory(), yh.pin_memory()
    for i, X in enumerate(Xs):
        xh[x_off[i]:x_off[i] + X.nbytes].copy_(torch.from_numpy(X.view(np.uint8).reshape(-1)))
    xd = torch.empty(x_bytes, dtype=torch.uint8, device="cuda")
    yd = torch.empty(y_bytes, dtype=torch.uint8, device="cuda")
    arr = (B.GemmLayer * 2)()
    for i, ((p, s, z), (M, K, N)) in enumerate(zip(weights, shapes)):
        arr[i] = B.GemmLayer(M, N, K, p.data_ptr(), s.data_ptr(), z.data_ptr(), x_off[i], y_off[i])
    st = B.lib().w4_gemm_host_batch(ctypes.cast(arr, ctypes.c_void_p), 2, 128, ctypes.c_void_p(xh.data_ptr()),
                                    ctypes.c_void_p(xd.data_ptr()), ctypes.c_size_t(x_bytes),
                                    ctypes.c_void_p(yh.data_ptr()), ctypes.c_void_p(yd.data_ptr()),
                                    ctypes.c_size_t(y_bytes), None, ctypes.c_size_t(0), 0,
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.current_stream().synchronize()
    for i, (M, K, N) in enumerate(shapes):
        got = yh[y_off[i]:y_off[i] + 2 * M * N].view(torch.float16).view(M, N)
        ref = B.w4_gemm(torch.from_numpy(Xs[i]).cuda(), *weights[i]).cpu()
        assert torch.equal(got, ref), shapes[i]
    assert B.w4_check_device_status() == 0
