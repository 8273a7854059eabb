"""The bounded waits on a GPU: a wait that nothing can satisfy gives up after its limit, the
device status reports W4_ERR_DEVICE_TIMEOUT, and the context stays usable (a quantise + GEMM right
after still matches the oracle)."""
import time

import numpy as np
import pytest
import torch

import oracle
from weight_only_int4_06_b200 import synth
from weight_only_int4_06_b200 import w4a16 as B

pytestmark = pytest.mark.gpu


def test_wait_without_arrival_times_out_and_the_context_survives():
    assert B.w4_check_device_status() == 0
    t0 = time.perf_counter()
    B.w4_selftest_bounded_wait(200_000_000)  # 0.2 s
    assert B.w4_check_device_status() == 7  # W4_ERR_DEVICE_TIMEOUT (reading it also clears it)
    assert 0.15 <= time.perf_counter() - t0 < 30.0
    assert B.w4_check_device_status() == 0
    X, W = synth.single_layer_case()
    p, s, z = B.w4_quantize_pack(torch.from_numpy(W).cuda())
    Y = B.w4_gemm(torch.from_numpy(X).cuda(), p, s, z).cpu().numpy().astype(np.float64)
    po, so, zo = oracle.quantize_pack(W)
    assert np.array_equal(p.cpu().numpy().view(np.uint32), po)
    Yref = oracle.gemm(X, po, so, zo)
    rms = np.sqrt(np.mean(Yref ** 2))
    assert np.all(np.abs(Y - Yref) <= 5e-3 * (np.abs(Yref) + rms))
    assert B.w4_check_device_status() == 0
