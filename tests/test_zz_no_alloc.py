"""awq_scale_search_noalloc: the AWQ search for callers that cannot allocate device memory.

Some callers (an engine plugin that owns no device memory, a service under a fixed memory budget,
a path that must not trigger cudaMalloc's implicit synchronisation) cannot supply a workspace.
This entry point uses the library's built-in scratch array instead.  These tests call it through
the C ABI and compare it with awq_scale_search (caller-supplied workspace), twice in a row, since
the shared scratch keeps the previous call's contents.  The file sorts last so that a run that
stops at the first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from weight_only_int4_06_b200 import synth
from weight_only_int4_06_b200 import w4a16 as B

SCRATCH = 16 * 1024 * 1024  # W4_NOALLOC_SCRATCH_BYTES


def _raw_noalloc(Xd, Wd, n_alpha):
    T, K = Xd.shape
    N = Wd.shape[0]
    mse = torch.full((n_alpha,), float("nan"), dtype=torch.float64, device="cuda")
    best = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    best_s = torch.full((K,), float("nan"), dtype=torch.float32, device="cuda")
    st = B.lib().awq_scale_search_noalloc(
        ctypes.c_void_p(Xd.data_ptr()), T, ctypes.c_void_p(Wd.data_ptr()), N, K, 128, n_alpha,
        ctypes.c_void_p(mse.data_ptr()), ctypes.c_void_p(best.data_ptr()), ctypes.c_void_p(best_s.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, B.STATUS_NAMES.get(st, st)
    assert B.w4_check_device_status() == 0
    return mse.cpu().numpy(), int(best.cpu().item()), best_s.cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("T,K,N", [(512, 1024, 512), (4096, 2048, 2048)])
def test_noalloc_matches_workspace_entry_twice(T, K, N):
    X, W = synth.awq_case(T=T, K=K, N=N, case_id=61)
    Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda()
    assert B.awq_workspace_size(T, N, K) <= SCRATCH
    mse_ref, best_ref, s_ref = (t.cpu().numpy() for t in B.awq_scale_search(Xd, Wd, 20))
    best_ref = int(best_ref[0])
    for _ in range(2):  # the second call starts from the first call's leftover scratch contents
        mse, best, s = _raw_noalloc(Xd, Wd, 20)
        assert np.all(np.abs(mse - mse_ref) <= 1e-3 * mse_ref)
        assert best == best_ref
        assert np.array_equal(s, s_ref)


def test_noalloc_rejects_problems_beyond_the_scratch():
    """K = N = 4096 needs more than the 16 MiB scratch: rejected on the host, nothing enqueued."""
    n = ctypes.c_size_t(0)
    assert B.lib().awq_workspace_size(4096, 4096, 4096, 128, 20, ctypes.byref(n)) == 0
    assert n.value > SCRATCH
    P = ctypes.c_void_p(1 << 20)
    st = B.lib().awq_scale_search_noalloc(P, 4096, P, 4096, 4096, 128, 20, P, P, P, None)
    assert st == 5  # W4_ERR_WORKSPACE
