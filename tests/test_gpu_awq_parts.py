"""GPU check of the row-split AWQ search's library calls (awq_colsum, awq_scales_from_colsum,
awq_sse, awq_select) against awq_scale_search on all rows, with the parts emulated in one process
on one GPU (no kernel waits on another).  Column sums add exactly; the scales are bit-identical;
the MSEs differ only by the grouping of rows into fp32 tensor-core tiles (parts do not start on
tile boundaries), well inside 1e-5 relative."""
import numpy as np
import pytest
import torch

import oracle
from weight_only_int4_06_b200 import synth
from weight_only_int4_06_b200 import w4a16 as B

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,K,N,cuts", [(300, 256, 64, (0, 130, 130, 300)), (2000, 512, 136, (0, 777, 1500, 2000))])
def test_parts_equal_the_whole(T, K, N, cuts):
    X, W = synth.awq_case(T=T, K=K, N=N, case_id=43)
    Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda()
    parts = [Xd[a:b].contiguous() for a, b in zip(cuts[:-1], cuts[1:])]
    col = torch.zeros(K, dtype=torch.int64, device="cuda")
    for P in parts:
        col += B.awq_colsum(P) if P.shape[0] else 0
    assert torch.equal(col, B.awq_colsum(Xd))  # integers: exact in any order
    s_all = B.awq_scales_from_colsum(col, T, 20)
    sse = torch.stack([B.awq_sse(P, Wd, s_all) if P.shape[0] else torch.zeros(20, dtype=torch.float64, device="cuda")
                       for P in parts])
    mse, best, best_s = B.awq_select(sse, T, N, s_all)
    mse_w, best_w, s_w = B.awq_scale_search(Xd, Wd, 20)
    assert B.w4_check_device_status() == 0
    mse, mse_w = mse.cpu().numpy(), mse_w.cpu().numpy()
    assert np.all(np.abs(mse - mse_w) <= 1e-5 * mse_w)
    b, bw = int(best.item()), int(best_w.item())
    assert b == bw or abs(mse_w[b] - mse_w[bw]) <= 1e-4 * mse_w[bw]
    assert torch.equal(s_all[bw], s_w)
    _, best_o, _, s_o = oracle.awq_scale_search(X, W, 20)
    assert np.array_equal(s_all.cpu().numpy(), s_o)  # the scales are the oracle's, bit for bit
