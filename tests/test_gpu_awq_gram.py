"""GPU parity of awq_scale_search_gram (the AWQ scale search through the Gram matrix X^T X)
against the CPU oracle, with the same bar as the direct form: per-alpha MSE within 1e-3 relative,
the same argmin (either index of an oracle near-tie within 2e-3), the exact scales; the 9000-row
case spans three chunks of the Gram accumulation with a ragged last one.  At the full calibration
size the two device forms are compared with each other (the oracle's direct product over 65536
rows is too slow): their MSEs agree within the same 1e-3 relative.

Page: "GPTQ, AWQ and the rules of post-training quantization", section "AWQ: find the one percent
that matters" (grid search of the exponent on the output error of the calibration activations)."""
import numpy as np
import pytest
import torch

import oracle
from weight_only_int4_06_b200 import synth
from weight_only_int4_06_b200 import w4a16 as B

pytestmark = pytest.mark.gpu


def run_gram(X, W, n_alpha=20):
    mse, best, s = B.awq_scale_search_gram(torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda(), n_alpha)
    assert B.w4_check_device_status() == 0
    return mse.cpu().numpy(), int(best.cpu().item()), s.cpu().numpy()


def check_against_oracle(X, W, n_alpha=20):
    mse_g, best_g, s_g = run_gram(X, W, n_alpha)
    mse_o, best_o, _, s_all = oracle.awq_scale_search(X, W, n_alpha)
    rel = np.abs(mse_g - mse_o) / mse_o
    assert np.all(rel <= 1e-3), f"max rel err {rel.max():.3g} at alpha {np.argmax(rel)}"
    order = np.argsort(mse_o, kind="stable")
    if n_alpha > 1 and (mse_o[order[1]] - mse_o[order[0]]) <= 2e-3 * mse_o[order[0]]:
        assert best_g in (int(order[0]), int(order[1]))
    else:
        assert best_g == best_o
    assert np.array_equal(s_g, s_all[best_g])


def test_gram_small():
    X, W = synth.awq_case(T=256, K=512, N=64)
    check_against_oracle(X, W)


@pytest.mark.parametrize("T,K,N,n_alpha", [(1, 128, 8, 1), (130, 256, 264, 3), (700, 384, 136, 20),
                                           (512, 1024, 512, 20), (9000, 256, 64, 5)])
def test_gram_ragged(T, K, N, n_alpha):
    X, W = synth.awq_case(T=T, K=K, N=N, case_id=52)
    check_against_oracle(X, W, n_alpha)


def test_gram_zero_channel():
    """A channel that is zero in every calibration row has G_kk = 0: its diagonal factor is 1 and
    its weights cannot change the output error."""
    X, W = synth.awq_case(T=300, K=256, N=64, case_id=53)
    X = X.copy()
    X[:, 7] = 0
    X[:, 200] = 0
    check_against_oracle(X, W, 10)


def test_gram_calibration_subsample_matches_oracle():
    X, W = synth.awq_case()
    rows = synth.awq_subsample_rows()
    check_against_oracle(np.ascontiguousarray(X[rows]), W)


def test_gram_full_size_agrees_with_direct_form():
    X, W = synth.awq_case()
    Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda()
    mse_g, best_g, s_g = B.awq_scale_search_gram(Xd, Wd)
    mse_d, best_d, s_d = B.awq_scale_search(Xd, Wd)
    assert B.w4_check_device_status() == 0
    mse_g, mse_d = mse_g.cpu().numpy(), mse_d.cpu().numpy()
    rel = np.abs(mse_g - mse_d) / mse_d
    print(f"gram vs direct, max rel diff of the MSEs: {rel.max():.3g}")
    assert np.all(rel <= 1e-3), f"max rel diff {rel.max():.3g}"
    bg, bd = int(best_g.item()), int(best_d.item())
    if bg != bd:  # only a near-tie may flip
        assert abs(mse_d[bg] - mse_d[bd]) <= 2e-3 * mse_d[bd]
    else:
        assert torch.equal(s_g, s_d)
    mse_g2, best_g2, _ = B.awq_scale_search_gram(Xd, Wd)
    assert np.array_equal(mse_g.view(np.uint64), mse_g2.cpu().numpy().view(np.uint64))  # deterministic
