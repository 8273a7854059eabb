"""The binding never computes on the host: host tensors, wrong dtypes and non-contiguous views are
rejected before any work, for every entry point (CPU only; the library is loaded, nothing runs)."""
import pytest
import torch

from weight_only_int4_06_b200 import w4a16 as B

H = torch.float16
W = torch.zeros(64, 256, dtype=H)
X = torch.zeros(4, 256, dtype=H)
P = torch.zeros(64, 32, dtype=torch.int32)
S = torch.zeros(64, 2, dtype=H)
Z = torch.zeros(64, 2, dtype=torch.uint8)

CALLS = {
    "w4_quantize_pack": lambda: B.w4_quantize_pack(W),
    "w4_quantize_pack_bits": lambda: B.w4_quantize_pack_bits(W, 3, 128),
    "w4_gemm": lambda: B.w4_gemm(X, P, S, Z),
    "wb_gemm": lambda: B.wb_gemm(X, torch.zeros(64, 24, dtype=torch.int32), S, Z, 3, 128),
    "w4_act_prepare": lambda: B.w4_act_prepare(X),
    "awq_scale_search": lambda: B.awq_scale_search(X, W, 4),
    "awq_scale_search_gram": lambda: B.awq_scale_search_gram(X, W, 4),
    "awq_clip_search": lambda: B.awq_clip_search(X, W),
    "awq_colsum": lambda: B.awq_colsum(X),
    "gptq_quantize": lambda: B.gptq_quantize(X, W),
    "gptq_quantize_ex": lambda: B.gptq_quantize_ex(X, W, 3, 128),
}


@pytest.mark.parametrize("name", sorted(CALLS))
def test_host_tensors_are_rejected(name):
    # w4_gemm accepts a host X (it copies it to the weights' device), so with host weights it
    # fails on the missing device instead of a type check: either way nothing is computed
    with pytest.raises((ValueError, TypeError, AssertionError, RuntimeError)):
        CALLS[name]()


def test_wrong_dtype_and_layout_are_rejected():
    with pytest.raises(TypeError):
        B.w4_quantize_pack(W.float())
    with pytest.raises(ValueError):
        B._dev(torch.zeros(8, 8, dtype=H).t(), H, "X")  # non-contiguous
