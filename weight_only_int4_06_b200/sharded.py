"""The AWQ scale search with the calibration rows split across ranks.

One process per GPU (torch.distributed; NCCL between GPUs), each holding a slice of the
calibration rows X_local and the whole weight matrix W.  The exchange follows the structure of
the search ("GPTQ, AWQ and the rules of post-training quantization", section "AWQ: find the one
percent that matters": the scales depend on the activations only through per-channel means, and
the error of each alpha is a sum over calibration rows):

    colsum  = all-reduce(sum) of every rank's exact integer column sums   (K int64, exact)
    T_total = all-reduce(sum) of the row counts
    s_all   = scales from colsum and T_total                             (identical on every rank)
    sse     = all-gather of every rank's per-alpha sums of squares        ([world, n_alpha] fp64)
    mse, best, best_s = the part-ordered sums / (T_total N), lowest argmin

All arithmetic runs in the library's kernels (awq_colsum, awq_scales_from_colsum, awq_sse,
awq_select); the collectives only move integers and per-rank partial sums.  Every rank takes the
same collective steps in the same order, including a rank that holds no rows.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class DeviceOps:
    """The library calls the search is built from (a test may substitute host stand-ins)."""

    def __init__(self):
        from . import w4a16 as B
        self.B = B

    def colsum(self, X):
        return self.B.awq_colsum(X)

    def scales(self, colsum, T_total, n_alpha):
        return self.B.awq_scales_from_colsum(colsum, T_total, n_alpha)

    def sse(self, X, W, s_all, group):
        return self.B.awq_sse(X, W, s_all, group)

    def select(self, sse_by_part, T_total, N, s_all):
        return self.B.awq_select(sse_by_part, T_total, N, s_all)


def awq_scale_search_sharded(X_local: torch.Tensor, W: torch.Tensor, n_alpha: int = 20, group: int = 128,
                             process_group=None, ops=None):
    """Returns (mse [n_alpha] fp64, best [1] int32, best_s [K] fp32) on every rank, equal (up to the
    association of fp64 sums) to awq_scale_search on the concatenation of all ranks' rows."""
    ops = ops or DeviceOps()
    T_local, K = X_local.shape
    N = W.shape[0]
    dev = W.device
    world = dist.get_world_size(process_group)
    if T_local > 0:
        colsum = ops.colsum(X_local)
    else:
        colsum = torch.zeros(K, dtype=torch.int64, device=dev)
    dist.all_reduce(colsum, op=dist.ReduceOp.SUM, group=process_group)
    t = torch.tensor([T_local], dtype=torch.int64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=process_group)
    T_total = int(t.item())
    if T_total < 1:
        raise ValueError("no calibration rows on any rank")
    s_all = ops.scales(colsum, T_total, n_alpha)
    if T_local > 0:
        sse = ops.sse(X_local, W, s_all, group)
    else:
        sse = torch.zeros(n_alpha, dtype=torch.float64, device=dev)
    parts = [torch.empty_like(sse) for _ in range(world)]
    dist.all_gather(parts, sse, group=process_group)
    return ops.select(torch.stack(parts), T_total, N, s_all)
