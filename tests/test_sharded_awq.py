"""The row-split AWQ search's host orchestration on CPU: two and three gloo ranks on 127.0.0.1,
each holding a slice of the calibration rows (one rank holds none in the three-rank case).

The per-part arithmetic is the library's on a GPU; here host stand-ins written from the oracle
take its place (exact column sums, the oracle's scales, the literal per-row squared errors, the
part-ordered sum and lowest argmin), so what is checked is the exchange: integer all-reduce of
the column sums and row counts, gather of the per-part sums in rank order, normalisation by the
total row count.  The result must equal the oracle's search on all rows."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
T, K, N, N_ALPHA = 90, 256, 16, 6


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _HostOps:
    def __init__(self, O):
        self.O = O

    def colsum(self, X):
        units = (np.abs(X.numpy().astype(np.float64)) * 2.0 ** 24).astype(np.int64)
        return torch.from_numpy(units.sum(axis=0))

    def scales(self, colsum, T_total, n_alpha):
        m = colsum.numpy().astype(np.float64) * 2.0 ** -24 / T_total
        return torch.from_numpy(np.stack([self.O.awq_scales(m, i / n_alpha).astype(np.float32)
                                          for i in range(n_alpha)]))

    def sse(self, X, W, s_all, group):
        X64 = X.numpy().astype(np.float64)
        W16 = W.numpy()
        ref = X64 @ W16.astype(np.float64).T
        out = []
        for s32 in s_all.numpy():
            q, s16, z = self.O.quantize_rtn(W16, s32, group)
            Wq = self.O.dequantize(self.O.pack_nibbles(q), s16, z, group)
            out.append(np.sum(((X64 / s32.astype(np.float64)) @ Wq.T - ref) ** 2))
        return torch.tensor(out, dtype=torch.float64)

    def select(self, sse_by_part, T_total, N, s_all):
        tot = np.zeros(sse_by_part.shape[1])
        for p in range(sse_by_part.shape[0]):  # part order
            tot = tot + sse_by_part[p].numpy()
        mse = tot / (T_total * N)
        b = int(np.argmin(mse))
        return torch.from_numpy(mse), torch.tensor([b], dtype=torch.int32), s_all[b].clone()


def _case(synth):
    """Channel 3 is zero in every row, so its mean is floored (1e-6) and the scales depend on the
    total row count (elsewhere the normalisation cancels any common factor of the means)."""
    X, W = synth.awq_case(T=T, K=K, N=N, case_id=41)
    X = X.copy()
    X[:, 3] = 0
    return X, W


def _rows(rank, world):
    if world == 3:
        return [(0, 50), (50, 50), (50, T)][rank]  # rank 1 holds no rows
    return [(0, 37), (37, T)][rank]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from oracle import w4a16_oracle as O
    from weight_only_int4_06_b200 import synth
    from weight_only_int4_06_b200.sharded import awq_scale_search_sharded
    dist.init_process_group("gloo", rank=rank, world_size=world)
    X, W = _case(synth)
    a, b = _rows(rank, world)
    mse, best, s = awq_scale_search_sharded(torch.from_numpy(np.ascontiguousarray(X[a:b])), torch.from_numpy(W),
                                            N_ALPHA, ops=_HostOps(O))
    q.put((rank, mse.numpy(), int(best.item()), s.numpy()))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_row_split_search_equals_the_oracle(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    from oracle import w4a16_oracle as O
    from weight_only_int4_06_b200 import synth
    X, W = _case(synth)
    mse_o, best_o, s_o, _ = O.awq_scale_search(X, W, N_ALPHA)
    for rank, mse, best, s in got:
        assert np.allclose(mse, mse_o, rtol=1e-12, atol=0), rank
        assert best == best_o and np.array_equal(s, s_o), rank
