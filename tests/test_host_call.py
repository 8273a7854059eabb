"""HostGemmCall marshals exactly the arguments w4_gemm_host passes (host logic only: the C library
is replaced by a recorder, device tensors by host tensors)."""
import ctypes

import pytest
import torch

from weight_only_int4_06_b200 import w4a16 as B


def _plain(a):
    if a is None:
        return None
    if isinstance(a, ctypes.c_void_p):
        return a.value
    if isinstance(a, ctypes._SimpleCData):
        return a.value
    return a


class _Recorder:
    def __init__(self):
        self.calls = []

    def w4_gemm_host(self, *args):
        self.calls.append(tuple(_plain(a) for a in args))
        return 0


@pytest.fixture
def fake(monkeypatch):
    rec = _Recorder()
    monkeypatch.setattr(B, "lib", lambda: rec)
    monkeypatch.setattr(B, "_dev", lambda t, dtype, name: ctypes.c_void_p(t.data_ptr()))
    monkeypatch.setattr(B, "_stream", lambda s: ctypes.c_void_p(1234))
    monkeypatch.setattr(B, "_ws_size", lambda M, N, K, g: 0)
    return rec


def test_prepared_call_passes_the_same_arguments(fake):
    M, K, N = 2, 256, 64
    X = torch.zeros(M, K, dtype=torch.float16)
    out = torch.zeros(M, N, dtype=torch.float16)
    packed = torch.zeros(N, K // 8, dtype=torch.int32)
    scales = torch.zeros(N, K // 128, dtype=torch.float16)
    zeros = torch.zeros(N, K // 128, dtype=torch.uint8)
    xd = torch.zeros(M, K, dtype=torch.float16)
    yd = torch.zeros(M, N, dtype=torch.float16)
    ws = torch.zeros(64, dtype=torch.uint8)
    B.w4_gemm_host(X, packed, scales, zeros, out, xd, yd, workspace=ws, variant=3)
    call = B.HostGemmCall(X, packed, scales, zeros, out, xd, yd, workspace=ws, variant=3)
    assert call.run() is out
    call.run()
    assert len(fake.calls) == 3
    assert fake.calls[0] == fake.calls[1] == fake.calls[2]
    B.w4_gemm_host(X, packed, scales, zeros, out, xd, yd)
    B.HostGemmCall(X, packed, scales, zeros, out, xd, yd).run()
    assert fake.calls[3] == fake.calls[4] and fake.calls[3][11] is None  # no workspace


def test_prepared_call_validates_once(fake):
    X = torch.zeros(2, 256, dtype=torch.float16)
    with pytest.raises(ValueError):
        B.HostGemmCall(X, torch.zeros(64, 32, dtype=torch.int32), torch.zeros(64, 2, dtype=torch.float16),
                       torch.zeros(64, 2, dtype=torch.uint8), torch.zeros(2, 63, dtype=torch.float16),
                       torch.zeros(2, 256, dtype=torch.float16), torch.zeros(2, 64, dtype=torch.float16))
    assert fake.calls == []


def test_prepared_call_raises_on_a_status(fake, monkeypatch):
    monkeypatch.setattr(fake, "w4_gemm_host", lambda *a: 2)
    X = torch.zeros(1, 128, dtype=torch.float16)
    call = B.HostGemmCall(X, torch.zeros(8, 16, dtype=torch.int32), torch.zeros(8, 1, dtype=torch.float16),
                          torch.zeros(8, 1, dtype=torch.uint8), torch.zeros(1, 8, dtype=torch.float16),
                          torch.zeros(1, 128, dtype=torch.float16), torch.zeros(1, 8, dtype=torch.float16))
    with pytest.raises(B.W4Error):
        call.run()
