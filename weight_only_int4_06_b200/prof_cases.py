"""Small, self-checking workloads for ncu captures of single kernels (profiles/ cites these).

    python -m weight_only_int4_06_b200.prof_cases decode-layer N K [n_launch] [variant]
        one decode layer (M = 1) through w4_gemm, n_launch launches over 8 rotating weight sets
        (random packed codes, scales and zero points: the GEMV's work does not depend on values),
        so a capture that skips the first launches sees weights that are not L2-resident
    python -m weight_only_int4_06_b200.prof_cases clip T K N
        awq_clip_search twice on a seeded calibration-like layer (10 ratios)
    python -m weight_only_int4_06_b200.prof_cases skinny-quant
        w4_quantize_pack of W[16384, 8192] twice and of W[28672, 8192], then w4_gemm at M = 16 on
        the latter twice (both operands larger than L2)

Each ends by checking the device status word and prints one "ok" line.
"""
from __future__ import annotations

import sys


def decode_layer(N: int, K: int, n_launch: int = 8, variant: int = 0):
    import torch
    from . import w4a16 as w
    G = K // 128
    nb = 8
    Ws = [(torch.randint(-2 ** 31, 2 ** 31 - 1, (N, K // 8), dtype=torch.int32, device="cuda"),
           (torch.rand(N, G, device="cuda") * 0.01 + 0.001).half(),
           torch.randint(0, 16, (N, G), dtype=torch.uint8, device="cuda")) for _ in range(nb)]
    X = torch.randn(1, K, device="cuda").half()
    Y = None
    for i in range(n_launch):
        p, s, z = Ws[i % nb]
        Y = w.w4_gemm(X, p, s, z, variant=variant) if variant else w.w4_gemm(X, p, s, z)
    torch.cuda.synchronize()
    assert w.w4_check_device_status() == 0
    print("ok", N, K, float(Y.float().abs().mean()))


def clip(T: int, K: int, N: int):
    import torch
    from . import synth
    from . import w4a16 as B
    X, W = synth.awq_case(T=T, K=K, N=N, case_id=70)
    Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda()
    best = None
    for _ in range(2):
        best, _, p, s, z = B.awq_clip_search(Xd, Wd, None, 10)
    torch.cuda.synchronize()
    assert B.w4_check_device_status() == 0
    print("ok", T, K, N, torch.bincount(best.flatten().long(), minlength=10).tolist())


def skinny_quant():
    import torch
    from . import w4a16 as B
    torch.manual_seed(0)
    Wq = (torch.randn(16384, 8192, device="cuda") * 0.02).half()
    for _ in range(2):
        B.w4_quantize_pack(Wq)
    del Wq
    W = (torch.randn(28672, 8192, device="cuda") * 0.02).half()
    p, s, z = B.w4_quantize_pack(W)
    del W
    X = torch.randn(16, 8192, device="cuda").half()
    for _ in range(2):
        B.w4_gemm(X, p, s, z)
    torch.cuda.synchronize()
    assert B.w4_check_device_status() == 0
    print("ok")


def main(argv):
    if not argv:
        raise SystemExit(__doc__)
    cmd, rest = argv[0], [int(a) for a in argv[1:]]
    if cmd == "decode-layer":
        decode_layer(*rest)
    elif cmd == "clip":
        clip(*rest)
    elif cmd == "skinny-quant":
        skinny_quant()
    else:
        raise SystemExit(f"unknown case {cmd!r}\n{__doc__}")


if __name__ == "__main__":
    main(sys.argv[1:])
