"""CPU oracle for the other weight widths and column orders: INT2/INT3/INT8 round-to-nearest
groups, their packed bit streams, GPTQ at any of those widths with optional act-order (desc_act),
the matmuls that serve them, and a matmul whose activations are divided by a per-channel scale.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check and the benchmark's
CPU-baseline leg may import this module.  It shares no code with the CUDA library.

Pages: "AutoGPTQ vs The Stack v2" (GPTQ to 2/3/4/8-bit codes with per-group scales and zero
points, optional act-order, desc_act); "GPTQ, AWQ and the rules of post-training
quantization", sections "AWQ: find the one percent that matters" (INT3 with group size 128) and
"What activation-awareness buys and what it does not" (INT2 with group size 64; AWQ's scaling
applied before GPTQ).

Readings adopted where the pages are silent:
* a b-bit group has L = 2^b - 1 steps: the rules of the INT4 quantiser with 15 replaced by L
  (zero-inclusive range, s32 = (hi - lo) / L in fp32, fp16 scale rounded up, z = clamp(rint(-lo /
  s16), 0, L), q = clamp(rint(v / s16) + z, 0, L), half to even, one rounding per fp32 step);
* packing: each row's codes form one little-endian bit stream, code k in bits b k .. b k + b - 1,
  stream bit j in bit j % 32 of the row's word j / 32 (for b = 4 this is the INT4 nibble layout;
  a 3-bit code may straddle two words); K b must be a multiple of 32;
* act-order: the columns are processed in decreasing order of diag(X^T X) (a stable sort, so
  equal diagonals keep their index order); groups are consecutive in that order; the outputs are
  stored in processing order together with perm (perm[i] = the original column processed i-th),
  and the matmul gathers activations by perm: Y = X[:, perm] dequant(W_perm)^T.  The equivalent
  per-column group index of the original order is g_idx[perm[i]] = i // group;
* scaled activations: X' = fp16(fp32(x) / s) per element (one fp32 division, round to nearest,
  then one rounding to fp16), then the usual matmul.

Parity pins: every function here is pinned by the non-GPU tests in ``tests/test_oracle_wbits.py``
(the 4-bit case against the INT4 oracle, bit strings, a hand-worked 3-bit stream, brute force,
closed forms and permutation invariants).
"""
from __future__ import annotations

import numpy as np

from .w4a16_oracle import QuantRangeError, fp16_round_up

BITS = (2, 3, 4, 8)


def levels(bits: int) -> int:
    """L = 2^bits - 1 quantisation steps ("AutoGPTQ vs The Stack v2": 2/3/4/8-bit codes)."""
    assert bits in BITS, bits
    return (1 << bits) - 1


# ----------------------------------------------------------------------------
# Round-to-nearest groups of any width
# ----------------------------------------------------------------------------
def _params(v32: np.ndarray, L: int):
    """Scale and zero point of groups of fp32 values v32 [..., group] (last axis is the group): the
    INT4 quantiser's rules with L steps (the first reading in this module's header)."""
    lo = np.minimum(v32.min(axis=-1), np.float32(0))
    hi = np.maximum(v32.max(axis=-1), np.float32(0))
    d = hi - lo
    s16 = fp16_round_up(d / np.float32(L))
    s16 = np.where(d == 0, np.float16(1.0), s16).astype(np.float16)
    if np.isinf(s16).any():
        raise QuantRangeError("fp16 group scale overflow")
    sf = s16.astype(np.float32)
    z = np.clip(np.rint(-lo / sf), 0, L)
    return s16, sf, z


def quantize_rtn_bits(W: np.ndarray, bits: int, group: int, act_scale: np.ndarray | None = None):
    """Round-to-nearest b-bit groups ("GPTQ, AWQ and the rules of post-training quantization", section
    "The problem both methods solve"; INT3 g128 and INT2 g64 in its AWQ sections).
    Returns (q [N, K] uint8 codes 0..L, scales [N, K/group] fp16, zeros [N, K/group] uint8)."""
    L = levels(bits)
    W = np.asarray(W, dtype=np.float16)
    N, K = W.shape
    assert K % group == 0
    G = K // group
    v = W.astype(np.float32)
    if act_scale is not None:
        v = v * np.asarray(act_scale).astype(np.float32)[None, :]
    vg = v.reshape(N, G, group)
    s16, sf, z = _params(vg, L)
    q = np.clip(np.rint(vg / sf[:, :, None]) + z[:, :, None], 0, L)
    return q.reshape(N, K).astype(np.uint8), s16, z.astype(np.uint8)


# ----------------------------------------------------------------------------
# Bit streams
# ----------------------------------------------------------------------------
def pack_bits(q: np.ndarray, bits: int) -> np.ndarray:
    """[N, K] codes -> [N, K * bits / 32] uint32 (little-endian bit stream per row; the pages fix no
    layout, this is the packing reading in this module's header)."""
    q = np.asarray(q, dtype=np.uint64)
    N, K = q.shape
    assert (K * bits) % 32 == 0
    words = np.zeros((N, K * bits // 32), dtype=np.uint64)
    mask = np.uint64((1 << bits) - 1)
    for k in range(K):
        pos = bits * k
        w, off = pos // 32, pos % 32
        c = q[:, k] & mask
        words[:, w] |= (c << np.uint64(off)) & np.uint64(0xFFFFFFFF)
        if off + bits > 32:  # the code's upper bits start the next word
            words[:, w + 1] |= c >> np.uint64(32 - off)
    return words.astype(np.uint32)


def unpack_bits(packed: np.ndarray, bits: int, K: int) -> np.ndarray:
    """Inverse of pack_bits."""
    p = np.asarray(packed, dtype=np.uint64)
    N = p.shape[0]
    assert p.shape[1] * 32 == K * bits
    mask = np.uint64((1 << bits) - 1)
    q = np.zeros((N, K), dtype=np.uint8)
    for k in range(K):
        pos = bits * k
        w, off = pos // 32, pos % 32
        c = p[:, w] >> np.uint64(off)
        if off + bits > 32:
            c |= p[:, w + 1] << np.uint64(32 - off)
        q[:, k] = (c & mask).astype(np.uint8)
    return q


def quantize_pack_bits(W: np.ndarray, bits: int, group: int, act_scale: np.ndarray | None = None):
    """quantize_rtn_bits followed by pack_bits."""
    q, s16, z = quantize_rtn_bits(W, bits, group, act_scale)
    return pack_bits(q, bits), s16, z


def dequantize_bits(packed: np.ndarray, scales: np.ndarray, zeros: np.ndarray, bits: int, group: int,
                    K: int) -> np.ndarray:
    """w[n, k] = (q - z[n, k // group]) * s16[n, k // group], exact in fp64 (dequantisation for fp16
    compute, "AutoAWQ vs The Stack v2")."""
    q = unpack_bits(packed, bits, K).astype(np.float64)
    s = np.repeat(np.asarray(scales, dtype=np.float16).astype(np.float64), group, axis=1)
    z = np.repeat(np.asarray(zeros).astype(np.float64), group, axis=1)
    return (q - z) * s


def gemm_bits(X: np.ndarray, packed: np.ndarray, scales: np.ndarray, zeros: np.ndarray, bits: int,
              group: int) -> np.ndarray:
    """Y = X . dequant(W)^T in fp64."""
    X64 = np.asarray(X).astype(np.float64)
    return X64 @ dequantize_bits(packed, scales, zeros, bits, group, X64.shape[1]).T


# ----------------------------------------------------------------------------
# Act-order layout
# ----------------------------------------------------------------------------
def act_order_perm(X: np.ndarray) -> np.ndarray:
    """perm[i] = original column processed i-th: decreasing diag(X^T X), stable (desc_act,
    "AutoGPTQ vs The Stack v2"; the order criterion is the act-order reading in this header)."""
    X64 = np.asarray(X).astype(np.float64)
    d = np.einsum("tk,tk->k", X64, X64)
    return np.argsort(-d, kind="stable")


def g_idx_from_perm(perm: np.ndarray, group: int) -> np.ndarray:
    """Group of every original column: g_idx[perm[i]] = i // group."""
    g = np.empty(len(perm), dtype=np.int32)
    g[np.asarray(perm)] = np.arange(len(perm)) // group
    return g


def gemm_act_order(X: np.ndarray, packed: np.ndarray, scales: np.ndarray, zeros: np.ndarray,
                   perm: np.ndarray, bits: int, group: int) -> np.ndarray:
    """Y = X[:, perm] dequant(W_perm)^T (W stored in processing order)."""
    Xp = np.asarray(X)[:, np.asarray(perm)]
    return gemm_bits(Xp, packed, scales, zeros, bits, group)


def dequantize_g_idx(q_orig: np.ndarray, scales: np.ndarray, zeros: np.ndarray, g_idx: np.ndarray) -> np.ndarray:
    """Dequantisation in the original column order with a per-column group index."""
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)[:, g_idx]
    z = np.asarray(zeros).astype(np.float64)[:, g_idx]
    return (np.asarray(q_orig).astype(np.float64) - z) * s


# ----------------------------------------------------------------------------
# GPTQ at any width, natural or act-order
# ----------------------------------------------------------------------------
def _gptq_bits(X, W, bits, group, damp, act_order, stop_after, act_scale=None):
    L = levels(bits)
    X64 = np.asarray(X).astype(np.float64)
    Wc = np.asarray(W, dtype=np.float16).astype(np.float64).copy()
    N, K = Wc.shape
    assert K % group == 0
    if act_scale is not None:  # AWQ's scaling first: X / s and W * s (both in fp64)
        s64 = np.asarray(act_scale, dtype=np.float32).astype(np.float64)
        X64 = X64 / s64[None, :]
        Wc = Wc * s64[None, :]
    if act_order:
        d = np.einsum("tk,tk->k", X64, X64)
        perm = np.argsort(-d, kind="stable")
    else:
        perm = np.arange(K)
    X64 = X64[:, perm]
    Wc = Wc[:, perm]
    H = X64.T @ X64
    H[np.diag_indices(K)] += damp * np.mean(np.diag(H))
    U = np.linalg.cholesky(np.linalg.inv(H)).T
    G = K // group
    q = np.zeros((N, K), dtype=np.uint8)
    s16 = np.zeros((N, G), dtype=np.float16)
    z = np.zeros((N, G), dtype=np.uint8)
    sf = zg = None
    for k in range(K if stop_after is None else stop_after):
        if k % group == 0:
            sg, sf, zg = _params(Wc[:, k:k + group].astype(np.float32), L)
            s16[:, k // group] = sg
            z[:, k // group] = zg.astype(np.uint8)
        v = Wc[:, k].astype(np.float32)
        qk = np.clip(np.rint(v / sf) + zg, 0, L)
        q[:, k] = qk.astype(np.uint8)
        w_hat = (qk.astype(np.float64) - zg.astype(np.float64)) * sf.astype(np.float64)
        e = (Wc[:, k] - w_hat) / U[k, k]
        Wc[:, k + 1:] -= np.outer(e, U[k, k + 1:])
    return q, s16, z, Wc, perm


def gptq_quantize_bits(X: np.ndarray, W: np.ndarray, bits: int = 4, group: int = 128, damp: float = 0.01,
                       act_order: bool = False, act_scale: np.ndarray | None = None):
    """GPTQ ("GPTQ, AWQ and the rules of post-training quantization", section "GPTQ: pay for the error
    with the other weights") with b-bit groups, columns in natural or act-order.

    H = X^T X + damp * mean(diag) I in fp64; with act-order, columns, H's rows and columns and W's
    columns are first permuted by perm.  U = upper Cholesky factor of H^-1.  For each column k in
    processing order: at a group's first column its scale and zero point come from the group's
    current weights rounded to fp32; q_k = clamp(rint(fp32(w_k) / s) + z, 0, L);
    e = (w_k - (q_k - z) s) / U_kk; w_j -= e U_kj for later j.
    act_scale [K] (fp32): AWQ's per-channel scale applied first ("GPTQ, AWQ and the rules of
    post-training quantization", section "What activation-awareness buys and what it does not":
    the scaling is independent of the second-order update and goes before it): GPTQ then runs on
    X / s and W * s, both formed in fp64, and the layer computes (X / s) dequant(W)^T.
    Returns (packed, scales, zeros, perm), outputs in processing order (perm = arange when
    act_order is False).
    """
    q, s16, z, _, perm = _gptq_bits(X, W, bits, group, damp, act_order, None, act_scale)
    return pack_bits(q, bits), s16, z, perm


def gptq_state_bits(X: np.ndarray, W: np.ndarray, bits: int, group: int, damp: float, act_order: bool,
                    stop_after: int, act_scale: np.ndarray | None = None):
    """The weights in processing order after the first stop_after columns (for tests), and perm."""
    _, _, _, Wc, perm = _gptq_bits(X, W, bits, group, damp, act_order, stop_after, act_scale)
    return Wc, perm


# ----------------------------------------------------------------------------
# Activations divided by a per-channel scale inside the matmul
# ----------------------------------------------------------------------------
def scale_activations(X: np.ndarray, s: np.ndarray) -> np.ndarray:
    """X' = fp16(fp32(x) / s) per element."""
    x32 = np.asarray(X, dtype=np.float16).astype(np.float32)
    return (x32 / np.asarray(s, dtype=np.float32)[None, :]).astype(np.float16)
