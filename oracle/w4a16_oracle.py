"""CPU oracle for group-wise INT4 weight-only quantisation, the W4A16 matmul and the
AWQ activation-aware scale search.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check and
the benchmark's CPU-baseline leg may import this module.  It shares no code,
constants or tables with the CUDA library and never imports it.

Everything here is written for a reader to check by eye against the pages:

* "GPTQ, AWQ and the rules of post-training quantization" -- section "The problem
  both methods solve" (round-to-nearest rounding of weights to a small integer
  format) and section "AWQ: find the one percent that matters" (INT4 with group
  size 128; per-channel scale = the channel's mean |x| to the power alpha;
  alpha on a 20-point grid over [0, 1]; multiply a channel's weights by s and
  divide its activation by s, so the layer computes the same function).
* "AutoGPTQ vs The Stack v2" -- the GPTQ quantisation blurb (per-group
  quantisation, group size typically 128, scales and zero points).
* "When to Use AWQ vs GPTQ" -- section "Practical Usage"
  (quant_config w_bit 4, q_group_size 128).
* "AutoAWQ vs The Stack v2" -- the WQLinear blurb (INT4 storage, FP16 compute,
  weights dequantised on the fly inside the matmul).

Readings adopted where the pages are silent:

* the group range includes zero: lo = min(0, min v), hi = max(0, max v);
* scale: s32 = (hi - lo) / 15 in fp32 (IEEE round to nearest), then the fp16 scale
  is s32 rounded toward +infinity, so that the 16 levels cover [lo, hi];
* zero point z = clamp(rint(-lo / s16), 0, 15); code q = clamp(rint(v / s16) + z, 0, 15);
  rint rounds half to even; every step is one correctly rounded fp32 operation;
* an all-zero group gets s16 = 1 (then z = 0 and q = 0);
* dequantised weight w = (q - z) * s16 (exact in fp64);
* packing: 8 codes per uint32, the code of the lowest k in the lowest nibble;
* AWQ: m_j = mean_t |X_tj| (exact sum), s_j = max(m_j, 1e-6) ** alpha_i with
  alpha_i = i / n_alpha, i = 0 .. n_alpha - 1, then s <- s / sqrt(max(s) * min(s));
  s is rounded to fp32 before it scales W, and the same fp32 s divides X;
  MSE_i = mean over (t, n) of ((X / s) Wq^T - X W^T)^2 with unquantised W in the
  reference term; the chosen alpha is the lowest index among the minima.

Parity pins: every function here is pinned by the non-GPU tests in
``tests/test_oracle.py`` (closed forms, brute force, exact rational arithmetic,
invariants and library special cases).
"""
from __future__ import annotations

import numpy as np

GROUP = 128
QMAX = 15  # 4-bit codes 0 .. 15


class QuantRangeError(ValueError):
    """A group's fp16 scale overflowed to +inf (|W * act_scale| too large for fp16)."""


# ----------------------------------------------------------------------------
# fp16 rounding toward +infinity
# ----------------------------------------------------------------------------
def fp16_round_up(x32: np.ndarray) -> np.ndarray:
    """Round fp32 values to fp16 toward +infinity (the scale's rounding: the pages fix an fp16
    scale but not how it is rounded; rounding up keeps the 16 levels over the group's range).

    numpy's float32 -> float16 cast rounds to nearest (ties to even); where that
    result lies below the fp32 value, step one fp16 ulp up.
    """
    x32 = np.asarray(x32, dtype=np.float32)
    with np.errstate(over="ignore"):
        h = x32.astype(np.float16)
        low = h.astype(np.float32) < x32
        h = h.copy()
        h[low] = np.nextafter(h[low], np.float16(np.inf))
    return h


# ----------------------------------------------------------------------------
# Round-to-nearest group quantisation (one row group of 128 along K)
# ----------------------------------------------------------------------------
def quantize_rtn(W: np.ndarray, act_scale: np.ndarray | None = None, group: int = GROUP,
                 clip_ratio: np.ndarray | None = None):
    """Group-wise asymmetric INT4 round-to-nearest quantisation of W (or of W * diag(act_scale)).

    "GPTQ, AWQ and the rules of post-training quantization", section "The problem both methods solve" (round to the nearest
    level of a small integer format); "AutoGPTQ vs The Stack v2" (a scale and a zero point per group,
    group size 128); the steps the pages leave open follow the readings in this module's header.

    W: [N, K] fp16.  act_scale: [K] (cast to fp32) or None.
    clip_ratio: [N, K/group] fp32 or None.  When given, both ends of each group's zero-inclusive
    range are multiplied by the ratio (one fp32 multiply each) before the scale and zero point
    are derived; codes of weights outside the shrunk range saturate at 0 or 15.
    Returns (q [N, K] uint8 codes, scales [N, K/group] fp16, zeros [N, K/group] uint8).
    """
    W = np.asarray(W, dtype=np.float16)
    N, K = W.shape
    assert K % group == 0
    G = K // group
    v = W.astype(np.float32)
    if act_scale is not None:
        a = np.asarray(act_scale).astype(np.float32)
        v = v * a[None, :]  # one fp32 multiply per element
    vg = v.reshape(N, G, group)

    lo = np.minimum(vg.min(axis=2), np.float32(0))
    hi = np.maximum(vg.max(axis=2), np.float32(0))
    if clip_ratio is not None:
        r = np.asarray(clip_ratio, dtype=np.float32).reshape(N, G)
        lo = lo * r
        hi = hi * r
    d = hi - lo  # fp32, rounded to nearest
    s32 = d / np.float32(QMAX)  # fp32 IEEE division
    s16 = fp16_round_up(s32)
    s16[d == 0] = np.float16(1.0)  # all-zero group
    if np.isinf(s16).any():
        raise QuantRangeError("fp16 group scale overflow")
    sf = s16.astype(np.float32)

    z = np.clip(np.rint(-lo / sf), 0, QMAX)  # fp32 division, round half to even
    q = np.clip(np.rint(vg / sf[:, :, None]) + z[:, :, None], 0, QMAX)
    return (q.reshape(N, K).astype(np.uint8), s16, z.astype(np.uint8))


# ----------------------------------------------------------------------------
# Packing: 8 nibbles per uint32, lowest k in the lowest nibble
# ----------------------------------------------------------------------------
def pack_nibbles(q: np.ndarray) -> np.ndarray:
    """8 codes per uint32, the lowest k in the lowest nibble ("AutoAWQ vs The Stack v2": INT4
    storage; the pages do not fix the nibble order)."""
    q = np.asarray(q, dtype=np.uint32)
    N, K = q.shape
    assert K % 8 == 0
    q8 = q.reshape(N, K // 8, 8)
    word = np.zeros((N, K // 8), dtype=np.uint32)
    for i in range(8):
        word |= (q8[:, :, i] & np.uint32(0xF)) << np.uint32(4 * i)
    return word


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_nibbles."""
    packed = np.asarray(packed, dtype=np.uint32)
    N, W8 = packed.shape
    q = np.zeros((N, W8, 8), dtype=np.uint8)
    for i in range(8):
        q[:, :, i] = (packed >> np.uint32(4 * i)) & np.uint32(0xF)
    return q.reshape(N, W8 * 8)


def quantize_pack(W: np.ndarray, act_scale: np.ndarray | None = None, group: int = GROUP):
    """Returns (packed [N, K/8] uint32, scales [N, K/group] fp16, zeros [N, K/group] uint8)."""
    q, s16, z = quantize_rtn(W, act_scale, group)
    return pack_nibbles(q), s16, z


# ----------------------------------------------------------------------------
# Dequantisation and the fp64 matmul
# ----------------------------------------------------------------------------
def dequantize(packed: np.ndarray, scales: np.ndarray, zeros: np.ndarray, group: int = GROUP) -> np.ndarray:
    """w[n, k] = (q[n, k] - z[n, k // group]) * s16[n, k // group], exact in fp64 ("AutoAWQ vs The
    Stack v2": the weights are dequantised for FP16 compute)."""
    q = unpack_nibbles(packed).astype(np.float64)
    N, K = q.shape
    s = np.repeat(np.asarray(scales, dtype=np.float16).astype(np.float64), group, axis=1)
    z = np.repeat(np.asarray(zeros).astype(np.float64), group, axis=1)
    assert s.shape == (N, K)
    return (q - z) * s


def gemm(X: np.ndarray, packed: np.ndarray, scales: np.ndarray, zeros: np.ndarray,
         group: int = GROUP) -> np.ndarray:
    """Y = X . dequant(W)^T in fp64 (the W4A16 matmul of "AutoAWQ vs The Stack v2": activations stay
    fp16, weights are INT4).  X: [M, K] fp16.  Returns [M, N] float64."""
    Wd = dequantize(packed, scales, zeros, group)
    return np.asarray(X).astype(np.float64) @ Wd.T


def gemm_entries(X: np.ndarray, packed: np.ndarray, scales: np.ndarray, zeros: np.ndarray,
                 rows: np.ndarray, cols: np.ndarray, group: int = GROUP) -> np.ndarray:
    """Selected outputs Y[rows[i], cols[i]], each as its own fp64 dot product."""
    rows = np.asarray(rows)
    cols = np.asarray(cols)
    out = np.empty(len(rows), dtype=np.float64)
    ucols, inv = np.unique(cols, return_inverse=True)
    Wd = dequantize(np.asarray(packed)[ucols], np.asarray(scales)[ucols], np.asarray(zeros)[ucols], group)
    X64 = np.asarray(X)[rows].astype(np.float64)
    for i in range(len(rows)):
        out[i] = float(np.dot(X64[i], Wd[inv[i]]))
    return out


# ----------------------------------------------------------------------------
# AWQ activation-aware scale search
# ----------------------------------------------------------------------------
def channel_mean_abs(X: np.ndarray) -> np.ndarray:
    """m_j = (1/T) sum_t |X[t, j]|, with the sum taken exactly ("GPTQ, AWQ and the rules of post-training quantization",
    section "AWQ: find the one percent that matters": a channel's mean activation magnitude).

    Every fp16 value is an integer multiple of 2**-24 below 2**16, so |X| * 2**24 is an
    exact int64 and the column sums (at most 2**16 * 2**40 < 2**63) are exact; the one
    rounding is the final conversion to fp64.
    """
    X = np.asarray(X, dtype=np.float16)
    T = X.shape[0]
    units = (np.abs(X.astype(np.float64)) * 2.0 ** 24).astype(np.int64)
    tot = units.sum(axis=0, dtype=np.int64)
    return tot.astype(np.float64) * 2.0 ** -24 / T


def awq_alpha_grid(n_alpha: int = 20) -> np.ndarray:
    """alpha_i = i / n_alpha, i < n_alpha (the 20-point grid on [0, 1] of "GPTQ, AWQ and the rules of post-training quantization",
    section "AWQ: find the one percent that matters"; 1.0 itself is not a grid point)."""
    return np.array([i / n_alpha for i in range(n_alpha)], dtype=np.float64)


def awq_scales(m: np.ndarray, alpha: float) -> np.ndarray:
    """s_j = max(m_j, 1e-6) ** alpha, normalised by sqrt(max(s) * min(s)) (fp64; "GPTQ, AWQ and the rules of post-training quantization",
    section "AWQ: find the one percent that matters"; the floor and the normaliser are readings)."""
    s = np.maximum(np.asarray(m, dtype=np.float64), 1e-6) ** alpha
    return s / np.sqrt(s.max() * s.min())


def awq_scale_search(X: np.ndarray, W: np.ndarray, n_alpha: int = 20, group: int = GROUP,
                     quantizer=None):
    """Grid search of the AWQ per-channel scale exponent alpha ("GPTQ, AWQ and the rules of post-training quantization",
    section "AWQ: find the one percent that matters": scale W's channels by s, divide X's by s, and
    keep the alpha whose quantised layer output is closest to the original).

    X: [T, K] fp16 calibration activations; W: [N, K] fp16 weights.
    quantizer(W16, s32) -> fake-quantised W * diag(s32) as fp64 [N, K]; the default is
    quantize_rtn followed by dequantize (a test may pass an exact identity instead).
    Returns (mse [n_alpha] fp64, best index, s_best [K] fp32, all s [n_alpha, K] fp32).
    """
    X64 = np.asarray(X).astype(np.float64)
    W16 = np.asarray(W, dtype=np.float16)
    W64 = W16.astype(np.float64)
    T = X64.shape[0]
    N = W64.shape[0]
    m = channel_mean_abs(X)
    Y_ref = X64 @ W64.T
    mse = np.empty(n_alpha, dtype=np.float64)
    s_all = np.empty((n_alpha, X64.shape[1]), dtype=np.float32)
    for i, alpha in enumerate(awq_alpha_grid(n_alpha)):
        s32 = awq_scales(m, alpha).astype(np.float32)
        s_all[i] = s32
        s64 = s32.astype(np.float64)
        if quantizer is None:
            q, s16, z = quantize_rtn(W16, s32, group)
            Wq = dequantize(pack_nibbles(q), s16, z, group)
        else:
            Wq = quantizer(W16, s32)
        Y_q = (X64 / s64[None, :]) @ Wq.T
        mse[i] = np.mean((Y_q - Y_ref) ** 2)
        assert Y_q.shape == (T, N)
    best = int(np.argmin(mse))  # first occurrence = lowest index among the minima
    return mse, best, s_all[best].copy(), s_all


# ----------------------------------------------------------------------------
# AWQ clip search: per-group shrinking of the quantisation range
# ----------------------------------------------------------------------------
def clip_ratio_grid(n_ratios: int = 10) -> np.ndarray:
    """Shrink ratios r_j = 1 - j/20, j = 0 .. n_ratios-1 (fp32; 1.0 first).  The pages name the
    clipping ("AutoAWQ vs The Stack v2") without a grid; this grid is a reading."""
    return np.array([1.0 - j / 20.0 for j in range(n_ratios)], dtype=np.float64).astype(np.float32)


def awq_clip_search(X: np.ndarray, W: np.ndarray, act_scale: np.ndarray | None = None,
                    n_ratios: int = 10, group: int = GROUP):
    """Choose, for every (row n, group g), the range shrink ratio with the least output error
    (activation-guided clipping, "AutoAWQ vs The Stack v2"; the objective is a reading: each
    group's own contribution to the output error).

    The layer sees activations X diag(1/a) and quantises W diag(a) (a = act_scale, or 1).  For
    ratio r_j the group is quantised with its range shrunk by r_j (quantize_rtn's clip_ratio) and
        err[n, g, j] = sum_t ( sum_{k in g} (X[t,k] / a_k) * (w_hat[n,k] - v[n,k]) )^2
    with v = W a as the quantiser sees it (fp32) and w_hat = (q - z) * s16 (fp64); the output
    error of the group's own columns, every group on its own.  best = lowest j among the minima.
    Returns (err [N, G, R] fp64, best [N, G] int64, packed, scales, zeros) where the last three
    are the quantisation of W diag(a) with every group's best ratio.
    """
    X64 = np.asarray(X).astype(np.float64)
    W16 = np.asarray(W, dtype=np.float16)
    N, K = W16.shape
    G = K // group
    v = W16.astype(np.float32)
    if act_scale is not None:
        a32 = np.asarray(act_scale).astype(np.float32)
        v = v * a32[None, :]
        Xs = X64 / a32.astype(np.float64)[None, :]
    else:
        Xs = X64
    v64 = v.astype(np.float64)
    ratios = clip_ratio_grid(n_ratios)
    err = np.empty((N, G, n_ratios), dtype=np.float64)
    for j, r in enumerate(ratios):
        q, s16, z = quantize_rtn(W16, act_scale, group, np.full((N, G), r, dtype=np.float32))
        E = dequantize(pack_nibbles(q), s16, z, group) - v64  # [N, K]
        for g in range(G):
            cols = slice(g * group, (g + 1) * group)
            out = Xs[:, cols] @ E[:, cols].T  # [T, N]: the group's contribution to the output error
            err[:, g, j] = np.sum(out * out, axis=0)
    best = np.argmin(err, axis=2)  # first occurrence = lowest j among the minima
    q, s16, z = quantize_rtn(W16, act_scale, group, ratios[best])
    return err, best, pack_nibbles(q), s16, z


# ----------------------------------------------------------------------------
# GPTQ: quantise one column at a time and let the later columns absorb the error
# ----------------------------------------------------------------------------
def _group_params_rtn(v32: np.ndarray):
    """Scale and zero point of quantize_rtn for one group per row: v32 [N, group] fp32 (the same
    steps as quantize_rtn)."""
    lo = np.minimum(v32.min(axis=1), np.float32(0))
    hi = np.maximum(v32.max(axis=1), np.float32(0))
    d = hi - lo
    s16 = fp16_round_up(d / np.float32(QMAX))
    s16[d == 0] = np.float16(1.0)
    if np.isinf(s16).any():
        raise QuantRangeError("fp16 group scale overflow")
    sf = s16.astype(np.float32)
    z = np.clip(np.rint(-lo / sf), 0, QMAX)
    return s16, sf, z


def gptq_quantize(X: np.ndarray, W: np.ndarray, damp: float = 0.01, group: int = GROUP,
                  stop_after: int | None = None):
    """GPTQ on one layer ("GPTQ, AWQ and the rules of post-training quantization", section "GPTQ: pay
    for the error with the other weights"): columns are quantised in order, and after each one the
    not-yet-quantised columns are corrected so that the layer's output on the calibration data
    moves as little as possible.

    H = X^T X (fp64) plus damp * mean(diag H) on the diagonal; U = the upper Cholesky factor of H^-1.
    For column k: q_k = RTN code of the current W[:, k] with its group's scale and zero point, which
    are taken (quantize_rtn's rule) from the current, already corrected weights of the group when
    its first column is reached; e = (W[:, k] - (q_k - z) s) / U[k, k]; W[:, j] -= e U[k, j], j > k.
    The weights are carried in fp64; the group parameters see them rounded to fp32.
    stop_after: return after that many columns (for tests), with the corrected W.
    Returns (packed, scales, zeros, W_corrected fp64).
    """
    X64 = np.asarray(X).astype(np.float64)
    Wc = np.asarray(W, dtype=np.float16).astype(np.float64).copy()
    N, K = Wc.shape
    G = K // group
    H = X64.T @ X64
    H[np.diag_indices(K)] += damp * np.mean(np.diag(H))
    Hinv = np.linalg.inv(H)
    U = np.linalg.cholesky(Hinv).T  # upper: Hinv = U^T U
    q = np.zeros((N, K), dtype=np.uint8)
    s16 = np.zeros((N, G), dtype=np.float16)
    z = np.zeros((N, G), dtype=np.uint8)
    sf = zg = None
    ncols = K if stop_after is None else stop_after
    for k in range(ncols):
        g = k // group
        if k % group == 0:
            s_g, sf, zg = _group_params_rtn(Wc[:, k:k + group].astype(np.float32))
            s16[:, g] = s_g
            z[:, g] = zg.astype(np.uint8)
        v = Wc[:, k].astype(np.float32)
        qk = np.clip(np.rint(v / sf) + zg, 0, QMAX)
        q[:, k] = qk.astype(np.uint8)
        w_hat = (qk.astype(np.float64) - zg.astype(np.float64)) * sf.astype(np.float64)
        e = (Wc[:, k] - w_hat) / U[k, k]
        Wc[:, k + 1:] -= np.outer(e, U[k, k + 1:])
    return pack_nibbles(q), s16, z, Wc
