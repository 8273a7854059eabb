"""Seeded synthetic inputs for the W4A16 layer workloads.

This module only draws random numbers and casts them; it holds none of the
method's arithmetic (no quantisation, packing, dequantisation or matmul).  Both
the CUDA path's tests/bench and the CPU oracle's tests take their inputs from
here, so the two sides always see the same bits.

Recipe (stand-in for the real models and calibration corpora the pages measure
on, which are not available here):

* weights ``W`` [N, K] ~ N(0, 0.02) drawn in fp32, cast to fp16 (round to nearest);
* activations ``X`` [M, K] ~ N(0, 1) in fp32, 1 % of the K channels (chosen
  without replacement) multiplied by 20 -- the "activation-salient" outlier
  channels of "GPTQ, AWQ and the rules of post-training quantization",
  section "AWQ: find the one percent that matters" -- then cast to fp16;
* AWQ calibration activations ``X_calib`` [T, K]: a per-channel standard
  deviation ``exp(N(0, 1))`` (log-normal), times N(0, 1) per element, the same
  1 % x20 outlier channels, cast to fp16.  T = 65536 mirrors the
  "128 sequences" calibration set of the same page (128 x 512 tokens).

* correlated calibration activations (GPTQ cases): X = Z A * 0.3 + 0.1 E with Z [T, r] and
  E [T, K] ~ N(0, 1) and a mixing matrix A [r, K] ~ N(0, 1), r = K / 8, cast to fp16.  Real
  activations have strongly correlated channels, which is what GPTQ's compensation exploits; the
  independent-channel recipe above leaves it almost nothing to exploit.

Seeds: the single-layer smoke case uses ``seed = 0``; every other case uses the
sequence seed ``[case_id, M, K, N]`` and draws, in this fixed order, W, X and
then the outlier channel set.
"""
from __future__ import annotations

import numpy as np

W_STD = 0.02
OUTLIER_FRACTION = 0.01
OUTLIER_GAIN = 20.0

# Layer shapes of the workloads.  (K, N) pairs; M is the number of activation rows.
DECODE_7B_SHAPES = ((4096, 4096), (4096, 12288), (4096, 11008), (11008, 4096))
SMALL_BATCH_70B_SHAPES = ((8192, 8192), (8192, 28672), (28672, 8192))
SMALL_BATCH_MS = (4, 8, 16, 32)
PREFILL_SHAPES = ((4096, 11008), (4096, 4096), (8192, 28672))
PREFILL_MS = (512, 2048, 4096)
AWQ_T, AWQ_K, AWQ_N, AWQ_SUBSAMPLE = 65536, 4096, 4096, 4096


def _to_f16(a32: np.ndarray) -> np.ndarray:
    return a32.astype(np.float16)


def single_layer_case():
    """The 512x512 smoke case: X [1, 512] ~ N(0,1), W [512, 512] ~ N(0, 0.02), seed 0.

    Returns (X, W) as fp16 numpy arrays.
    """
    rng = np.random.default_rng(0)
    W = _to_f16(rng.standard_normal((512, 512), dtype=np.float32) * np.float32(W_STD))
    X = _to_f16(rng.standard_normal((1, 512), dtype=np.float32))
    return X, W


def outlier_channels(rng: np.random.Generator, K: int) -> np.ndarray:
    n = int(round(OUTLIER_FRACTION * K))
    return np.sort(rng.choice(K, n, replace=False))


def layer_case(case_id: int, M: int, K: int, N: int):
    """A linear layer: W [N, K] ~ N(0, 0.02); X [M, K] ~ N(0, 1) with 1 % x20 channels.

    Returns (X, W) as fp16 numpy arrays.  Draw order: W, X, outlier set.
    """
    rng = np.random.default_rng([case_id, M, K, N])
    W = _to_f16(rng.standard_normal((N, K), dtype=np.float32) * np.float32(W_STD))
    X32 = rng.standard_normal((M, K), dtype=np.float32)
    idx = outlier_channels(rng, K)
    X32[:, idx] *= np.float32(OUTLIER_GAIN)
    return _to_f16(X32), W


def weights_only(case_id: int, K: int, N: int, copy: int = 0) -> np.ndarray:
    """Extra independent weight matrices of one shape (distinct buffers for cold-L2 timing)."""
    rng = np.random.default_rng([case_id, 0, K, N, 1000 + copy])
    return _to_f16(rng.standard_normal((N, K), dtype=np.float32) * np.float32(W_STD))


def awq_case(T: int = AWQ_T, K: int = AWQ_K, N: int = AWQ_N, case_id: int = 5):
    """AWQ calibration layer: X_calib [T, K] (log-normal channel std, 1 % x20), W [N, K].

    Returns (X_calib, W) as fp16 numpy arrays.  Draw order: W, channel std, X, outlier set.
    """
    rng = np.random.default_rng([case_id, T, K, N])
    W = _to_f16(rng.standard_normal((N, K), dtype=np.float32) * np.float32(W_STD))
    sigma = np.exp(rng.standard_normal(K, dtype=np.float32)).astype(np.float32)
    X32 = rng.standard_normal((T, K), dtype=np.float32)
    X32 *= sigma[None, :]
    idx = outlier_channels(rng, K)
    X32[:, idx] *= np.float32(OUTLIER_GAIN)
    return _to_f16(X32), W


def awq_subsample_rows(T: int = AWQ_T, n: int = AWQ_SUBSAMPLE, case_id: int = 5) -> np.ndarray:
    """Seeded row subsample (sorted, without replacement) used to check the search on the CPU."""
    rng = np.random.default_rng([case_id, T, n, 7])
    return np.sort(rng.choice(T, n, replace=False))


def correlated_case(T: int, K: int, N: int, case_id: int = 9):
    """GPTQ calibration layer with correlated channels: X [T, K] (rank K/8 plus noise), W [N, K].

    Returns (X, W) as fp16 numpy arrays.  Draw order: W, Z, A, E.
    """
    rng = np.random.default_rng([case_id, T, K, N, 77])
    W = _to_f16(rng.standard_normal((N, K), dtype=np.float32) * np.float32(W_STD))
    r = max(1, K // 8)
    Z = rng.standard_normal((T, r), dtype=np.float32)
    A = rng.standard_normal((r, K), dtype=np.float32)
    E = rng.standard_normal((T, K), dtype=np.float32)
    X = (Z @ A) * np.float32(0.3) + np.float32(0.1) * E
    return _to_f16(X), W
