"""Seeded synthetic inputs shared by the CPU oracle, the tests and the benchmark.

This module only draws random numbers and casts them to the storage dtypes of the
workloads; it contains none of the quantization or matmul arithmetic. Both the oracle
(``oracle/``) and the CUDA path are fed from here, so both see identical bits.

Recipes (all from numpy ``default_rng``, float64 normals as in the demos of
"LLM Weight Quantization - GPTQ, AWQ, SmoothQuant, FP8 & INT4/INT8 Trade-offs",
section "Granularity and outliers", then cast to the storage dtype):

* tiny RTN config: W fp32 256x512 ~N(0, 0.02) seed 0; X bf16 1x512 ~N(0, 1) seed 1.
* 7B-class decode: W bf16 N x K in {4096x4096, 11008x4096, 4096x11008} ~N(0, 0.02)
  seed 0; X bf16 M x K ~N(0, 1) seed 1, M in {1, 4, 16}.
* 70B-class decode: W bf16 28672x8192 and 8192x28672 ~N(0, 0.015); M in {1, 8, 32}.
* prefill: X bf16 2048x4096 ~N(0, 1); W bf16 11008x4096 ~N(0, 0.02).
* outlier stress: W bf16 4096x4096 ~N(0, 0.02) with round(0.001*K) input columns
  (chosen without replacement, seed 2) multiplied by U(20, 100); X bf16 8x4096 ~N(0, 1)
  with the same channels multiplied by independent U(20, 100) draws. The 0.1% share and
  the 20-100x range follow "DL S067 - Quantization", section "The origin story".

bf16 values are produced by torch's float64 -> bfloat16 cast and returned as uint16 bit
patterns; fp32 values by numpy's float64 -> float32 cast.
"""
from __future__ import annotations

import numpy as np

SEED_W = 0
SEED_X = 1
SEED_OUTLIER = 2

# (N, K) weight shapes standing in for Llama-2-7B / Llama-2/3-70B projection layers.
SHAPES_7B = ((4096, 4096), (11008, 4096), (4096, 11008))
SHAPES_70B = ((28672, 8192), (8192, 28672))
M_7B = (1, 4, 16)
M_70B = (1, 8, 32)
PREFILL = dict(M=2048, N=11008, K=4096)


def normal_f64(shape, sigma, seed):
    """float64 N(0, sigma) draws from ``default_rng(seed)``."""
    return np.random.default_rng(seed).normal(0.0, sigma, shape)


def to_f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64).astype(np.float32))


def to_bf16_bits(a):
    """Cast float64 values to bfloat16 with torch and return the uint16 bit patterns."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.float64)))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f64(bits):
    """Widen bfloat16 bit patterns to float64 (exact)."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u32.view(np.float32).astype(np.float64)


def f16_bits_to_f64(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def weight_bf16(N, K, sigma=0.02, seed=SEED_W):
    return to_bf16_bits(normal_f64((N, K), sigma, seed))


def act_bf16(M, K, sigma=1.0, seed=SEED_X):
    return to_bf16_bits(normal_f64((M, K), sigma, seed))


def tiny_config():
    """W fp32 256x512 ~N(0,0.02) seed 0, X bf16 1x512 ~N(0,1) seed 1."""
    W = to_f32(normal_f64((256, 512), 0.02, SEED_W))
    X = act_bf16(1, 512)
    return W, X


def outlier_config(N=4096, K=4096, M=8, sigma=0.02, frac=0.001):
    """Outlier-stress inputs: returns (W bf16 bits, X bf16 bits, outlier column indices)."""
    n_out = int(round(frac * K))
    rng = np.random.default_rng(SEED_OUTLIER)
    cols = np.sort(rng.choice(K, n_out, replace=False))
    w_mult = rng.uniform(20.0, 100.0, n_out)
    x_mult = rng.uniform(20.0, 100.0, n_out)
    W = normal_f64((N, K), sigma, SEED_W)
    W[:, cols] *= w_mult
    X = normal_f64((M, K), 1.0, SEED_X)
    X[:, cols] *= x_mult
    return to_bf16_bits(W), to_bf16_bits(X), cols


def granularity_demo_tensors():
    """The synthetic tensors of the granularity/outlier demo on the study-docs page
    ("LLM Weight Quantization ...", section "Granularity and outliers"), drawn in the
    same order from ``default_rng(0)``: W 1024x1024 ~N(0,0.02) with its first 8 rows
    x6, X 256x1024 ~N(0,1) with 6 distinct channels x50. float64."""
    rng = np.random.default_rng(0)
    W = rng.normal(0, 0.02, (1024, 1024))
    W[:8] *= 6
    X = rng.normal(0, 1, (256, 1024))
    ch = rng.choice(1024, 6, replace=False)
    X[:, ch] *= 50
    return W, X


def calibration_toy_tensors():
    """The calibration toy on the study-docs page ("LLM Weight Quantization ...",
    section "GPTQ vs AWQ: two ways to choose what error to keep"), drawn in the same
    order from ``default_rng(1)``: a d x d mixing matrix N(0,1)/sqrt(d) (d = 128), 4
    distinct "salient" channels whose activations are 8x larger, a calibration set and a
    held-out set of 1024 correlated activations each (standard normals times the mixing
    matrix, plus 0.3 times independent standard normals, times the channel factors), and
    W 64x128 ~N(0, 0.05). Returns (W, X_cal, X_test), float64. The mixing only shapes the
    synthetic activations; no quantization arithmetic happens here."""
    rng = np.random.default_rng(1)
    d, rows, n = 128, 64, 1024
    mix = rng.normal(0, 1, (d, d)) / np.sqrt(d)
    chan = np.ones(d)
    chan[rng.choice(d, 4, replace=False)] = 8.0

    def draw(m):
        base = rng.normal(0, 1, (m, d)) @ mix
        return (base + 0.3 * rng.normal(0, 1, (m, d))) * chan

    X_cal = draw(n)
    X_test = draw(n)
    W = rng.normal(0, 0.05, (rows, d))
    return W, X_cal, X_test
