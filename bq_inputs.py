"""Seeded synthetic inputs for the bit-plane quantized linear layer.

This module only draws random tensors and rounds them to the storage types the
layer consumes (fp32 weights, bf16 activations). It contains none of the
quantization or layer arithmetic, so both the CUDA path's tests/bench and the
CPU oracle can use it without sharing method code.

Every tensor comes from ``numpy.random.default_rng([seed, tensor_id])`` (PCG64)
drawn in float64, then cast. The workload table below gives the shapes and
value distributions of the five weight formats (Llama-7B / Llama-13B
projection shapes stand in for the pages' models; no model or dataset is read).
"""
from __future__ import annotations

import numpy as np

# tensor ids: one independent stream per tensor role
TID_W, TID_X, TID_H2, TID_LORA_A, TID_LORA_B, TID_W_OUTLIER, TID_X_CHANNEL = 1, 2, 3, 4, 5, 6, 7
TID_COMP_A, TID_COMP_B = 8, 9
TID_H3 = 10


def rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tensor_id)])


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float values to the nearest bfloat16 (ties to even); returns float32."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).reshape(f.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """The uint16 storage of bf16-exact float32 values (e.g. from bf16_round)."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    return (f.view(np.uint32) >> 16).astype(np.uint16).reshape(f.shape)


def gaussian(shape, std: float, seed: int, tid: int) -> np.ndarray:
    return (rng(seed, tid).standard_normal(shape) * std).astype(np.float32)


def weights(N: int, K: int, seed: int = 0, std: float = 0.02,
            outlier_frac: float = 0.0, outlier_scale: float = 20.0) -> np.ndarray:
    """W [N,K] float32 ~ N(0, std^2); optionally a seeded choice (without
    replacement) of ``outlier_frac`` of the entries multiplied by ``outlier_scale``."""
    W = rng(seed, TID_W).standard_normal((N, K)) * std
    n_out = int(round(outlier_frac * N * K))
    if n_out > 0:
        idx = rng(seed, TID_W_OUTLIER).choice(N * K, size=n_out, replace=False)
        W.reshape(-1)[idx] *= outlier_scale
    return W.astype(np.float32)


def activations(M: int, K: int, seed: int = 0, std: float = 1.0,
                channel_frac: float = 0.0, channel_scale: float = 10.0) -> np.ndarray:
    """x [M,K] ~ N(0, std^2), rounded to bf16 (returned as bf16-exact float32);
    optionally a seeded ``channel_frac`` of the K channels scaled for all rows."""
    x = rng(seed, TID_X).standard_normal((M, K)) * std
    n_ch = int(round(channel_frac * K))
    if n_ch > 0:
        ch = rng(seed, TID_X_CHANNEL).choice(K, size=n_ch, replace=False)
        x[:, ch] *= channel_scale
    return bf16_round(x)


def uniform(n: int, lo: float, hi: float, seed: int, tid: int) -> np.ndarray:
    return rng(seed, tid).uniform(lo, hi, size=n).astype(np.float32)


def compensation_vectors(N: int, K: int, seed: int = 0, std: float = 0.1):
    """The ABQ distribution-compensation vectors a [N] and b [K], float32, each
    ~ N(0, std^2), so a b^T has std std^2 (0.01 by default, half the weights' 0.02).
    The pages fit a and b by calibration on data; these seeded draws stand in."""
    return gaussian(N, std, seed, TID_COMP_A), gaussian(K, std, seed, TID_COMP_B)


# ---------------------------------------------------------------------------
# Workload table: the five weight formats with their shapes and distributions.
# ---------------------------------------------------------------------------
WORKLOADS = {
    "rabit": dict(shapes=[(256, 512)], Ms=[1], w_std=0.02, h2=(0.5, 1.5)),
    "rabit3": dict(shapes=[(256, 512)], Ms=[1], w_std=0.02, h2=(0.5, 1.5), h3=(0.5, 1.5)),
    "bitnet": dict(shapes=[(4096, 4096), (11008, 4096), (4096, 11008)], Ms=[1], w_std=0.02),
    "ternary": dict(shapes=[(2048, 2048)], Ms=[1, 4, 16], w_std=0.02, lora_rank=32,
                    lora_alpha=0.1, a_std=0.02, b_std=0.01),
    "abq": dict(shapes=[(4096, 4096), (11008, 4096)], Ms=[1, 8, 64], w_std=0.02,
                w_outlier=(0.001, 20.0), x_channel=(0.01, 10.0),
                wa=[(2, 8), (4, 4), (6, 6), (8, 8)]),
    "bvsr": dict(shapes=[(5120, 5120), (13824, 5120), (5120, 13824)], Ms=[1], w_std=0.02),
}


def layer_inputs(fmt: str, N: int, K: int, M: int, seed: int = 0, lora_rank: int = 32) -> dict:
    """All tensors one layer call of format ``fmt`` needs, drawn per the workload table."""
    wl = WORKLOADS[fmt]
    out = {}
    if fmt == "abq":
        frac, sc = wl["w_outlier"]
        out["W"] = weights(N, K, seed, wl["w_std"], frac, sc)
        cf, cs = wl["x_channel"]
        out["x"] = activations(M, K, seed, 1.0, cf, cs)
    else:
        out["W"] = weights(N, K, seed, wl["w_std"])
        out["x"] = activations(M, K, seed, 1.0)
    if fmt in ("rabit", "rabit3"):
        lo, hi = wl["h2"]
        out["h2"] = uniform(K, lo, hi, seed, TID_H2)
    if fmt == "rabit3":
        lo, hi = wl["h3"]
        out["h3"] = uniform(K, lo, hi, seed, TID_H3)
    if fmt == "ternary":
        out["lora_A"] = gaussian((K, lora_rank), wl["a_std"], seed, TID_LORA_A)
        out["lora_B"] = gaussian((lora_rank, N), wl["b_std"], seed, TID_LORA_B)
    return out
