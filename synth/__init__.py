"""Seeded synthetic inputs shared by the CPU oracle, the tests and the benchmark.

This module holds input generation only: random numbers, an input cast to
bf16, and shape recipes.  It contains none of the attention method's
arithmetic (no projection, no selection, no softmax, no calibration), so the
oracle and the CUDA path can both draw from it without sharing any of the
computation they are compared on.

The law of the activations follows the workload description that accompanies
the AQUA pages (AQUA: Attention via QUery mAgnitudes, arXiv 2509.11155,
abstract): queries and keys are anisotropic,

    x = z R^T + 0.05 n,   z_j ~ N(0, exp(-j/32)) (second argument = variance),
    n ~ N(0, 1),          R a seeded random orthogonal d x d matrix,

and values are V ~ N(0, 1).  The calibration matrix stacks 8192 query rows
and 8192 key rows drawn from the same law.  Seeds: R uses 0, calibration 1,
runtime queries 2, keys 3, values 4.
"""
from __future__ import annotations

import numpy as np

D_HEAD = 128
SEED_R, SEED_CAL, SEED_Q, SEED_K, SEED_V = 0, 1, 2, 3, 4
NOISE_STD = 0.05
DECAY = 32.0


def orthogonal_R(d: int = D_HEAD, seed: int = SEED_R) -> np.ndarray:
    """Random orthogonal matrix: QR of a d x d N(0,1) matrix with diag(R_qr) > 0."""
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((d, d))
    q, r = np.linalg.qr(a)
    return q * np.sign(np.diag(r))[None, :]


def anisotropic_rows(n: int, d: int, R: np.ndarray, rng: np.random.Generator) -> np.ndarray:
    """n rows of x = z R^T + 0.05 N(0,1) with z_j ~ N(0, exp(-j/32)), float64."""
    std = np.sqrt(np.exp(-np.arange(d) / DECAY))
    z = rng.standard_normal((n, d)) * std[None, :]
    return z @ R.T + NOISE_STD * rng.standard_normal((n, d))


def calibration_matrix(d: int = D_HEAD, n_q: int = 8192, n_k: int = 8192,
                       seed: int = SEED_CAL) -> np.ndarray:
    """Stacked calibration queries and keys, [n_q + n_k, d] float32."""
    R = orthogonal_R(d)
    rng = np.random.default_rng(seed)
    xq = anisotropic_rows(n_q, d, R, rng)
    xk = anisotropic_rows(n_k, d, R, rng)
    return np.vstack([xq, xk]).astype(np.float32)


def qk_tensor(shape: tuple, seed: int, d: int = D_HEAD) -> np.ndarray:
    """Anisotropic query/key activations of the given shape (last axis = d), float32."""
    assert shape[-1] == d
    R = orthogonal_R(d)
    rng = np.random.default_rng(seed)
    n = int(np.prod(shape[:-1]))
    return anisotropic_rows(n, d, R, rng).reshape(shape).astype(np.float32)


def v_tensor(shape: tuple, seed: int = SEED_V) -> np.ndarray:
    """Values V ~ N(0,1) of the given shape, float32."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal(shape).astype(np.float32)


def cast_bf16(x: np.ndarray) -> np.ndarray:
    """Cast float32 inputs to bf16 (round to nearest even); returns float32 holding
    bf16-exact values so both sides of a comparison see the same input numbers."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((u >> 16) & 1)
    u = ((u + bias) & 0xFFFF0000).astype(np.uint32)
    return u.view(np.float32)


def bf16_bits(x_bf16_exact: np.ndarray) -> np.ndarray:
    """Upper 16 bits of bf16-exact float32 values (the raw bf16 encoding)."""
    u = np.ascontiguousarray(x_bf16_exact, dtype=np.float32).view(np.uint32)
    return (u >> 16).astype(np.uint16)


def decode_inputs(B: int, Hq: int, Hkv: int, T: int, d: int = D_HEAD, bf16: bool = True,
                  steps: int = 1):
    """History + per-step inputs for a decode workload.

    Returns dict with
      k_hist [B, T, Hkv, d], v_hist [B, T, Hkv, d]  (T history tokens),
      q      [steps, B, Hq, d], k_new [steps, B, Hkv, d], v_new [steps, B, Hkv, d].
    Keys and values are drawn as one stream of T + steps tokens per sequence.
    """
    kk = qk_tensor((B, T + steps, Hkv, d), SEED_K, d)
    vv = v_tensor((B, T + steps, Hkv, d), SEED_V)
    q = qk_tensor((steps, B, Hq, d), SEED_Q, d)
    if bf16:
        kk, vv, q = cast_bf16(kk), cast_bf16(vv), cast_bf16(q)
    return {
        "k_hist": kk[:, :T], "v_hist": vv[:, :T],
        "k_new": np.ascontiguousarray(kk[:, T:].transpose(1, 0, 2, 3)),
        "v_new": np.ascontiguousarray(vv[:, T:].transpose(1, 0, 2, 3)),
        "q": q,
    }


def prefill_inputs(L_total: int, Hq: int, Hkv: int, d: int = D_HEAD, bf16: bool = True, B: int = 1):
    """A prompt of L_total tokens: q [B, L, Hq, d], k [B, L, Hkv, d], v [B, L, Hkv, d]."""
    q = qk_tensor((B, L_total, Hq, d), SEED_Q, d)
    k = qk_tensor((B, L_total, Hkv, d), SEED_K, d)
    v = v_tensor((B, L_total, Hkv, d), SEED_V)
    if bf16:
        q, k, v = cast_bf16(q), cast_bf16(k), cast_bf16(v)
    return {"q": q, "k": k, "v": v}
