"""Seeded synthetic inputs shared by the tests, the bench and the oracle runs.

Holds random draws only (none of the method's arithmetic).  Shapes and
distributions follow the workloads the method is aimed at: batch-1 decode
matvecs of Mistral-7B-shaped projections with weights i.i.d. N(0, 0.02^2)
rounded to fp16, and activations that are either N(0, 1) or Student-t with
3 degrees of freedom scaled to unit variance (outlier-heavy).
"""
import math

import numpy as np

SIGMA_W = 0.02


def weights(in_dim, out_dim, seed, sigma=SIGMA_W):
    """W [in_dim x out_dim] float16: N(0, sigma^2) drawn in float32, rounded to nearest fp16."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((in_dim, out_dim), dtype=np.float32) * np.float32(sigma)).astype(np.float16)


def vector(in_dim, seed, dist="normal", dtype=np.float32):
    """v [in_dim]: N(0, 1) ("normal") or t_3 / sqrt(3) ("t3"), cast to dtype."""
    rng = np.random.default_rng(seed)
    if dist == "normal":
        v = rng.standard_normal(in_dim)
    elif dist == "t3":
        v = rng.standard_t(3, in_dim) / math.sqrt(3.0)
    else:
        raise ValueError(dist)
    return v.astype(np.float32).astype(dtype)


def gate(n_experts, in_dim, seed, scale=1.0 / 64):
    """Router matrix [n_experts x in_dim] float32, N(0, 1) * scale."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n_experts, in_dim)) * scale).astype(np.float32)


def q8_weights(in_dim, out_dim, seed, sigma=SIGMA_W):
    """Q8 weights of the same draw as `weights`: (q int8 [in_dim x out_dim],
    s float16 [in_dim]) with s_i = fp16(max_j |w_ij| / 127) and q_ij =
    round(w_ij / s_i) clipped to [-127, 127] (per-row symmetric absmax
    quantisation of a N(0, sigma^2) float32 draw).  A row that is all zero
    gets s_i = 1."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((in_dim, out_dim), dtype=np.float32) * np.float32(sigma)
    amax = np.abs(w).max(axis=1)
    s = (amax / np.float32(127.0)).astype(np.float16)
    s[s == 0] = np.float16(1.0)
    q = np.clip(np.rint(w / s.astype(np.float32)[:, None]), -127, 127).astype(np.int8)
    return q, s
