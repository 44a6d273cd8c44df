"""CPU oracle for the Effort matvec on Q8 weights.

TEST INFRASTRUCTURE ONLY, under the same rules as ``effort_oracle``: nothing
on the product path may import or call it, it shares nothing with the CUDA
library, and it never takes an input or an expected value from it.

Source: [SHOW-HN] Hacker News thread "Show HN: Speeding up LLM inference 2x
times (possibly)", item 40067677: the post text says the implementation is
for FP16 and that Q8 is in the works; the author adds that the algorithm
should work on top of Q8; the exchange on embedding position bits describes
a Q8 bucket word of 1 sign bit, 3 location bits and 4 weight bits.

Reading (the pages fix no Q8 format; each point is also listed in the
design notes of the repository):

* A Q8 matrix is int8 values q [in_dim x out_dim] and one binary16 scale s_i
  per row (the row that multiplies v[i]); the weight is w_ij = s_i * q_ij,
  taken exactly (11 + 8 significant bits: exact in float32 and float64).
  Per-row scales keep each row's order a property of q alone.
* The method then runs on those weights unchanged, as the author says it
  should: row order |w| descending with ties to the lower column, keep,
  probes, chart x_ik = fl32(|v_i| * p_ik) (p_ik = |w| at the probe rank,
  exact in float32), K, the weighted order statistic c, the selection
  fl32(|v_i| * |w_ij|) >= c, and out as the float64 sum over the used pairs
  (each product v_i * w_ij is exact in float64: 24 + 11 + 8 bits).
* The 1 + 3 + 4 bit bucket word is a storage idea for the weights, not a
  different computation: it keeps 4 of q's bits, which is lossless only
  when a bucket's magnitudes span at most 16 levels.  The oracle defines the
  results on the full q; a packed store must reproduce them.
"""
from __future__ import annotations

import numpy as np

from oracle import effort_oracle as F

P_PROBES = F.P_PROBES


def q8_to_float64(q: np.ndarray, s_bits: np.ndarray) -> np.ndarray:
    """w_ij = s_i * q_ij in float64 (exact: 11 + 8 significant bits)."""
    q = np.asarray(q)
    if q.dtype != np.int8:
        raise ValueError("q must be int8")
    s = F.fp16_bits_to_float64(np.asarray(s_bits, dtype=np.uint16))
    return s[:, None] * q.astype(np.float64)


class PreparedQ8:
    """``precompute(W)`` for a Q8 matrix: the same sort, keep and probes as
    the fp16 oracle, on the exact dequantised weights."""

    def __init__(self, q, s_bits, keep_fraction: float = 1.0, P: int = P_PROBES):
        q = np.asarray(q)
        s_bits = np.asarray(s_bits, dtype=np.uint16)
        if q.ndim != 2 or q.size == 0 or q.dtype != np.int8:
            raise ValueError("q must be a non-empty 2-D int8 array")
        if s_bits.shape != (q.shape[0],):
            raise ValueError("one scale per row")
        s = F.fp16_bits_to_float64(s_bits)
        if not np.all(np.isfinite(s)):
            raise ValueError("a scale is not finite")
        kf = float(np.float32(keep_fraction))
        if not (kf > 0.0 and kf <= 1.0):
            raise ValueError("keep_fraction must be in (0, 1]")
        self.in_dim, self.out_dim = q.shape
        self.n = F.kept_count(self.out_dim, keep_fraction)
        if self.n < 1:
            raise ValueError("keep_fraction keeps no weight of a row")
        self.q = q
        self.s_bits = s_bits
        self.W = q8_to_float64(q, s_bits)
        mag = np.abs(self.W)
        # |w| descending, ties by the lower column (a stable sort on -|w|)
        self.W_idx = np.argsort(-mag, axis=1, kind="stable")
        self.W_val = np.take_along_axis(self.W, self.W_idx, axis=1)
        self.W_mag = np.abs(self.W_val)
        self.probes, self.weights = F.get_probes(self.W_mag, self.n, P)
        self.kept = np.zeros((self.in_dim, self.out_dim), dtype=bool)
        np.put_along_axis(self.kept, self.W_idx[:, : self.n], True, axis=1)


def selected_mask(prep: PreparedQ8, v32: np.ndarray, c: np.float32) -> np.ndarray:
    """S = {(i, j) kept : fl32(|v_i| * |w_ij|) >= c}; |w_ij| is exact in float32."""
    a = np.abs(v32.astype(np.float32))[:, None]
    wabs = np.abs(prep.W).astype(np.float32)
    prod = (a * wabs).astype(np.float32)
    return prep.kept & (prod >= np.float32(c))


def approx_mul(prep: PreparedQ8, v32: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """out_j = sum over used (i, j) of v_i * w_ij, float64, i ascending."""
    contrib = np.where(mask, v32.astype(np.float64)[:, None] * prep.W, 0.0)
    out = np.zeros(prep.out_dim, dtype=np.float64)
    for i in range(prep.in_dim):
        out += contrib[i]
    return out


def effort_gemv(prep: PreparedQ8, v, effort: float) -> F.Result:
    """One approximate matvec on Q8 weights: chart -> topK cutoff -> select -> multiply."""
    ef = float(np.float32(effort))
    if not (ef > 0.0 and ef <= 1.0):
        raise ValueError("effort must be in (0, 1]")
    v32 = F.as_f32_vector(v)
    if v32.shape != (prep.in_dim,):
        raise ValueError("v has the wrong length")
    if not np.all(np.isfinite(v32)):
        raise ValueError("v holds a non-finite value")
    chart = F.cutoff_chart(v32, prep.probes)
    K = F.effort_K(effort, prep.in_dim, prep.out_dim)
    c = F.top_k_cutoff(chart, prep.weights, K, prep.in_dim * prep.n)
    mask = selected_mask(prep, v32, c)
    out = approx_mul(prep, v32, mask)
    return F.Result(c, K, mask, out)


def dense_gemv(q, s_bits, v) -> np.ndarray:
    """Plain out = W^T v in float64 with W = s * q."""
    return q8_to_float64(q, s_bits).T @ F.as_f32_vector(v).astype(np.float64)
