"""CPU oracle for the Effort approximate matrix-vector multiply.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code, constants generator or helper with the CUDA library, and it
never reads anything the CUDA library produced as an input or an expected
value.

Sources (cited by page title and the part of the page):

* [SHOW-HN] Hacker News thread "Show HN: Speeding up LLM inference 2x times
  (possibly)", item 40067677 (HN Gopher archive of 2024-04-17):
  - the post text: only part of the weight multiplications are done, the
    fraction is adjustable per call ("effort"), and the data format lets the
    loader skip the least important weights;
  - a commenter's question quoting the pseudo-code of the equations page:
    ``precompute(W)`` transposes W, takes probes, sorts the rows into
    ``W_idx, W_val``; ``approxMul`` forms ``cutoff_chart = v * probes``, takes
    ``cutoff = topK(cutoff_chart, effort)`` and multiplies with that cutoff;
  - the author's reply contrasting the format with CSR: every weight of a
    row is stored, sorted from the largest absolute value down, and only a
    leading part of each row, set by the input vector, is used;
  - the CSR passage quoted by a commenter: take an element of the vector,
    multiply it by a weight and add the product into the output at the
    weight's position.
* [HN-40095016] Hacker News item 40095016, the author's reply on complexity:
  O(effort * inDim * outDim) multiplications, O(inDim) for the dispatch and
  about O(inDim * log inDim) to find the cutoff.

Readings of points the pages leave open (each is also listed in the design
notes of the repository):

* W is given as [in_dim x out_dim] (already "flipped"): row i holds the
  weights that multiply v[i]; out[j] = sum_i v[i] * W[i, j].
* Row order: |w| descending, ties by the lower column index first.
* keep_fraction kappa keeps the first n = floor(kappa * out_dim + 1/2)
  entries of every row's order; the rest are never used.
* Probes: P = 16 per row.  Split the kept list into P segments with
  boundaries b_k = floor(k * n / P); probe k is |w| at the midpoint rank
  floor((b_{k-1} + b_k) / 2) and carries the integer weight b_k - b_{k-1}
  (the number of entries it stands for).  Empty segments carry weight 0.
* Chart: x_ik = fl32(|v_i| * p_ik), single precision, round to nearest even.
* K = llround(effort * in_dim * out_dim) computed in double.  topK is the
  weighted order statistic c = max{x in chart : sum of weights of chart
  entries >= x is >= K}.  If K >= the kept count, c = 0 (everything kept is
  used); if K == 0, c = +inf (nothing is used).
* Selection: (i, j) is used iff it is kept and fl32(|v_i| * |w_ij|) >= c.
  The product, not a division, decides; ties at c are used.
* out is the float64 sum of v_i * w_ij over the used pairs (each such product
  is exact in float64: 24 + 11 significant bits).
"""
from __future__ import annotations

import math

import numpy as np

P_PROBES = 16  # probes per row (reading of ``get_probes`` in [SHOW-HN])


# --------------------------------------------------------------------------
# Step 0: decode binary16 weights exactly (IEEE 754-2008 binary16 layout)
# --------------------------------------------------------------------------
def fp16_bits_to_float64(bits) -> np.ndarray:
    """Decode IEEE-754 binary16 bit patterns into exact float64 values.

    Layout: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
    exponent 0 -> subnormal (fraction * 2**-24); exponent 31 -> inf / NaN.
    Written from the format definition, not from any conversion routine.
    """
    b = np.asarray(bits, dtype=np.uint16).astype(np.int64)
    sign = np.where((b >> 15) & 1, -1.0, 1.0)
    expo = (b >> 10) & 0x1F
    frac = (b & 0x3FF).astype(np.float64)
    normal = sign * (1.0 + frac / 1024.0) * np.exp2((expo - 15).astype(np.float64))
    subnormal = sign * frac * 2.0 ** -24
    out = np.where(expo == 0, subnormal, normal)
    out = np.where((expo == 31) & (frac == 0), sign * np.inf, out)
    out = np.where((expo == 31) & (frac != 0), np.nan, out)
    return out


def fp16_magnitude_key(bits) -> np.ndarray:
    """|w| as the 15-bit integer of its binary16 pattern (sign dropped).

    For finite binary16 numbers this integer orders exactly like |w|, which
    is how ties in magnitude are recognised (equal keys <=> equal |w|).
    """
    return (np.asarray(bits, dtype=np.uint16).astype(np.int64)) & 0x7FFF


# --------------------------------------------------------------------------
# precompute(W): sortMatrixRows and get_probes            ([SHOW-HN] pseudo-code)
# --------------------------------------------------------------------------
def kept_count(out_dim: int, keep_fraction: float) -> int:
    """n = floor(kappa * out_dim + 1/2): entries of each row that are kept.

    The post text of [SHOW-HN] says the format lets the loader skip a chosen
    share of the least important weights; the rounding is this oracle's
    reading.  kappa is taken as the single-precision number the caller
    passes, widened exactly to double.
    """
    x = float(np.float32(keep_fraction)) * out_dim + 0.5
    return int(math.floor(x))


def sort_matrix_rows(W_bits: np.ndarray):
    """``W_idx, W_val = sortMatrixRows(W)`` of the [SHOW-HN] pseudo-code.

    For each row i, order the column indices j by |w_ij| descending and, for
    equal magnitudes, by j ascending (the author's CSR reply: rows stored
    sorted from the highest absolute value to the lowest).
    Returns (W_idx int64 [I, O], W_val float64 [I, O] signed values in that
    order, W_mag float64 [I, O] = |W_val|).
    """
    W_bits = np.asarray(W_bits, dtype=np.uint16)
    I, O = W_bits.shape
    mag = fp16_magnitude_key(W_bits)
    # primary key: magnitude descending; secondary: j ascending.  lexsort
    # sorts by the last key first; a stable sort on -mag keeps j ascending.
    W_idx = np.argsort(-mag, axis=1, kind="stable")
    vals = fp16_bits_to_float64(W_bits)
    W_val = np.take_along_axis(vals, W_idx, axis=1)
    return W_idx, W_val, np.abs(W_val)


def probe_layout(n: int, P: int = P_PROBES):
    """Ranks and integer weights of the P probes of a kept list of length n.

    Segment k (1-based) spans ranks [b_{k-1}, b_k) with b_k = floor(k*n/P);
    its probe sits at rank floor((b_{k-1}+b_k)/2) and weighs b_k - b_{k-1}.
    Empty segments get weight 0 and no rank (returned as -1).
    """
    b = [(k * n) // P for k in range(P + 1)]
    ranks, weights = [], []
    for k in range(1, P + 1):
        w = b[k] - b[k - 1]
        weights.append(w)
        ranks.append((b[k - 1] + b[k]) // 2 if w > 0 else -1)
    return np.array(ranks, dtype=np.int64), np.array(weights, dtype=np.int64)


def get_probes(W_mag_sorted: np.ndarray, n: int, P: int = P_PROBES):
    """``probes = get_probes(W)``: per-row |w| samples at the probe ranks.

    Returns (probes float64 [I, P] exact magnitudes, weights int64 [P]).
    Probes of empty segments are 0 with weight 0.
    """
    ranks, weights = probe_layout(n, P)
    I = W_mag_sorted.shape[0]
    probes = np.zeros((I, P), dtype=np.float64)
    for k in range(P):
        if weights[k] > 0:
            probes[:, k] = W_mag_sorted[:, ranks[k]]
    return probes, weights


class Prepared:
    """Result of ``precompute(W)`` plus the kept count (oracle form)."""

    def __init__(self, W_bits, keep_fraction: float = 1.0, P: int = P_PROBES):
        W_bits = np.asarray(W_bits, dtype=np.uint16)
        if W_bits.ndim != 2 or W_bits.size == 0:
            raise ValueError("W must be a non-empty 2-D array of binary16 bits")
        vals = fp16_bits_to_float64(W_bits)
        if not np.all(np.isfinite(vals)):
            raise ValueError("W holds a non-finite value")
        kf = float(np.float32(keep_fraction))
        if not (kf > 0.0 and kf <= 1.0):
            raise ValueError("keep_fraction must be in (0, 1]")
        self.in_dim, self.out_dim = W_bits.shape
        self.n = kept_count(self.out_dim, keep_fraction)
        if self.n < 1:
            raise ValueError("keep_fraction keeps no weight of a row")
        self.W_bits = W_bits
        self.W_idx, self.W_val, self.W_mag = sort_matrix_rows(W_bits)
        self.probes, self.weights = get_probes(self.W_mag, self.n, P)
        # kept[i, j]: True iff column j is among the first n of row i's order
        self.kept = np.zeros((self.in_dim, self.out_dim), dtype=bool)
        np.put_along_axis(self.kept, self.W_idx[:, : self.n], True, axis=1)


# --------------------------------------------------------------------------
# approxMul: chart, topK cutoff, multiply                  ([SHOW-HN] pseudo-code)
# --------------------------------------------------------------------------
def as_f32_vector(v) -> np.ndarray:
    """v as single precision (a binary16 v widens exactly)."""
    v = np.asarray(v)
    if v.dtype == np.float16:
        v = fp16_bits_to_float64(v.view(np.uint16)).astype(np.float32)
    return v.astype(np.float32)


def cutoff_chart(v32: np.ndarray, probes: np.ndarray) -> np.ndarray:
    """``cutoff_chart = v * probes``: x_ik = fl32(|v_i| * p_ik).

    Single-precision multiply, one rounding (numpy float32 x float32).
    """
    a = np.abs(v32.astype(np.float32))[:, None]
    return (a * probes.astype(np.float32)).astype(np.float32)


def effort_K(effort: float, in_dim: int, out_dim: int) -> int:
    """K = llround(effort * in_dim * out_dim), the product taken in double.

    The author's complexity reply [HN-40095016] puts the multiplication count
    at effort * inDim * outDim; K is that count, rounded half away from zero.
    """
    x = float(np.float32(effort)) * float(in_dim * out_dim)
    fl = math.floor(x)
    return int(fl) + (1 if (x - fl) >= 0.5 else 0)


def top_k_cutoff(chart: np.ndarray, weights: np.ndarray, K: int, kept_total: int) -> np.float32:
    """``cutoff = topK(cutoff_chart, effort)`` as a weighted order statistic.

    c = max{x in chart : sum of weights of chart entries >= x is >= K}.
    Special cases: K >= kept_total -> 0 (all kept products used);
    K == 0 -> +inf (none used).
    """
    if K >= kept_total:
        return np.float32(0.0)
    if K == 0:
        return np.float32(np.inf)
    x = chart.reshape(-1)
    w = np.broadcast_to(weights[None, :], chart.shape).reshape(-1).astype(np.int64)
    order = np.argsort(-x.astype(np.float64), kind="stable")
    cum = np.cumsum(w[order])
    m = int(np.searchsorted(cum, K, side="left"))  # first position with cum >= K
    return np.float32(x[order][m])


def selected_mask(prep: Prepared, v32: np.ndarray, c: np.float32) -> np.ndarray:
    """S = {(i, j) kept : fl32(|v_i| * |w_ij|) >= c} as a boolean [I, O] mask."""
    a = np.abs(v32.astype(np.float32))[:, None]
    wabs = np.abs(fp16_bits_to_float64(prep.W_bits)).astype(np.float32)
    prod = (a * wabs).astype(np.float32)
    return prep.kept & (prod >= np.float32(c))


def approx_mul(prep: Prepared, v32: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """out_j = sum over used (i, j) of v_i * w_ij, in float64, i ascending.

    This is the CSR-style step of [SHOW-HN]: each vector element multiplies
    the used weights of its row and the products are added into the output
    at the weights' column positions.
    """
    W = fp16_bits_to_float64(prep.W_bits)
    contrib = np.where(mask, v32.astype(np.float64)[:, None] * W, 0.0)
    out = np.zeros(prep.out_dim, dtype=np.float64)
    for i in range(prep.in_dim):  # i ascending, as written out in the pages' example
        out += contrib[i]
    return out


class Result:
    def __init__(self, c, K, mask, out):
        self.c = c              # float32 cutoff
        self.K = K              # target count
        self.mask = mask        # [I, O] used pairs
        self.count = int(mask.sum())
        self.L = mask.sum(axis=1).astype(np.int64)  # per-row prefix lengths
        self.out = out          # float64 [O]


def effort_gemv(prep: Prepared, v, effort: float) -> Result:
    """One approximate matvec: chart -> topK cutoff -> select -> multiply."""
    ef = float(np.float32(effort))
    if not (ef > 0.0 and ef <= 1.0):
        raise ValueError("effort must be in (0, 1]")
    v32 = as_f32_vector(v)
    if v32.shape != (prep.in_dim,):
        raise ValueError("v has the wrong length")
    if not np.all(np.isfinite(v32)):
        raise ValueError("v holds a non-finite value")
    chart = cutoff_chart(v32, prep.probes)
    K = effort_K(effort, prep.in_dim, prep.out_dim)
    c = top_k_cutoff(chart, prep.weights, K, prep.in_dim * prep.n)
    mask = selected_mask(prep, v32, c)
    out = approx_mul(prep, v32, mask)
    return Result(c, K, mask, out)


def row_prefix_lengths(prep: Prepared, mask: np.ndarray) -> np.ndarray:
    """L_i and a check that row i's used set is the first L_i of its order.

    Raises AssertionError if some row's used set is not a prefix.
    """
    in_order = np.take_along_axis(mask, prep.W_idx, axis=1)
    L = in_order.sum(axis=1)
    ranks = np.arange(prep.out_dim)[None, :]
    assert np.array_equal(in_order, ranks < L[:, None]), "used set is not a prefix"
    return L.astype(np.int64)


def dense_gemv(W_bits: np.ndarray, v) -> np.ndarray:
    """Plain out = W^T v in float64 (the dense baseline of the method)."""
    return fp16_bits_to_float64(W_bits).T @ as_f32_vector(v).astype(np.float64)
