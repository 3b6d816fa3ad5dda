"""Plain fp64 CPU oracle of the compressed linear layer.

    y = deq(Q (.) M) x  +  S_csr x  +  deq(L_q) (deq(R_q) x)

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline leg
of the benchmark may import this module.  It shares no code with the CUDA
library: it re-derives every step from the method's definition and from the
packed-format specification written in ``include/cql.h``.

Sources (web pages summarising the methods):

* SLiM: One-shot Quantization and Sparsity with Low-rank Approximation for LLM
  Weight Compression -- review summary, bullets "SLIM-Quant" (symmetric
  quantisation with weights clipped before round-to-nearest), "Low-rank
  adapter quantization" (AbsMax, groups of 128); rebuttal sections
  "Unstructured vs. 2:4 Sparsity" and "Order of Pruning and Quantization".
* SqueezeLLM: Dense-and-Sparse Quantization -- "Approach" (non-uniform LUT
  quantisation whose k-means centroids are weighted by a diagonal Fisher
  information; the top 0.45% outliers go to a full-precision CSR matrix so
  the dense part has a narrower range).
* SLiM review summary, "SLIM-Quant", and rebuttal, "Assumptions in
  Theoretical Derivations": the clip threshold alpha is found by a grid
  search over a probabilistic (histogram-based) model of the quantisation
  error.
* SLiM (same page), review summary "SLIM-LoRA" and rebuttal "Assumptions in
  Theoretical Derivations": the adapters minimise the saliency-weighted
  error norm ||F(W - W_C - L R)|| for an additive, invertible saliency F
  built from the layer's (positive) average input; the solution is the SVD
  of F(W - W_C), mapped back through F^-1.  Naive-LoRA is the plain SVD.
* SLiM (same page), rebuttal "Output Error Minimization in SLiM-Quant": the
  output-error variant scales the weights of the ~1% most salient input
  channels up by a factor and the matching activations down by it; a
  channel's saliency is the product of the normalised mean magnitudes of its
  activations and of its weights.

Where the pages are silent the plainest reading is taken; every such reading
is listed in the design notes and repeated at the function that makes it.
Every function works in fp64 on exact widenings of the inputs.  Rounding to
fp16 uses NumPy's float64 -> float16 conversion, a single round-to-nearest-
even step (pinned in the tests).

Pin status: every function below is pinned by at least one CPU test against
brute force, an invariant, a closed form or a library routine (see
``tests/test_oracle_pins.py``).  The published accuracy and perplexity figures
are "parity unpinned": they need model checkpoints and text corpora that are
not available.
"""
from __future__ import annotations

import math
import struct
from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np

__all__ = [
    "MASK_NONE", "MASK_2_4", "MASK_BITMAP50",
    "CODEC_INT4", "CODEC_INT3", "CODEC_LUT3", "CODEC_LUT4",
    "GROUP", "ROWBLK", "PAIRS_2OF4", "META_NIBBLE_2OF4",
    "OracleDesc", "desc_for",
    "fp16_round", "n_outliers", "select_outliers",
    "mask_2of4", "mask_bitmap50",
    "quantize_uniform", "lut_centroids", "lut_assign",
    "quantize_adapter_rows", "quantize_adapter_cols",
    "build_csr", "compress", "packed_layout", "pack_bytes",
    "channel_saliency", "select_salient_channels", "scale_activations",
    "compressed_matrix", "slim_lora", "lowrank_objective", "build_adapters",
    "ALPHA_GRID", "ALPHA_BINS", "clip_histogram", "alpha_objective", "search_clip_alpha",
    "KMEANS_MAX_ITERS", "fisher_kmeans",
    "forward", "forward_terms", "dense_reconstruction",
    "rel_err", "pack_and_forward", "HEADER_BYTES", "NPLANES",
    "P_HEADER", "P_VALUES", "P_META", "P_SCALES", "P_VOFF", "P_CSR_ROWPTR",
    "P_CSR_COL", "P_CSR_VAL", "P_R_VALUES", "P_R_SCALES", "P_L_VALUES", "P_L_SCALES",
    "P_SALIENT", "FORMAT_VERSION",
]

# ---------------------------------------------------------------------------
# enumerations (values fixed by the packed-format specification)
# ---------------------------------------------------------------------------
MASK_NONE, MASK_2_4, MASK_BITMAP50 = 0, 1, 2
CODEC_INT4, CODEC_INT3, CODEC_LUT3, CODEC_LUT4 = 0, 1, 2, 3
GROUP = 128            # weight and adapter quantisation group
ROWBLK = 32            # rows per interleaved row block
SLAB = 16              # bytes each row contributes to one slab

# 2:4 pattern index p -> kept positions (i0, i1), i0 < i1, lexicographic.
PAIRS_2OF4 = ((0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3))
# Byte-format code of a 2:4 group in the META plane: the two kept positions
# themselves, i0 | (i1 << 2) (a format choice: the pages fix no byte layout;
# this is the 2-bit-index form that sparse tensor cores read).
META_NIBBLE_2OF4 = tuple(i0 | (i1 << 2) for i0, i1 in PAIRS_2OF4)

_CODEC_BITS = {CODEC_INT4: 4, CODEC_INT3: 3, CODEC_LUT3: 3, CODEC_LUT4: 4}


@dataclass
class OracleDesc:
    """Mirror of the C descriptor (fields with the same meaning)."""
    n_out: int
    k_in: int
    mask: int
    codec: int
    clip_alpha: float = 0.9     # stored as float32, widened exactly
    outlier_frac: float = 0.0   # stored as float32, widened exactly
    rank: int = 0
    group: int = GROUP
    adapter_bits: int = 4
    adapter_group: int = GROUP
    flags: int = 0
    salient_channels: int = 0   # SLiM^O: channels scaled (0 = plain SLiM)
    salient_log2: int = 0       # SLiM^O: the factor is 2**salient_log2


def desc_for(wl) -> OracleDesc:
    """Descriptor for a ``workloads.Workload``."""
    mask = {"2:4": MASK_2_4, "bitmap50": MASK_BITMAP50, "none": MASK_NONE}[wl.mask]
    codec = {"int4": CODEC_INT4, "int3": CODEC_INT3, "lut3": CODEC_LUT3,
             "lut4": CODEC_LUT4}[wl.codec]
    return OracleDesc(wl.n, wl.k, mask, codec, wl.clip_alpha, wl.outlier_frac, wl.rank,
                      salient_channels=getattr(wl, "salient_channels", 0),
                      salient_log2=getattr(wl, "salient_log2", 0))


def _f32(v: float) -> float:
    """The fp64 value of the float32 nearest to v (descriptor fields are fp32)."""
    return float(np.float32(v))


# ---------------------------------------------------------------------------
# elementary rounding
# ---------------------------------------------------------------------------

def fp16_round(a) -> np.ndarray:
    """Round fp64 values to the nearest fp16 (ties to even); return them as fp64.

    The pages fix no scale dtype; fp16 is the reading taken for every stored
    scale, centroid and outlier value (SqueezeLLM keeps outliers in "FP16";
    SLiM's kernels run in FP16)."""
    return np.asarray(a, dtype=np.float64).astype(np.float16).astype(np.float64)


# ---------------------------------------------------------------------------
# outlier extraction (SqueezeLLM, "Approach": dense-and-sparse decomposition)
# ---------------------------------------------------------------------------

def n_outliers(desc: OracleDesc) -> int:
    """Number of CSR outliers: floor(f * N * K) with f the fp32 fraction.
    (Reading: floor, over the whole matrix.)"""
    if desc.outlier_frac <= 0:
        return 0
    return int(math.floor(_f32(desc.outlier_frac) * float(desc.n_out) * float(desc.k_in)))


def select_outliers(w: np.ndarray, count: int) -> np.ndarray:
    """Linear indices (ascending) of the ``count`` entries of largest |w|.

    Order: |w| descending, ties to the lower row-major index (reading: the
    pages name no tie rule).  The selection is global over the matrix."""
    if count <= 0:
        return np.zeros(0, dtype=np.int64)
    a = np.abs(np.asarray(w, dtype=np.float64)).reshape(-1)
    order = np.argsort(-a, kind="stable")
    return np.sort(order[:count])


# ---------------------------------------------------------------------------
# masks (SLiM rebuttal "Unstructured vs. 2:4 Sparsity"; magnitude pruning)
# ---------------------------------------------------------------------------

def mask_2of4(w: np.ndarray):
    """2:4 magnitude mask along K.

    In every aligned group of 4 consecutive columns of a row keep the 2 entries
    of largest |w|; ties go to the lower column (reading).  Returns
    (keep bool [N][K], pattern index p uint8 [N][K/4]) with
    PAIRS_2OF4[p] = (i0, i1) the kept positions."""
    a = np.abs(np.asarray(w, dtype=np.float64))
    n, k = a.shape
    g = a.reshape(n, k // 4, 4)
    # rank of element i inside its group: how many others precede it in the
    # order (|w| desc, index asc)
    ai = g[..., :, None]
    aj = g[..., None, :]
    idx = np.arange(4)
    before = (aj > ai) | ((aj == ai) & (idx[None, :] < idx[:, None]))
    rank = before.sum(axis=-1)
    keep_g = rank < 2
    keep = keep_g.reshape(n, k)
    # pattern index from the two kept positions
    pos = np.argsort(~keep_g, axis=-1, kind="stable")[..., :2]  # kept positions, ascending
    lut = np.full((4, 4), 255, dtype=np.uint8)
    for p, (i0, i1) in enumerate(PAIRS_2OF4):
        lut[i0, i1] = p
    pat = lut[pos[..., 0], pos[..., 1]]
    return keep, pat


def mask_bitmap50(w: np.ndarray) -> np.ndarray:
    """Unstructured 50% magnitude mask: per row keep the K/2 entries of largest
    |w|, ties to the lower column (reading: per row, not per layer; a random
    magnitude mask on random weights)."""
    a = np.abs(np.asarray(w, dtype=np.float64))
    n, k = a.shape
    order = np.argsort(-a, axis=1, kind="stable")
    keep = np.zeros((n, k), dtype=bool)
    np.put_along_axis(keep, order[:, : k // 2], True, axis=1)
    return keep


# ---------------------------------------------------------------------------
# uniform codec: SLiM-Quant style symmetric clipped round-to-nearest
# ---------------------------------------------------------------------------

def quantize_uniform(w: np.ndarray, bits: int, alpha: float,
                     exclude: Optional[np.ndarray] = None):
    """Symmetric clipped RTN with one scale per 128 consecutive columns.

    SLiM review summary, "SLIM-Quant": symmetric weight quantisation, weights
    clipped before rounding to the nearest integer.  Readings:
      * qmax = 2^(bits-1) - 1 (no -2^(bits-1) level, the grid is symmetric);
      * amax is taken over the group's non-outlier entries (all of them,
        before masking: quantise-first, which the pages' ablation finds
        equivalent; for magnitude masks the maximum is always kept anyway);
      * s = fp16( (alpha * amax) / qmax ), evaluated in fp64;
      * q = clamp(rint(w / s), -qmax, qmax), round half to even; s == 0 gives
        q == 0.
    Returns (q int8 [N][K], s fp64 [N][K/128] holding fp16 values)."""
    w = np.asarray(w, dtype=np.float64)
    n, k = w.shape
    qmax = (1 << (bits - 1)) - 1
    a = np.abs(w)
    if exclude is not None:
        a = np.where(exclude, 0.0, a)
    amax = a.reshape(n, k // GROUP, GROUP).max(axis=2)
    s = fp16_round((_f32(alpha) * amax) / float(qmax))
    sb = np.repeat(s, GROUP, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.rint(w / np.where(sb > 0, sb, 1.0))
    q = np.where(sb > 0, np.clip(r, -qmax, qmax), 0.0).astype(np.int8)
    return q, s


ALPHA_GRID = tuple(i / 100 for i in range(30, 101))   # candidate clip thresholds 0.30 .. 1.00
ALPHA_BINS = 1024


def clip_histogram(w: np.ndarray, keep: np.ndarray, exclude: Optional[np.ndarray] = None) -> np.ndarray:
    """Empirical distribution of the normalised magnitudes t = |w| / amax_g
    (amax_g over the group's non-outlier entries, as the codec takes it) of
    the entries the codec's error reaches: kept by the mask, not outliers, in
    groups with amax_g > 0.  Bin b = min(floor((|w| / amax_g) * 1024), 1023),
    evaluated in fp64.  Returns int64 counts [1024]."""
    a = np.abs(np.asarray(w, dtype=np.float64))
    n, k = a.shape
    ae = np.where(exclude, 0.0, a) if exclude is not None else a
    amax = np.repeat(ae.reshape(n, k // GROUP, GROUP).max(axis=2), GROUP, axis=1)
    use = keep & (amax > 0)
    if exclude is not None:
        use &= ~exclude
    with np.errstate(divide="ignore", invalid="ignore"):
        b = np.floor((a / np.where(amax > 0, amax, 1.0)) * ALPHA_BINS)
    b = np.minimum(b, ALPHA_BINS - 1).astype(np.int64)
    return np.bincount(b[use], minlength=ALPHA_BINS).astype(np.int64)


def alpha_objective(counts: np.ndarray, bits: int, alpha: float) -> float:
    """Expected squared error (in units of amax^2, up to the entry count) of
    symmetric clipped RTN with threshold alpha over the histogram: bin b
    stands for its centre c_b = (b + 1/2) / 1024, quantised to
    Q(c) = min(rint((c qmax) / alpha), qmax) * alpha / qmax; the sum
    sum_b count_b (c_b - Q(c_b))^2 runs over b in order (fp64; alpha is the
    fp32 value)."""
    qmax = float((1 << (bits - 1)) - 1)
    al = _f32(alpha)
    c = (np.arange(ALPHA_BINS, dtype=np.float64) + 0.5) / ALPHA_BINS
    q = np.minimum(np.rint((c * qmax) / al), qmax)
    d = c - (q * al) / qmax
    return float(np.cumsum(np.asarray(counts, dtype=np.float64) * (d * d))[-1])


def search_clip_alpha(counts: np.ndarray, bits: int) -> float:
    """SLiM-Quant's grid search: the candidate of ALPHA_GRID (as fp32) with
    the least alpha_objective, ties to the smaller alpha.  Readings: the
    pages give neither the grid nor the bin count; a layer-wide alpha (the
    descriptor holds one) from a 1024-bin histogram of |w| / amax_g over
    0.30 .. 1.00 in steps of 0.01."""
    best, best_v = None, None
    for a in ALPHA_GRID:
        v = alpha_objective(counts, bits, a)
        if best_v is None or v < best_v:
            best, best_v = a, v
    return float(np.float32(best))


# ---------------------------------------------------------------------------
# LUT codec: SqueezeLLM-style non-uniform per-row table
# ---------------------------------------------------------------------------

def lut_centroids(w: np.ndarray, bits: int, exclude: Optional[np.ndarray] = None) -> np.ndarray:
    """Per-row table of 2^bits centroids.

    SqueezeLLM "Approach": non-uniform LUT quantisation.  Readings (the
    sensitivity-weighted k-means needs gradients on data, which are not
    available): centroid j of a row is the linearly interpolated quantile of
    the row's non-outlier values at p_j = (j + 1/2) / 2^bits,
        h = (n_r - 1) p_j,  c_j = v[floor h] + (h - floor h)(v[floor h + 1] - v[floor h])
    with v the sorted values, evaluated in fp64 in exactly that order, then
    rounded to fp16.  A zero centroid is +0 (the sign of a zero from a sort
    is not defined).  A row with no values gets all-zero centroids.
    Returns fp64 [N][2^bits] holding fp16 values."""
    w = np.asarray(w, dtype=np.float64)
    n, k = w.shape
    nc = 1 << bits
    vals = np.where(exclude, np.inf, w) if exclude is not None else w.copy()
    v = np.sort(vals, axis=1)
    nr = (k - exclude.sum(axis=1)) if exclude is not None else np.full(n, k)
    out = np.zeros((n, nc), dtype=np.float64)
    rows = np.arange(n)
    for j in range(nc):
        p = (j + 0.5) / nc
        h = (nr - 1).astype(np.float64) * p
        lo = np.floor(h).astype(np.int64)
        lo = np.clip(lo, 0, k - 1)
        frac = h - np.floor(h)
        hi = np.minimum(lo + 1, np.maximum(nr - 1, 0))
        vlo = v[rows, lo]
        vhi = v[rows, hi]
        c = vlo + frac * (vhi - vlo)
        out[:, j] = np.where(nr > 0, c, 0.0) + 0.0      # -0 -> +0
    return fp16_round(out)


KMEANS_MAX_ITERS = 32


def fisher_kmeans(w: np.ndarray, cent0: np.ndarray, fisher: np.ndarray,
                  exclude: Optional[np.ndarray] = None, max_iters: int = KMEANS_MAX_ITERS,
                  round_fp16: bool = True) -> np.ndarray:
    """Sensitivity-weighted k-means of every row (SqueezeLLM "Approach":
    centroids weighted by the diagonal Fisher information).

    Lloyd iterations from the initial table cent0 [N][2^b]: each non-outlier
    value of the row goes to its nearest centroid (fp64 |v - c_j|, ties to the
    lower j); each centroid becomes sum f v / sum f over its members (f the
    fp32 Fisher diagonal; a centroid with no weight keeps its value).  A row
    stops when an assignment repeats the previous one, or after max_iters
    updates.  Readings: the initial table is the quantile table; sums run in
    column order (sequentially, fp64, products f v exact); the result is
    rounded to fp16 (+0 for a zero).  Returns fp64 [N][2^b] of fp16 values
    (unrounded fp64 with round_fp16=False)."""
    v = np.asarray(w, dtype=np.float64)
    f = np.asarray(fisher, dtype=np.float32).astype(np.float64)
    n, k = v.shape
    c = np.array(cent0, dtype=np.float64, copy=True)
    nc = c.shape[1]
    member = np.ones((n, k), dtype=bool) if exclude is None else ~exclude
    fv = f * v
    prev = None
    active = np.ones(n, dtype=bool)
    for _ in range(max_iters):
        best = np.abs(v - c[:, 0:1])
        asg = np.zeros((n, k), dtype=np.int64)
        for j in range(1, nc):
            dj = np.abs(v - c[:, j:j + 1])
            better = dj < best                           # strict: ties to the lower j
            asg[better] = j
            best = np.where(better, dj, best)
        if prev is not None:
            same = np.all((asg == prev) | ~member, axis=1)
            active &= ~same
        if not active.any():
            break
        for j in range(nc):
            m = member & (asg == j)
            num = np.cumsum(np.where(m, fv, 0.0), axis=1)[:, -1]
            den = np.cumsum(np.where(m, f, 0.0), axis=1)[:, -1]
            upd = active & (den > 0)
            c[upd, j] = num[upd] / den[upd]
        prev = asg
    return fp16_round(c) + 0.0 if round_fp16 else c


def lut_assign(w: np.ndarray, cent: np.ndarray) -> np.ndarray:
    """Code of every entry: the centroid at least |w - c_j| (fp64), ties to the
    lower j (reading).  Outliers are assigned too; the CSR stores the
    residual."""
    w = np.asarray(w, dtype=np.float64)
    best = np.abs(w - cent[:, 0:1])
    code = np.zeros(w.shape, dtype=np.uint8)
    for j in range(1, cent.shape[1]):
        d = np.abs(w - cent[:, j:j + 1])
        upd = d < best
        code[upd] = j
        best = np.where(upd, d, best)
    return code


# ---------------------------------------------------------------------------
# adapters: AbsMax int4 in groups of 128 (SLiM "Low-rank adapter quantization")
# ---------------------------------------------------------------------------

def _absmax_q(v: np.ndarray, bits: int):
    """AbsMax symmetric quantisation of each row of ``v`` (one scale per row):
    s = fp16(amax / qmax) in fp64, q = clamp(rint(v / s), -qmax, qmax)."""
    qmax = (1 << (bits - 1)) - 1
    amax = np.abs(v).max(axis=1)
    s = fp16_round(amax / float(qmax))
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.rint(v / np.where(s > 0, s, 1.0)[:, None])
    q = np.where((s > 0)[:, None], np.clip(r, -qmax, qmax), 0.0).astype(np.int8)
    return q, s


def quantize_adapter_rows(R: np.ndarray, bits: int = 4):
    """R_q: R is [r][K]; groups are 128 consecutive K entries of one row j
    (reading: groups run along the model dimension).  Returns
    (q int8 [r][K], s fp64 [r][K/128])."""
    R = np.asarray(R, dtype=np.float64)
    r, k = R.shape
    q, s = _absmax_q(R.reshape(r * (k // GROUP), GROUP), bits)
    return q.reshape(r, k), s.reshape(r, k // GROUP)


def quantize_adapter_cols(L: np.ndarray, bits: int = 4):
    """L_q: L is [N][r]; groups are 128 consecutive N entries of one column j.
    Returns (q int8 [N][r], s fp64 [N/128][r])."""
    L = np.asarray(L, dtype=np.float64)
    n, r = L.shape
    t = L.reshape(n // GROUP, GROUP, r).transpose(0, 2, 1).reshape(-1, GROUP)
    q, s = _absmax_q(t, bits)
    q = q.reshape(n // GROUP, r, GROUP).transpose(0, 2, 1).reshape(n, r)
    return q, s.reshape(n // GROUP, r)


# ---------------------------------------------------------------------------
# CSR of outliers
# ---------------------------------------------------------------------------

def build_csr(w: np.ndarray, out_idx: np.ndarray, dense_val: np.ndarray):
    """CSR of the outliers.  Value = fp16(w - dense part at that position)
    (reading: the sparse and dense parts add back to the original outlier, the
    dense-and-sparse decomposition's intent).  Rows ascending, columns
    ascending within a row.  Returns (row_ptr int64 [N+1], col int64, val fp64)."""
    n, k = w.shape
    rows = out_idx // k
    cols = out_idx % k
    w64 = np.asarray(w, dtype=np.float64).reshape(-1)
    val = fp16_round(w64[out_idx] - dense_val.reshape(-1)[out_idx])
    counts = np.bincount(rows, minlength=n)
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    return row_ptr, cols.astype(np.int64), val  # out_idx is sorted: row-major order


# ---------------------------------------------------------------------------
# salient-channel scaling (SLiM rebuttal, "Output Error Minimization in
# SLiM-Quant"; the variant is called SLiM^O there)
# ---------------------------------------------------------------------------

SALIENT_ROW_BLOCK = 64      # rows per partial sum of a channel's |w|


def channel_saliency(w: np.ndarray, act_absmean: np.ndarray) -> np.ndarray:
    """Saliency of every input channel c: mean|x_c| * sum_n |w[n, c]|, fp64.

    The page defines it as the product of the normalised average magnitudes
    of the channel's activations and weights.  Dividing either factor by a
    positive constant (its mean, its maximum, or N for the weight average)
    does not change which channels rank highest, so the plain product of the
    activation statistic and the column's |w| sum is kept (reading).  The
    activation statistic is an input (measured on calibration data by the
    caller; synthetic here), taken as float32 and widened exactly.

    Summation order (fixed so that an implementation can reproduce the fp64
    result bit for bit): rows in consecutive blocks of 64, each block summed
    from its first row on, then the block sums added from the first block
    on."""
    w = np.abs(np.asarray(w, dtype=np.float64))
    n, k = w.shape
    assert n % SALIENT_ROW_BLOCK == 0
    nb = n // SALIENT_ROW_BLOCK
    blocks = w.reshape(nb, SALIENT_ROW_BLOCK, k)
    part = np.zeros((nb, k))
    for i in range(SALIENT_ROW_BLOCK):
        part += blocks[:, i, :]
    colsum = np.zeros(k)
    for b in range(nb):
        colsum += part[b]
    a = np.asarray(act_absmean, dtype=np.float32).astype(np.float64)
    assert a.shape == (k,)
    return a * colsum


def select_salient_channels(w: np.ndarray, act_absmean: np.ndarray, count: int) -> np.ndarray:
    """Ascending indices of the ``count`` channels of highest saliency (ties
    to the lower channel index; reading: the page names no tie rule)."""
    sal = channel_saliency(w, act_absmean)
    order = np.lexsort((np.arange(sal.size), -sal))   # saliency descending, then index
    return np.sort(order[:count]).astype(np.int64)


def scale_activations(x: np.ndarray, salient: np.ndarray, log2: int) -> np.ndarray:
    """x with the salient channels divided by the factor 2**log2 (the inverse
    of the weights' scaling; exact in fp64)."""
    x = np.array(x, dtype=np.float64, copy=True)
    x[:, salient] = x[:, salient] / float(2 ** log2)
    return x


# ---------------------------------------------------------------------------
# the whole encoding
# ---------------------------------------------------------------------------

def compress(desc: OracleDesc, w: np.ndarray, L: Optional[np.ndarray] = None,
             R: Optional[np.ndarray] = None, act_absmean: Optional[np.ndarray] = None,
             fisher: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Run the encoding steps in order: (SLiM^O) salient-channel scaling,
    outliers, mask, codec, CSR, adapters.

    With ``desc.salient_channels`` > 0 the chosen columns of W are multiplied
    by 2**salient_log2 before every other step, which then all work on the
    scaled matrix W'; the forward pass divides the same activation channels
    by the factor, so W' x' = W x before compression.  (Reading: the page
    leaves the factor's value unstated; a power of two keeps both scalings
    exact.  The adapters L, R are taken as given, acting on x'.)

    Returns the decoded parts the forward pass needs plus the raw codes the
    packer serialises."""
    w = np.asarray(w, dtype=np.float64)
    n, k = w.shape
    assert (n, k) == (desc.n_out, desc.k_in)
    parts: Dict[str, np.ndarray] = {}
    if desc.salient_channels > 0:
        assert act_absmean is not None and desc.salient_log2 > 0
        sal = select_salient_channels(w, act_absmean, desc.salient_channels)
        w = w.copy()
        w[:, sal] = w[:, sal] * float(2 ** desc.salient_log2)
        parts["salient"] = sal
        parts["salient_log2"] = np.int64(desc.salient_log2)
    ns = n_outliers(desc)
    out_idx = select_outliers(w, ns)
    is_out = np.zeros(n * k, dtype=bool)
    is_out[out_idx] = True
    is_out = is_out.reshape(n, k)
    parts["out_idx"] = out_idx

    # mask on the original magnitudes
    if desc.mask == MASK_2_4:
        keep, pat = mask_2of4(w)
        parts["pattern"] = pat
    elif desc.mask == MASK_BITMAP50:
        keep = mask_bitmap50(w)
    else:
        keep = np.ones((n, k), dtype=bool)
    parts["keep"] = keep

    bits = _CODEC_BITS[desc.codec]
    if desc.codec in (CODEC_INT4, CODEC_INT3):
        alpha = desc.clip_alpha
        if alpha == 0:                                  # SLiM-Quant alpha search
            alpha = search_clip_alpha(clip_histogram(w, keep, is_out if ns else None), bits)
        parts["clip_alpha"] = np.float64(np.float32(alpha))
        q, s = quantize_uniform(w, bits, alpha, exclude=is_out if ns else None)
        dense = np.where(keep, q.astype(np.float64) * np.repeat(s, GROUP, axis=1), 0.0)
        parts["q"] = q
        parts["scales"] = s
        parts["codes"] = (q.astype(np.int16) + (1 << (bits - 1))).astype(np.uint8)
    else:
        cent = lut_centroids(w, bits, exclude=is_out if ns else None)
        if fisher is not None:                          # SqueezeLLM sensitivity-weighted k-means
            cent = fisher_kmeans(w, cent, fisher, exclude=is_out if ns else None)
        code = lut_assign(w, cent)
        dense = np.where(keep, np.take_along_axis(cent, code.astype(np.int64), axis=1), 0.0)
        parts["centroids"] = cent
        parts["codes"] = code
    parts["w_dense"] = dense

    if desc.outlier_frac > 0:
        rp, col, val = build_csr(w, out_idx, dense)
        parts["csr_row_ptr"], parts["csr_col"], parts["csr_val"] = rp, col, val

    if desc.rank > 0:
        assert L is not None and R is not None
        rq, rs = quantize_adapter_rows(R, desc.adapter_bits)
        lq, ls = quantize_adapter_cols(L, desc.adapter_bits)
        parts["R_q"], parts["R_s"], parts["L_q"], parts["L_s"] = rq, rs, lq, ls
        parts["R_hat"] = rq.astype(np.float64) * np.repeat(rs, GROUP, axis=1)
        parts["L_hat"] = lq.astype(np.float64) * np.repeat(ls, GROUP, axis=0)
    return parts


# ---------------------------------------------------------------------------
# forward pass (fp64)
# ---------------------------------------------------------------------------

def forward_terms(parts: Dict[str, np.ndarray], x: np.ndarray, rows=None):
    """The three terms of y separately, in fp64.  x is [B][K].

    ``rows`` optionally restricts the output to a subset of output rows (used
    for sampled parity at full size).  Returns (main, csr, lowrank), each
    [B][len(rows)].  A SLiM^O layer first divides its salient activation
    channels by the factor."""
    x = np.asarray(x, dtype=np.float64)
    if "salient" in parts:
        x = scale_activations(x, parts["salient"], int(parts["salient_log2"]))
    wd = parts["w_dense"]
    sel = np.arange(wd.shape[0]) if rows is None else np.asarray(rows)
    main = x @ wd[sel].T
    csr = np.zeros_like(main)
    if "csr_row_ptr" in parts:
        rp, col, val = parts["csr_row_ptr"], parts["csr_col"], parts["csr_val"]
        for oi, n in enumerate(sel):
            a, b = rp[n], rp[n + 1]
            if b > a:
                csr[:, oi] = x[:, col[a:b]] @ val[a:b]
    lr = np.zeros_like(main)
    if "R_hat" in parts:
        t = x @ parts["R_hat"].T                      # [B][r]
        lr = t @ parts["L_hat"][sel].T                # [B][rows]
    return main, csr, lr


def forward(parts: Dict[str, np.ndarray], x: np.ndarray, rows=None, flags: int = 0) -> np.ndarray:
    """y = main + csr + lowrank (fp64).  ``flags`` drops terms like the C
    descriptor's term toggles (bit 0 main, bit 1 csr, bit 2 low-rank)."""
    m, c, l = forward_terms(parts, x, rows)
    y = np.zeros_like(m)
    if not flags & 1:
        y += m
    if not flags & 2:
        y += c
    if not flags & 4:
        y += l
    return y


def dense_reconstruction(parts: Dict[str, np.ndarray]) -> np.ndarray:
    """W_hat = deq(Q (.) M) + S + deq(L) deq(R) as one dense fp64 matrix, in
    the original channel scale (a SLiM^O layer's salient columns divided by
    the factor), so that forward(x) = x W_hat^T."""
    wd = parts["w_dense"].copy()
    if "csr_row_ptr" in parts:
        rp, col, val = parts["csr_row_ptr"], parts["csr_col"], parts["csr_val"]
        rows = np.repeat(np.arange(len(rp) - 1), np.diff(rp))
        np.add.at(wd, (rows, col), val)
    if "R_hat" in parts:
        wd = wd + parts["L_hat"] @ parts["R_hat"]
    if "salient" in parts:
        sal = parts["salient"]
        wd[:, sal] = wd[:, sal] / float(2 ** int(parts["salient_log2"]))
    return wd


# ---------------------------------------------------------------------------
# adapter construction (SLiM review summary, "SLIM-LoRA"; rebuttal,
# "Assumptions in Theoretical Derivations")
# ---------------------------------------------------------------------------

def compressed_matrix(parts: Dict[str, np.ndarray]) -> np.ndarray:
    """W_C: what the sparse quantised part and the CSR outliers represent,
    in the space the codec encoded (W' for a SLiM^O layer), fp64.  The
    adapters are built to compensate W(') - W_C."""
    wd = parts["w_dense"].copy()
    if "csr_row_ptr" in parts:
        rp, col, val = parts["csr_row_ptr"], parts["csr_col"], parts["csr_val"]
        rows = np.repeat(np.arange(len(rp) - 1), np.diff(rp))
        np.add.at(wd, (rows, col), val)
    return wd


def slim_lora(err: np.ndarray, rank: int, act_absmean: Optional[np.ndarray] = None):
    """Rank-r adapters (L [N][r], R [r][K]) of the compression error
    E = W - W_C.

    SLiM-LoRA: with F(M) = M diag(xbar) (xbar the layer's average input
    magnitude, positive, so F is additive and invertible), minimise
    ||F(E - L R)||_F; by Eckart-Young the optimum is L R = F^-1((F(E))_r),
    (.)_r the rank-r truncated SVD.  Reading of the garbled formulas: F
    scales the input columns by xbar, and the singular values are split as
    L = U_r Sigma_r^(1/2), R = Sigma_r^(1/2) V_r^T diag(xbar)^-1 (the page
    fixes only the product).  Naive-LoRA (act_absmean None): xbar = 1."""
    e = np.asarray(err, dtype=np.float64)
    k = e.shape[1]
    xbar = np.ones(k) if act_absmean is None else np.asarray(act_absmean, dtype=np.float32).astype(np.float64)
    assert (xbar > 0).all()
    u, sv, vt = np.linalg.svd(e * xbar[None, :], full_matrices=False)
    root = np.sqrt(sv[:rank])
    L = u[:, :rank] * root[None, :]
    R = (root[:, None] * vt[:rank]) / xbar[None, :]
    return L, R


def build_adapters(desc: OracleDesc, w: np.ndarray, act_absmean: Optional[np.ndarray] = None,
                   naive: bool = False):
    """SLiM-LoRA (or Naive-LoRA) adapters of rank desc.rank for W.

    Compresses W without adapters (every encoding step but the last), forms
    E = W(') - W_C in the space the codec encoded, and returns slim_lora(E).
    The saliency weight is the average input the adapters see: act_absmean,
    divided by the factor on a SLiM^O layer's salient channels (reading)."""
    d0 = OracleDesc(desc.n_out, desc.k_in, desc.mask, desc.codec, desc.clip_alpha, desc.outlier_frac, 0,
                    salient_channels=desc.salient_channels, salient_log2=desc.salient_log2)
    parts = compress(d0, w, act_absmean=act_absmean)
    wp = np.array(w, dtype=np.float64, copy=True)
    xbar = None if act_absmean is None else np.asarray(act_absmean, dtype=np.float32).astype(np.float64)
    if "salient" in parts:
        f = float(2 ** desc.salient_log2)
        wp[:, parts["salient"]] *= f
        if xbar is not None:
            xbar[parts["salient"]] /= f
    err = wp - compressed_matrix(parts)
    return slim_lora(err, desc.rank, None if naive else xbar)


def lowrank_objective(err: np.ndarray, L: np.ndarray, R: np.ndarray, act_absmean=None) -> float:
    """||F(E - L R)||_F^2 with F as in slim_lora."""
    e = np.asarray(err, dtype=np.float64)
    xbar = np.ones(e.shape[1]) if act_absmean is None else np.asarray(act_absmean, dtype=np.float32).astype(np.float64)
    d = (e - np.asarray(L, dtype=np.float64) @ np.asarray(R, dtype=np.float64)) * xbar[None, :]
    return float(np.sum(d * d))


def rel_err(y: np.ndarray, ref: np.ndarray) -> float:
    """max_i |y_i - r_i| / max(|r_i|, rms(r)) -- the error metric of the
    parity tests (reading of "max relative error": plain |r_i| is undefined
    near zero, so it is floored at the rms of the reference)."""
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    den = np.maximum(np.abs(ref), rms)
    den = np.where(den > 0, den, 1.0)
    return float(np.max(np.abs(y - ref) / den)) if ref.size else 0.0


# ---------------------------------------------------------------------------
# packed byte layout (the specification in include/cql.h, re-derived here)
# ---------------------------------------------------------------------------

HEADER_BYTES = 512
FORMAT_VERSION = 2
NPLANES = 13
(P_HEADER, P_VALUES, P_META, P_SCALES, P_VOFF, P_CSR_ROWPTR, P_CSR_COL,
 P_CSR_VAL, P_R_VALUES, P_R_SCALES, P_L_VALUES, P_L_SCALES, P_SALIENT) = range(NPLANES)


def _pad16(x: int) -> int:
    return (x + 15) // 16 * 16


def _align256(x: int) -> int:
    return (x + 255) // 256 * 256


def _kept_per_row(desc: OracleDesc) -> int:
    return desc.k_in // 2 if desc.mask in (MASK_2_4, MASK_BITMAP50) else desc.k_in


def _row_bytes(desc: OracleDesc) -> Dict[int, int]:
    """Bytes each row contributes to each interleaved plane (padded to 16)."""
    k, r = desc.k_in, desc.rank
    bits = _CODEC_BITS[desc.codec]
    rb = {P_VALUES: _pad16((_kept_per_row(desc) * bits + 7) // 8)}
    rb[P_META] = _pad16(k // 8) if desc.mask in (MASK_2_4, MASK_BITMAP50) else 0
    if desc.codec in (CODEC_INT4, CODEC_INT3):
        rb[P_SCALES] = _pad16(2 * (k // GROUP))
    else:
        rb[P_SCALES] = 2 * (1 << bits)
    rb[P_VOFF] = _pad16(2 * (k // GROUP)) if desc.mask == MASK_BITMAP50 else 0
    rb[P_R_VALUES] = k // 2 if r else 0
    rb[P_R_SCALES] = _pad16(2 * (k // GROUP)) if r else 0
    rb[P_L_VALUES] = _pad16(r // 2) if r else 0
    return rb


def packed_layout(desc: OracleDesc, nnz: Optional[int] = None) -> dict:
    """Offsets and lengths of every plane.  Planes follow the header in index
    order, each starting on a 256-byte boundary; absent planes have length 0."""
    n, k, r = desc.n_out, desc.k_in, desc.rank
    if nnz is None:
        nnz = n_outliers(desc)
    rb = _row_bytes(desc)
    rpad = (r + ROWBLK - 1) // ROWBLK * ROWBLK
    ln = [0] * NPLANES
    ln[P_HEADER] = HEADER_BYTES
    ln[P_VALUES] = n * rb[P_VALUES]
    ln[P_META] = n * rb[P_META]
    ln[P_SCALES] = n * rb[P_SCALES]
    ln[P_VOFF] = n * rb[P_VOFF]
    if desc.outlier_frac > 0:
        ln[P_CSR_ROWPTR] = 4 * (n + 1)
        ln[P_CSR_COL] = 2 * nnz
        ln[P_CSR_VAL] = 2 * nnz
    if r:
        ln[P_R_VALUES] = rpad * rb[P_R_VALUES]
        ln[P_R_SCALES] = rpad * rb[P_R_SCALES]
        ln[P_L_VALUES] = n * rb[P_L_VALUES]
        ln[P_L_SCALES] = 2 * (n // GROUP) * r
    ln[P_SALIENT] = 2 * desc.salient_channels
    off = [0] * NPLANES
    pos = 0
    for i in range(NPLANES):
        pos = _align256(pos)
        off[i] = pos
        pos += ln[i]
    total = _align256(pos)
    return {"off": off, "len": ln, "total": total, "nnz": nnz, "row_bytes": rb}


def _bitstream(codes: np.ndarray, bits: int, row_bytes: int) -> np.ndarray:
    """Row-wise little-endian bit stream: code i of a row occupies stream bits
    [bits*i, bits*i + bits), stream bit j is bit (j mod 8) of byte j // 8.
    Rows are zero-padded to ``row_bytes``."""
    n, m = codes.shape
    c = codes.astype(np.uint8)
    bit_planes = ((c[:, :, None] >> np.arange(bits, dtype=np.uint8)) & 1).reshape(n, m * bits)
    packed = np.packbits(bit_planes, axis=1, bitorder="little")
    out = np.zeros((n, row_bytes), dtype=np.uint8)
    out[:, : packed.shape[1]] = packed
    return out


def _interleave(rows: np.ndarray) -> np.ndarray:
    """Row-interleaved layout: rows in blocks of 32; block b is a run of
    512-byte slabs, slab s holding bytes [16 s, 16 s + 16) of each of the 32
    rows, row by row.  Byte j of row i sits at
        ((i // 32) * (row_bytes // 16) + j // 16) * 512 + (i % 32) * 16 + j % 16."""
    n, rb = rows.shape
    assert n % ROWBLK == 0 and rb % SLAB == 0
    t = rows.reshape(n // ROWBLK, ROWBLK, rb // SLAB, SLAB).transpose(0, 2, 1, 3)
    return np.ascontiguousarray(t).reshape(-1)


def _u16le(a: np.ndarray) -> np.ndarray:
    """uint16 [..., m] -> its little-endian bytes uint8 [..., 2m]."""
    return np.ascontiguousarray(np.asarray(a, dtype="<u2")).view(np.uint8)


def _f16_bits(v: np.ndarray) -> np.ndarray:
    return np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)


def _header(desc: OracleDesc, lay: dict, alpha=None) -> np.ndarray:
    d = struct.pack(
        "<iiiiiffiiiIii12x",
        desc.n_out, desc.k_in, desc.mask, desc.codec, desc.group,
        np.float32(desc.clip_alpha if alpha is None else alpha), np.float32(desc.outlier_frac), desc.rank,
        desc.adapter_bits, desc.adapter_group, desc.flags, desc.salient_channels, desc.salient_log2)
    assert len(d) == 64
    body = b"CQL1" + struct.pack("<I", FORMAT_VERSION) + d
    body += struct.pack("<QQ", lay["total"], lay["nnz"])
    body += struct.pack(f"<{NPLANES}Q", *lay["off"]) + struct.pack(f"<{NPLANES}Q", *lay["len"])
    out = np.zeros(HEADER_BYTES, dtype=np.uint8)
    out[: len(body)] = np.frombuffer(body, dtype=np.uint8)
    return out


def pack_bytes(desc: OracleDesc, parts: Dict[str, np.ndarray]) -> np.ndarray:
    """Serialise the encoding into the packed buffer (uint8 [total])."""
    n, k, r = desc.n_out, desc.k_in, desc.rank
    nnz = len(parts["out_idx"]) if desc.outlier_frac > 0 else 0
    lay = packed_layout(desc, nnz)
    rb = lay["row_bytes"]
    buf = np.zeros(lay["total"], dtype=np.uint8)

    def put(plane, data):
        data = np.asarray(data, dtype=np.uint8).reshape(-1)
        assert data.size == lay["len"][plane], (plane, data.size, lay["len"][plane])
        buf[lay["off"][plane]: lay["off"][plane] + data.size] = data

    put(P_HEADER, _header(desc, lay, parts.get("clip_alpha")))
    bits = _CODEC_BITS[desc.codec]
    keep = parts["keep"]
    codes = parts["codes"]
    kept = _kept_per_row(desc)
    if desc.mask == MASK_NONE:
        kept_codes = codes
    else:
        kept_codes = codes[keep].reshape(n, kept)   # row-major boolean index keeps column order
    put(P_VALUES, _interleave(_bitstream(kept_codes, bits, rb[P_VALUES])))
    if desc.mask == MASK_2_4:
        nib = np.asarray(META_NIBBLE_2OF4, dtype=np.uint8)[parts["pattern"]]
        put(P_META, _interleave(_bitstream(nib, 4, rb[P_META])))
    elif desc.mask == MASK_BITMAP50:
        put(P_META, _interleave(_bitstream(keep.astype(np.uint8), 1, rb[P_META])))
    if desc.codec in (CODEC_INT4, CODEC_INT3):
        sc = _u16le(_f16_bits(parts["scales"]))
    else:
        sc = _u16le(_f16_bits(parts["centroids"]))
    sc_rows = np.zeros((n, rb[P_SCALES]), dtype=np.uint8)
    sc_rows[:, : sc.shape[1]] = sc
    put(P_SCALES, _interleave(sc_rows))
    if desc.mask == MASK_BITMAP50:
        cnt = keep.reshape(n, k // GROUP, GROUP).sum(axis=2)
        voff = np.zeros((n, k // GROUP), dtype=np.int64)
        voff[:, 1:] = np.cumsum(cnt, axis=1)[:, :-1]
        vrows = np.zeros((n, rb[P_VOFF]), dtype=np.uint8)
        vb = _u16le(voff.astype(np.uint16))
        vrows[:, : vb.shape[1]] = vb
        put(P_VOFF, _interleave(vrows))
    if desc.outlier_frac > 0:
        put(P_CSR_ROWPTR, np.asarray(parts["csr_row_ptr"], dtype="<i4").view(np.uint8))
        put(P_CSR_COL, np.asarray(parts["csr_col"], dtype="<u2").view(np.uint8))
        put(P_CSR_VAL, _f16_bits(parts["csr_val"]).astype("<u2").view(np.uint8))
    if r:
        rpad = (r + ROWBLK - 1) // ROWBLK * ROWBLK
        rc = np.zeros((rpad, k), dtype=np.uint8)
        rc[:r] = (parts["R_q"].astype(np.int16) + 8).astype(np.uint8)
        rrows = _bitstream(rc, 4, rb[P_R_VALUES])
        rrows[r:] = 0
        put(P_R_VALUES, _interleave(rrows))
        rs = np.zeros((rpad, rb[P_R_SCALES]), dtype=np.uint8)
        rsb = _u16le(_f16_bits(parts["R_s"]))
        rs[:r, : rsb.shape[1]] = rsb
        put(P_R_SCALES, _interleave(rs))
        lc = (parts["L_q"].astype(np.int16) + 8).astype(np.uint8)
        put(P_L_VALUES, _interleave(_bitstream(lc, 4, rb[P_L_VALUES])))
        put(P_L_SCALES, _u16le(_f16_bits(parts["L_s"])).reshape(-1))
    if desc.salient_channels > 0:
        put(P_SALIENT, _u16le(parts["salient"].astype(np.uint16)))
    return buf


def pack_and_forward(desc: OracleDesc, w, L, R, x, act_absmean=None, fisher=None):
    """Convenience: (packed bytes, parts, y fp64)."""
    parts = compress(desc, w, L, R, act_absmean, fisher)
    return pack_bytes(desc, parts), parts, forward(parts, x)
