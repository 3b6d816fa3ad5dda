"""Synthetic workloads shaped like the layers the pages measure.

The pages evaluate on LLaMA / OPT checkpoints and on C4 / WikiText2 text,
none of which exists on this machine.  These generators stand in for them with
random weights of the same shapes (LLaMA-7B attention and MLP projections) and
the same value structure the workload descriptions ask for:

* Gaussian weights of standard deviation 0.02 with a small fraction of entries
  multiplied by 20 (heavy outliers, the situation SqueezeLLM's dense-and-sparse
  split and SLiM's clipping are designed for);
* Student-t(4) weights for the dense-and-sparse LUT workload (heavier tails);
* rank-r adapter factors drawn as 0.01 N(0, 1);
* activations drawn as N(0, 1);
* for the output-error (SLiM^O) variant, a per-channel activation statistic
  mean|x_c| drawn as exp(0.5 N(0, 1)) with 0.5% of the channels multiplied by
  30 (the few "massive" activation channels LLMs show), from its own stream
  (PCG64 seeded with (seed, 1)) so the other draws are unchanged;
* for the sensitivity-weighted LUT (SqueezeLLM), a diagonal Fisher
  information drawn as squared N(0, 1) gradients (chi-square, 1 degree of
  freedom; heavy-tailed positive weights), stream (seed, 2).

Every array is drawn from ``numpy.random.default_rng(seed)`` (PCG64) in a fixed
order: W, the spike positions, L, R, x.  Nothing here masks, quantises or
multiplies: rounding an input to the dtype it is delivered in (bf16 or fp16) is
the only transformation.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Dict, Optional, Tuple

import numpy as np


# ----------------------------------------------------------------------------
# storage-type helpers (input delivery only)
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return the
    16-bit patterns.  NaN is not produced by the generators and not handled."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    u = u + np.uint32(0x7FFF) + lsb          # finite inputs: no 32-bit overflow
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to the fp32 values they denote (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _deliver(a64: np.ndarray, dtype: str) -> Tuple[np.ndarray, Optional[np.ndarray]]:
    """Round fp64 draws to the delivery dtype.

    Returns (values as float32 holding the exact delivered values, raw 16-bit
    patterns or None for fp32)."""
    if dtype == "f32":
        return a64.astype(np.float32), None
    if dtype == "f16":
        h = a64.astype(np.float16)
        return h.astype(np.float32), h.view(np.uint16)
    if dtype == "bf16":
        bits = f32_to_bf16_bits(a64.astype(np.float32))
        return bf16_bits_to_f32(bits), bits
    raise ValueError(f"unknown dtype {dtype!r}")


# ----------------------------------------------------------------------------
# workload descriptions
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    """One synthetic layer: shapes, value recipe and compression settings."""

    name: str
    seed: int
    n: int                      # output rows N
    k: int                      # input columns K
    w_dist: str = "normal"      # "normal" or "student_t4"
    w_std: float = 0.02
    w_dtype: str = "f32"        # dtype W is delivered in: "f32" or "bf16"
    spike_frac: float = 0.0     # fraction of W entries multiplied by spike_mult
    spike_mult: float = 20.0
    mask: str = "2:4"           # "2:4", "bitmap50", "none"
    codec: str = "int4"         # "int4", "int3", "lut3", "lut4"
    clip_alpha: float = 0.9
    outlier_frac: float = 0.0   # fraction of entries sent to the CSR matrix
    rank: int = 0
    lr_std: float = 0.01
    x_dtype: str = "bf16"       # "f16" or "bf16"
    batches: Tuple[int, ...] = (1,)
    note: str = ""
    salient_channels: int = 0   # SLiM^O: channels scaled (0 = plain SLiM)
    salient_log2: int = 0       # SLiM^O: factor 2**salient_log2
    fisher: bool = False        # draw a Fisher diagonal (LUT k-means weights)


WORKLOADS: Dict[str, Workload] = {
    # Tiny single layer: small enough for pure-Python brute force.
    "tiny": Workload(
        name="tiny", seed=0, n=256, k=512, w_dtype="f32",
        spike_frac=0.005, mask="2:4", codec="int4", clip_alpha=0.9,
        rank=16, x_dtype="f16", batches=(1,),
        note="W 256x512 fp32 0.02N(0,1), 0.5% of entries x20; 2:4; int4 g128 "
             "clip 0.9; rank-16 int4 adapters; x fp16 batch 1"),
    # LLaMA-7B MLP up/gate projection, decode.
    "mlp_up": Workload(
        name="mlp_up", seed=2, n=11008, k=4096, w_dtype="bf16",
        spike_frac=0.001, mask="2:4", codec="int4", clip_alpha=0.9,
        rank=128, x_dtype="bf16", batches=(1, 4, 16),
        note="W 11008x4096 bf16 0.02N(0,1) + 0.1% entries x20; 2:4; int4 g128 "
             "clip 0.9; rank-128 int4 adapters; x bf16 batch 1/4/16"),
    # SqueezeLLM-style dense-and-sparse decode.
    "lut_dense_sparse": Workload(
        name="lut_dense_sparse", seed=3, n=4096, k=4096, w_dist="student_t4",
        w_dtype="f32", mask="none", codec="lut3", outlier_frac=0.0045,
        rank=0, x_dtype="f16", batches=(1, 8),
        note="W 4096x4096 0.02 Student-t(4); 3-bit per-row LUT; top 0.45% |w| "
             "to fp16 CSR; no mask; x fp16 batch 1/8"),
    # LLaMA-7B down projection with an unstructured 50% mask.
    "down_unstructured": Workload(
        name="down_unstructured", seed=4, n=4096, k=11008, w_dtype="f32",
        mask="bitmap50", codec="int3", clip_alpha=0.9, rank=64,
        x_dtype="bf16", batches=(1, 2, 4, 8, 16),
        note="W 4096x11008 fp32 0.02N(0,1); per-row magnitude 50% bitmap; "
             "int3 g128 clip 0.9; rank-64 adapters; x bf16 batch 1..16"),
    # Prefill GEMMs, 2048 tokens.
    "prefill_up": Workload(
        name="prefill_up", seed=5, n=11008, k=4096, w_dtype="bf16",
        mask="2:4", codec="int4", clip_alpha=0.9, rank=64, x_dtype="bf16",
        batches=(2048,),
        note="2048 tokens x (4096 -> 11008); 2:4 int4 g128 + rank-64 adapters"),
    # Output-error variant (SLiM^O) of the MLP up projection: the 1% most
    # salient input channels (41 of 4096) scaled by 2.
    "mlp_up_slimo": Workload(
        name="mlp_up_slimo", seed=7, n=11008, k=4096, w_dtype="bf16",
        spike_frac=0.001, mask="2:4", codec="int4", clip_alpha=0.9,
        rank=128, x_dtype="bf16", batches=(1, 16), salient_channels=41, salient_log2=1,
        note="mlp_up with SLiM^O: top 1% salient channels (41) x2, activations /2"),
    "prefill_down": Workload(
        name="prefill_down", seed=6, n=4096, k=11008, w_dtype="bf16",
        mask="2:4", codec="int4", clip_alpha=0.9, rank=64, x_dtype="bf16",
        batches=(2048,),
        note="2048 tokens x (11008 -> 4096); 2:4 int4 g128 + rank-64 adapters"),
}


def workload(name: str, **overrides) -> Workload:
    """Look up a named workload, optionally overriding fields (e.g. sizes for
    a scaled-down parity case)."""
    wl = WORKLOADS[name]
    return replace(wl, **overrides) if overrides else wl


# 32-layer LLaMA-7B-shaped decode stack: per layer q, k, v, o (4096x4096),
# gate, up (11008x4096) and down (4096x11008).
_STACK_SHAPES = (
    ("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
    ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008),
)


def stack_layer_specs(n_layers: int = 32):
    """Workloads of the decode stack, in execution order.  The seed of linear
    j of layer l is 5000 + 16 l + j."""
    out = []
    for layer in range(n_layers):
        for j, (nm, n, k) in enumerate(_STACK_SHAPES):
            out.append(Workload(
                name=f"stack.l{layer}.{nm}", seed=5000 + 16 * layer + j, n=n, k=k,
                w_dtype="bf16", mask="2:4", codec="int4", clip_alpha=0.9,
                rank=64, x_dtype="bf16", batches=(1,)))
    return out


# ----------------------------------------------------------------------------
# drawing
# ----------------------------------------------------------------------------

def make_layer_inputs(wl: Workload, max_batch: Optional[int] = None) -> dict:
    """Draw W, L, R and x for a workload.

    Returns a dict with
      ``w``      float32 [N][K], the exact delivered weight values,
      ``w_bits`` uint16 [N][K] bf16 patterns when W is delivered as bf16,
      ``L``      float32 [N][r] (or None when rank == 0),
      ``R``      float32 [r][K] (or None),
      ``x``      float32 [B][K], the exact delivered activation values,
      ``x_bits`` uint16 [B][K] (fp16 or bf16 patterns),
      ``act_absmean`` float32 [K] per-channel mean |x| statistic (SLiM^O
                 workloads; None otherwise),
      ``fisher`` float32 [N][K] Fisher diagonal (workloads with fisher=True;
                 None otherwise).
    """
    rng = np.random.default_rng(wl.seed)
    n, k = wl.n, wl.k
    if wl.w_dist == "normal":
        w = rng.standard_normal((n, k)) * wl.w_std
    elif wl.w_dist == "student_t4":
        w = rng.standard_t(4.0, size=(n, k)) * wl.w_std
    else:
        raise ValueError(wl.w_dist)
    n_spikes = int(np.floor(wl.spike_frac * n * k))
    if n_spikes:
        idx = rng.choice(n * k, size=n_spikes, replace=False)
        w.reshape(-1)[idx] *= wl.spike_mult
    w32, w_bits = _deliver(w, wl.w_dtype)
    L = R = None
    if wl.rank > 0:
        L = (rng.standard_normal((n, wl.rank)) * wl.lr_std).astype(np.float32)
        R = (rng.standard_normal((wl.rank, k)) * wl.lr_std).astype(np.float32)
    bmax = max_batch if max_batch is not None else max(wl.batches)
    x32, x_bits = _deliver(rng.standard_normal((bmax, k)), wl.x_dtype)
    act = None
    if wl.salient_channels > 0:
        arng = np.random.default_rng((wl.seed, 1))
        a = np.exp(0.5 * arng.standard_normal(k))
        heavy = arng.choice(k, size=max(1, k // 200), replace=False)
        a[heavy] *= 30.0
        act = a.astype(np.float32)
    fis = None
    if wl.fisher:
        g = np.random.default_rng((wl.seed, 2)).standard_normal((n, k))
        fis = (g * g).astype(np.float32)
    return {"w": w32, "w_bits": w_bits, "L": L, "R": R, "x": x32, "x_bits": x_bits, "act_absmean": act,
            "fisher": fis}


def make_activations(k: int, batch: int, dtype: str, seed: int):
    """Fresh N(0,1) activations [batch][k] in the delivery dtype.

    Returns (float32 exact values, raw 16-bit patterns)."""
    rng = np.random.default_rng(seed)
    return _deliver(rng.standard_normal((batch, k)), dtype)
