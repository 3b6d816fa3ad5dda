"""GPU adapter construction (cql_build_adapters: SLiM-LoRA and Naive-LoRA;
SLiM review summary, "SLIM-LoRA") against the CPU oracle.

The adapters are a truncated SVD, computed on the GPU by randomized
subspace iteration, so L and R themselves are not unique (signs, rotations
inside a singular-value cluster).  What is unique is checked:
* a planted case whose compression error is exactly of rank r (a lossless
  int4 grid matrix plus a small rank-r perturbation): L R must equal the
  error, element by element;
* noise-like compression errors of real layers: the weighted objective
  ||(E - L R) diag(xbar)||^2 must lie between the oracle's exact optimum and
  that optimum plus a small relative margin, and obey the projection
  identity ||F(E)||^2 - ||F(L R)||^2 (which holds for any orthogonal
  projection, at any size);
* the whole flow (pack, build, pack again) gives a layer whose packed bytes
  equal the oracle's packing of the same L, R and whose forward matches.
"""
import numpy as np
import pytest

import oracle as O
import sparse_quantized_rank_b200 as C
from tests.gpu_util import c_desc, check_close, device_inputs
from workloads import make_layer_inputs, workload

pytestmark = pytest.mark.gpu


def _gpu_adapters(desc_o, W, act, dev, naive=False):
    import torch
    d = c_desc(desc_o)
    layer = C.CompressedLinear.with_adapters(d, W, act_absmean=act, naive=naive)
    torch.cuda.synchronize()
    return layer, layer.L.cpu().numpy().astype(np.float64), layer.R.cpu().numpy().astype(np.float64)


def _error(desc_o, w, act):
    """E in the space the codec encoded and the weight xbar' (oracle)."""
    d0 = O.OracleDesc(desc_o.n_out, desc_o.k_in, desc_o.mask, desc_o.codec, desc_o.clip_alpha, desc_o.outlier_frac,
                      0, salient_channels=desc_o.salient_channels, salient_log2=desc_o.salient_log2)
    parts = O.compress(d0, w, act_absmean=act)
    wp = np.array(w, dtype=np.float64)
    xb = None if act is None else np.asarray(act, dtype=np.float32).astype(np.float64)
    if "salient" in parts:
        f = float(2 ** desc_o.salient_log2)
        wp[:, parts["salient"]] *= f
        if xb is not None:
            xb[parts["salient"]] /= f
    return wp - O.compressed_matrix(parts), xb


@pytest.mark.parametrize("weighted", [False, True])
def test_planted_low_rank_error_is_recovered(weighted, cuda_dev):
    import torch
    rng = np.random.default_rng(31)
    n, k, r = 256, 512, 16
    s = 2.0 ** -6
    q = rng.integers(-6, 7, size=(n, k)).astype(np.float64)
    q[:, ::128] = 7.0                                   # every group's maximum, unperturbed
    A = rng.standard_normal((n, r))
    B = rng.standard_normal((r, k))
    B[:, ::128] = 0.0
    delta = A @ B
    delta *= 0.4 * s / np.abs(delta).max()              # below half a grid step: codes unchanged
    w = (q * s + delta).astype(np.float32)
    act = np.exp(0.5 * rng.standard_normal(k)).astype(np.float32) if weighted else None
    d = O.OracleDesc(n, k, O.MASK_NONE, O.CODEC_INT4, clip_alpha=1.0, rank=r)
    e, _ = _error(d, w, act)
    assert np.abs(e - delta).max() < 1e-5 * np.abs(delta).max()
    W = torch.from_numpy(w).to(cuda_dev)
    actd = None if act is None else torch.from_numpy(act).to(cuda_dev)
    _, L, R = _gpu_adapters(d, W, actd, cuda_dev)
    lr = L @ R
    assert np.abs(lr - e).max() <= 1e-4 * np.abs(e).max(), np.abs(lr - e).max() / np.abs(e).max()


CASES = {
    "tiny_r16": workload("tiny", rank=16),
    "mlp_up_mid_r64": workload("mlp_up", n=2048, k=1024, rank=64),
    "bitmap_int3_r32": workload("down_unstructured", n=512, k=1408, rank=32),
    "lut_csr_r32": workload("lut_dense_sparse", n=512, k=1024, rank=32),
    "slimo_r32": workload("mlp_up_slimo", n=1024, k=1024, rank=32, salient_channels=10),
}


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("naive", [False, True])
def test_objective_near_the_exact_optimum(name, naive, cuda_dev):
    import torch
    wl = CASES[name]
    inp = make_layer_inputs(wl, max_batch=1)
    act = inp["act_absmean"]
    if act is None:
        act = np.exp(0.5 * np.random.default_rng(wl.seed).standard_normal(wl.k)).astype(np.float32)
    d = O.desc_for(wl)
    W, _, _, _ = device_inputs(inp, wl, cuda_dev)
    _, L, R = _gpu_adapters(d, W, torch.from_numpy(act).to(cuda_dev), cuda_dev, naive=naive)
    e, xb = _error(d, inp["w"], act)
    xw = None if naive else xb
    Lo, Ro = O.slim_lora(e, wl.rank, xw)
    opt = O.lowrank_objective(e, Lo, Ro, xw)
    got = O.lowrank_objective(e, L, R, xw)
    base = O.lowrank_objective(e, np.zeros((wl.n, 1)), np.zeros((1, wl.k)), xw)
    assert got >= opt * (1 - 1e-6), (got, opt)
    print(f"{name} naive={naive}: captured-energy deficit {(got - opt) / (base - opt):.2e}, "
          f"objective excess {(got - opt) / opt:.2e}")
    assert got <= opt + 0.02 * (base - opt) + 1e-9 * base, (got, opt, base)
    # projection identity (any orthogonal projection of F(E))
    f = np.ones(wl.k) if xw is None else xw
    flr = (L @ R) * f[None, :]
    assert abs(got - (base - np.sum(flr * flr))) <= 1e-4 * base


def test_pack_build_pack_flow_matches_the_oracle(cuda_dev):
    """with_adapters packs W with the adapters it built: the packed bytes are
    the oracle's packing of the same L and R, and the forward matches."""
    import torch
    wl = workload("mlp_up", n=1024, k=2048, rank=64)
    inp = make_layer_inputs(wl, max_batch=4)
    d = O.desc_for(wl)
    act = np.exp(0.5 * np.random.default_rng(9).standard_normal(wl.k)).astype(np.float32)
    W, _, _, x = device_inputs(inp, wl, cuda_dev)
    layer, L, R = _gpu_adapters(d, W, torch.from_numpy(act).to(cuda_dev), cuda_dev)
    parts = O.compress(d, inp["w"], L.astype(np.float32), R.astype(np.float32))
    assert np.array_equal(layer.packed.cpu().numpy(), O.pack_bytes(d, parts))
    y = layer.forward(x[:4].contiguous(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    check_close(y, O.forward(parts, inp["x"][:4].astype(np.float64)), "f32", what="built adapters forward")
