"""Degenerate and boundary cases against the CPU oracle (GPU).

* an all-zero weight matrix: every scale 0, every code the zero code, the
  output the adapter term alone;
* the largest CSR fraction the descriptor allows (1/16 of all entries);
* the smallest layer (one 128 x 128 tile) at batch 1, 16 (the largest decode
  batch) and 17 (the smallest prefill);
* SLiM^O at its limits: K/8 salient channels scaled by 2^8.
"""
import numpy as np
import pytest

import oracle as O
import sparse_quantized_rank_b200 as C
from tests.gpu_util import Case, c_desc, check_close
from workloads import make_layer_inputs, workload

pytestmark = pytest.mark.gpu


def test_all_zero_weights(cuda_dev):
    import torch
    wl = workload("mlp_up", n=256, k=512, rank=16)
    inp = make_layer_inputs(wl, max_batch=4)
    w0 = np.zeros_like(inp["w"])
    d = O.desc_for(wl)
    parts = O.compress(d, w0, inp["L"], inp["R"])
    assert (parts["scales"] == 0).all() and (parts["q"] == 0).all()
    W = torch.zeros(wl.n, wl.k, dtype=torch.bfloat16, device=cuda_dev)
    L = torch.from_numpy(inp["L"]).to(cuda_dev)
    R = torch.from_numpy(inp["R"]).to(cuda_dev)
    layer = C.CompressedLinear(c_desc(d), W, L, R)
    torch.cuda.synchronize()
    assert np.array_equal(layer.packed.cpu().numpy(), O.pack_bytes(d, parts))
    x = torch.from_numpy(inp["x_bits"].view(np.int16)).to(cuda_dev).view(torch.bfloat16)
    for b in (1, 4):
        y = layer.forward(x[:b].contiguous(), out_dtype=torch.float32)
        torch.cuda.synchronize()
        ref = O.forward(parts, inp["x"][:b].astype(np.float64))
        _, _, lr = O.forward_terms(parts, inp["x"][:b].astype(np.float64))
        assert np.array_equal(ref, lr)                  # the adapter term alone
        check_close(y, ref, "f32", what=f"zero W B={b}")


@pytest.mark.parametrize("wl", [
    workload("lut_dense_sparse", n=256, k=512, outlier_frac=0.0625),
    workload("mlp_up", n=256, k=512, mask="none", outlier_frac=0.0625, rank=16),
], ids=["lut3", "int4_dense"])
def test_largest_outlier_fraction(wl, cuda_dev):
    import torch
    case = Case(wl, cuda_dev, max_batch=3)
    assert len(case.parts["csr_col"]) == int(np.floor(np.float32(0.0625) * 256 * 512))
    assert np.array_equal(case.packed_bytes(), case.ref_bytes)
    for b in (1, 3):
        y = case.forward(b, torch.float32)
        torch.cuda.synchronize()
        check_close(y, case.reference(b), "f32", what=f"csr 1/16 B={b}")


def test_smallest_layer_across_the_decode_prefill_boundary(cuda_dev):
    import torch
    case = Case(workload("mlp_up", n=128, k=128, rank=16), cuda_dev, max_batch=17)
    assert np.array_equal(case.packed_bytes(), case.ref_bytes)
    for b in (1, 16, 17):
        y = case.forward(b, torch.float32)
        torch.cuda.synchronize()
        check_close(y, case.reference(b), "f32", what=f"128x128 B={b}")
        assert case.layer.device_status(b) == C.CQL_OK


def test_slimo_at_its_limits(cuda_dev):
    import torch
    wl = workload("mlp_up_slimo", n=256, k=1024, rank=16, salient_channels=128, salient_log2=8)
    case = Case(wl, cuda_dev, max_batch=20)
    assert np.array_equal(case.packed_bytes(), case.ref_bytes)
    for b in (1, 20):
        y = case.forward(b, torch.float32)
        torch.cuda.synchronize()
        check_close(y, case.reference(b), "f32", what=f"SLiM^O K/8 x256 B={b}")
