"""GPU parity of the output-error variant (SLiM^O; SLiM rebuttal, "Output
Error Minimization in SLiM-Quant") against the CPU oracle.

The packer's channel selection and the scaled encoding are compared byte for
byte with the oracle's packed buffer; the forward (which first divides the
salient activation channels by the factor) is compared element by element on
the tensor-core decode, the CUDA-core decode (every codec and mask, f16 and
bf16 activations), the prefill GEMM and the no-workspace entry point.
"""
import ctypes

import numpy as np
import pytest

import oracle as O
import sparse_quantized_rank_b200 as C
from tests.gpu_util import Case, check_close
from workloads import workload

pytestmark = pytest.mark.gpu

CASES = {
    # 2:4 int4 (tensor-core decode and prefill), bf16 x
    "slimo_small": (workload("mlp_up_slimo", n=1024, k=2048, rank=64, salient_channels=20), (1, 5, 16)),
    # f16 x, factor 8, rank 16, tiny
    "slimo_tiny_f16": (workload("tiny", salient_channels=6, salient_log2=3), (1, 3)),
    # bitmap int3 (CUDA-core decode)
    "slimo_bitmap_int3": (workload("down_unstructured", n=256, k=1408, salient_channels=14, salient_log2=1), (1, 8)),
    # LUT3 + CSR outliers (the CSR term reads x' too)
    "slimo_lut_csr": (workload("lut_dense_sparse", n=512, k=1024, salient_channels=10, salient_log2=2), (1, 2)),
    # int4 2:4 with CSR outliers on the tensor-core decode (CSR and R x read x')
    "slimo_2of4_csr": (workload("mlp_up", n=512, k=1152, outlier_frac=0.002, rank=48, salient_channels=12,
                                salient_log2=1), (1, 16)),
    # the full-size layer (1% of 4096 channels)
    "mlp_up_slimo": (workload("mlp_up_slimo"), (1, 16)),
}
PREFILL = {
    "slimo_small": 300,
    "mlp_up_slimo": 2048,
}
_cache = {}


def get_case(name, dev):
    if name not in _cache:
        wl, batches = CASES[name]
        mb = max(max(batches), PREFILL.get(name, 0))
        _cache[name] = Case(wl, dev, max_batch=mb)
    return _cache[name]


@pytest.mark.parametrize("name", list(CASES))
def test_slimo_pack_bit_exact(name, cuda_dev):
    case = get_case(name, cuda_dev)
    got = case.packed_bytes()
    assert got.size == case.ref_bytes.size
    lay = O.packed_layout(case.od)
    o, n = lay["off"][O.P_SALIENT], lay["len"][O.P_SALIENT]
    assert n == 2 * case.wl.salient_channels
    assert np.array_equal(got[o:o + n], case.ref_bytes[o:o + n]), "salient channel list"
    assert np.array_equal(got, case.ref_bytes)


@pytest.mark.parametrize("name", list(CASES))
def test_slimo_forward_matches_oracle(name, cuda_dev):
    import torch
    case = get_case(name, cuda_dev)
    xt = torch.float16 if case.wl.x_dtype == "f16" else torch.bfloat16
    for b in CASES[name][1]:
        ref = case.reference(b)
        for odt, dn in ((torch.float32, "f32"), (xt, case.wl.x_dtype)):
            y = case.forward(b, odt)
            torch.cuda.synchronize()
            check_close(y, ref, dn, what=f"{name} B={b} out={dn}")
        assert case.layer.device_status(b) == C.CQL_OK


@pytest.mark.parametrize("name", ["slimo_small", "slimo_2of4_csr"])
def test_slimo_cuda_core_decode(name, cuda_dev):
    import torch
    case = get_case(name, cuda_dev)
    for b in CASES[name][1]:
        y = case.forward(b, torch.float32, flags=C.CQL_FLAG_CUDA_CORE)
        torch.cuda.synchronize()
        check_close(y, case.reference(b), "f32", what=f"{name} CUDA cores B={b}")


@pytest.mark.parametrize("name", list(PREFILL))
def test_slimo_prefill(name, cuda_dev):
    import torch
    case = get_case(name, cuda_dev)
    m = PREFILL[name]
    y = case.forward(m, torch.float32)
    torch.cuda.synchronize()
    check_close(y, case.reference(m), "f32", what=f"{name} prefill M={m}")
    assert case.layer.device_status(m) == C.CQL_OK


def test_slimo_activations_left_untouched(cuda_dev):
    """The caller's x is not modified (x' lives in the workspace)."""
    import torch
    case = get_case("slimo_small", cuda_dev)
    x = case.x[:5].contiguous()
    before = x.clone()
    case.layer.forward(x, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(x, before)


def test_slimo_noalloc(cuda_dev):
    import torch
    case = get_case("slimo_small", cuda_dev)
    b = 5
    x = case.x[:b].contiguous()
    y = torch.empty((b, case.wl.n), dtype=torch.float32, device=cuda_dev)
    st = C.lib().compressed_linear_forward_noalloc(
        ctypes.byref(case.layer.desc), case.layer.packed.data_ptr(), x.data_ptr(), C._dt_of(x), y.data_ptr(),
        C.CQL_DT_F32, b, torch.cuda.current_stream().cuda_stream)
    assert st == C.CQL_OK
    torch.cuda.synchronize()
    check_close(y, case.reference(b), "f32", what="SLiM^O no-workspace B=5")
    assert C.cql_get_device_status(None) == C.CQL_OK
