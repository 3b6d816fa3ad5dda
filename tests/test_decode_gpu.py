"""GPU parity of the device packer (bit-exact) and the decode forward pass
(within tolerance) against the CPU oracle, through the C ABI.

Sizes: every named workload at full size, plus reduced cases that still span
several row blocks, several K tiles and ragged tails (odd unit counts, rank not
a multiple of 32, batches that are not powers of two)."""
import numpy as np
import pytest

import oracle as O
import sparse_quantized_rank_b200 as C
from tests.gpu_util import Case, check_close
from workloads import workload

pytestmark = pytest.mark.gpu

REDUCED = {
    "tiny": workload("tiny"),
    "mlp_up_small": workload("mlp_up", n=1024, k=2048),
    "lut_small": workload("lut_dense_sparse", n=512, k=1024),
    "down_small": workload("down_unstructured", n=512, k=1408),
    "int3_2of4": workload("mlp_up", n=384, k=1152, codec="int3", rank=48, x_dtype="f16"),
    "int4_dense_csr": workload("mlp_up", n=256, k=640, mask="none", outlier_frac=0.003, rank=16),
    "int3_dense": workload("down_unstructured", n=256, k=384, mask="none", rank=0),
    "lut4_lr": workload("lut_dense_sparse", n=384, k=768, codec="lut4", rank=32),
    "bitmap_int4_csr": workload("down_unstructured", n=256, k=896, codec="int4", outlier_frac=0.002, rank=16),
    # tensor-core path with every term: CSR rows and R x as side work, a K
    # that ends in a one-group x chunk (33 groups), rank 48 (a half adapter
    # chunk), fp16 x; 16 row tiles x 33 groups = 528 tiles, so CTAs hold
    # several tiles and cross row tiles and x chunks
    "int4_2of4_csr_ragged": workload("mlp_up", n=2048, k=4224, outlier_frac=0.002, rank=48, x_dtype="f16"),
}
FULL = {
    "mlp_up": workload("mlp_up"),
    "lut_dense_sparse": workload("lut_dense_sparse"),
    "down_unstructured": workload("down_unstructured"),
}

_cache = {}


def get_case(name, cuda_dev):
    if name not in _cache:
        wl = REDUCED.get(name) or FULL[name]
        _cache[name] = Case(wl, cuda_dev, max_batch=16)
    return _cache[name]


def out_dtypes(case):
    import torch
    xt = torch.float16 if case.wl.x_dtype == "f16" else torch.bfloat16
    return [(torch.float32, "f32"), (xt, case.wl.x_dtype)]


@pytest.mark.parametrize("name", list(REDUCED) + list(FULL))
def test_pack_bit_exact(name, cuda_dev):
    case = get_case(name, cuda_dev)
    got = case.packed_bytes()
    ref = case.ref_bytes
    assert got.shape == ref.shape
    if not np.array_equal(got, ref):
        diff = np.nonzero(got != ref)[0]
        lay = O.packed_layout(case.od)
        planes = sorted({max(i for i in range(12) if lay["off"][i] <= d and lay["len"][i] > 0) for d in diff[:1000]})
        raise AssertionError(f"{len(diff)} bytes differ; first at {diff[:8]}; planes {planes}")


@pytest.mark.parametrize("name,batches", [
    ("tiny", (1, 2, 3, 16)),
    ("mlp_up_small", (1, 4, 5, 16)),
    ("lut_small", (1, 8)),
    ("down_small", (1, 2, 7, 16)),
    ("int3_2of4", (1, 3)),
    ("int4_dense_csr", (1, 6)),
    ("int3_dense", (1, 2)),
    ("lut4_lr", (1, 4)),
    ("bitmap_int4_csr", (1, 9)),
    ("int4_2of4_csr_ragged", (1, 3, 8, 13)),
    ("mlp_up", (1, 4, 16)),
    ("lut_dense_sparse", (1, 8)),
    ("down_unstructured", (1, 2, 4, 8, 16)),
])
def test_forward_matches_oracle(name, batches, cuda_dev):
    import torch
    case = get_case(name, cuda_dev)
    for b in batches:
        ref = case.reference(b)
        for odt, dn in out_dtypes(case):
            y = case.forward(b, odt)
            torch.cuda.synchronize()
            check_close(y, ref, dn, what=f"{name} B={b} out={dn}")
        assert case.layer.device_status(b) == C.CQL_OK


@pytest.mark.parametrize("name", ["tiny", "mlp_up_small", "lut_small", "down_small", "int4_dense_csr",
                                  "lut4_lr", "bitmap_int4_csr", "int4_2of4_csr_ragged"])
def test_each_term_alone(name, cuda_dev):
    """Every term checked on its own scale (a bug in the small adapter or CSR
    term cannot hide inside the tolerance of the sum)."""
    import torch
    case = get_case(name, cuda_dev)
    main_, csr_, lr_ = O.forward_terms(case.parts, case.inp["x"][:3].astype(np.float64))
    terms = {
        "main": (C.CQL_FLAG_NO_CSR | C.CQL_FLAG_NO_LOWRANK, main_),
        "csr": (C.CQL_FLAG_NO_MAIN | C.CQL_FLAG_NO_LOWRANK, csr_),
        "lowrank": (C.CQL_FLAG_NO_MAIN | C.CQL_FLAG_NO_CSR, lr_),
    }
    for tname, (flags, ref) in terms.items():
        y = case.forward(3, torch.float32, flags=flags)
        torch.cuda.synchronize()
        if not np.any(ref):
            assert not torch.any(y).item(), f"{name}: {tname} should be zero"
            continue
        check_close(y, ref, "f32", what=f"{name} term {tname}")


def test_repeated_calls_stay_clean(cuda_dev):
    """The workspace is self-cleaning: many calls in a row give the same
    result (accumulators and counters are reset by the epilogue)."""
    import torch
    case = get_case("mlp_up_small", cuda_dev)
    y0 = case.forward(4, torch.float32)
    for _ in range(20):
        y = case.forward(4, torch.float32)
    torch.cuda.synchronize()
    check_close(y, case.reference(4), "f32", what="repeat")
    assert torch.allclose(y, y0, rtol=1e-5, atol=1e-6)


def test_corrupt_header_reported(cuda_dev):
    """A packed buffer whose header does not match the descriptor is reported
    through the device error word, not by a fault."""
    import torch
    case = get_case("tiny", cuda_dev)
    saved = case.layer.packed[:4].clone()
    case.layer.packed[0] = 0
    try:
        case.forward(1, torch.float32)
        assert case.layer.device_status(1) == C.CQL_ERR_FORMAT
    finally:
        case.layer.packed[:4] = saved
    case.forward(1, torch.float32)
    assert case.layer.device_status(1) == C.CQL_OK
