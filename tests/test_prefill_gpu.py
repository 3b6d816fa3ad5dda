"""GPU parity of the tcgen05 prefill path (batch > 16) against the CPU oracle.

Small cases cover a ragged token tile (M not a multiple of 256), fp16 and bf16
activations, ranks whose adapter extension is padded, no adapters, no mask and
3-bit codes; the two full-size prefill GEMMs (2048 tokens, 4096 -> 11008 and
11008 -> 4096) are compared on every output."""
import numpy as np
import pytest

import oracle as O
import sparse_quantized_rank_b200 as C
from tests.gpu_util import Case, check_close
from workloads import workload

pytestmark = pytest.mark.gpu

CASES = {
    "pf_small": (workload("prefill_up", n=256, k=512, rank=64), 300),
    "pf_small_f16_r16": (workload("prefill_up", n=384, k=640, rank=16, x_dtype="f16"), 77),
    "pf_norank": (workload("prefill_up", n=256, k=1024, rank=0), 512),
    "pf_dense_int4": (workload("prefill_up", n=128, k=256, mask="none", rank=32), 40),
    "pf_int3_2of4": (workload("prefill_up", n=128, k=384, codec="int3", rank=48), 600),
    # int3 2:4 on the sparse tensor cores: 24-byte code groups, an odd group
    # count (17), a ragged token tile
    "pf_int3_2of4_sparse": (workload("prefill_up", n=1024, k=2176, codec="int3", rank=64), 333),
    "prefill_up": (workload("prefill_up"), 2048),
    "prefill_down": (workload("prefill_down"), 2048),
}
_cache = {}


def get_case(name, dev):
    if name not in _cache:
        wl, m = CASES[name]
        _cache[name] = (Case(wl, dev, max_batch=m), m)
    return _cache[name]


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_matches_oracle(name, cuda_dev):
    import torch
    case, m = get_case(name, cuda_dev)
    assert np.array_equal(case.packed_bytes(), case.ref_bytes)
    ref = case.reference(m)
    xt = torch.float16 if case.wl.x_dtype == "f16" else torch.bfloat16
    for odt, dn in ((torch.float32, "f32"), (xt, case.wl.x_dtype)):
        y = case.forward(m, odt)
        torch.cuda.synchronize()
        check_close(y, ref, dn, what=f"{name} M={m} out={dn}")
    assert case.layer.device_status(m) == C.CQL_OK


@pytest.mark.parametrize("name", ["pf_small", "pf_small_f16_r16"])
def test_prefill_terms(name, cuda_dev):
    import torch
    case, m = get_case(name, cuda_dev)
    main_, _, lr_ = O.forward_terms(case.parts, case.inp["x"][:m].astype(np.float64))
    for flags, ref, tn in ((C.CQL_FLAG_NO_LOWRANK, main_, "main"), (C.CQL_FLAG_NO_MAIN, lr_, "lowrank")):
        y = case.forward(m, torch.float32, flags=flags)
        torch.cuda.synchronize()
        check_close(y, ref, "f32", what=f"{name} term {tn}")


def test_prefill_repeat_and_batch_sizes(cuda_dev):
    """Several token counts through one layer, twice each (the adapter
    accumulator is cleared per call)."""
    import torch
    case, m = get_case("pf_small", cuda_dev)
    for b in (17, 255, 256, 257, 300):
        ref = case.reference(b)
        for _ in range(2):
            y = case.forward(b, torch.float32)
            torch.cuda.synchronize()
            check_close(y, ref, "f32", what=f"pf_small M={b}")


def test_prefill_unsupported_is_reported(cuda_dev):
    import torch
    case = Case(workload("lut_dense_sparse", n=128, k=256), cuda_dev, max_batch=32)
    with pytest.raises(C.CqlError) as ei:
        case.forward(32, torch.float32)
    assert ei.value.status == C.CQL_ERR_UNSUPPORTED
