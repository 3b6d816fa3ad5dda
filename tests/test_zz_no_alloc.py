"""The no-workspace entry point, compressed_linear_forward_noalloc.

It exists for callers that cannot allocate device memory (a plugin enqueue
path that may not allocate, a runtime with a fixed device-memory budget, a
binding that passes only raw pointers); it uses a fixed scratch array inside
the library instead of a caller workspace.  Checked here through the C ABI:
two calls in a row must match the CPU oracle within the tolerance of every
other parity test and give the regular entry point's fp32 output up to the
order of its fp32 reductions (the same kernels run on the same inputs); consecutive calls with different layers
and batch sizes reuse the array after its partial clear; the device error
word of the array is readable; a layer whose workspace would not fit the
fixed scratch is refused before anything runs.
"""
import ctypes

import pytest

import sparse_quantized_rank_b200 as C
from tests.gpu_util import Case, check_close
from workloads import workload

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": (workload("tiny"), 1),
    "mlp_up_small": (workload("mlp_up", n=1024, k=2048), 4),
    "lut_small": (workload("lut_dense_sparse", n=512, k=1024), 8),
    "down_small": (workload("down_unstructured", n=512, k=1408), 16),
}
_cache = {}


def _case(name, dev):
    if name not in _cache:
        wl, b = CASES[name]
        _cache[name] = Case(wl, dev, max_batch=16)
    return _cache[name]


def _noalloc(case, batch, dev):
    import torch
    x = case.x[:batch].contiguous()
    y = torch.full((batch, case.wl.n), float("nan"), dtype=torch.float32, device=dev)
    st = C.lib().compressed_linear_forward_noalloc(
        ctypes.byref(case.layer.desc), case.layer.packed.data_ptr(), x.data_ptr(), C._dt_of(x), y.data_ptr(),
        C.CQL_DT_F32, batch, torch.cuda.current_stream().cuda_stream)
    assert st == C.CQL_OK, C.cql_status_string(st)
    return y


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_oracle_and_regular_entry_point(name, cuda_dev):
    import torch
    case = _case(name, cuda_dev)
    batch = CASES[name][1]
    ref = case.reference(batch)
    regular = case.layer.forward(case.x[:batch].contiguous(), out_dtype=torch.float32)
    for _ in range(2):                       # two calls in a row: the scratch is reused
        y = _noalloc(case, batch, cuda_dev)
        torch.cuda.synchronize()
        check_close(y, ref, "f32", what=f"noalloc {name} B={batch}")
        # the same kernels on the same inputs; only the order of the fp32
        # reductions at L2 (split-K, adapter partials) may differ between runs
        check_close(y, regular.double().cpu().numpy(), "f32", tol=1e-5, what=f"noalloc {name} vs regular")
        assert C.cql_get_device_status(None) == C.CQL_OK


def test_noalloc_alternating_layers_and_batches(cuda_dev):
    """Consecutive calls whose scratch layouts differ (batch 16, then 1, then
    a different layer): each clears the part it uses, so none sees the
    previous call's leftovers."""
    import torch
    seq = [("down_small", 16), ("down_small", 1), ("mlp_up_small", 16), ("tiny", 3), ("mlp_up_small", 1),
           ("lut_small", 8), ("down_small", 2)]
    outs = []
    for name, b in seq:
        case = _case(name, cuda_dev)
        outs.append((name, b, case, _noalloc(case, b, cuda_dev)))
    torch.cuda.synchronize()
    for name, b, case, y in outs:
        check_close(y, case.reference(b), "f32", what=f"noalloc sequence {name} B={b}")
    assert C.cql_get_device_status(None) == C.CQL_OK


def test_noalloc_refuses_oversized_workspace(cuda_dev):
    """A 2048-token prefill needs far more than the fixed scratch: refused
    with CQL_ERR_SIZE, nothing launched."""
    d = C.make_desc(11008, 4096, rank=64)
    st = C.lib().compressed_linear_forward_noalloc(ctypes.byref(d), 1 << 40, 1 << 40, C.CQL_DT_BF16, 1 << 40,
                                                   C.CQL_DT_BF16, 2048, None)
    assert st == C.CQL_ERR_SIZE
