"""The no-workspace entry point, compressed_linear_forward_noalloc.

It exists for callers that cannot allocate device memory (a plugin enqueue
path that may not allocate, a runtime with a fixed device-memory budget, a
binding that passes only raw pointers); it uses a fixed scratch array inside
the library instead of a caller workspace.  Checked here through the C ABI:
two calls in a row must match the regular entry point's output within the
same tolerance as every other parity test, and a layer whose workspace would
not fit the fixed scratch is refused before anything runs.
"""
import ctypes

import pytest

import sparse_quantized_rank_b200 as C
from tests.gpu_util import Case, check_close
from workloads import workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,over,batch", [
    ("tiny", {}, 1),
    ("mlp_up", dict(n=1024, k=2048), 4),
    ("lut_dense_sparse", dict(n=512, k=1024), 8),
    ("down_unstructured", dict(n=512, k=1408), 16),
])
def test_noalloc_matches_regular_entry_point(name, over, batch, cuda_dev):
    import torch
    case = Case(workload(name, **over), cuda_dev, max_batch=batch)
    x = case.x[:batch].contiguous()
    ref = case.layer.forward(x, out_dtype=torch.float32)
    torch.cuda.synchronize()
    refv = ref.double().cpu().numpy()
    lib = C.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):                       # two calls in a row: the scratch is reused
        y = torch.full((batch, case.wl.n), float("nan"), dtype=torch.float32, device=cuda_dev)
        st = lib.compressed_linear_forward_noalloc(ctypes.byref(case.layer.desc), case.layer.packed.data_ptr(),
                                                   x.data_ptr(), C._dt_of(x), y.data_ptr(), C.CQL_DT_F32, batch,
                                                   stream)
        assert st == C.CQL_OK, C.cql_status_string(st)
        torch.cuda.synchronize()
        check_close(y, refv, "f32", what=f"noalloc {name} B={batch}")


def test_noalloc_refuses_oversized_workspace(cuda_dev):
    """A 2048-token prefill needs far more than the fixed scratch: refused
    with CQL_ERR_SIZE, nothing launched."""
    d = C.make_desc(11008, 4096, rank=64)
    st = C.lib().compressed_linear_forward_noalloc(ctypes.byref(d), 1 << 40, 1 << 40, C.CQL_DT_BF16, 1 << 40,
                                                   C.CQL_DT_BF16, 2048, None)
    assert st == C.CQL_ERR_SIZE
