"""Parity under the range-checked build (libcql_checked.so, -DCQL_CHECKED).

Every plane read, activation read, workspace access and output store of the
forward kernels, and every plane store of the pack kernels, checks its index
against its buffer; an index outside
records CQL_ERR_RANGE (with the site) and skips the access.  With a memory
checker unavailable, this is the library's own guard against out-of-bounds
indexing: these cases run every forward path (tensor-core decode with CSR
and ragged shapes, the CUDA-core codecs and masks, the sparse prefill with a
ragged token tile, SLiM^O, the no-workspace entry point) and every packer
path (top-k outliers, both masks, the clip search, quantile and Fisher LUTs,
the salient channel list, adapters), and require clean error words, packed
bytes equal to the oracle's and parity with the oracle.
"""
import ctypes

import pytest

import sparse_quantized_rank_b200 as C
from tests.gpu_util import Case, check_close
from workloads import workload

pytestmark = pytest.mark.gpu

CASES = {
    "mlp_up_small": (workload("mlp_up", n=1024, k=2048), (1, 16)),
    "tc_csr_ragged": (workload("mlp_up", n=2048, k=4224, outlier_frac=0.002, rank=48, x_dtype="f16"), (1, 8, 13)),
    "lut_small": (workload("lut_dense_sparse", n=512, k=1024), (1, 8)),
    "down_small": (workload("down_unstructured", n=512, k=1408), (1, 7, 16)),
    "int3_2of4": (workload("mlp_up", n=384, k=1152, codec="int3", rank=48, x_dtype="f16"), (1, 3)),
    "int4_dense_csr": (workload("mlp_up", n=256, k=640, mask="none", outlier_frac=0.003, rank=16), (1, 6)),
    "prefill_small": (workload("prefill_up", n=256, k=512, rank=64), (300,)),
    "slimo_small": (workload("mlp_up_slimo", n=1024, k=1024, rank=32, salient_channels=10), (1, 5, 40)),
    # packer paths the cases above do not reach: the clip search (2:4 and
    # bitmap), bitmap int4 with CSR outliers, Fisher k-means LUT4
    "alpha_2of4": (workload("mlp_up", n=512, k=1024, clip_alpha=0.0), (1,)),
    "alpha_bitmap_csr": (workload("down_unstructured", n=256, k=768, codec="int4", outlier_frac=0.002,
                                  clip_alpha=0.0), (1, 4)),
    "fisher_lut4": (workload("lut_dense_sparse", n=256, k=512, codec="lut4", fisher=True), (1, 2)),
}


@pytest.fixture(scope="module")
def checked_lib():
    C.use_library(True)
    yield C.lib()
    C.use_library(False)


@pytest.mark.parametrize("name", list(CASES))
def test_checked_build_parity(name, checked_lib, cuda_dev):
    import torch
    wl, batches = CASES[name]
    case = Case(wl, cuda_dev, max_batch=max(batches))
    # the pack ran under the checked library too: clean error word, every
    # byte equal to the oracle's
    assert case.layer.pack_status() == C.CQL_OK, f"{name}: checked build recorded an error in the pack"
    assert (case.packed_bytes() == case.ref_bytes).all(), f"{name}: packed bytes differ from the oracle's"
    for b in batches:
        y = case.forward(b, torch.float32)
        torch.cuda.synchronize()
        assert case.layer.device_status(b) == C.CQL_OK, f"{name} B={b}: checked build recorded an error"
        check_close(y, case.reference(b), "f32", what=f"checked {name} B={b}")


def test_checked_build_noalloc(checked_lib, cuda_dev):
    import torch
    case = Case(workload("mlp_up", n=1024, k=2048), cuda_dev, max_batch=4)
    x = case.x[:4].contiguous()
    y = torch.empty((4, case.wl.n), dtype=torch.float32, device=cuda_dev)
    st = C.lib().compressed_linear_forward_noalloc(
        ctypes.byref(case.layer.desc), case.layer.packed.data_ptr(), x.data_ptr(), C._dt_of(x), y.data_ptr(),
        C.CQL_DT_F32, 4, torch.cuda.current_stream().cuda_stream)
    assert st == C.CQL_OK
    torch.cuda.synchronize()
    assert C.cql_get_device_status(None) == C.CQL_OK
    check_close(y, case.reference(4), "f32", what="checked no-workspace B=4")
