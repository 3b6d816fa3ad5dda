"""GPU packer searches against the CPU oracle, byte for byte.

* SLiM-Quant clip search (SLiM review summary, "SLIM-Quant"): a descriptor
  with clip_alpha = 0 has the packer histogram |w| / amax_g and pick the
  grid alpha of least modelled error; the packed bytes (codes, scales, CSR,
  and the header's recorded alpha) equal the oracle's.
* SqueezeLLM sensitivity-weighted k-means ("Approach"): LUT layers packed
  with a Fisher diagonal get per-row weighted Lloyd centroids; the packed
  bytes equal the oracle's.
The forward of each layer matches the oracle.
"""
import numpy as np
import pytest

import oracle as O
from tests.gpu_util import Case, check_close
from workloads import workload

pytestmark = pytest.mark.gpu

CASES = {
    "alpha_2of4_int4": (workload("mlp_up", n=1024, k=2048, clip_alpha=0.0), (1, 16)),
    "alpha_bitmap_int3": (workload("down_unstructured", n=512, k=1408, clip_alpha=0.0), (1, 8)),
    "alpha_dense_int4_csr": (workload("mlp_up", n=256, k=640, mask="none", outlier_frac=0.003, rank=16,
                                      clip_alpha=0.0), (1, 3)),
    "alpha_mlp_up_full": (workload("mlp_up", clip_alpha=0.0), (1,)),
    "fisher_lut3_csr": (workload("lut_dense_sparse", n=512, k=1024, fisher=True), (1, 8)),
    "fisher_lut4_lr": (workload("lut_dense_sparse", n=384, k=768, codec="lut4", rank=32, fisher=True), (1, 2)),
    "fisher_lut_full": (workload("lut_dense_sparse", fisher=True), (1,)),
}
_cache = {}


def get_case(name, dev):
    if name not in _cache:
        wl, batches = CASES[name]
        _cache[name] = Case(wl, dev, max_batch=max(batches))
    return _cache[name]


@pytest.mark.parametrize("name", list(CASES))
def test_search_pack_bit_exact(name, cuda_dev):
    case = get_case(name, cuda_dev)
    got = case.packed_bytes()
    ref = case.ref_bytes
    assert got.size == ref.size
    assert np.array_equal(got[:512], ref[:512]), "header (incl. the recorded alpha)"
    lay = O.packed_layout(case.od)
    for p in range(O.NPLANES):
        o, n = lay["off"][p], lay["len"][p]
        assert np.array_equal(got[o:o + n], ref[o:o + n]), f"plane {p}"
    if case.wl.clip_alpha == 0.0:
        a = case.layer.clip_alpha()
        assert a == float(case.parts["clip_alpha"]) and 0.3 <= a <= 1.0


@pytest.mark.parametrize("name", list(CASES))
def test_search_forward_matches_oracle(name, cuda_dev):
    import torch
    case = get_case(name, cuda_dev)
    for b in CASES[name][1]:
        y = case.forward(b, torch.float32)
        torch.cuda.synchronize()
        check_close(y, case.reference(b), "f32", what=f"{name} B={b}")
