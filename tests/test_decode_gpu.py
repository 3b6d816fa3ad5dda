"""GPU parity of the device packer (bit-exact) and the decode forward pass
(within tolerance) against the CPU oracle, through the C ABI.

Sizes: every named workload at full size, plus reduced cases that still span
several row blocks, several K tiles and ragged tails (odd unit counts, rank not
a multiple of 32, batches that are not powers of two)."""
import numpy as np
import pytest

import oracle as O
import sparse_quantized_rank_b200 as C
from tests.gpu_util import Case, c_desc, check_close, device_inputs
from workloads import make_layer_inputs, stack_layer_specs, workload

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
    # int3 2:4 on the tensor cores: 24-byte code groups straddling slabs,
    # an odd group count (the last group at byte offset 0 of its slabs), CSR
    "int3_2of4_tc": workload("mlp_up", n=1536, k=2176, codec="int3", outlier_frac=0.001, rank=64),
    "mlp_up_int3": workload("mlp_up", codec="int3"),
}
FULL = {
    "mlp_up": workload("mlp_up"),
    "lut_dense_sparse": workload("lut_dense_sparse"),
    "down_unstructured": workload("down_unstructured"),
}
# The other shapes of the 32-layer LLaMA-7B decode stack (2:4 int4 g128,
# rank 64, bf16, batch 1), drawn by the stack's own per-linear seeds: q
# (4096x4096), gate (11008x4096) and down (4096x11008) of layer 0.
_STACK0 = {wl.name.split(".")[-1]: wl for wl in stack_layer_specs(1)}
STACK = {f"stack_{k}": _STACK0[k] for k in ("q", "gate", "down")}
FULL.update(STACK)

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
        planes = sorted({max(i for i in range(O.NPLANES) if lay["off"][i] <= d and lay["len"][i] > 0)
                         for d in diff[:1000]})
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
    ("int3_2of4_tc", (1, 4, 9, 16)),
    ("mlp_up_int3", (1, 16)),
    ("mlp_up", (1, 4, 16)),
    ("lut_dense_sparse", (1, 8)),
    ("down_unstructured", (1, 2, 4, 8, 16)),
    ("stack_q", (1,)),
    ("stack_gate", (1,)),
    ("stack_down", (1,)),
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


def test_layers_chained_without_sync(cuda_dev):
    """Several different layers called back to back on one stream with no
    synchronisation in between (each forward is launched programmatically
    dependent on the kernel before it, which belongs to another layer); every
    output is then checked against the oracle."""
    import torch
    names = ["mlp_up_small", "int4_2of4_csr_ragged", "down_small", "tiny", "mlp_up_small"]
    cases = [get_case(n, cuda_dev) for n in names]
    torch.cuda.synchronize()
    outs = []
    for case, b in zip(cases, (1, 3, 2, 1, 16)):
        outs.append((case, b, case.forward(b, torch.float32)))
    torch.cuda.synchronize()
    for case, b, y in outs:
        check_close(y, case.reference(b), "f32", what=f"chained {case.wl.name} B={b}")
        assert case.layer.device_status(b) == C.CQL_OK


def test_pack_then_forward_without_sync(cuda_dev):
    """Packing and the first forward on one stream with no synchronisation in
    between: the forward must see every packed byte (its first kernel reads
    weights before waiting for the kernel that precedes it)."""
    import torch
    for wl, b in ((workload("mlp_up", n=1024, k=2048, seed=41), 1),
                  (workload("mlp_up", n=512, k=1024, seed=42, outlier_frac=0.002, rank=32), 4)):
        inp = make_layer_inputs(wl, max_batch=b)
        od = O.desc_for(wl)
        parts = O.compress(od, inp["w"], inp["L"], inp["R"])
        W, L, R, x = device_inputs(inp, wl, cuda_dev)
        torch.cuda.synchronize()
        layer = C.CompressedLinear(c_desc(od), W, L, R)      # pack: queued, not waited for
        y = layer.forward(x[:b].contiguous(), out_dtype=torch.float32)
        torch.cuda.synchronize()
        check_close(y, O.forward(parts, inp["x"][:b].astype(np.float64)), "f32", what=f"pack+forward {wl.n}x{wl.k}")
        assert np.array_equal(layer.packed.cpu().numpy(), O.pack_bytes(od, parts))
        assert layer.device_status(b) == C.CQL_OK


@pytest.mark.parametrize("batch", [1, 16])
def test_bounded_wait_runs_out_and_is_reported(batch, cuda_dev):
    """A call whose x load is skipped (test flag) lets the tensor-core decode's
    bounded waits on x run out: the call completes, the device error word says
    CQL_ERR_TIMEOUT, and the next ordinary call on the same workspace is clean
    and correct.  No GPU fault is involved: nothing that waits on x has issued
    a copy or an MMA when the waits give up."""
    import torch
    case = get_case("mlp_up_small", cuda_dev)
    case.forward(batch, torch.float32)
    assert case.layer.device_status(batch) == C.CQL_OK
    case.forward(batch, torch.float32, flags=C.CQL_FLAG_DEBUG_SKIP_X)
    assert case.layer.device_status(batch) == C.CQL_ERR_TIMEOUT
    ws, nbytes = case.layer.workspace(batch)
    C.cql_workspace_init(ws, nbytes)                 # the rule after any device error
    y = case.forward(batch, torch.float32)
    assert case.layer.device_status(batch) == C.CQL_OK
    check_close(y, case.reference(batch), "f32", what=f"after timeout B={batch}")


@pytest.mark.parametrize("name,batches", [("mlp_up_small", (1, 4, 16)), ("int4_2of4_csr_ragged", (1, 13)),
                                          ("int3_2of4_tc", (1, 16)), ("int3_2of4", (3,))])
def test_cuda_core_decode_of_2of4_int4(name, batches, cuda_dev):
    """The CUDA-core decode of a 2:4 int4 or int3 layer (selected by flag; the
    tensor-core decode is the default for these layers) against the oracle."""
    import torch
    case = get_case(name, cuda_dev)
    for b in batches:
        y = case.forward(b, torch.float32, flags=C.CQL_FLAG_CUDA_CORE)
        torch.cuda.synchronize()
        check_close(y, case.reference(b), "f32", what=f"{name} cuda-core B={b}")
        assert case.layer.device_status(b) == C.CQL_OK
