"""Host-side checks of the C ABI (no GPU needed).

* libcql.so loads and exports every function include/cql.h declares;
* the host layout computation agrees with the oracle's independent one;
* argument, alignment and size errors come back before anything launches.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
import sparse_quantized_rank_b200 as C
from sparse_quantized_rank_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return C.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "cql.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\*?\s+\**([a-z_0-9]+)\s*\(", src, flags=re.M)))


def test_exports_every_declared_symbol(lib):
    names = header_functions()
    assert set(names) == set(C.EXPORTED), names
    for n in names:
        assert hasattr(lib, n), n
    assert C.cql_version() == O.FORMAT_VERSION == 2
    assert C.cql_status_string(C.CQL_ERR_SIZE).startswith("CQL_ERR_SIZE")


def test_checked_build_exports_every_declared_symbol():
    """The range-checked variant (-DCQL_CHECKED) builds and exports the same
    C ABI; selecting it routes the binding's calls to it."""
    path = B.build(checked=True)
    assert path.endswith("libcql_checked.so")
    L = ctypes.CDLL(path)
    for n in header_functions():
        assert hasattr(L, n), n
    C.use_library(True)
    try:
        assert C.cql_status_string(C.CQL_ERR_RANGE).startswith("CQL_ERR_RANGE")
        assert C.lib()._name == path
    finally:
        C.use_library(False)
    assert C.lib()._name.endswith("libcql.so")


def test_desc_struct_size():
    assert ctypes.sizeof(C.cql_desc) == 64
    assert ctypes.sizeof(C.cql_layout) == 16 + 2 * 8 * 13


DESCS = [
    dict(n_out=256, k_in=512, mask=1, codec=0, rank=16),
    dict(n_out=11008, k_in=4096, mask=1, codec=0, rank=128),
    dict(n_out=4096, k_in=4096, mask=0, codec=2, outlier_frac=0.0045),
    dict(n_out=4096, k_in=11008, mask=2, codec=1, rank=64),
    dict(n_out=128, k_in=384, mask=1, codec=1, rank=48),
    dict(n_out=384, k_in=256, mask=0, codec=3, outlier_frac=0.01, rank=32),
    dict(n_out=128, k_in=128, mask=2, codec=0, outlier_frac=0.001),
    dict(n_out=11008, k_in=4096, mask=1, codec=0, rank=128, salient_channels=41, salient_log2=1),
    dict(n_out=256, k_in=1024, mask=0, codec=2, outlier_frac=0.01, salient_channels=128, salient_log2=8),
]


@pytest.mark.parametrize("kw", DESCS)
def test_layout_matches_oracle(lib, kw):
    d = C.make_desc(**kw)
    lay = C.cql_packed_layout(d)
    od = O.OracleDesc(kw["n_out"], kw["k_in"], kw["mask"], kw["codec"], 0.9, kw.get("outlier_frac", 0.0),
                      kw.get("rank", 0), salient_channels=kw.get("salient_channels", 0),
                      salient_log2=kw.get("salient_log2", 0))
    ol = O.packed_layout(od)
    assert list(lay.off) == ol["off"]
    assert list(lay.len) == ol["len"]
    assert lay.total_bytes == ol["total"] and lay.nnz == ol["nnz"]


def test_descriptor_validation(lib):
    ok = dict(n_out=256, k_in=512, mask=1, codec=0, rank=16)
    C.cql_packed_layout(C.make_desc(**ok))
    bad = [
        (dict(ok, n_out=200), C.CQL_ERR_ARG),
        (dict(ok, k_in=100), C.CQL_ERR_ARG),
        (dict(ok, mask=3), C.CQL_ERR_ARG),
        (dict(ok, codec=7), C.CQL_ERR_ARG),
        (dict(ok, rank=8), C.CQL_ERR_ARG),
        (dict(ok, rank=512), C.CQL_ERR_ARG),
        (dict(ok, clip_alpha=-0.1), C.CQL_ERR_ARG),
        (dict(ok, clip_alpha=1.5), C.CQL_ERR_ARG),
        (dict(ok, outlier_frac=-0.1), C.CQL_ERR_ARG),
        (dict(ok, codec=2), C.CQL_ERR_UNSUPPORTED),          # LUT needs no mask
        (dict(ok, mask=0, codec=2, k_in=32768), C.CQL_ERR_UNSUPPORTED),
        (dict(ok, salient_channels=-1, salient_log2=1), C.CQL_ERR_ARG),
        (dict(ok, salient_channels=65, salient_log2=1), C.CQL_ERR_ARG),     # more than K/8
        (dict(ok, salient_channels=5, salient_log2=0), C.CQL_ERR_ARG),      # factor 1 is no scaling
        (dict(ok, salient_channels=5, salient_log2=9), C.CQL_ERR_ARG),
        (dict(ok, salient_channels=0, salient_log2=1), C.CQL_ERR_ARG),      # factor without channels
    ]
    for kw, st in bad:
        with pytest.raises(C.CqlError) as ei:
            C.cql_packed_layout(C.make_desc(**kw))
        assert ei.value.status == st, kw
    d = C.make_desc(**ok)
    d.group = 64
    with pytest.raises(C.CqlError) as ei:
        C.cql_packed_layout(d)
    assert ei.value.status == C.CQL_ERR_UNSUPPORTED


def test_call_errors_return_before_launch(lib):
    """Null, misaligned and undersized arguments are rejected on the host."""
    d = C.make_desc(256, 512, rank=16)
    lay = C.cql_packed_layout(d)
    ws = C.cql_workspace_size(d, 1)
    fake = 1 << 40                                  # never dereferenced
    L = lib
    st = L.compressed_linear_forward(ctypes.byref(d), None, fake, C.CQL_DT_F16, fake, C.CQL_DT_F16, 1, fake, ws, None)
    assert st == C.CQL_ERR_ARG
    st = L.compressed_linear_forward(ctypes.byref(d), fake + 16, fake, C.CQL_DT_F16, fake, C.CQL_DT_F16, 1, fake, ws,
                                     None)
    assert st == C.CQL_ERR_ALIGN
    st = L.compressed_linear_forward(ctypes.byref(d), fake, fake, C.CQL_DT_F16, fake, C.CQL_DT_F16, 1, fake, ws - 256,
                                     None)
    assert st == C.CQL_ERR_SIZE
    st = L.compressed_linear_forward(ctypes.byref(d), fake, fake, C.CQL_DT_F32, fake, C.CQL_DT_F16, 1, fake, ws, None)
    assert st == C.CQL_ERR_ARG                       # fp32 activations are not accepted
    st = L.compressed_linear_forward(ctypes.byref(d), fake, fake, C.CQL_DT_F16, fake, C.CQL_DT_F16, 0, fake, ws, None)
    assert st == C.CQL_ERR_ARG
    pw = C.cql_pack_workspace_size(d)
    st = L.pack_compressed_weight(ctypes.byref(d), fake, C.CQL_DT_F32, None, None, None, None, fake, lay.total_bytes, fake, pw,
                                  None)
    assert st == C.CQL_ERR_ARG                       # rank 16 needs L and R
    st = L.pack_compressed_weight(ctypes.byref(d), fake, C.CQL_DT_F32, fake, fake, None, None, fake, lay.total_bytes - 1, fake, pw,
                                  None)
    assert st == C.CQL_ERR_SIZE
    st = L.pack_compressed_weight(ctypes.byref(d), fake + 8, C.CQL_DT_F32, fake, fake, None, None, fake, lay.total_bytes, fake, pw,
                                  None)
    assert st == C.CQL_ERR_ALIGN
    ds = C.make_desc(256, 512, rank=16, salient_channels=5, salient_log2=1)
    lay_s = C.cql_packed_layout(ds)
    pws = C.cql_pack_workspace_size(ds)
    st = L.pack_compressed_weight(ctypes.byref(ds), fake, C.CQL_DT_F32, fake, fake, None, None, fake, lay_s.total_bytes,
                                  fake, pws, None)
    assert st == C.CQL_ERR_ARG                       # SLiM^O needs the activation statistic
    assert L.cql_get_device_status(None, None, None) == C.CQL_ERR_ARG


def test_adapter_construction_argument_errors(lib):
    """cql_build_adapters checks its arguments on the host, before anything
    is launched."""
    fake = 1 << 40
    d0 = C.make_desc(256, 512, rank=0)
    with pytest.raises(C.CqlError) as ei:
        C.cql_adapter_workspace_size(d0)                 # no adapters to build
    assert ei.value.status == C.CQL_ERR_ARG
    d = C.make_desc(256, 512, rank=16)
    nb = C.cql_adapter_workspace_size(d)
    assert nb >= 256 * 512 * 4 and nb % 256 == 0
    L = lib
    assert L.cql_build_adapters(ctypes.byref(d), None, C.CQL_DT_F32, fake, None, fake, fake, fake, nb, None) == \
        C.CQL_ERR_ARG
    assert L.cql_build_adapters(ctypes.byref(d), fake, C.CQL_DT_F16, fake, None, fake, fake, fake, nb, None) == \
        C.CQL_ERR_ARG                                    # W must be fp32 or bf16
    assert L.cql_build_adapters(ctypes.byref(d), fake, C.CQL_DT_F32, fake + 16, None, fake, fake, fake, nb, None) == \
        C.CQL_ERR_ALIGN
    assert L.cql_build_adapters(ctypes.byref(d), fake, C.CQL_DT_F32, fake, None, fake, fake, fake, nb - 256, None) == \
        C.CQL_ERR_SIZE


def test_workspace_sizes_grow_with_batch(lib):
    d = C.make_desc(11008, 4096, rank=128)
    sizes = [C.cql_workspace_size(d, b) for b in (1, 4, 16)]
    assert sizes[0] < sizes[1] < sizes[2]
    assert all(s % 256 == 0 for s in sizes)


@pytest.mark.parametrize("name,over", [
    ("tiny", dict(n=128, k=256, rank=16)),
    ("lut_dense_sparse", dict(n=128, k=256)),
    ("mlp_up_slimo", dict(n=128, k=512, rank=16, salient_channels=5, salient_log2=1)),
    ("down_unstructured", dict(n=128, k=384, rank=16, clip_alpha=0.0)),
])
def test_saved_buffer_header_and_checksums(lib, name, over):
    """A host copy of a packed buffer (the oracle's, byte-identical to the
    GPU packer's) gives back its descriptor and layout, and every plane's
    CRC-32 equals zlib's."""
    import zlib
    from workloads import make_layer_inputs, workload
    wl = workload(name, **over)
    inp = make_layer_inputs(wl, max_batch=1)
    od = O.desc_for(wl)
    parts = O.compress(od, inp["w"], inp["L"], inp["R"], inp["act_absmean"])
    buf = bytes(O.pack_bytes(od, parts))
    d, lay = C.cql_read_header(buf)
    assert (d.n_out, d.k_in, d.mask, d.codec, d.rank) == (od.n_out, od.k_in, od.mask, od.codec, od.rank)
    assert (d.salient_channels, d.salient_log2) == (od.salient_channels, od.salient_log2)
    if od.clip_alpha == 0.0:                              # the searched alpha is what the header holds
        assert d.clip_alpha == np.float32(parts["clip_alpha"])
    ol = O.packed_layout(od)
    assert list(lay.off) == ol["off"] and list(lay.len) == ol["len"] and lay.total_bytes == len(buf)
    crc = C.cql_plane_checksums(buf)
    for i in range(O.NPLANES):
        seg = buf[ol["off"][i]: ol["off"][i] + ol["len"][i]]
        assert crc[i] == (zlib.crc32(seg) if ol["len"][i] else 0), i


def test_saved_buffer_corruption_is_reported(lib):
    from workloads import make_layer_inputs, workload
    wl = workload("tiny", n=128, k=256, rank=16)
    inp = make_layer_inputs(wl, max_batch=1)
    od = O.desc_for(wl)
    buf = bytearray(O.pack_bytes(od, O.compress(od, inp["w"], inp["L"], inp["R"])))

    def status(b):
        try:
            C.cql_read_header(bytes(b))
            return C.CQL_OK
        except C.CqlError as e:
            return e.status
    assert status(buf) == C.CQL_OK
    assert status(buf[:-256]) == C.CQL_ERR_SIZE           # truncated
    assert status(buf[:100]) == C.CQL_ERR_SIZE            # not even a header
    bad = bytearray(buf); bad[0] ^= 1                     # magic
    assert status(bad) == C.CQL_ERR_FORMAT
    bad = bytearray(buf); bad[4] ^= 1                     # version
    assert status(bad) == C.CQL_ERR_FORMAT
    bad = bytearray(buf); bad[8] ^= 1                     # n_out no longer a multiple of 128
    assert status(bad) == C.CQL_ERR_FORMAT
    bad = bytearray(buf); bad[88 + 8 * 13 + 8] ^= 1       # a stored plane length
    assert status(bad) == C.CQL_ERR_FORMAT


def test_layout_matches_oracle_on_random_descriptors(lib):
    """Property check over many valid descriptors (every mask / codec pair the
    format allows, ragged shapes, adapter ranks, CSR fractions, SLiM^O
    fields): the library's layout equals the oracle's, planes are 256-byte
    aligned, in order and disjoint, and the header's size rule holds."""
    from hypothesis import given, settings, strategies as st

    @st.composite
    def descs(draw):
        codec = draw(st.sampled_from([O.CODEC_INT4, O.CODEC_INT3, O.CODEC_LUT3, O.CODEC_LUT4]))
        lut = codec in (O.CODEC_LUT3, O.CODEC_LUT4)
        mask = O.MASK_NONE if lut else draw(st.sampled_from([O.MASK_NONE, O.MASK_2_4, O.MASK_BITMAP50]))
        n = 128 * draw(st.integers(1, 96))
        k = 128 * draw(st.integers(1, 128 if lut else 512))
        rank = 16 * draw(st.integers(0, 16))
        frac = draw(st.sampled_from([0.0, 0.0005, 0.002, 0.0045, 0.0625]))
        m = draw(st.integers(0, k // 8))
        e = draw(st.integers(1, 8)) if m else 0
        return dict(n_out=n, k_in=k, mask=mask, codec=codec, rank=rank, outlier_frac=frac,
                    salient_channels=m, salient_log2=e)

    @settings(max_examples=400, derandomize=True, deadline=None)
    @given(descs())
    def check(kw):
        lay = C.cql_packed_layout(C.make_desc(**kw))
        od = O.OracleDesc(kw["n_out"], kw["k_in"], kw["mask"], kw["codec"], 0.9, float(np.float32(kw["outlier_frac"])),
                          kw["rank"], salient_channels=kw["salient_channels"], salient_log2=kw["salient_log2"])
        ol = O.packed_layout(od)
        assert list(lay.off) == ol["off"] and list(lay.len) == ol["len"], kw
        assert lay.total_bytes == ol["total"] and lay.nnz == ol["nnz"], kw
        end = 0
        for i in range(O.NPLANES):
            assert lay.off[i] % 256 == 0 and lay.off[i] >= end, (kw, i)
            end = lay.off[i] + lay.len[i]
        assert lay.len[0] == 512 and lay.total_bytes >= end and lay.total_bytes % 256 == 0

    check()


def test_binding_refuses_mis_shaped_tensors():
    """The C entry point sees raw pointers only, so the binding checks the
    tensors' shapes, dtypes, layout and devices before calling it."""
    import torch
    d = C.make_desc(256, 512)
    x = torch.zeros(3, 512, dtype=torch.bfloat16)
    C.check_forward_args(d, x, torch.zeros(3, 256), torch.device("cpu"))      # valid
    C.check_forward_args(d, x.half(), None, None)
    bad = [
        (torch.zeros(3, 384, dtype=torch.bfloat16), None),                         # K mismatch
        (torch.zeros(512, 3, dtype=torch.bfloat16).t(), None),                     # not contiguous
        (torch.zeros(3, 512), None),                                                # fp32 activations
        (x, torch.zeros(2, 256)),                                                   # out rows
        (x, torch.zeros(3, 128)),                                                   # out columns
        (x, torch.zeros(256, 3).t()),                                               # out not contiguous
        (x, torch.zeros(3, 256, dtype=torch.int32)),                                # out dtype
    ]
    for xi, oi in bad:
        with pytest.raises(ValueError):
            C.check_forward_args(d, xi, oi, torch.device("cpu"))
    with pytest.raises(ValueError):                                                 # another device
        C.check_forward_args(d, x, None, torch.device("cuda", 0))


def test_binding_refuses_mis_shaped_pack_inputs():
    import torch
    d = C.make_desc(256, 512, rank=16, salient_channels=4, salient_log2=1)
    W = torch.zeros(256, 512, dtype=torch.bfloat16)
    L, R, a = torch.zeros(256, 16), torch.zeros(16, 512), torch.ones(512)
    C.check_pack_args(d, W, L, R, a)                                            # valid
    C.check_pack_args(C.make_desc(256, 512), W.float())                         # rank 0, no SLiM^O
    bad = [
        (W[:128], L, R, a, None),                                               # W rows
        (W.half(), L, R, a, None),                                              # W dtype
        (W, None, R, a, None),                                                  # rank needs L
        (W, L.t().contiguous(), R, a, None),                                    # L transposed
        (W, L, R.double(), a, None),                                            # R dtype
        (W, L, R, None, None),                                                  # SLiM^O needs the statistic
        (W, L, R, torch.ones(256), None),                                       # statistic length
        (W, L, R, a, torch.ones(512, 256)),                                     # Fisher shape
    ]
    for args in bad:
        with pytest.raises(ValueError):
            C.check_pack_args(d, *args)
