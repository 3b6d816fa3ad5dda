"""The C ABI from a plain C99 program (tests/abi_consumer.c; no GPU needed).

include/cql.h must compile as C under -std=c99 -pedantic -Werror, and a C
program linked against libcql.so must read back, from host copies of packed
layers the oracle wrote, the same descriptor, layout and per-plane CRC-32
that the oracle and zlib compute, and get the documented argument errors.
"""
import os
import shutil
import subprocess
import zlib

import numpy as np
import pytest

import oracle as O
import sparse_quantized_rank_b200 as C
from sparse_quantized_rank_b200 import build as B
from workloads import make_layer_inputs, workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_quantized_rank_b200")

LAYERS = [
    ("tiny", {}),
    ("mlp_up", dict(n=256, k=512, rank=32, outlier_frac=0.002)),
    ("mlp_up", dict(n=128, k=384, clip_alpha=0.0)),                       # searched alpha in the header
    ("down_unstructured", dict(n=256, k=640, codec="int4", rank=16)),    # bitmap mask, VOFF plane
    ("lut_dense_sparse", dict(n=128, k=256, rank=0)),                     # LUT3 + CSR
    ("mlp_up_slimo", dict(n=256, k=512, rank=16, salient_channels=9)),   # SALIENT plane
]


@pytest.fixture(scope="module")
def consumer(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    B.build()
    out = str(tmp_path_factory.mktemp("abi") / "abi_consumer")
    cmd = ["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "abi_consumer.c"), "-L", PKG, "-lcql", f"-Wl,-rpath,{PKG}", "-o", out]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return out


def _layer(name, over):
    wl = workload(name, **over)
    inp = make_layer_inputs(wl, max_batch=1)
    od = O.desc_for(wl)
    parts = O.compress(od, inp["w"], inp["L"], inp["R"], inp["act_absmean"])
    return od, parts, bytes(O.pack_bytes(od, parts))


def test_c_program_reads_oracle_buffers(consumer, tmp_path):
    layers, files = [], []
    for i, (name, over) in enumerate(LAYERS):
        od, parts, buf = _layer(name, over)
        f = tmp_path / f"layer{i}.cql"
        f.write_bytes(buf)
        layers.append((od, parts, buf))
        files.append(str(f))
    r = subprocess.run([consumer] + files, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    lines = r.stdout.strip().splitlines()
    assert len(lines) == len(layers)
    P = O.NPLANES
    for (od, parts, buf), f, line in zip(layers, files, lines):
        tok = line.split()
        assert tok[0] == f
        n, k, mask, codec, rank = (int(t) for t in tok[1:6])
        assert (n, k, mask, codec, rank) == (od.n_out, od.k_in, od.mask, od.codec, od.rank)
        alpha = np.float32(parts["clip_alpha"]) if od.clip_alpha == 0.0 else np.float32(od.clip_alpha)
        assert np.float32(float(tok[6])) == alpha
        assert (int(tok[7]), int(tok[8])) == (od.salient_channels, od.salient_log2)
        ol = O.packed_layout(od)
        total, nnz = int(tok[9]), int(tok[10])
        off = [int(t) for t in tok[11:11 + P]]
        ln = [int(t) for t in tok[11 + P:11 + 2 * P]]
        crc = [int(t) for t in tok[11 + 2 * P:11 + 3 * P]]
        assert total == len(buf) and nnz == O.n_outliers(od)
        assert off == ol["off"] and ln == ol["len"]
        for i in range(P):
            seg = buf[off[i]:off[i] + ln[i]]
            assert crc[i] == (zlib.crc32(seg) if ln[i] else 0), i
        # the C program's struct layout agrees with the Python binding's
        assert int(tok[11 + 3 * P]) == C.cql_pack_workspace_size(C.cql_read_header(buf)[0])


def test_c_program_rejects_a_corrupt_copy(consumer, tmp_path):
    _, _, buf = _layer("tiny", {})
    bad = bytearray(buf)
    bad[5] ^= 1                                         # format version
    f = tmp_path / "bad.cql"
    f.write_bytes(bytes(bad))
    good = tmp_path / "good.cql"
    good.write_bytes(buf)
    r = subprocess.run([consumer, str(good), str(f)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 1
    assert "CQL_ERR_FORMAT" in r.stderr
