"""Pins of the oracle's packed bytes against the format specification.

The decoder here is written independently from the specification comment in
include/cql.h: it reads every field element by element through the byte
address formula, in pure Python, and compares with the oracle's decoded
parts.  A hand-worked fixture pins the bytes of one small layer.
"""
import json
import os
import struct

import numpy as np
import pytest

import oracle as O
from workloads import make_layer_inputs, workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rit_addr(i, j, row_bytes):
    """Address of byte j of row i in a row-interleaved plane."""
    return ((i // 32) * (row_bytes // 16) + j // 16) * 512 + (i % 32) * 16 + (j % 16)


def read_bits(plane, i, row_bytes, bitpos, nbits):
    v = 0
    for t in range(nbits):
        sb = bitpos + t
        byte = plane[rit_addr(i, sb // 8, row_bytes)]
        v |= ((int(byte) >> (sb % 8)) & 1) << t
    return v


def u16(plane, i, j, row_bytes):
    """Little-endian uint16 at row bytes [j, j+2) of row i."""
    return int(plane[rit_addr(i, j, row_bytes)]) | (int(plane[rit_addr(i, j + 1, row_bytes)]) << 8)


def f16(bits):
    return float(np.array([bits], dtype=np.uint16).view(np.float16)[0])


def parse_header(buf):
    assert bytes(buf[:4]) == b"CQL1"
    (ver,) = struct.unpack_from("<I", bytes(buf[:8]), 4)
    d = struct.unpack_from("<iiiiiffiiiIii", bytes(buf[:72]), 8)
    assert not any(buf[60:72])                      # reserved descriptor words
    total, nnz = struct.unpack_from("<QQ", bytes(buf[:88]), 72)
    off = struct.unpack_from("<13Q", bytes(buf[:296]), 88)
    ln = struct.unpack_from("<13Q", bytes(buf[:296]), 192)
    assert not any(buf[296:512])
    return ver, d, total, nnz, list(off), list(ln)


CASES = [
    ("tiny", dict(n=128, k=256, rank=16)),
    ("tiny", dict(n=128, k=256, rank=32, codec="int3")),
    ("tiny", dict(n=128, k=256, rank=0, mask="none")),
    ("down_unstructured", dict(n=128, k=384, rank=16)),
    ("lut_dense_sparse", dict(n=128, k=256)),
    ("lut_dense_sparse", dict(n=128, k=256, codec="lut4")),
    ("mlp_up_slimo", dict(n=128, k=512, rank=16, salient_channels=5, salient_log2=1)),
    ("lut_dense_sparse", dict(n=128, k=256, salient_channels=32, salient_log2=3)),
]


@pytest.mark.parametrize("name,over", CASES)
def test_packed_bytes_decode_to_parts(name, over):
    wl = workload(name, **over)
    inp = make_layer_inputs(wl, max_batch=1)
    d = O.desc_for(wl)
    parts = O.compress(d, inp["w"], inp["L"], inp["R"], inp["act_absmean"])
    buf = O.pack_bytes(d, parts)
    ver, hd, total, nnz, off, ln = parse_header(buf)
    assert ver == 2 and total == buf.size
    assert hd[:5] == (d.n_out, d.k_in, d.mask, d.codec, 128) and hd[7] == d.rank
    assert hd[11:13] == (d.salient_channels, d.salient_log2)
    n, k, r = d.n_out, d.k_in, d.rank
    bits = {0: 4, 1: 3, 2: 3, 3: 4}[d.codec]
    plane = lambda p: buf[off[p]: off[p] + ln[p]]
    for p in range(13):
        assert off[p] % 256 == 0
    if d.salient_channels:
        sal = np.frombuffer(bytes(plane(O.P_SALIENT)), dtype="<u2")
        assert len(sal) == d.salient_channels and (np.diff(sal.astype(int)) > 0).all()
        assert (sal == parts["salient"]).all()
    else:
        assert ln[O.P_SALIENT] == 0
    keep = parts["keep"]

    vals = plane(O.P_VALUES)
    vrb = ln[O.P_VALUES] // n
    sc = plane(O.P_SCALES)
    srb = ln[O.P_SCALES] // n
    for i in range(0, n, 7):                       # every 7th row, all columns
        cols = [c for c in range(k) if keep[i, c]]
        for ci, c in enumerate(cols):
            u = read_bits(vals, i, vrb, bits * ci, bits)
            if d.codec in (O.CODEC_INT4, O.CODEC_INT3):
                assert u - (1 << (bits - 1)) == parts["q"][i, c]
            else:
                assert u == parts["codes"][i, c]
        if d.mask == O.MASK_2_4:
            meta = plane(O.P_META)
            for g in range(k // 4):
                nib = read_bits(meta, i, k // 8, 4 * g, 4)
                i0, i1 = nib & 3, nib >> 2
                assert [c - 4 * g for c in cols if 4 * g <= c < 4 * g + 4] == [i0, i1]
        elif d.mask == O.MASK_BITMAP50:
            meta = plane(O.P_META)
            voff = plane(O.P_VOFF)
            vorb = ln[O.P_VOFF] // n
            for c in range(k):
                assert read_bits(meta, i, k // 8, c, 1) == int(keep[i, c])
            for g in range(k // 128):
                lo = u16(voff, i, 2 * g, vorb)
                assert lo == int(keep[i, : 128 * g].sum())
        if d.codec in (O.CODEC_INT4, O.CODEC_INT3):
            for g in range(k // 128):
                b = u16(sc, i, 2 * g, srb)
                assert f16(b) == parts["scales"][i, g]
        else:
            for j in range(1 << bits):
                b = u16(sc, i, 2 * j, srb)
                assert f16(b) == parts["centroids"][i, j]
    if d.outlier_frac > 0:
        rp = np.frombuffer(bytes(plane(O.P_CSR_ROWPTR)), dtype="<i4")
        col = np.frombuffer(bytes(plane(O.P_CSR_COL)), dtype="<u2")
        val = np.frombuffer(bytes(plane(O.P_CSR_VAL)), dtype="<f2")
        assert nnz == len(col) == rp[-1]
        assert (rp == parts["csr_row_ptr"]).all() and (col == parts["csr_col"]).all()
        assert (val.astype(np.float64) == parts["csr_val"]).all()
    if r:
        rv, rs = plane(O.P_R_VALUES), plane(O.P_R_SCALES)
        rrb = k // 2
        rsrb = ln[O.P_R_SCALES] // ((r + 31) // 32 * 32)
        for j in range(r):
            for c in range(0, k, 5):
                assert read_bits(rv, j, rrb, 4 * c, 4) - 8 == parts["R_q"][j, c]
            for g in range(k // 128):
                b = u16(rs, j, 2 * g, rsrb)
                assert f16(b) == parts["R_s"][j, g]
        lv = plane(O.P_L_VALUES)
        lrb = ln[O.P_L_VALUES] // n
        for i in range(0, n, 3):
            for j in range(r):
                assert read_bits(lv, i, lrb, 4 * j, 4) - 8 == parts["L_q"][i, j]
        ls = np.frombuffer(bytes(plane(O.P_L_SCALES)), dtype="<f2").astype(np.float64)
        assert (ls.reshape(n // 128, r) == parts["L_s"]).all()


def test_handworked_fixture():
    g = json.load(open(os.path.join(GOLDEN, "handworked_2of4_int4.json")))
    n, k = 128, 128
    w = np.zeros((n, k))
    for i in range(n):
        grp = g["group_values_by_rotation"][str(i % 4)]
        w[i] = np.tile(grp, k // 4)
    d = O.OracleDesc(n, k, O.MASK_2_4, O.CODEC_INT4, clip_alpha=1.0)
    parts = O.compress(d, w)
    buf = O.pack_bytes(d, parts)
    lay = O.packed_layout(d)
    assert lay["off"] == g["layout"]["off"] and lay["len"] == g["layout"]["len"]
    assert lay["total"] == g["layout"]["total"] == buf.size
    off = lay["off"]
    for i in range(n):
        rot = str(i % 4)
        vb = int(g["values_byte_by_rotation"][rot], 16)
        mb = int(g["meta_byte_by_rotation"][rot], 16)
        for j in range(g["values_row_bytes"]):
            assert buf[off[1] + rit_addr(i, j, 32)] == vb
        for j in range(g["meta_row_bytes"]):
            assert buf[off[2] + rit_addr(i, j, 16)] == mb
        s0 = u16(buf[off[3]:], i, 0, 16)
        assert s0 == int(g["scale_fp16_bits"], 16)
        assert not any(buf[off[3] + rit_addr(i, j, 16)] for j in range(2, 16))


@pytest.mark.parametrize("name,over", [
    ("tiny", dict(n=128, k=256, rank=16, outlier_frac=0.003)),                 # 2:4 int4 + CSR
    ("down_unstructured", dict(n=128, k=384, rank=0)),                         # bitmap int3
    ("lut_dense_sparse", dict(n=128, k=256)),                                  # LUT3 + CSR
    ("mlp_up_slimo", dict(n=128, k=512, rank=16, salient_channels=5, salient_log2=2)),
])
def test_compressed_matrix_is_what_the_bytes_hold(name, over):
    """W_C (the codes' values plus the CSR outliers, in the space the codec
    encoded), which the adapter construction compensates, equals a
    reconstruction of each weight read field by field from the packed bytes:
    its code (at its rank among the row's kept columns), its group scale or
    row centroid, and its CSR entry if it has one."""
    wl = workload(name, **over)
    inp = make_layer_inputs(wl, max_batch=1)
    d = O.desc_for(wl)
    parts = O.compress(d, inp["w"], inp["L"], inp["R"], inp["act_absmean"])
    buf = O.pack_bytes(d, parts)
    _, _, _, _, off, ln = parse_header(buf)
    plane = lambda p: buf[off[p]: off[p] + ln[p]]
    n, k = d.n_out, d.k_in
    bits = {0: 4, 1: 3, 2: 3, 3: 4}[d.codec]
    vals, sc = plane(O.P_VALUES), plane(O.P_SCALES)
    vrb, srb = ln[O.P_VALUES] // n, ln[O.P_SCALES] // n
    csr = {}
    if ln[O.P_CSR_COL]:
        rp = np.frombuffer(bytes(plane(O.P_CSR_ROWPTR)), dtype="<i4")
        col = np.frombuffer(bytes(plane(O.P_CSR_COL)), dtype="<u2")
        val = np.frombuffer(bytes(plane(O.P_CSR_VAL)), dtype="<f2")
        for i in range(n):
            for e in range(rp[i], rp[i + 1]):
                csr[(i, int(col[e]))] = float(val[e])
    wc = O.compressed_matrix(parts)
    for i in range(0, n, 9):
        if d.mask == O.MASK_2_4:
            meta = plane(O.P_META)
            kept = []
            for g in range(k // 4):
                nib = read_bits(meta, i, k // 8, 4 * g, 4)
                kept += [4 * g + (nib & 3), 4 * g + (nib >> 2)]
        elif d.mask == O.MASK_BITMAP50:
            meta = plane(O.P_META)
            kept = [c for c in range(k) if read_bits(meta, i, k // 8, c, 1)]
        else:
            kept = list(range(k))
        slot = {c: j for j, c in enumerate(kept)}
        for c in range(k):
            v = 0.0
            if c in slot:
                u = read_bits(vals, i, vrb, bits * slot[c], bits)
                if d.codec in (O.CODEC_INT4, O.CODEC_INT3):
                    v = (u - (1 << (bits - 1))) * f16(u16(sc, i, 2 * (c // 128), srb))
                else:
                    v = f16(u16(sc, i, 2 * u, srb))
            v += csr.get((i, c), 0.0)
            assert wc[i, c] == v, (i, c)
