"""Python binding of libcql, the B200 compressed linear layer.

    y = deq(Q (.) M) x + S_csr x + deq(L_q) (deq(R_q) x)

Argument marshalling only: every function below calls the C ABI declared in
``include/cql.h`` with the same name, passing device pointers taken from torch
tensors (torch supplies device memory and streams, nothing else).  There is no
CPU fallback: if ``libcql.so`` is missing or cannot be loaded, the first call
raises.

``CompressedLinear`` is a small convenience owner of the packed buffer and
workspace for one layer.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcql.so")
LIB_CHECKED_PATH = os.path.join(HERE, "libcql_checked.so")   # the range-checked build

# enums (include/cql.h)
CQL_OK, CQL_ERR_ARG, CQL_ERR_ALIGN, CQL_ERR_FORMAT, CQL_ERR_SIZE, CQL_ERR_UNSUPPORTED, \
    CQL_ERR_CUDA, CQL_ERR_TIMEOUT, CQL_ERR_RANGE = range(9)
CQL_MASK_NONE, CQL_MASK_2_4, CQL_MASK_BITMAP50 = 0, 1, 2
CQL_CODEC_INT4_SYM, CQL_CODEC_INT3_SYM, CQL_CODEC_LUT3_ROW, CQL_CODEC_LUT4_ROW = 0, 1, 2, 3
CQL_DT_F32, CQL_DT_F16, CQL_DT_BF16 = 0, 1, 2
CQL_FLAG_NO_MAIN, CQL_FLAG_NO_CSR, CQL_FLAG_NO_LOWRANK = 1, 2, 4
CQL_FLAG_DEBUG_SKIP_X = 0x100
CQL_FLAG_CUDA_CORE = 0x200
CQL_NPLANES = 13
CQL_MAX_DECODE_BATCH = 16

EXPORTED = (
    "cql_status_string", "cql_version", "cql_packed_layout", "cql_pack_workspace_size",
    "pack_compressed_weight", "cql_workspace_size", "cql_workspace_init",
    "compressed_linear_forward", "cql_get_device_status", "compressed_linear_forward_noalloc",
    "cql_adapter_workspace_size", "cql_build_adapters", "cql_read_header", "cql_plane_checksums",
)


class cql_desc(ctypes.Structure):
    _fields_ = [
        ("n_out", ctypes.c_int32), ("k_in", ctypes.c_int32), ("mask", ctypes.c_int32),
        ("codec", ctypes.c_int32), ("group", ctypes.c_int32), ("clip_alpha", ctypes.c_float),
        ("outlier_frac", ctypes.c_float), ("rank", ctypes.c_int32), ("adapter_bits", ctypes.c_int32),
        ("adapter_group", ctypes.c_int32), ("flags", ctypes.c_uint32), ("salient_channels", ctypes.c_int32),
        ("salient_log2", ctypes.c_int32), ("reserved", ctypes.c_int32 * 3),
    ]


class cql_layout(ctypes.Structure):
    _fields_ = [
        ("total_bytes", ctypes.c_uint64), ("nnz", ctypes.c_uint64),
        ("off", ctypes.c_uint64 * CQL_NPLANES), ("len", ctypes.c_uint64 * CQL_NPLANES),
    ]


class CqlError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {cql_status_string(status)} ({status})")
        self.status = status


_libs = {}
_active = LIB_PATH


def use_library(checked: bool) -> None:
    """Route every call of this module to the range-checked library
    (libcql_checked.so, built with -DCQL_CHECKED) or back to libcql.so.
    Objects keep the buffers they made with either; both libraries share the
    packed format and the workspace layout."""
    global _active
    _active = LIB_CHECKED_PATH if checked else LIB_PATH


def lib():
    """The loaded library (raises if it is missing: there is no fallback)."""
    if _active not in _libs:
        if not os.path.exists(_active):
            raise RuntimeError(f"{_active} is missing: build it with "
                               "`python -m sparse_quantized_rank_b200.build`"
                               + (" --checked" if _active == LIB_CHECKED_PATH else ""))
        L = ctypes.CDLL(_active)
        P, U64, I32 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int32
        L.cql_status_string.restype = ctypes.c_char_p
        L.cql_status_string.argtypes = [ctypes.c_int]
        L.cql_version.restype = I32
        L.cql_packed_layout.argtypes = [ctypes.POINTER(cql_desc), ctypes.POINTER(cql_layout)]
        L.cql_pack_workspace_size.argtypes = [ctypes.POINTER(cql_desc), ctypes.POINTER(U64)]
        L.pack_compressed_weight.argtypes = [ctypes.POINTER(cql_desc), P, ctypes.c_int, P, P, P, P, P, U64, P,
                                             U64, P]
        L.cql_workspace_size.argtypes = [ctypes.POINTER(cql_desc), I32, ctypes.POINTER(U64)]
        L.cql_workspace_init.argtypes = [P, U64, P]
        L.compressed_linear_forward.argtypes = [ctypes.POINTER(cql_desc), P, P, ctypes.c_int, P, ctypes.c_int,
                                                I32, P, U64, P]
        L.cql_get_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int)]
        L.compressed_linear_forward_noalloc.argtypes = [ctypes.POINTER(cql_desc), P, P, ctypes.c_int, P,
                                                        ctypes.c_int, I32, P]
        L.cql_adapter_workspace_size.argtypes = [ctypes.POINTER(cql_desc), ctypes.POINTER(U64)]
        L.cql_build_adapters.argtypes = [ctypes.POINTER(cql_desc), P, ctypes.c_int, P, P, P, P, P, U64, P]
        L.cql_read_header.argtypes = [P, U64, ctypes.POINTER(cql_desc), ctypes.POINTER(cql_layout)]
        L.cql_plane_checksums.argtypes = [P, U64, ctypes.POINTER(ctypes.c_uint32 * CQL_NPLANES)]
        for fn in EXPORTED[2:]:
            getattr(L, fn).restype = ctypes.c_int
        _libs[_active] = L
    return _libs[_active]


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st: int, where: str):
    if st != CQL_OK:
        raise CqlError(st, where)


def make_desc(n_out: int, k_in: int, mask: int = CQL_MASK_2_4, codec: int = CQL_CODEC_INT4_SYM,
              clip_alpha: float = 0.9, outlier_frac: float = 0.0, rank: int = 0, flags: int = 0,
              salient_channels: int = 0, salient_log2: int = 0) -> cql_desc:
    d = cql_desc()
    d.n_out, d.k_in, d.mask, d.codec, d.group = n_out, k_in, mask, codec, 128
    d.clip_alpha, d.outlier_frac, d.rank = clip_alpha, outlier_frac, rank
    d.adapter_bits, d.adapter_group, d.flags = 4, 128, flags
    d.salient_channels, d.salient_log2 = salient_channels, salient_log2
    return d


# ---------------------------------------------------------------------------
# the C ABI, same names
# ---------------------------------------------------------------------------

def cql_status_string(s: int) -> str:
    return lib().cql_status_string(int(s)).decode()


def cql_version() -> int:
    return int(lib().cql_version())


def cql_packed_layout(desc: cql_desc) -> cql_layout:
    out = cql_layout()
    _check(lib().cql_packed_layout(ctypes.byref(desc), ctypes.byref(out)), "cql_packed_layout")
    return out


def cql_pack_workspace_size(desc: cql_desc) -> int:
    v = ctypes.c_uint64()
    _check(lib().cql_pack_workspace_size(ctypes.byref(desc), ctypes.byref(v)), "cql_pack_workspace_size")
    return int(v.value)


def pack_compressed_weight(desc, W, w_dt, L, R, act_absmean, fisher, packed, packed_bytes, workspace, ws_bytes,
                           stream=None):
    _check(lib().pack_compressed_weight(ctypes.byref(desc), _ptr(W), int(w_dt), _ptr(L), _ptr(R), _ptr(act_absmean),
                                        _ptr(fisher), _ptr(packed), int(packed_bytes), _ptr(workspace),
                                        int(ws_bytes), _stream(stream)),
           "pack_compressed_weight")


def cql_workspace_size(desc: cql_desc, batch: int) -> int:
    v = ctypes.c_uint64()
    _check(lib().cql_workspace_size(ctypes.byref(desc), int(batch), ctypes.byref(v)), "cql_workspace_size")
    return int(v.value)


def cql_workspace_init(workspace, ws_bytes, stream=None):
    _check(lib().cql_workspace_init(_ptr(workspace), int(ws_bytes), _stream(stream)), "cql_workspace_init")


def compressed_linear_forward(desc, packed, x, x_dt, y, y_dt, batch, workspace, ws_bytes, stream=None):
    _check(lib().compressed_linear_forward(ctypes.byref(desc), _ptr(packed), _ptr(x), int(x_dt), _ptr(y), int(y_dt),
                                           int(batch), _ptr(workspace), int(ws_bytes), _stream(stream)),
           "compressed_linear_forward")


def compressed_linear_forward_noalloc(desc, packed, x, x_dt, y, y_dt, batch, stream=None):
    """Forward without a workspace (the library's fixed 4 MiB scratch array is
    used instead); for callers that cannot allocate device memory."""
    _check(lib().compressed_linear_forward_noalloc(ctypes.byref(desc), _ptr(packed), _ptr(x), int(x_dt), _ptr(y),
                                                   int(y_dt), int(batch), _stream(stream)),
           "compressed_linear_forward_noalloc")


def cql_adapter_workspace_size(desc: cql_desc) -> int:
    v = ctypes.c_uint64()
    _check(lib().cql_adapter_workspace_size(ctypes.byref(desc), ctypes.byref(v)), "cql_adapter_workspace_size")
    return int(v.value)


def cql_build_adapters(desc, W, w_dt, packed, act_absmean, L, R, workspace, ws_bytes, stream=None):
    _check(lib().cql_build_adapters(ctypes.byref(desc), _ptr(W), int(w_dt), _ptr(packed), _ptr(act_absmean), _ptr(L),
                                    _ptr(R), _ptr(workspace), int(ws_bytes), _stream(stream)),
           "cql_build_adapters")


def cql_read_header(packed_host: bytes):
    """(cql_desc, cql_layout) stored in a host copy of a packed buffer."""
    buf = ctypes.create_string_buffer(bytes(packed_host), len(packed_host))
    d, lay = cql_desc(), cql_layout()
    _check(lib().cql_read_header(ctypes.cast(buf, ctypes.c_void_p), len(packed_host), ctypes.byref(d),
                                 ctypes.byref(lay)), "cql_read_header")
    return d, lay


def cql_plane_checksums(packed_host: bytes):
    """CRC-32 of every plane of a host copy of a packed buffer."""
    buf = ctypes.create_string_buffer(bytes(packed_host), len(packed_host))
    out = (ctypes.c_uint32 * CQL_NPLANES)()
    _check(lib().cql_plane_checksums(ctypes.cast(buf, ctypes.c_void_p), len(packed_host), ctypes.byref(out)),
           "cql_plane_checksums")
    return list(out)


def cql_get_device_status(workspace, stream=None) -> int:
    """Device error word of a workspace (None: the fixed scratch of the
    no-workspace entry point on the current device)."""
    v = ctypes.c_int()
    _check(lib().cql_get_device_status(_ptr(workspace), _stream(stream), ctypes.byref(v)), "cql_get_device_status")
    return int(v.value)


# ---------------------------------------------------------------------------
# convenience owner of one packed layer
# ---------------------------------------------------------------------------

def check_forward_args(desc: cql_desc, x, out=None, device=None) -> None:
    """Raise ValueError unless x is a contiguous [B][K] fp16/bf16 tensor and
    out (if given) a contiguous [B][N] fp32/fp16/bf16 tensor, both on
    ``device`` (the packed layer's).  The C entry point receives raw
    pointers and cannot see a tensor's size, so a wrong shape would make the
    kernels read or write past its end: it is refused here."""
    import torch
    if x.dim() != 2 or x.shape[1] != desc.k_in or not x.is_contiguous():
        raise ValueError(f"x must be a contiguous [batch][{desc.k_in}] tensor, got {tuple(x.shape)}")
    if x.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError(f"x must be float16 or bfloat16, got {x.dtype}")
    if device is not None and x.device != device:
        raise ValueError(f"x is on {x.device}, the packed layer on {device}")
    if out is not None:
        if tuple(out.shape) != (x.shape[0], desc.n_out) or not out.is_contiguous():
            raise ValueError(f"out must be a contiguous [{x.shape[0]}][{desc.n_out}] tensor, got {tuple(out.shape)}")
        if out.dtype not in (torch.float32, torch.float16, torch.bfloat16):
            raise ValueError(f"out must be float32, float16 or bfloat16, got {out.dtype}")
        if out.device != x.device:
            raise ValueError(f"out is on {out.device}, x on {x.device}")


def check_pack_args(desc: cql_desc, W, L=None, R=None, act_absmean=None, fisher=None) -> None:
    """Raise ValueError unless the packer's inputs have the shapes and dtypes
    the descriptor implies (W [N][K] fp32/bf16; L [N][r], R [r][K],
    act_absmean [K], fisher [N][K] fp32) and share W's device.  The C entry
    point reads them through raw pointers and cannot check their sizes."""
    import torch
    n, k, r = desc.n_out, desc.k_in, desc.rank
    want = [("W", W, (n, k), (torch.float32, torch.bfloat16))]
    if r > 0:
        if L is None or R is None:
            raise ValueError(f"rank {r} needs L [{n}][{r}] and R [{r}][{k}]")
        want += [("L", L, (n, r), (torch.float32,)), ("R", R, (r, k), (torch.float32,))]
    if act_absmean is not None:
        want.append(("act_absmean", act_absmean, (k,), (torch.float32,)))
    elif desc.salient_channels > 0:
        raise ValueError("salient_channels > 0 needs act_absmean [K]")
    if fisher is not None:
        want.append(("fisher", fisher, (n, k), (torch.float32,)))
    for name, t, shape, dts in want:
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
        if t.dtype not in dts:
            raise ValueError(f"{name} must be one of {dts}, got {t.dtype}")
        if t.device != W.device:
            raise ValueError(f"{name} is on {t.device}, W on {W.device}")


def _dt_of(t) -> int:
    import torch
    return {torch.float32: CQL_DT_F32, torch.float16: CQL_DT_F16, torch.bfloat16: CQL_DT_BF16}[t.dtype]


class CompressedLinear:
    """Packs one layer on the GPU and runs its forward pass.

    ``W`` is a CUDA tensor [N][K] (fp32 or bf16), ``L`` [N][r] and ``R`` [r][K]
    fp32 CUDA tensors (or None when rank is 0), ``act_absmean`` a fp32 CUDA
    tensor [K] of per-channel mean |x| (SLiM^O layers only), ``fisher`` a
    fp32 CUDA tensor [N][K] Fisher diagonal (LUT codecs: weighted k-means).
    A descriptor with clip_alpha 0 has the packer search alpha; the chosen
    value is in ``clip_alpha()``.  Buffers are torch tensors: the packed
    layer once, and one forward workspace per distinct batch size, on the
    first call at that size (its layout depends on the batch, and the
    kernels leave it ready for the next call at the same size); later calls
    allocate only the output tensor (or none, given ``out``)."""

    def __init__(self, desc: cql_desc, W, L=None, R=None, stream=None, act_absmean=None, fisher=None):
        import torch
        check_pack_args(desc, W, L, R, act_absmean, fisher)
        self.desc = desc
        self.layout = cql_packed_layout(desc)
        dev = W.device
        self.packed = torch.empty(self.layout.total_bytes, dtype=torch.uint8, device=dev)
        pw = cql_pack_workspace_size(desc)
        pws = torch.empty(max(pw, 256), dtype=torch.uint8, device=dev)
        args = [None if t is None else t.contiguous() for t in (W, L, R, act_absmean, fisher)]
        if isinstance(stream, torch.cuda.Stream):
            # the pack runs on a side stream: keep the allocator from reusing
            # the inputs' memory (the caller may drop W right away, and the
            # contiguous copies are temporaries) before that stream is done
            for t in args:
                if t is not None:
                    t.record_stream(stream)
        Wc, Lc, Rc, ac, fc = args
        pack_compressed_weight(desc, Wc, _dt_of(Wc), Lc, Rc, ac, fc, self.packed, self.layout.total_bytes, pws, pw,
                               stream)
        self._pack_ws = pws            # kept alive until the pack kernels ran
        self._ws = {}

    def clip_alpha(self) -> float:
        """The clip threshold the layer was encoded with (read from the packed
        header: the searched value when the descriptor asked for a search)."""
        return float(self.packed[28:32].cpu().view(__import__("torch").float32).item())

    @classmethod
    def with_adapters(cls, desc: cql_desc, W, act_absmean=None, naive: bool = False, stream=None, fisher=None):
        """Pack W with adapters built on the GPU from its own compression
        error: SLiM-LoRA weighted by ``act_absmean`` (Naive-LoRA when
        ``naive`` or when no statistic is given).  Packs with zero adapters,
        builds L and R (cql_build_adapters), packs again with them.  The
        built factors are kept as ``.L`` and ``.R``."""
        import torch
        dev = W.device
        r = desc.rank
        zL = torch.zeros(desc.n_out, r, dtype=torch.float32, device=dev)
        zR = torch.zeros(r, desc.k_in, dtype=torch.float32, device=dev)
        first = cls(desc, W, zL, zR, stream=stream, act_absmean=act_absmean, fisher=fisher)
        nb = cql_adapter_workspace_size(desc)
        ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev)
        stat = None if (naive or act_absmean is None) else act_absmean.contiguous()
        cql_build_adapters(desc, W.contiguous(), _dt_of(W), first.packed, stat, zL, zR, ws, nb, stream)
        layer = cls(desc, W, zL, zR, stream=stream, act_absmean=act_absmean, fisher=fisher)
        layer.L, layer.R = zL, zR
        layer._build_ws = (ws, first)            # alive until the queued kernels ran
        return layer

    def workspace(self, batch: int, stream=None):
        import torch
        nbytes = cql_workspace_size(self.desc, batch)
        ws = self._ws.get(batch)
        if ws is None:
            ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.packed.device)
            cql_workspace_init(ws, nbytes, stream)
            self._ws[batch] = ws
        return ws, nbytes

    def forward(self, x, out_dtype=None, out=None, flags: Optional[int] = None, stream=None):
        import torch
        check_forward_args(self.desc, x, out, self.packed.device)
        batch = x.shape[0]
        if out is None:
            out = torch.empty(batch, self.desc.n_out, dtype=out_dtype or x.dtype, device=x.device)
        ws, nbytes = self.workspace(batch, stream)
        d = self.desc
        if flags is not None:
            d = cql_desc.from_buffer_copy(self.desc)
            d.flags = flags
        compressed_linear_forward(d, self.packed, x, _dt_of(x), out, _dt_of(out), batch, ws, nbytes, stream)
        return out

    def device_status(self, batch: int, stream=None) -> int:
        ws, _ = self.workspace(batch, stream)
        return cql_get_device_status(ws, stream)

    def pack_status(self, stream=None) -> int:
        """Device error word of the pack that built this layer: CQL_OK, or
        CQL_ERR_RANGE when the range-checked library saw a pack kernel index
        outside its plane."""
        return cql_get_device_status(self._pack_ws, stream)
