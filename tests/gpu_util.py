"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
library through its C ABI, and compare with the oracle."""
import math
import os
import time

import numpy as np

import oracle as O
import sparse_quantized_rank_b200 as C
from workloads import make_layer_inputs

DT_NAME = {C.CQL_DT_F32: "f32", C.CQL_DT_F16: "f16", C.CQL_DT_BF16: "bf16"}

# Per-config metrics of this session (written as JSON lines by conftest when
# CQL_METRICS_JSONL names a file): every parity comparison's max relative
# error, and the oracle's time for every reference forward.
METRICS = []


def c_desc(od: O.OracleDesc, flags: int = 0):
    return C.make_desc(od.n_out, od.k_in, od.mask, od.codec, od.clip_alpha, od.outlier_frac, od.rank, flags,
                       od.salient_channels, od.salient_log2)


def device_inputs(inp, wl, dev):
    import torch
    if wl.w_dtype == "bf16":
        W = torch.from_numpy(inp["w_bits"].view(np.int16)).to(dev).view(torch.bfloat16)
    else:
        W = torch.from_numpy(inp["w"]).to(dev)
    L = torch.from_numpy(inp["L"]).to(dev) if inp["L"] is not None else None
    R = torch.from_numpy(inp["R"]).to(dev) if inp["R"] is not None else None
    xt = torch.float16 if wl.x_dtype == "f16" else torch.bfloat16
    x = torch.from_numpy(inp["x_bits"].view(np.int16)).to(dev).view(xt)
    return W, L, R, x


class Case:
    """One workload: oracle parts/bytes (CPU) and the packed layer (GPU)."""

    def __init__(self, wl, dev, max_batch=None):
        import torch
        self.wl = wl
        self.inp = make_layer_inputs(wl, max_batch=max_batch)
        self.od = O.desc_for(wl)
        self.parts = O.compress(self.od, self.inp["w"], self.inp["L"], self.inp["R"], self.inp["act_absmean"],
                                self.inp["fisher"])
        self.ref_bytes = O.pack_bytes(self.od, self.parts)
        self.W, self.L, self.R, self.x = device_inputs(self.inp, wl, dev)
        act = self.inp["act_absmean"]
        self.act = None if act is None else torch.from_numpy(act).to(dev)
        fis = self.inp["fisher"]
        self.fisher = None if fis is None else torch.from_numpy(fis).to(dev)
        self.layer = C.CompressedLinear(c_desc(self.od), self.W, self.L, self.R, act_absmean=self.act,
                                        fisher=self.fisher)
        torch.cuda.synchronize()

    def packed_bytes(self):
        return self.layer.packed.cpu().numpy()

    def forward(self, batch, out_dtype, flags=0):
        x = self.x[:batch].contiguous()
        y = self.layer.forward(x, out_dtype=out_dtype, flags=flags)
        return y

    def reference(self, batch, flags=0):
        t0 = time.perf_counter()
        y = O.forward(self.parts, self.inp["x"][:batch].astype(np.float64), flags=flags)
        METRICS.append({"kind": "oracle_time", "workload": self.wl.name, "n": self.wl.n, "k": self.wl.k,
                        "batch": int(batch), "flags": int(flags), "oracle_ms": (time.perf_counter() - t0) * 1e3,
                        "threads": os.cpu_count()})
        return y


def half_ulp(ref: np.ndarray, dt: str) -> np.ndarray:
    """Half an ulp of the output format at |ref| (the rounding the output
    conversion itself may add)."""
    a = np.abs(ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1e-300)))
    if dt == "bf16":
        e = np.maximum(e, -126)
        return np.exp2(e - 8)
    if dt == "f16":
        e = np.maximum(e, -14)
        return np.exp2(e - 11)
    return np.zeros_like(a)


def check_close(y, ref, dt: str, tol: float = 2e-3, what: str = ""):
    """|y - r| <= tol * max(|r|, rms(r)) (+ half an output ulp for 16-bit
    outputs).  Returns the rel_err metric."""
    yv = y.float().cpu().numpy().astype(np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert yv.shape == ref.shape, (yv.shape, ref.shape)
    rms = math.sqrt(float(np.mean(ref * ref))) if ref.size else 0.0
    den = np.maximum(np.abs(ref), rms)
    bound = tol * den + half_ulp(ref, dt)
    err = np.abs(yv - ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err / np.maximum(bound, 1e-300)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {err.size} outside tolerance; worst at {i}: "
                             f"y={yv[i]!r} ref={ref[i]!r} err={err[i]:.3e} bound={bound[i]:.3e} "
                             f"rel_err={O.rel_err(yv, ref):.3e}")
    r = O.rel_err(yv, ref)
    METRICS.append({"kind": "parity", "what": what, "out_dtype": dt, "max_rel_err": r, "tol": tol,
                    "elements": int(err.size)})
    return r
