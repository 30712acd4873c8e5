"""Seeded synthetic inputs for the gated delta-rule recurrence.

This module is shared by the CUDA path's tests/bench and by the fp64 oracle's
tests. It holds only the random draws and the workload recipes (shapes, value
distributions, gate modes); none of the recurrence's arithmetic lives here.

The generator itself is C (``gen.c``, counter-based splitmix64 + Box-Muller,
OpenMP over elements); this file builds it with gcc on first use and wraps it
with ctypes.

Workloads (the five synthetic configurations of the gated delta-rule pages:
GDN scalar gates, KDA channel decay, FG2-GDN+ with OSDN preconditioner, decode):

  gdn_fp32_small   B=1  H=2  T=256   d=64  fp32  alpha~U(0.9,1) scalar, beta=sigmoid(N) scalar, S0=0
  gdn_prefill      B=8  H=16 T=4096  d=128 bf16  alpha=exp(-softplus(N)*0.1) scalar, beta scalar, S0=0
  kda              B=4  H=32 T=8192  d=128 bf16  alpha=exp(-softplus(N)*0.05) per key channel, beta scalar,
                                                 S0~N(0,0.02^2)
  fg2_osdn_long    B=2  H=16 T=32768 d=128 bf16  channel alpha, beta_k in R^dk, beta_v in R^dv (sigmoid(N)),
                                                 preconditioner d=1+0.1*N per key channel, S0~N(0,0.02^2)
  decode           1024 sequences, H=32, d=128: resident S~N(0,0.02^2) fp32, one bf16 token per step,
                   channel alpha, beta_k, beta_v as in fg2_osdn_long, 100 steps
  (backward)       every workload above also draws the backward's cotangents: dO ~ N(0,1) like o,
                   dS_T ~ N(0, 0.1^2) fp32 (make_bwd_inputs)
  osdn_phase1      the OSDN preconditioner scan on fg2_osdn_long's keys (same seed): B=2 H=16 T=32768
                   d_k=128 bf16 k, beta=sigmoid(N) per token, retention r~U(0.95,1) per token, eta=0.5,
                   d_0 = 1

q and k are drawn N(0,1) per element and L2-normalised per (b, t, h) row in fp64
before rounding to the storage dtype; v ~ N(0,1).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libdngen.so")
_lock = threading.Lock()
_lib = None

GEN_NORMAL, GEN_UNIFORM, GEN_SIGMOID, GEN_EXP_NEG_SOFTPLUS, GEN_L2ROWS = 0, 1, 2, 3, 4
OUT_F64, OUT_F32, OUT_BF16 = 0, 1, 2

# gate modes, same numbering as the C ABI (absent / one value per token / one per channel)
GATE_ONE, GATE_SCALAR, GATE_CHANNEL = 0, 1, 2

SEED_BASE = 20260000
TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "alpha": 3, "beta_k": 4, "beta_v": 5, "key_scale": 6, "S0": 7,
              "beta": 8, "retention": 9, "dO": 10, "dS_T": 11}


def build(force: bool = False) -> str:
    """Compile gen.c into libdngen.so next to this file (gcc, -O2, OpenMP)."""
    src = os.path.join(_HERE, "gen.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _LIB_PATH, src, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            lib.dn_gen_fill.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int,
                                        ctypes.c_double, ctypes.c_double, ctypes.c_int64, ctypes.c_int,
                                        ctypes.c_void_p]
            lib.dn_gen_fill.restype = ctypes.c_int
            lib.dn_gen_splitmix_at.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
            lib.dn_gen_splitmix_at.restype = ctypes.c_uint64
            lib.dn_gen_normal_at.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
            lib.dn_gen_normal_at.restype = ctypes.c_double
            _lib = lib
    return _lib


def splitmix_at(seed: int, ctr: int) -> int:
    return int(_load().dn_gen_splitmix_at(seed, ctr))


def normal_at(seed: int, i: int) -> float:
    return float(_load().dn_gen_normal_at(seed, i))


_OUT = {"f64": (OUT_F64, np.float64), "f32": (OUT_F32, np.float32), "bf16": (OUT_BF16, np.uint16)}


def fill(shape, seed: int, kind: int, p0: float = 0.0, p1: float = 1.0, dtype: str = "f32",
         offset: int = 0, row: int = 0, out: np.ndarray | None = None) -> np.ndarray:
    """Draw a tensor. bf16 tensors come back as np.uint16 bit patterns."""
    code, npdt = _OUT[dtype]
    n = int(np.prod(shape)) if len(shape) else 1
    if out is None:
        out = np.empty(shape, dtype=npdt)
    assert out.dtype == npdt and out.flags["C_CONTIGUOUS"] and out.size == n
    rc = _load().dn_gen_fill(seed, offset, n, kind, p0, p1, row, code, out.ctypes.data)
    if rc != 0:
        raise ValueError("dn_gen_fill rejected its arguments")
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (np.uint16) to float32."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_to_f32(x).astype(np.float64)
    return x.astype(np.float64)


@dataclass
class Workload:
    """One synthetic configuration: shapes, storage dtype and gate recipe."""
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    io: str                      # "f32" or "bf16" for q, k, v, o
    alpha: int                   # GATE_* mode
    alpha_kind: tuple            # (GEN_*, p0, p1)
    beta_k: int
    beta_v: int
    key_scale: int
    s0_std: float                # 0 -> S0 absent (zero)
    chunk: int = 64
    steps: int = 0               # >0: decode workload with this many steps
    cfg_index: int = 0           # selects the seed block
    extra: dict = field(default_factory=dict)

    def seed(self, tensor: str) -> int:
        return SEED_BASE + self.cfg_index * 16 + TENSOR_IDS[tensor]

    def scaled(self, **kw) -> "Workload":
        """Same recipe and seeds with different sizes (used for small parity cases)."""
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "gdn_fp32_small": Workload("gdn_fp32_small", B=1, T=256, H=2, dk=64, dv=64, io="f32",
                               alpha=GATE_SCALAR, alpha_kind=(GEN_UNIFORM, 0.9, 1.0),
                               beta_k=GATE_SCALAR, beta_v=GATE_ONE, key_scale=GATE_ONE,
                               s0_std=0.0, cfg_index=1),
    "gdn_prefill": Workload("gdn_prefill", B=8, T=4096, H=16, dk=128, dv=128, io="bf16",
                            alpha=GATE_SCALAR, alpha_kind=(GEN_EXP_NEG_SOFTPLUS, 0.1, 0.0),
                            beta_k=GATE_SCALAR, beta_v=GATE_ONE, key_scale=GATE_ONE,
                            s0_std=0.0, cfg_index=2),
    "kda": Workload("kda", B=4, T=8192, H=32, dk=128, dv=128, io="bf16",
                    alpha=GATE_CHANNEL, alpha_kind=(GEN_EXP_NEG_SOFTPLUS, 0.05, 0.0),
                    beta_k=GATE_SCALAR, beta_v=GATE_ONE, key_scale=GATE_ONE,
                    s0_std=0.02, cfg_index=3),
    "fg2_osdn_long": Workload("fg2_osdn_long", B=2, T=32768, H=16, dk=128, dv=128, io="bf16",
                              alpha=GATE_CHANNEL, alpha_kind=(GEN_EXP_NEG_SOFTPLUS, 0.05, 0.0),
                              beta_k=GATE_CHANNEL, beta_v=GATE_CHANNEL, key_scale=GATE_CHANNEL,
                              s0_std=0.02, cfg_index=4),
    "decode": Workload("decode", B=1024, T=1, H=32, dk=128, dv=128, io="bf16",
                       alpha=GATE_CHANNEL, alpha_kind=(GEN_EXP_NEG_SOFTPLUS, 0.05, 0.0),
                       beta_k=GATE_CHANNEL, beta_v=GATE_CHANNEL, key_scale=GATE_ONE,
                       s0_std=0.02, steps=100, cfg_index=5),
    "osdn_phase1": Workload("osdn_phase1", B=2, T=32768, H=16, dk=128, dv=128, io="bf16",
                            alpha=GATE_ONE, alpha_kind=(GEN_UNIFORM, 1.0, 1.0),
                            beta_k=GATE_SCALAR, beta_v=GATE_ONE, key_scale=GATE_ONE,
                            s0_std=0.0, cfg_index=4,
                            extra={"eta": 0.5, "retention": (GEN_UNIFORM, 0.95, 1.0)}),
}


def _gate_shape(w: Workload, mode: int, width: int, T: int):
    if mode == GATE_ONE:
        return None
    if mode == GATE_SCALAR:
        return (w.B, T, w.H)
    return (w.B, T, w.H, width)


def make_inputs(w: Workload, step: int = 0) -> dict:
    """Draw every input of one forward call (or of decode step `step`) as numpy arrays.

    Keys: q, k, v (io dtype; bf16 as uint16 bits), alpha, beta_k, beta_v, key_scale
    (float32 or None when the gate is absent), S0 (float32 [B,H,dk,dv] or None).
    For a decode workload S0 is the resident state and T is 1; `step` selects
    fresh per-step draws through the counter offset.
    """
    T = w.T
    out = {}
    n_qk = w.B * T * w.H * w.dk
    n_v = w.B * T * w.H * w.dv
    off_qk = step * n_qk
    off_v = step * n_v
    out["q"] = fill((w.B, T, w.H, w.dk), w.seed("q"), GEN_L2ROWS, dtype=w.io, offset=off_qk, row=w.dk)
    out["k"] = fill((w.B, T, w.H, w.dk), w.seed("k"), GEN_L2ROWS, dtype=w.io, offset=off_qk, row=w.dk)
    out["v"] = fill((w.B, T, w.H, w.dv), w.seed("v"), GEN_NORMAL, 0.0, 1.0, dtype=w.io, offset=off_v)
    shp = _gate_shape(w, w.alpha, w.dk, T)
    if shp is None:
        out["alpha"] = None
    else:
        kind, p0, p1 = w.alpha_kind
        out["alpha"] = fill(shp, w.seed("alpha"), kind, p0, p1, dtype="f32", offset=step * int(np.prod(shp)))
    shp = _gate_shape(w, w.beta_k, w.dk, T)
    out["beta_k"] = None if shp is None else fill(shp, w.seed("beta_k"), GEN_SIGMOID, dtype="f32",
                                                  offset=step * int(np.prod(shp)))
    shp = _gate_shape(w, w.beta_v, w.dv, T)
    out["beta_v"] = None if shp is None else fill(shp, w.seed("beta_v"), GEN_SIGMOID, dtype="f32",
                                                  offset=step * int(np.prod(shp)))
    shp = _gate_shape(w, w.key_scale, w.dk, T)
    out["key_scale"] = None if shp is None else fill(shp, w.seed("key_scale"), GEN_NORMAL, 1.0, 0.1,
                                                     dtype="f32", offset=step * int(np.prod(shp)))
    if w.s0_std > 0.0:
        if step == 0 or w.steps == 0:
            out["S0"] = fill((w.B, w.H, w.dk, w.dv), w.seed("S0"), GEN_NORMAL, 0.0, w.s0_std, dtype="f32")
        else:
            out["S0"] = None  # decode steps after the first continue from the resident state
    else:
        out["S0"] = None
    return out


def make_bwd_inputs(w: Workload, ds_std: float = 0.1) -> dict:
    """Cotangents of the backward pass for workload w: dO [B,T,H,dv] ~ N(0,1) in the storage dtype
    (the gradient of the loss with respect to o) and dS_T [B,H,dk,dv] ~ N(0, ds_std^2) fp32 (with
    respect to the final state)."""
    return {"dO": fill((w.B, w.T, w.H, w.dv), w.seed("dO"), GEN_NORMAL, 0.0, 1.0, dtype=w.io),
            "dS_T": fill((w.B, w.H, w.dk, w.dv), w.seed("dS_T"), GEN_NORMAL, 0.0, ds_std, dtype="f32")}


def make_osdn_inputs(w: Workload) -> dict:
    """Inputs of the OSDN preconditioner scan: k (as make_inputs draws it for the same seed block),
    beta [B,T,H] = sigmoid(N(0,1)), retention [B,T,H] (None when the recipe has none), eta."""
    shp = (w.B, w.T, w.H)
    out = {"k": fill((w.B, w.T, w.H, w.dk), w.seed("k"), GEN_L2ROWS, dtype=w.io, row=w.dk),
           "beta": fill(shp, w.seed("beta"), GEN_SIGMOID, dtype="f32"),
           "retention": None, "eta": float(w.extra.get("eta", 0.5))}
    rk = w.extra.get("retention")
    if rk is not None:
        kind, p0, p1 = rk
        out["retention"] = fill(shp, w.seed("retention"), kind, p0, p1, dtype="f32")
    return out
