"""CPU oracle for ART run-time-terminated decode attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does; the
two share no code.  The arithmetic lives in ``art_oracle.c`` (plain C, IEEE
double); this module only builds it with gcc, marshals CPU tensors into its
argument struct and unpacks the results.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "art_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
BAND = 1e-4   # relative half-width of the "undecided" band around a threshold

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile art_oracle.c into liboracle.so next to it (gcc, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "art_oracle.h"))):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32), ("B", ctypes.c_int32), ("Hq", ctypes.c_int32),
        ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32), ("page", ctypes.c_int32),
        ("max_blocks", ctypes.c_int32), ("num_pages", ctypes.c_int32),
        ("q", ctypes.c_void_p), ("q_stride", ctypes.c_int64 * 3),
        ("k", ctypes.c_void_p), ("k_stride", ctypes.c_int64 * 4),
        ("v", ctypes.c_void_p), ("v_stride", ctypes.c_int64 * 4),
        ("page_table", ctypes.c_void_p), ("block_order", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p), ("scale", ctypes.c_double),
        ("eps_m", ctypes.c_void_p), ("eps_d", ctypes.c_void_p),
        ("P", ctypes.c_void_p), ("min_blocks", ctypes.c_void_p), ("band", ctypes.c_double),
    ]


class _Result(ctypes.Structure):
    _fields_ = [
        ("stop", ctypes.c_void_p), ("adm_count", ctypes.c_void_p), ("adm", ctypes.c_void_p),
        ("adm_cap", ctypes.c_int32), ("amb_count", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("ds", ctypes.c_void_p), ("dd", ctypes.c_void_p), ("flag", ctypes.c_void_p),
    ]


_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.art_oracle_run.argtypes = [ctypes.POINTER(_Problem), ctypes.POINTER(_Result), ctypes.c_int]
        _lib.art_oracle_run.restype = ctypes.c_int
        _lib.art_oracle_prefix_out.argtypes = [ctypes.POINTER(_Problem), ctypes.c_int32, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        _lib.art_oracle_prefix_out.restype = ctypes.c_int
    return _lib


@dataclass
class OracleResult:
    stop: np.ndarray          # [B, Hkv] canonical stop
    admissible: list          # [B*Hkv] lists of admissible stops
    amb_count: np.ndarray     # [B, Hkv]
    out: Optional[np.ndarray] # [B, Hq, d] float64 at the canonical stop
    ds: Optional[np.ndarray]  # [B, Hkv, max_blocks]
    dd: Optional[np.ndarray]
    flag: Optional[np.ndarray]


def _cpu(t: torch.Tensor) -> torch.Tensor:
    return t.detach().to("cpu")


class Problem:
    """Holds CPU copies of a workload's arrays and the ctypes struct over them."""

    def __init__(self, w, scale: Optional[float] = None, band: float = BAND,
                 eps_m=None, eps_d=None, P=None, min_blocks=None):
        q, k, v = _cpu(w.q), _cpu(w.k_cache), _cpu(w.v_cache)
        if q.dtype == torch.float32:
            self.dtype = F32
        elif q.dtype == torch.bfloat16:
            self.dtype = BF16
        else:
            raise TypeError(q.dtype)
        assert k.dtype == q.dtype and v.dtype == q.dtype
        if self.dtype == BF16:
            q, k, v = (x.view(torch.int16) for x in (q, k, v))
        self.q, self.k, self.v = q, k, v
        self.pt = _cpu(w.page_table).to(torch.int32).contiguous()
        self.bo = _cpu(w.block_order).to(torch.int32).contiguous()
        self.sl = _cpu(w.seq_lens).to(torch.int32).contiguous()
        B = q.shape[0]

        def arr(x, default, dt):
            x = default if x is None else x
            t = torch.as_tensor(_cpu(x) if isinstance(x, torch.Tensor) else x)
            # thresholds are given to the kernel as binary32: use the same values
            t = t.to(torch.float32).to(dt) if dt == torch.float64 else t.to(dt)
            return (t.expand(B) if t.dim() == 0 else t.reshape(B)).contiguous()

        self.eps_m = arr(eps_m, w.eps_m, torch.float64)
        self.eps_d = arr(eps_d, w.eps_d, torch.float64)
        self.P = arr(P, w.P, torch.int32)
        self.mb = arr(min_blocks, w.min_blocks, torch.int32)
        d = q.shape[2]
        p = _Problem()
        p.dtype = self.dtype
        p.B, p.Hq, p.d = B, q.shape[1], d
        p.Hkv, p.page = k.shape[1], k.shape[2]
        p.max_blocks = self.pt.shape[1]
        p.num_pages = k.shape[0]
        p.q = q.data_ptr()
        p.q_stride = (ctypes.c_int64 * 3)(*q.stride())
        p.k = k.data_ptr()
        p.k_stride = (ctypes.c_int64 * 4)(*k.stride())
        p.v = v.data_ptr()
        p.v_stride = (ctypes.c_int64 * 4)(*v.stride())
        p.page_table = self.pt.data_ptr()
        p.block_order = self.bo.data_ptr()
        p.seq_lens = self.sl.data_ptr()
        p.scale = (1.0 / math.sqrt(d)) if scale is None else float(scale)
        p.eps_m = self.eps_m.data_ptr()
        p.eps_d = self.eps_d.data_ptr()
        p.P = self.P.data_ptr()
        p.min_blocks = self.mb.data_ptr()
        p.band = band
        self.struct = p
        self.B, self.Hq, self.Hkv, self.d = B, p.Hq, p.Hkv, d
        self.G = p.Hq // p.Hkv
        self.max_blocks = p.max_blocks


_ERR = {-1: "invalid arguments", -2: "block order or page table entry out of range", -3: "out of memory"}


def run(w, *, scale=None, band=BAND, eps_m=None, eps_d=None, P=None, min_blocks=None,
        want_out=True, want_stats=False, nthreads=0, adm_cap=64) -> OracleResult:
    """Run the ART walk with the stop rule for every (b, kv-head) unit."""
    lib = _load()
    pb = Problem(w, scale=scale, band=band, eps_m=eps_m, eps_d=eps_d, P=P, min_blocks=min_blocks)
    U = pb.B * pb.Hkv
    stop = np.zeros(U, np.int32)
    adm_count = np.zeros(U, np.int32)
    adm = np.zeros((U, adm_cap), np.int32)
    amb = np.zeros(U, np.int32)
    out = np.zeros((pb.B, pb.Hq, pb.d), np.float64) if want_out else None
    ds = np.zeros((U, pb.max_blocks), np.float64) if want_stats else None
    dd = np.zeros((U, pb.max_blocks), np.float64) if want_stats else None
    flag = np.zeros((U, pb.max_blocks), np.int8) if want_stats else None
    r = _Result()
    r.stop, r.adm_count, r.adm = stop.ctypes.data, adm_count.ctypes.data, adm.ctypes.data
    r.adm_cap = adm_cap
    r.amb_count = amb.ctypes.data
    r.out = out.ctypes.data if out is not None else None
    r.ds = ds.ctypes.data if ds is not None else None
    r.dd = dd.ctypes.data if dd is not None else None
    r.flag = flag.ctypes.data if flag is not None else None
    rc = lib.art_oracle_run(ctypes.byref(pb.struct), ctypes.byref(r), int(nthreads))
    if rc != 0:
        raise ValueError(f"art_oracle_run failed: {_ERR.get(rc, rc)}")
    admissible = [list(adm[u, :min(adm_count[u], adm_cap)]) for u in range(U)]
    sh = (pb.B, pb.Hkv)
    return OracleResult(stop.reshape(sh), admissible, amb.reshape(sh), out,
                        None if ds is None else ds.reshape(pb.B, pb.Hkv, -1),
                        None if dd is None else dd.reshape(pb.B, pb.Hkv, -1),
                        None if flag is None else flag.reshape(pb.B, pb.Hkv, -1))


def prefix_out(w, units: Sequence[int], s: Sequence[int], *, scale=None, nthreads=0) -> np.ndarray:
    """Output after the first s[i] walk steps of unit units[i] (= b*Hkv + h): [n, G, d] float64."""
    lib = _load()
    pb = Problem(w, scale=scale)
    units = np.ascontiguousarray(np.asarray(units, np.int32))
    s = np.ascontiguousarray(np.asarray(s, np.int32))
    out = np.zeros((len(units), pb.G, pb.d), np.float64)
    if len(units) == 0:
        return out
    rc = lib.art_oracle_prefix_out(ctypes.byref(pb.struct), int(len(units)), units.ctypes.data,
                                   s.ctypes.data, out.ctypes.data, int(nthreads))
    if rc != 0:
        raise ValueError(f"art_oracle_prefix_out failed: {_ERR.get(rc, rc)}")
    return out
