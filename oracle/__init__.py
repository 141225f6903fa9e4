"""ctypes wrapper of the plain-C MoE layer oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The CUDA library never imports, links
or runs anything in this directory, and this wrapper imports nothing from the
CUDA package.  ``build()`` compiles the C file with gcc (OpenMP, no fast-math,
no FP contraction) into ``liboracle.so`` next to it.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

FMT = {"mxfp4": 0, "nvfp4": 1, "int4g128": 2, "fp8b128": 3}
NUMERICS = {"exact": 0, "a4": 1}


def build(force: bool = False) -> str:
    """Compile the oracle if the shared object is missing or older than the source."""
    with _lock:
        if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
            tmp = _SO + f".tmp{os.getpid()}"
            cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                   "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _SO)
    return _SO


class _Layer(C.Structure):
    _fields_ = [
        ("H", C.c_int), ("I", C.c_int), ("E", C.c_int), ("k", C.c_int), ("Is", C.c_int),
        ("fmt", C.c_int), ("numerics", C.c_int),
        ("router_w", C.c_void_p), ("router_bias", C.c_void_p),
        ("codes", C.c_void_p * 3), ("scales", C.c_void_p * 3),
        ("global_scale", C.c_void_p), ("shared_w", C.c_void_p * 3),
        ("scoring", C.c_int), ("renorm", C.c_int), ("n_sinks", C.c_int), ("shared_gate_w", C.c_void_p),
    ]

SCORING = {"softmax": 0, "sigmoid": 1}


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_SO)
        L.orc_e2m1.restype = C.c_double
        L.orc_e2m1.argtypes = [C.c_uint]
        L.orc_e8m0.restype = C.c_double
        L.orc_e8m0.argtypes = [C.c_uint]
        L.orc_e4m3.restype = C.c_double
        L.orc_e4m3.argtypes = [C.c_uint]
        L.orc_rne_e2m1.restype = C.c_uint
        L.orc_rne_e2m1.argtypes = [C.c_float]
        L.orc_rn_e4m3.restype = C.c_uint
        L.orc_rn_e4m3.argtypes = [C.c_float]
        L.orc_admit_scales.restype = C.c_long
        L.orc_admit_scales.argtypes = [C.c_int, C.c_void_p, C.c_long]
        L.orc_admit_fp8_codes.restype = C.c_long
        L.orc_admit_fp8_codes.argtypes = [C.c_void_p, C.c_long]
        L.orc_int4.restype = C.c_double
        L.orc_int4.argtypes = [C.c_uint]
        L.orc_quant_mx_block.restype = None
        L.orc_quant_mx_block.argtypes = [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p]
        L.orc_quant_nv_row.restype = None
        L.orc_quant_nv_row.argtypes = [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p]
        L.orc_a4_qdq_row.restype = None
        L.orc_a4_qdq_row.argtypes = [C.c_int, C.c_void_p, C.c_int, C.c_void_p]
        L.orc_dequant_row.restype = None
        L.orc_dequant_row.argtypes = [C.POINTER(_Layer), C.c_int, C.c_int, C.c_int, C.c_void_p]
        L.orc_permute.restype = None
        L.orc_permute.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]
        L.orc_forward.restype = C.c_int
        L.orc_forward.argtypes = [C.POINTER(_Layer), C.c_void_p, C.c_int, C.c_void_p, C.c_int,
                                  C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int]
        L.orc_route_all.restype = None
        L.orc_route_all.argtypes = [C.POINTER(_Layer), C.c_void_p, C.c_int, C.c_void_p, C.c_void_p,
                                    C.c_void_p, C.c_int]
        L.orc_route_row.restype = None
        L.orc_route_row.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p]
        L.orc_route_row_v.restype = None
        L.orc_route_row_v.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p]
        L.orc_max_threads.restype = C.c_int
        L.orc_expert_rows.restype = None
        L.orc_expert_rows.argtypes = [C.POINTER(_Layer), C.c_int, C.c_void_p, C.c_int, C.c_int, C.c_void_p]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


# ---------------------------------------------------------------- scalar decode
def e2m1(code: int) -> float:
    return lib().orc_e2m1(code)


def e8m0(code: int) -> float:
    return lib().orc_e8m0(code)


def e4m3(code: int) -> float:
    return lib().orc_e4m3(code)


def rne_e2m1(q: float) -> int:
    return lib().orc_rne_e2m1(q)


def rn_e4m3(t: float) -> int:
    return lib().orc_rn_e4m3(t)


def admit_scales(fmt: str, s: np.ndarray) -> int:
    """Index of the first scale the format rejects, or -1 (s holds the format's
    scale values: uint8 codes, bf16 bits as uint16, or fp32)."""
    s = np.ascontiguousarray(s)
    return lib().orc_admit_scales(FMT[fmt], _p(s.view(np.uint8)), s.size)


def admit_fp8_codes(q: np.ndarray) -> int:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    return lib().orc_admit_fp8_codes(_p(q), q.size)


def int4(nibble: int) -> float:
    return lib().orc_int4(nibble)


def quant_mx_block(v: np.ndarray):
    v = np.ascontiguousarray(v, dtype=np.float32)
    codes = np.zeros(v.size, dtype=np.uint8)
    sc = np.zeros(1, dtype=np.uint8)
    lib().orc_quant_mx_block(_p(v), v.size, _p(codes), _p(sc))
    return codes, int(sc[0])


def quant_nv_row(v: np.ndarray):
    v = np.ascontiguousarray(v, dtype=np.float32)
    codes = np.zeros(v.size, dtype=np.uint8)
    sc = np.zeros(v.size // 16, dtype=np.uint8)
    G = np.zeros(1, dtype=np.float32)
    lib().orc_quant_nv_row(_p(v), v.size, _p(codes), _p(sc), _p(G))
    return codes, sc, float(G[0])


def a4_qdq_row(fmt: str, v: np.ndarray) -> np.ndarray:
    """The A4 activation rule of the format applied to one row: quantise, then decode (fp64)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.zeros(v.size, dtype=np.float64)
    lib().orc_a4_qdq_row(FMT[fmt], _p(v), v.size, _p(out))
    return out


def permute(ids: np.ndarray, n_experts: int):
    ids = np.ascontiguousarray(ids, dtype=np.int32).reshape(-1)
    n = ids.size
    counts = np.zeros(n_experts, dtype=np.int32)
    offsets = np.zeros(n_experts + 1, dtype=np.int32)
    perm = np.zeros(n, dtype=np.int32)
    inv = np.zeros(n, dtype=np.int32)
    lib().orc_permute(_p(ids), n, n_experts, _p(counts), _p(offsets), _p(perm), _p(inv))
    return counts, offsets, perm, inv


def route_row(logits_row: np.ndarray, k: int, scoring: str = "softmax", renorm: bool = True):
    """Top-k ids and gates of one row of target logits (all targets, sinks included)."""
    l = np.ascontiguousarray(logits_row, dtype=np.float32)
    ids = np.zeros(k, dtype=np.int32)
    g = np.zeros(k, dtype=np.float32)
    lib().orc_route_row_v(_p(l), l.size, k, SCORING[scoring], 1 if renorm else 0, _p(ids), _p(g))
    return ids, g


class Layer:
    """The oracle's view of one layer: checkpoint arrays in the synthetic layout.

    ``codes[m]``/``scales[m]`` are uint8 arrays [E, rows, K/2] / [E, rows, K/G]
    for m = gate, up, down; ``shared_w`` three bf16-bit uint16 matrices or None.
    Router variants: ``router_w`` / ``router_bias`` cover the E experts and then
    ``n_sinks`` sink targets; ``scoring`` "softmax" | "sigmoid"; ``renorm``;
    ``shared_gate_w`` fp32 [H] or None.
    """

    def __init__(self, hidden, inter, n_experts, top_k, fmt, router_w, router_bias, codes, scales,
                 global_scale=None, shared_w=None, numerics="exact", scoring="softmax", renorm=True,
                 n_sinks=0, shared_gate_w=None):
        self._keep = []

        def keep(a, dt):
            if a is None:
                return None
            a = np.ascontiguousarray(a, dtype=dt)
            self._keep.append(a)
            return a

        self.H, self.I, self.E, self.k = hidden, inter, n_experts, top_k
        self.fmt = fmt
        s = _Layer()
        s.H, s.I, s.E, s.k = hidden, inter, n_experts, top_k
        s.Is = 0 if shared_w is None else shared_w[0].shape[0]
        self.Is = s.Is
        s.fmt = FMT[fmt]
        s.numerics = NUMERICS[numerics]
        s.router_w = _p(keep(router_w, np.float32))
        s.router_bias = _p(keep(router_bias, np.float32))
        for m in range(3):
            s.codes[m] = _p(keep(codes[m], np.uint8))
            # scales are passed as their bytes (uint8 codes, bf16 bits or fp32 by format)
            s.scales[m] = _p(keep(np.ascontiguousarray(scales[m]).view(np.uint8), np.uint8))
            s.shared_w[m] = None if shared_w is None else _p(keep(shared_w[m], np.uint16))
        s.global_scale = _p(keep(global_scale, np.float32))
        s.scoring = SCORING[scoring]
        s.renorm = 1 if renorm else 0
        s.n_sinks = n_sinks
        s.shared_gate_w = _p(keep(shared_gate_w, np.float32))
        self.n_targets = n_experts + n_sinks
        self._s = s

    @classmethod
    def from_weights(cls, lw, numerics="exact"):
        wl = lw.wl
        return cls(wl.hidden, wl.inter, wl.n_experts, wl.top_k, wl.fmt, lw.router_w, lw.router_bias,
                   lw.codes, lw.scales, lw.global_scale, lw.shared_w, numerics, wl.scoring, wl.renormalize,
                   wl.n_sinks, lw.shared_gate_w)

    def forward(self, x_bits: np.ndarray, rows=None, threads: int = 0):
        """y [n,H] fp32, logits [n, E + n_sinks], ids [n,k], gates [n,k] for the listed token rows."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        T = x.shape[0]
        r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
        n = T if r is None else r.size
        y = np.zeros((n, self.H), dtype=np.float32)
        lg = np.zeros((n, self.n_targets), dtype=np.float32)
        ids = np.zeros((n, self.k), dtype=np.int32)
        g = np.zeros((n, self.k), dtype=np.float32)
        rc = lib().orc_forward(C.byref(self._s), _p(x), T, _p(r), 0 if r is None else r.size,
                               _p(y), _p(lg), _p(ids), _p(g), threads)
        if rc != 0:
            raise ValueError(f"oracle forward failed ({rc})")
        return y, lg, ids, g

    def route_all(self, x_bits: np.ndarray, threads: int = 0):
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        T = x.shape[0]
        lg = np.zeros((T, self.n_targets), dtype=np.float32)
        ids = np.zeros((T, self.k), dtype=np.int32)
        g = np.zeros((T, self.k), dtype=np.float32)
        lib().orc_route_all(C.byref(self._s), _p(x), T, _p(lg), _p(ids), _p(g), threads)
        return lg, ids, g

    def expert_rows(self, e: int, x_row_bits: np.ndarray, i0: int, n: int, o: np.ndarray = None):
        """Timing sample: intermediate rows [i0, i0+n) of expert e on one token (EXACT)."""
        xt = (np.asarray(x_row_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
        xt = np.ascontiguousarray(xt, dtype=np.float64)
        if o is None:
            o = np.zeros(self.H, dtype=np.float64)
        lib().orc_expert_rows(C.byref(self._s), e, xt.ctypes.data, i0, n, o.ctypes.data)
        return o

    def dequant(self, m: int, e: int) -> np.ndarray:
        rows, K = (self.I, self.H) if m < 2 else (self.H, self.I)
        out = np.zeros((rows, K), dtype=np.float64)
        for r in range(rows):
            lib().orc_dequant_row(C.byref(self._s), m, e, r, out[r].ctypes.data)
        return out


def max_threads() -> int:
    return lib().orc_max_threads()
