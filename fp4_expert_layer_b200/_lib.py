"""ctypes binding of ``include/moe_layer.h`` (argument marshalling only).

Every step of the forward runs in the CUDA library; this module only converts
numpy arrays / torch tensors into the pointers and sizes the C ABI takes.  If
the shared library is missing or cannot be loaded the import of
:class:`MoELayer` fails loudly: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
# FP4MOE_CHECKED=1 loads the build with the device bounds checks compiled in
SO = os.path.join(HERE, "libfp4moe_checked.so" if os.environ.get("FP4MOE_CHECKED") == "1" else "libfp4moe.so")

MOE_OK = 0
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_ADMISSION", 3: "MOE_ERR_SLOT_TABLE",
          4: "MOE_ERR_OOM", 5: "MOE_ERR_CUDA", 6: "MOE_ERR_UNSUPPORTED"}
FMT = {"mxfp4": 0, "nvfp4": 1, "int4g128": 2, "fp8b128": 3}
NUMERICS = {"exact": 0, "a4": 1}
SCORING = {"softmax": 0, "sigmoid": 1}
OUT_DTYPE = {"f32": 0, "bf16": 1}

EXPORTED = ["moe_layer_plan", "moe_admit", "moe_layer_create", "moe_set_slot_table", "moe_forward",
            "moe_forward_host", "moe_get_stats", "moe_destroy", "moe_last_error", "moe_debug_inject",
            "moe_profile_enable", "moe_profile_read", "moe_route_topk_noalloc", "moe_debug_read",
            "moe_graph_capture", "moe_graph_launch", "moe_graph_destroy", "moe_set_policy", "moe_prefetch"]
POLICY = {"static": 0, "none": 1, "cache": 2, "hybrid": 3}


class MoEError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class Config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in (
        "hidden", "inter", "n_experts", "top_k", "shared_inter", "fmt", "renormalize", "numerics",
        "n_slots", "max_tokens", "n_staging", "device", "scoring", "n_sinks", "shared_gate", "out_dtype")]


class Weights(C.Structure):
    _fields_ = [
        ("router_w", C.c_void_p), ("router_bias", C.c_void_p),
        ("codes", C.c_void_p * 3), ("scales", C.c_void_p * 3),
        ("global_scale", C.c_void_p), ("shared_w", C.c_void_p * 3),
        ("shared_gate_w", C.c_void_p),
    ]


class Routing(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("logits", "ids", "gates", "counts", "offsets", "perm", "inv")]


class Stats(C.Structure):
    _fields_ = [
        ("forwards", C.c_uint64), ("misses", C.c_uint64), ("bytes_staged", C.c_uint64),
        ("last_misses", C.c_int32), ("last_waves", C.c_int32), ("last_active", C.c_int32),
        ("last_path", C.c_int32), ("launches", C.c_uint64), ("expert_bytes", C.c_uint64),
        ("device_bytes", C.c_uint64),
        ("pinned_bytes", C.c_uint64), ("device_error", C.c_int32),
        ("policy", C.c_int32), ("admitted", C.c_uint64), ("prefetched", C.c_uint64),
    ]


PROFILE_STAGES = ["router", "permute", "shared", "gateup", "down", "combine", "staging_wait", "forward",
                  "quantise", "unused"]


class Profile(C.Structure):
    _fields_ = [("forwards", C.c_uint64), ("ms", C.c_double * 10), ("launches", C.c_uint64 * 10)]


class Plan(C.Structure):
    _fields_ = [(n, C.c_uint64) for n in (
        "expert_bytes", "slot_bytes", "staging_bytes", "resident_bytes", "scratch_bytes", "pinned_bytes")]


_lib = None


def lib():
    """Load the CUDA library (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(SO):
            raise ImportError(f"CUDA library not built: {SO} (run fp4_expert_layer_b200/build.py)")
        L = C.CDLL(SO)
        L.moe_layer_plan.argtypes = [C.POINTER(Config), C.POINTER(Plan)]
        L.moe_admit.argtypes = [C.POINTER(Config), C.POINTER(Weights)]
        L.moe_layer_create.argtypes = [C.POINTER(Config), C.POINTER(Weights), C.c_void_p, C.POINTER(C.c_void_p)]
        L.moe_set_slot_table.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p]
        L.moe_set_policy.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_void_p]
        L.moe_prefetch.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p]
        L.moe_forward.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p, C.POINTER(Routing)]
        L.moe_forward_host.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p]
        L.moe_get_stats.argtypes = [C.c_void_p, C.POINTER(Stats)]
        L.moe_graph_capture.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p,
                                        C.POINTER(C.c_void_p)]
        L.moe_graph_launch.argtypes = [C.c_void_p, C.c_void_p]
        L.moe_graph_destroy.argtypes = [C.c_void_p]
        L.moe_destroy.argtypes = [C.c_void_p]
        L.moe_destroy.restype = None
        L.moe_last_error.restype = C.c_char_p
        L.moe_debug_inject.argtypes = [C.c_void_p, C.c_int32]
        L.moe_profile_enable.argtypes = [C.c_void_p, C.c_int32]
        L.moe_profile_read.argtypes = [C.c_void_p, C.POINTER(Profile)]
        L.moe_debug_read.argtypes = [C.c_void_p, C.c_int32, C.c_void_p, C.c_uint64]
        L.moe_route_topk_noalloc.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p,
                                             C.c_int32, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p,
                                             C.c_void_p]
        for n in EXPORTED:
            f = getattr(L, n)
            if n not in ("moe_destroy", "moe_last_error"):
                f.restype = C.c_int
        _lib = L
    return _lib


def check(status):
    if status != MOE_OK:
        raise MoEError(status, lib().moe_last_error().decode())


def make_config(hidden, inter, n_experts, top_k, shared_inter=0, fmt="mxfp4", numerics="exact",
                n_slots=None, max_tokens=1, n_staging=0, device=0, scoring="softmax", renormalize=True,
                n_sinks=0, shared_gate=False, out_dtype="f32") -> Config:
    return Config(hidden, inter, n_experts, top_k, shared_inter, FMT[fmt], 1 if renormalize else 0,
                  NUMERICS[numerics], n_experts if n_slots is None else n_slots, max_tokens, n_staging, device,
                  SCORING[scoring], n_sinks, 1 if shared_gate else 0, OUT_DTYPE[out_dtype])


def plan(cfg: Config) -> dict:
    p = Plan()
    check(lib().moe_layer_plan(C.byref(cfg), C.byref(p)))
    return {n: getattr(p, n) for n, _ in Plan._fields_}


class _HostWeights:
    """Keeps the numpy arrays alive and exposes them as a moe_weights_t."""

    def __init__(self, router_w, router_bias, codes, scales, global_scale, shared_w, shared_gate_w=None):
        self.keep = []
        w = Weights()

        def arr(a, dt):
            a = np.ascontiguousarray(a, dtype=dt)
            self.keep.append(a)
            return a

        w.router_w = arr(router_w, np.float32).ctypes.data
        w.router_bias = None if router_bias is None else arr(router_bias, np.float32).ctypes.data
        for m in range(3):
            cm = arr(codes[m], np.uint8)
            E = cm.shape[0]
            # scales go in as their bytes: uint8 codes, bf16 bits (uint16) or fp32, by format
            sm = np.ascontiguousarray(scales[m])
            sm = sm.view(np.uint8).reshape(E, -1)
            self.keep.append(sm)
            cp = (C.c_void_p * E)(*[cm[e].ctypes.data for e in range(E)])
            sp = (C.c_void_p * E)(*[sm[e].ctypes.data for e in range(E)])
            self.keep += [cp, sp]
            w.codes[m] = C.cast(cp, C.c_void_p)
            w.scales[m] = C.cast(sp, C.c_void_p)
        w.global_scale = None if global_scale is None else arr(global_scale, np.float32).ctypes.data
        for m in range(3):
            w.shared_w[m] = None if shared_w is None else arr(shared_w[m], np.uint16).ctypes.data
        w.shared_gate_w = None if shared_gate_w is None else arr(shared_gate_w, np.float32).ctypes.data
        self.w = w


def weights_from_layer(lw) -> _HostWeights:
    return _HostWeights(lw.router_w, lw.router_bias, lw.codes, lw.scales, lw.global_scale, lw.shared_w,
                        getattr(lw, "shared_gate_w", None))


def admit(cfg: Config, hw: _HostWeights):
    check(lib().moe_admit(C.byref(cfg), C.byref(hw.w)))


def route_topk_noalloc(x, router_w, router_bias, k, ids, gates, logits=None, stream=None):
    """Routing alone through the entry point that allocates nothing (see moe_layer.h).

    All arguments are caller-owned torch CUDA tensors: x bf16 [T, H], router_w fp32
    [E, H], router_bias fp32 [E] or None, ids int32 [T, k], gates fp32 [T, k],
    logits fp32 [T, E] or None.  For callers that must not allocate device memory
    when they call in; the library uses its fixed device scratch instead.
    """
    T, H = x.shape
    E = router_w.shape[0]
    check(lib().moe_route_topk_noalloc(
        x.data_ptr(), T, H, router_w.data_ptr(), None if router_bias is None else router_bias.data_ptr(),
        E, k, ids.data_ptr(), gates.data_ptr(), None if logits is None else logits.data_ptr(),
        _stream_ptr(stream)))


def _stream_ptr(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


class Graph:
    """A captured forward (moe_graph_t): launch() replays it; close() before the layer's."""

    def __init__(self, handle):
        self.handle = handle

    def launch(self, stream_ptr: int):
        check(lib().moe_graph_launch(self.handle, stream_ptr))

    def close(self):
        if self.handle:
            lib().moe_graph_destroy(self.handle)
            self.handle = None


class MoELayer:
    """One layer on one GPU.  ``forward`` takes and returns torch CUDA tensors."""

    def __init__(self, cfg: Config, hw: _HostWeights, stream=None):
        self.cfg = cfg
        self.handle = C.c_void_p()
        check(lib().moe_layer_create(C.byref(cfg), C.byref(hw.w), _stream_ptr(stream), C.byref(self.handle)))

    @classmethod
    def from_weights(cls, lw, n_slots=None, max_tokens=1, numerics="exact", n_staging=0, device=0,
                     stream=None, out_dtype="f32"):
        """The routing semantics (scoring, renormalisation, sinks, shared-expert
        gate) are the layer's own, as its workload declares them."""
        wl = lw.wl
        cfg = make_config(wl.hidden, wl.inter, wl.n_experts, wl.top_k, wl.shared_inter, wl.fmt, numerics,
                          wl.n_experts if n_slots is None else n_slots, max_tokens, n_staging, device,
                          getattr(wl, "scoring", "softmax"), getattr(wl, "renormalize", True),
                          getattr(wl, "n_sinks", 0), getattr(wl, "shared_gate", False), out_dtype)
        return cls(cfg, weights_from_layer(lw), stream)

    @property
    def out_torch_dtype(self):
        import torch
        return torch.bfloat16 if self.cfg.out_dtype == OUT_DTYPE["bf16"] else torch.float32

    def set_slot_table(self, table, stream=None):
        t = np.ascontiguousarray(table, dtype=np.int32)
        check(lib().moe_set_slot_table(self.handle, t.ctypes.data, _stream_ptr(stream)))

    def set_policy(self, policy: str, n_pinned: int = 0, stream=None):
        """Residency policy: "static" (the caller's table), "none", "cache" or "hybrid"."""
        check(lib().moe_set_policy(self.handle, POLICY[policy], n_pinned, _stream_ptr(stream)))

    def prefetch(self, experts, stream=None):
        """Copy predicted experts into evictable slots ahead of a forward (cache / hybrid)."""
        e = np.ascontiguousarray(experts, dtype=np.int32).reshape(-1)
        check(lib().moe_prefetch(self.handle, e.ctypes.data if e.size else None, e.size, _stream_ptr(stream)))

    def forward(self, x, y=None, routing: bool = False, stream=None):
        import torch
        T = x.shape[0]
        H = self.cfg.hidden
        assert x.dtype == torch.bfloat16 and x.is_cuda and x.is_contiguous() and x.shape[1] == H
        if y is None:
            y = torch.empty((T, H), dtype=self.out_torch_dtype, device=x.device)
        assert y.dtype == self.out_torch_dtype and y.is_contiguous()
        r = None
        rp = None
        if routing:
            E, k = self.cfg.n_experts + self.cfg.n_sinks, self.cfg.top_k   # routing targets
            dev = x.device
            r = {
                "logits": torch.empty((T, E), dtype=torch.float32, device=dev),
                "ids": torch.empty((T, k), dtype=torch.int32, device=dev),
                "gates": torch.empty((T, k), dtype=torch.float32, device=dev),
                "counts": torch.empty(E, dtype=torch.int32, device=dev),
                "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
                "perm": torch.empty(T * k, dtype=torch.int32, device=dev),
                "inv": torch.empty(T * k, dtype=torch.int32, device=dev),
            }
            rp = Routing(*[r[n].data_ptr() for n, _ in Routing._fields_])
        check(lib().moe_forward(self.handle, x.data_ptr(), T, y.data_ptr(), _stream_ptr(stream),
                                C.byref(rp) if rp is not None else None))
        return (y, r) if routing else y

    def forward_ptr(self, x_ptr: int, T: int, y_ptr: int, stream_ptr: int):
        check(lib().moe_forward(self.handle, x_ptr, T, y_ptr, stream_ptr, None))

    def forward_host(self, x_host: np.ndarray, y_host: np.ndarray = None, stream=None):
        x = np.ascontiguousarray(x_host, dtype=np.uint16)
        T = x.shape[0]
        if y_host is None:
            bf16 = self.cfg.out_dtype == OUT_DTYPE["bf16"]
            y_host = np.empty((T, self.cfg.hidden), dtype=np.uint16 if bf16 else np.float32)
        check(lib().moe_forward_host(self.handle, x.ctypes.data, T, y_host.ctypes.data, _stream_ptr(stream)))
        return y_host

    def forward_host_ptr(self, x_ptr: int, T: int, y_ptr: int, stream_ptr: int):
        check(lib().moe_forward_host(self.handle, x_ptr, T, y_ptr, stream_ptr))

    def capture_graph(self, x_ptr: int, T: int, y_ptr: int, stream_ptr: int) -> "Graph":
        """CUDA graph of one all-resident forward for these fixed buffers."""
        h = C.c_void_p()
        check(lib().moe_graph_capture(self.handle, x_ptr, T, y_ptr, stream_ptr, C.byref(h)))
        return Graph(h.value)

    def stats(self) -> dict:
        s = Stats()
        check(lib().moe_get_stats(self.handle, C.byref(s)))
        return {n: getattr(s, n) for n, _ in Stats._fields_}

    def profile_enable(self, on: bool = True):
        check(lib().moe_profile_enable(self.handle, 1 if on else 0))

    def profile_read(self) -> dict:
        p = Profile()
        check(lib().moe_profile_read(self.handle, C.byref(p)))
        return {"forwards": p.forwards,
                "ms": {n: p.ms[i] for i, n in enumerate(PROFILE_STAGES)},
                "launches": {n: p.launches[i] for i, n in enumerate(PROFILE_STAGES)}}

    def debug_read(self, which: int, dtype, count: int) -> np.ndarray:
        """Test hook: copy an internal buffer of the last forward to host."""
        out = np.empty(count, dtype=dtype)
        check(lib().moe_debug_read(self.handle, which, out.ctypes.data, out.nbytes))
        return out

    def inject(self, what: int):
        check(lib().moe_debug_inject(self.handle, what))

    def close(self):
        if self.handle:
            lib().moe_destroy(self.handle)
            self.handle = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
