"""Test-side helpers: margin-filtered token draws and independent numpy restatements.

The numpy restatements here (decode tables, dense evaluation) are written from
the format definitions, not from the oracle's code, so that they can pin it.
"""
from __future__ import annotations

import os

import numpy as np

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def e2m1_table():
    """16 code values from the hand-written fixture."""
    return np.array([float(v) for _, v in read_golden("e2m1_values.txt")], dtype=np.float64)


def top_margin_ok(logits: np.ndarray, k: int, margin: float = 1e-3) -> np.ndarray:
    """True for rows whose k+1 largest logits are pairwise >= margin apart."""
    kk = min(k + 1, logits.shape[1])
    s = -np.sort(-logits.astype(np.float64), axis=1)[:, :kk]
    if kk < 2:
        return np.ones(logits.shape[0], dtype=bool)
    return ((s[:, :-1] - s[:, 1:]) >= margin).all(axis=1)


def tokens_with_margin(orc_layer, wl, T, seed=None, stream=0, margin=1e-3, max_rounds=100,
                       threads=0):
    """Draw T tokens; redraw any whose top-(k+1) router logits are closer than ``margin``."""
    x = synth.make_tokens(wl, T, seed, stream)
    rng = synth.resample_rng(wl, seed, stream)
    redraws = 0
    bad = np.arange(T)
    for _ in range(max_rounds):
        lg, _, _ = orc_layer.route_all(x[bad], threads=threads)
        bad = bad[~top_margin_ok(lg, wl.top_k, margin)]
        if bad.size == 0:
            return x, redraws
        synth.redraw_rows(x, bad, rng)
        redraws += int(bad.size)
    raise RuntimeError("could not draw tokens with the requested top-k margin")


def int4_table():
    """16 code values from the hand-written fixture."""
    return np.array([float(v) for _, v in read_golden("int4_values.txt")], dtype=np.float64)


def _torch_e4m3(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).view(torch.float8_e4m3fn) \
        .to(torch.float64).numpy()


def np_decode(codes: np.ndarray, scales: np.ndarray, fmt: str, gscale: float = 1.0) -> np.ndarray:
    """Independent numpy decode of one code matrix ([rows, K/2] nibbles, or
    [rows, K] bytes for FP8) with its scales."""
    if fmt == "fp8b128":
        q = _torch_e4m3(codes)
        s = np.repeat(np.repeat(scales.astype(np.float64), 128, axis=0), 128, axis=1)
        return q * s
    tab = int4_table() if fmt == "int4g128" else e2m1_table()
    lo = codes & 0x0F
    hi = codes >> 4
    q = np.empty((codes.shape[0], codes.shape[1] * 2), dtype=np.float64)
    q[:, 0::2] = tab[lo]
    q[:, 1::2] = tab[hi]
    if fmt == "mxfp4":
        s = np.ldexp(1.0, scales.astype(np.int64) - 127)
        return q * np.repeat(s, 32, axis=1)
    if fmt == "int4g128":
        s = synth.bf16_bits_to_f32(scales).astype(np.float64)
        return q * np.repeat(s, 128, axis=1)
    s = _torch_e4m3(scales)
    return q * np.repeat(s, 16, axis=1) * gscale


def np_silu(a):
    return a / (1.0 + np.exp(-a))


def dense_layer(lw, x_bits, ids_from=None):
    """Dense evaluation: every expert on every token, gate 0 outside the top-k.

    Routing: numpy stable argsort on the negated fp32 logits of all targets
    (experts, then sinks; lower index first on ties); scores: full softmax over
    all targets, or an elementwise sigmoid; gates: the chosen scores, divided by
    their sum when the layer renormalises.  A chosen sink keeps its gate but has
    no FFN; the shared expert is scaled by sigmoid(fp32(x . w_sg)) when the
    layer has a shared-expert gate.
    """
    wl = lw.wl
    E, k = wl.n_experts, wl.top_k
    x = synth.bf16_bits_to_f32(x_bits).astype(np.float64)
    logits = x @ lw.router_w.astype(np.float64).T
    if lw.router_bias is not None:
        logits = logits + lw.router_bias.astype(np.float64)
    logits32 = logits.astype(np.float32)
    ids = np.argsort(-logits32, axis=1, kind="stable")[:, :k] if ids_from is None else ids_from
    l64 = logits32.astype(np.float64)
    if wl.scoring == "softmax":
        p = np.exp(l64 - l64.max(axis=1, keepdims=True))
        p = p / p.sum(axis=1, keepdims=True)
    else:
        p = 1.0 / (1.0 + np.exp(-l64))
    sel = np.take_along_axis(p, ids, axis=1)
    gates = (sel / sel.sum(axis=1, keepdims=True) if wl.renormalize else sel).astype(np.float32)
    G = np.zeros((x.shape[0], wl.n_targets), dtype=np.float64)
    np.put_along_axis(G, ids, gates.astype(np.float64), axis=1)
    y = np.zeros((x.shape[0], wl.hidden), dtype=np.float64)
    for e in range(E):
        gs = lw.global_scale[e] if lw.global_scale is not None else (1.0, 1.0, 1.0)
        Wg = np_decode(lw.codes[0][e], lw.scales[0][e], wl.fmt, float(gs[0]))
        Wu = np_decode(lw.codes[1][e], lw.scales[1][e], wl.fmt, float(gs[1]))
        Wd = np_decode(lw.codes[2][e], lw.scales[2][e], wl.fmt, float(gs[2]))
        a = (x @ Wg.T).astype(np.float32).astype(np.float64)
        u = (x @ Wu.T).astype(np.float32).astype(np.float64)
        h = (np_silu(a) * u).astype(np.float32).astype(np.float64)
        y += G[:, e:e + 1] * (h @ Wd.T)
    if lw.shared_w is not None:
        Wsg, Wsu, Wsd = (synth.bf16_bits_to_f32(w).astype(np.float64) for w in lw.shared_w)
        a = (x @ Wsg.T).astype(np.float32).astype(np.float64)
        u = (x @ Wsu.T).astype(np.float32).astype(np.float64)
        h = (np_silu(a) * u).astype(np.float32).astype(np.float64)
        gs = 1.0
        if lw.shared_gate_w is not None:
            sg = (x @ lw.shared_gate_w.astype(np.float64)).astype(np.float32).astype(np.float64)
            gs = (1.0 / (1.0 + np.exp(-sg)))[:, None]
        y += gs * (h @ Wsd.T)
    return y.astype(np.float32), logits32, ids.astype(np.int32), gates


def output_tolerance(ref: np.ndarray) -> float:
    """|gpu - oracle| <= 1e-2 * max|oracle| + 1e-3, per element."""
    return 1e-2 * float(np.max(np.abs(ref))) + 1e-3
