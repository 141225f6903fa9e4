"""Seeded synthetic inputs for one sparse MoE layer over 4-bit experts.

This module is shared by the CUDA path's tests, the benchmark and the CPU
oracle's tests.  It only draws random numbers and packs them into the
checkpoint byte layout; it holds none of the layer's arithmetic (no routing,
no decoding of FP4 values, no matrix products).

Workloads (shapes, formats, skew, resident budgets) follow the five layer
shapes the Strata pages discuss: an OLMoE-like layer, a Qwen3-30B-A3B-like
layer with Zipf-skewed routing, a DeepSeek-V4-Flash-like layer with one
always-on shared expert (page "ro99/strata", model table: 256 experts, top-6,
FP4 E2M1 experts), and a Qwen3.8-Flash-Next-like layer (page "Strata,
Explained", section 2: 512 experts, 10 routed plus 1 shared) with NVFP4
experts and a 9% resident budget (page strata.amperor.ai, memory-fit list:
"9% of experts hot").

Checkpoint byte layout (what ``moe_layer_create`` and the oracle both read):
  * codes[m]  uint8 [E, rows, K/2]: two E2M1 codes per byte, the element with
    the even column index in the low nibble (page "ro99/strata", "MXFP4 is read
    as MXFP4": two E2M1 codes per byte);
  * scales[m] uint8 [E, rows, K/32] E8M0 (MXFP4) or [E, rows, K/16] E4M3 (NVFP4),
    groups running along the input (reduction) dimension;
  * matrices are [out, in] row-major: gate and up are [I, H], down is [H, I].
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "workload", "LayerWeights", "make_layer",
    "make_tokens", "redraw_rows", "slot_table", "f32_to_bf16_bits",
    "bf16_bits_to_f32", "BASE_SEED",
]

BASE_SEED = 20261202

# Matrix indices used everywhere: 0 = gate [I, H], 1 = up [I, H], 2 = down [H, I].
GATE, UP, DOWN = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int            # seed offset
    hidden: int           # H
    inter: int            # I
    n_experts: int        # E
    top_k: int            # k
    shared_inter: int     # I_s (0 = no shared expert)
    fmt: str              # "mxfp4" | "nvfp4"
    zipf_s: Optional[float]
    decode_tokens: tuple
    prefill_tokens: Optional[int]
    n_slots: int          # resident budget S
    slot_policy: str      # "all" | "hottest" | "random"
    # router variants a checkpoint may declare (defaults: softmax, renormalised,
    # no sinks, shared expert with weight 1)
    scoring: str = "softmax"       # "softmax" | "sigmoid"
    renormalize: bool = True
    n_sinks: int = 0               # sink targets after the experts (no FFN)
    shared_gate: bool = False      # shared expert scaled by sigmoid(x . w_sg)

    @property
    def n_targets(self) -> int:
        return self.n_experts + self.n_sinks

    @property
    def group(self) -> int:
        """Weights per block scale along K (FP8 block-128: 128 x 128 blocks)."""
        return {"mxfp4": 32, "nvfp4": 16, "int4g128": 128, "fp8b128": 128}[self.fmt]

    def shape(self, m: int):
        """(rows, K) of matrix m."""
        H, I = self.hidden, self.inter
        return (I, H) if m in (GATE, UP) else (H, I)

    def code_shape(self, m: int):
        """(rows, bytes per row) of matrix m's codes."""
        r, k = self.shape(m)
        return (r, k) if self.fmt == "fp8b128" else (r, k // 2)

    def scale_shape(self, m: int):
        r, k = self.shape(m)
        return (r // 128, k // 128) if self.fmt == "fp8b128" else (r, k // self.group)

    @property
    def scale_dtype(self):
        return {"mxfp4": np.uint8, "nvfp4": np.uint8, "int4g128": np.uint16, "fp8b128": np.float32}[self.fmt]

    def expert_bytes(self) -> int:
        """Checkpoint bytes of one routed expert (codes + block scales [+ fp32 per-tensor])."""
        n = 0
        item = np.dtype(self.scale_dtype).itemsize
        for m in range(3):
            cr, cb = self.code_shape(m)
            sr, sc = self.scale_shape(m)
            n += cr * cb + sr * sc * item
        if self.fmt == "nvfp4":
            n += 3 * 4
        return n


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 0, 256, 128, 8, 2, 0, "mxfp4", None, (16,), None, 8, "all"),
        Workload("olmoe_like", 1, 2048, 1024, 64, 8, 0, "mxfp4", None, (1, 8, 32), None, 64, "all"),
        Workload("qwen3_30b_a3b_like", 2, 2048, 768, 128, 8, 0, "mxfp4", 1.1, (1, 16), 2048, 64, "hottest"),
        Workload("deepseek_v4_flash_like", 3, 4096, 2048, 256, 6, 2048, "mxfp4", None, (1, 64), 4096, 64, "random"),
        Workload("qwen3_8_flash_next_like", 4, 4096, 1024, 512, 10, 1024, "nvfp4", 1.1, (1, 4), 8192, 46, "hottest"),
        # supplementary compute-bound probe: DeepSeek-V4-Flash-like expert shapes, 16 resident
        # experts, 8192 tokens top-2 (about 1024 rows per expert)
        Workload("fp4_peak_probe", 5, 4096, 2048, 16, 2, 0, "mxfp4", None, (1,), 8192, 16, "all"),
    ]
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def custom_workload(hidden, inter, n_experts, top_k, shared_inter=0, fmt="mxfp4",
                    zipf_s=None, n_slots=None, name="custom", index=99, scoring="softmax",
                    renormalize=True, n_sinks=0, shared_gate=False) -> Workload:
    """A workload of arbitrary (small) shape, for tests."""
    return Workload(name, index, hidden, inter, n_experts, top_k, shared_inter, fmt,
                    zipf_s, (1,), None, n_experts if n_slots is None else n_slots,
                    "all" if n_slots is None else "hottest", scoring, renormalize, n_sinks, shared_gate)


# ----------------------------------------------------------------------------
# bf16 bit helpers (storage format of activations and shared-expert weights)
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16, nearest-even, returning the 16-bit patterns (finite inputs)."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# Layer weights
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class LayerWeights:
    wl: Workload
    router_w: np.ndarray                  # fp32 [E + n_sinks, H]
    router_bias: Optional[np.ndarray]     # fp32 [E + n_sinks] or None
    zipf_rank: Optional[np.ndarray]       # int64 [E + n_sinks], 1 = most popular (None without skew)
    codes: list                           # 3 x uint8 [E, rows, K/2]
    scales: list                          # 3 x uint8 [E, rows, K/G]
    global_scale: Optional[np.ndarray]    # fp32 [E, 3] (NVFP4) or None
    shared_w: Optional[list]              # 3 x uint16 bf16 bits: [Is,H], [Is,H], [H,Is]
    shared_gate_w: Optional[np.ndarray] = None   # fp32 [H] (shared-expert gate) or None


def _streams(seed: int, n: int):
    return np.random.SeedSequence(seed).spawn(n)


# substream slots
_S_X, _S_ROUTER, _S_BIAS, _S_EXPERTS, _S_SHARED, _S_RESAMPLE, _S_SLOTS, _S_SGATE = range(8)


def _seed(wl: Workload, seed: Optional[int]) -> int:
    return BASE_SEED + wl.index if seed is None else seed


def make_layer(wl: Workload, seed: Optional[int] = None, experts: Optional[int] = None) -> LayerWeights:
    """Draw one layer's weights.

    Recipe: router weights N(0, 0.02^2) fp32; E2M1 codes uniform over all 16
    values (uniform random bytes); E8M0 block exponents uniform in [118, 124];
    NVFP4 block scales are E4M3 codes with exponent field uniform in [7, 12] and
    any mantissa (values 1..60) and a per-tensor fp32 scale of 2^-9; shared
    expert weights N(0, 0.02^2) rounded to bf16; Zipf(s) skew as a per-target
    router bias -s*ln(rank) with ranks a seeded permutation of 1..E + n_sinks;
    sink targets get router rows like experts and no expert weights; the
    shared-expert gate vector (shared_gate) is N(0, 0.02^2) fp32.
    ``experts`` limits how many experts get distinct draws (the rest repeat
    them); only tests of host logic use it.
    """
    ss = _streams(_seed(wl, seed), 8)
    E, H = wl.n_experts, wl.hidden
    NT = wl.n_targets                      # experts, then sink targets (router rows only)
    rng_r = np.random.Generator(np.random.PCG64(ss[_S_ROUTER]))
    router_w = (rng_r.standard_normal((NT, H), dtype=np.float32) * np.float32(0.02)).astype(np.float32)

    router_bias = None
    rank = None
    if wl.zipf_s is not None:
        rng_b = np.random.Generator(np.random.PCG64(ss[_S_BIAS]))
        rank = rng_b.permutation(NT) + 1
        router_bias = (-wl.zipf_s * np.log(rank.astype(np.float64))).astype(np.float32)

    codes, scales = [], []
    for m in range(3):
        codes.append(np.empty((E,) + wl.code_shape(m), dtype=np.uint8))
        scales.append(np.empty((E,) + wl.scale_shape(m), dtype=wl.scale_dtype))
    expert_ss = ss[_S_EXPERTS].spawn(E)
    n_distinct = E if experts is None else min(E, experts)
    for e in range(E):
        if e >= n_distinct:
            for m in range(3):
                codes[m][e] = codes[m][e % n_distinct]
                scales[m][e] = scales[m][e % n_distinct]
            continue
        rng_e = np.random.Generator(np.random.PCG64(expert_ss[e]))
        for m in range(3):
            cr, cb = wl.code_shape(m)
            ssh = wl.scale_shape(m)
            codes[m][e] = np.frombuffer(rng_e.bytes(cr * cb), dtype=np.uint8).reshape(cr, cb)
            if wl.fmt == "mxfp4":
                scales[m][e] = rng_e.integers(118, 125, size=ssh, dtype=np.uint8)
            elif wl.fmt == "nvfp4":
                ex = rng_e.integers(7, 13, size=ssh, dtype=np.uint8)
                mant = rng_e.integers(0, 8, size=ssh, dtype=np.uint8)
                scales[m][e] = (ex << 3) | mant
            elif wl.fmt == "int4g128":
                # bf16 scales 2^u * [1, 2), u in -9..-5 (|w| up to 8 * 2^-4)
                v = np.ldexp(1.0 + rng_e.random(ssh), rng_e.integers(-9, -4, size=ssh)).astype(np.float32)
                scales[m][e] = f32_to_bf16_bits(v)
            else:
                # FP8 E4M3 weights over every finite code (NaN codes S.1111.111
                # redrawn as +-448), fp32 inverse scales 2^u * [1, 2), u in -14..-10
                q = codes[m][e]
                nan = (q & 0x7F) == 0x7F
                q[nan] = q[nan] & 0xFE
                scales[m][e] = np.ldexp(1.0 + rng_e.random(ssh), rng_e.integers(-14, -9, size=ssh)).astype(np.float32)
    global_scale = None
    if wl.fmt == "nvfp4":
        global_scale = np.full((E, 3), 2.0 ** -9, dtype=np.float32)

    shared_w = None
    if wl.shared_inter:
        Is = wl.shared_inter
        rng_s = np.random.Generator(np.random.PCG64(ss[_S_SHARED]))
        shared_w = [
            f32_to_bf16_bits(rng_s.standard_normal((Is, H), dtype=np.float32) * np.float32(0.02)),
            f32_to_bf16_bits(rng_s.standard_normal((Is, H), dtype=np.float32) * np.float32(0.02)),
            f32_to_bf16_bits(rng_s.standard_normal((H, Is), dtype=np.float32) * np.float32(0.02)),
        ]
    shared_gate_w = None
    if wl.shared_gate:
        rng_g = np.random.Generator(np.random.PCG64(ss[_S_SGATE]))
        shared_gate_w = (rng_g.standard_normal(H, dtype=np.float32) * np.float32(0.02)).astype(np.float32)
    return LayerWeights(wl, router_w, router_bias, rank, codes, scales, global_scale, shared_w, shared_gate_w)


def make_tokens(wl: Workload, T: int, seed: Optional[int] = None, stream: int = 0) -> np.ndarray:
    """T activation rows, N(0,1) fp32 rounded to bf16 (returned as bf16 bit patterns)."""
    ss = _streams(_seed(wl, seed), 7)[_S_X].spawn(stream + 1)[stream]
    rng = np.random.Generator(np.random.PCG64(ss))
    x = rng.standard_normal((T, wl.hidden), dtype=np.float32)
    return f32_to_bf16_bits(x)


def resample_rng(wl: Workload, seed: Optional[int] = None, stream: int = 0) -> np.random.Generator:
    ss = _streams(_seed(wl, seed), 7)[_S_RESAMPLE].spawn(stream + 1)[stream]
    return np.random.Generator(np.random.PCG64(ss))


def redraw_rows(x_bits: np.ndarray, rows, rng: np.random.Generator) -> None:
    """Replace the given rows of a bf16 activation matrix with fresh N(0,1) draws."""
    rows = np.asarray(rows, dtype=np.int64)
    if rows.size:
        x_bits[rows] = f32_to_bf16_bits(rng.standard_normal((rows.size, x_bits.shape[1]), dtype=np.float32))


def slot_table(lw: LayerWeights, n_slots: Optional[int] = None, seed: Optional[int] = None,
               policy: Optional[str] = None) -> np.ndarray:
    """Resident-slot table: int32 [E], slot index or -1 (expert kept in host memory).

    "all": every expert resident (slot = expert index); "hottest": the S experts
    with the lowest Zipf rank (a static warm fill); "coldest": the S experts with
    the highest Zipf rank (a cold start: most routed pairs miss); "random": a
    seeded random subset of S experts.
    """
    wl = lw.wl
    E = wl.n_experts
    S = wl.n_slots if n_slots is None else n_slots
    policy = wl.slot_policy if policy is None else policy
    table = np.full(E, -1, dtype=np.int32)
    if policy == "all" or S >= E:
        table[:] = np.arange(E, dtype=np.int32) if S >= E else -1
        if S < E:
            table[:S] = np.arange(S, dtype=np.int32)
        return table
    if policy in ("hottest", "coldest") and lw.zipf_rank is not None:
        order = np.argsort(lw.zipf_rank[:E], kind="stable")      # experts only (sinks hold no weights)
        if policy == "coldest":
            order = order[::-1]
    else:
        ss = _streams(_seed(wl, seed), 7)[_S_SLOTS]
        order = np.random.Generator(np.random.PCG64(ss)).permutation(E)
    chosen = order[:S]
    table[chosen] = np.arange(S, dtype=np.int32)
    return table
