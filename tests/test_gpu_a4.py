"""A4 numerics (activations quantised to the experts' FP4 format, tcgen05
block-scaled MMA) against the oracle's A4 mode.

Near a rounding boundary the GPU's fp32 h (different summation order) can pick
the neighbouring FP4 code where the oracle does not; each such flip moves one
element of h by one FP4 step, far inside the output tolerance.  The
quantisation of x is exact on both sides (bf16 inputs, identical fp32 steps).
"""
import numpy as np
import pytest

import oracle
import synth
from tests import _cases as cs
from tests import _gpu as G

pytestmark = pytest.mark.gpu

SHAPES = {
    "mx_small": dict(hidden=256, inter=128, n_experts=8, top_k=2),
    "nv_small": dict(hidden=512, inter=256, n_experts=8, top_k=2, fmt="nvfp4"),
    "mx_shared_zipf": dict(hidden=512, inter=256, n_experts=16, top_k=4, shared_inter=128, zipf_s=1.1),
    "nv_shared": dict(hidden=256, inter=384, n_experts=6, top_k=3, shared_inter=256, fmt="nvfp4"),
}


@pytest.mark.parametrize("T", [1, 7, 130, 300])
@pytest.mark.parametrize("name", list(SHAPES))
def test_a4_small_layers_vs_oracle_a4(name, T):
    wl = synth.custom_workload(**SHAPES[name])
    lw = synth.make_layer(wl, seed=31)
    L = oracle.Layer.from_weights(lw, numerics="a4")
    x, _ = cs.tokens_with_margin(L, wl, T, seed=31, stream=T)
    y_ref, lg, ids, g = L.forward(x)
    layer = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T, numerics="a4")
    y, r = G.run(layer, x)
    G.check_routing(r, lg, ids, g, wl.n_experts)
    G.check_output(y, y_ref)
    assert layer.stats()["last_path"] == 1
    layer.close()


def test_a4_paged_equals_resident_and_oracle():
    wl = synth.workload("qwen3_30b_a3b_like")
    lw = synth.make_layer(wl)
    L = oracle.Layer.from_weights(lw, numerics="a4")
    T = 2048
    x, _ = cs.tokens_with_margin(L, wl, T, stream=T)
    paged = G.make_layer(lw, max_tokens=T, numerics="a4", n_staging=8)
    resident = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T, numerics="a4")
    try:
        yp, rp = G.run(paged, x)
        yr, rr = G.run(resident, x)
        assert np.array_equal(yp, yr), "A4 paged output differs from the resident output"
        assert paged.stats()["last_waves"] > 1
        rows = np.array([0, 1, 777, 1500, T - 1], dtype=np.int32)
        y_ref, *_ = L.forward(x, rows=rows)
        G.check_output(yp[rows], y_ref)
    finally:
        paged.close()
        resident.close()


def test_a4_close_to_exact_mode():
    """A4 and EXACT outputs of the same layer agree to FP4 activation precision."""
    wl = synth.custom_workload(512, 256, 8, 2)
    lw = synth.make_layer(wl, seed=4)
    x = synth.make_tokens(wl, 64, seed=4)
    e = G.make_layer(lw, max_tokens=64)
    a = G.make_layer(lw, max_tokens=64, numerics="a4")
    ye, _ = G.run(e, x)
    ya, _ = G.run(a, x)
    rel = np.abs(ya - ye).max() / np.abs(ye).max()
    assert rel < 0.5, rel
    e.close()
    a.close()


@pytest.mark.parametrize("name", ["deepseek_v4_flash_like", "qwen3_8_flash_next_like"])
def test_a4_full_size_prefill_all_resident(name):
    """A4 at the prefill sizes the measurements quote (DeepSeek-V4-Flash-like
    4096 tokens, MXFP4; Qwen3.8-Flash-Next-like 8192 tokens, NVFP4), every
    expert resident: routing bit-exact against the oracle for every token,
    outputs against the oracle's A4 mode on the rows of the hottest and
    coldest experts' tiles, tile boundaries and ragged tails."""
    wl = synth.workload(name)
    lw = synth.make_layer(wl)
    L = oracle.Layer.from_weights(lw, numerics="a4")
    T = wl.prefill_tokens
    x, _ = cs.tokens_with_margin(L, wl, T, stream=T)
    layer = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T, numerics="a4")
    try:
        y, r = G.run(layer, x)
        assert layer.stats()["last_path"] == 1
        lg, ids, g = L.route_all(x)
        G.check_routing(r, lg, ids, g, wl.n_experts)
        rows = G.boundary_rows(layer, r, wl.top_k, rng=np.random.default_rng(9), extra=3)
        y_ref, *_ = L.forward(x, rows=rows)
        G.check_output(y[rows], y_ref)
    finally:
        layer.close()
