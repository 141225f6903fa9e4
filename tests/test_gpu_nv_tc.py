"""EXACT numerics of NVFP4 layers on the tensor core at prefill-sized batches:
each weight tile's E2M1 codes times their E4M3 block scales are decoded once per
token tile into shared memory as bf16 (exact), multiplied with tcgen05
kind::f16 against the bf16 x rows, the per-tensor scale applied to the fp32
accumulator; h is rounded to bf16 for the down pass.

Checks the path choice, full parity with the oracle on small shapes whose
tiles (64 or 128 tokens) end in ragged tails, agreement with the register
kernels that serve decode-sized batches of the same layer, and the full-size
Qwen3.8-Flash-Next-like prefill (8192 tokens, all resident) on rows chosen
from the tile list.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import _cases as cs
from tests import _gpu as G

pytestmark = pytest.mark.gpu

SHAPES = {
    "nv_basic": dict(hidden=512, inter=256, n_experts=8, top_k=2, fmt="nvfp4"),
    "nv_zipf_shared": dict(hidden=768, inter=384, n_experts=16, top_k=4, shared_inter=256, fmt="nvfp4",
                           zipf_s=1.1),
    "nv_k1": dict(hidden=256, inter=128, n_experts=4, top_k=1, fmt="nvfp4"),
}


@pytest.mark.parametrize("T", [100, 333, 700])
@pytest.mark.parametrize("name", list(SHAPES))
def test_nvfp4_prefill_tensor_core_parity(name, T):
    wl = synth.custom_workload(**SHAPES[name])
    lw = synth.make_layer(wl, seed=17)
    L = oracle.Layer.from_weights(lw)
    x, _ = cs.tokens_with_margin(L, wl, T, seed=17, stream=T)
    y_ref, lg, ids, g = L.forward(x)
    layer = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T)
    try:
        y, r = G.run(layer, x)
        assert layer.stats()["last_path"] == 3, "the NVFP4 prefill batch did not take the tensor-core path"
        G.check_routing(r, lg, ids, g, wl.n_experts)
        G.check_output(y, y_ref)
        tiles = G.tile_list(layer)
        assert tiles[:, 2].sum() == T * wl.top_k
        # repeated forwards are bit-identical (fixed work-item order per tile)
        y2, _ = G.run(layer, x)
        assert np.array_equal(y, y2)
    finally:
        layer.close()


def test_nvfp4_tensor_core_matches_register_path():
    """The same tokens through the tensor-core path (one forward of the whole
    batch) and through the register kernels (decode-sized slices of it) agree
    within the output tolerance of the oracle."""
    wl = synth.custom_workload(**SHAPES["nv_zipf_shared"])
    lw = synth.make_layer(wl, seed=23)
    L = oracle.Layer.from_weights(lw)
    T = 256
    x, _ = cs.tokens_with_margin(L, wl, T, seed=23, stream=1)
    y_ref, *_ = L.forward(x)
    layer = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T)
    try:
        y_tc, _ = G.run(layer, x)
        assert layer.stats()["last_path"] == 3
        parts = []
        for i in range(0, T, 2):
            yi, _ = G.run(layer, x[i:i + 2])
            assert layer.stats()["last_path"] == 0
            parts.append(yi)
        y_reg = np.concatenate(parts)
        G.check_output(y_tc, y_ref)
        G.check_output(y_reg, y_ref)
        tol = cs.output_tolerance(y_ref)
        assert float(np.abs(y_tc.astype(np.float64) - y_reg).max()) <= tol
    finally:
        layer.close()


def test_qwen3_8_flash_next_like_prefill_all_resident():
    """Full-size prefill, every expert resident: routing bit-exact against the
    oracle for all 8192 tokens, outputs against the oracle on the rows of the
    hottest and coldest experts' tiles, tile boundaries and ragged tails."""
    wl = synth.workload("qwen3_8_flash_next_like")
    lw = synth.make_layer(wl)
    L = oracle.Layer.from_weights(lw)
    T = wl.prefill_tokens
    x, _ = cs.tokens_with_margin(L, wl, T, stream=T)
    layer = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T)
    try:
        y, r = G.run(layer, x)
        assert layer.stats()["last_path"] == 3
        lg, ids, g = L.route_all(x)
        G.check_routing(r, lg, ids, g, wl.n_experts)
        rows = G.boundary_rows(layer, r, wl.top_k, rng=np.random.default_rng(8), extra=4)
        assert rows.size >= 8
        y_ref, *_ = L.forward(x, rows=rows)
        G.check_output(y[rows], y_ref)
    finally:
        layer.close()
