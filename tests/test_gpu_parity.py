"""CUDA path vs the CPU oracle, through the C ABI, on seeded synthetic layers.

Acceptance: bit-exact expert ids, counts, offsets and permutation (inputs drawn
with a top-k logit margin >= 1e-3); router logits within 1e-5; layer outputs
within |gpu - oracle| <= 1e-2 * max|oracle| + 1e-3 per element; paged outputs
bit-identical to all-resident outputs.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import _cases as cs
from tests import _gpu as G

pytestmark = pytest.mark.gpu

SMALL = {
    "mx_basic": dict(hidden=256, inter=128, n_experts=8, top_k=2),
    "mx_shared": dict(hidden=256, inter=256, n_experts=16, top_k=4, shared_inter=128),
    "nv_shared_zipf": dict(hidden=512, inter=128, n_experts=12, top_k=3, shared_inter=256, fmt="nvfp4",
                           zipf_s=1.1),
    "mx_wide": dict(hidden=768, inter=384, n_experts=32, top_k=8),
    "mx_k1": dict(hidden=256, inter=128, n_experts=4, top_k=1),
    "mx_k_eq_e": dict(hidden=256, inter=128, n_experts=3, top_k=3),
}


@pytest.mark.parametrize("T", [1, 3, 17, 64, 200])
@pytest.mark.parametrize("name", list(SMALL))
def test_small_layers_full_parity(name, T):
    wl = synth.custom_workload(**SMALL[name])
    lw = synth.make_layer(wl, seed=5)
    L = oracle.Layer.from_weights(lw)
    x, _ = cs.tokens_with_margin(L, wl, T, seed=5, stream=T)
    y_ref, lg, ids, g = L.forward(x)
    layer = G.make_layer(lw, max_tokens=T)
    y, r = G.run(layer, x)
    G.check_routing(r, lg, ids, g, wl.n_experts)
    G.check_output(y, y_ref)
    layer.close()


def test_tiny_workload_full_parity():
    wl = synth.workload("tiny")
    lw = synth.make_layer(wl)
    L = oracle.Layer.from_weights(lw)
    x, _ = cs.tokens_with_margin(L, wl, 16)
    y_ref, lg, ids, g = L.forward(x)
    layer = G.make_layer(lw, max_tokens=16)
    y, r = G.run(layer, x)
    G.check_routing(r, lg, ids, g, wl.n_experts)
    G.check_output(y, y_ref)
    # repeated forwards are bit-identical
    y2, _ = G.run(layer, x)
    assert np.array_equal(y, y2)
    layer.close()


# ---------------------------------------------------------------- OLMoE-like, all resident
@pytest.fixture(scope="module")
def olmoe():
    wl = synth.workload("olmoe_like")
    lw = synth.make_layer(wl)
    layer = G.make_layer(lw, max_tokens=32)
    yield lw, oracle.Layer.from_weights(lw), layer
    layer.close()


@pytest.mark.parametrize("T", [1, 8, 32])
def test_olmoe_decode_full_parity(olmoe, T):
    lw, L, layer = olmoe
    x, _ = cs.tokens_with_margin(L, lw.wl, T, stream=T)
    y_ref, lg, ids, g = L.forward(x)
    y, r = G.run(layer, x)
    G.check_routing(r, lg, ids, g, lw.wl.n_experts)
    G.check_output(y, y_ref)


def test_olmoe_forward_host_matches_device(olmoe):
    lw, L, layer = olmoe
    x = synth.make_tokens(lw.wl, 32, stream=77)
    y, _ = G.run(layer, x)
    yh = layer.forward_host(x)
    assert np.array_equal(y, yh)


# ---------------------------------------------------------------- paged workloads
def _paged_case(name, Ts, sample=8):
    wl = synth.workload(name)
    lw = synth.make_layer(wl)
    L = oracle.Layer.from_weights(lw)
    maxT = max(Ts)
    paged = G.make_layer(lw, max_tokens=maxT)                              # resident budget of the workload
    resident = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=maxT)    # every expert in HBM
    few = G.make_layer(lw, max_tokens=maxT, n_staging=4)                  # many staging waves
    rng = np.random.default_rng(3)
    try:
        for T in Ts:
            x, _ = cs.tokens_with_margin(L, wl, T, stream=T)
            yp, rp = G.run(paged, x)
            st = paged.stats()
            yr, rr = G.run(resident, x)
            assert np.array_equal(yp, yr), "paged output is not bit-identical to the resident output"
            for k in rr:
                assert np.array_equal(rp[k], rr[k])
            yf, _ = G.run(few, x)
            assert np.array_equal(yf, yr), "multi-wave paged output differs from the resident output"
            if T >= 64:
                assert few.stats()["last_waves"] > 1
            assert st["last_misses"] >= 0
            lg, ids, g = L.route_all(x)
            G.check_routing(rp, lg, ids, g, wl.n_experts)
            # tile-scheduler classes (hottest / coldest expert, tile boundaries,
            # ragged tails) plus random rows
            rows = G.boundary_rows(resident, rr, wl.top_k, rng=rng, extra=sample)
            y_ref, *_ = L.forward(x, rows=rows)
            G.check_output(yp[rows], y_ref)
        assert paged.stats()["misses"] > 0, "the paged layer never staged an expert"
        assert resident.stats()["misses"] == 0
    finally:
        for l in (paged, resident, few):
            l.close()


def test_qwen3_30b_like_paged():
    _paged_case("qwen3_30b_a3b_like", [1, 16, 2048])


def test_deepseek_v4_flash_like_paged_shared():
    _paged_case("deepseek_v4_flash_like", [1, 64, 4096])


def test_qwen3_8_flash_next_like_nvfp4_paged_shared():
    _paged_case("qwen3_8_flash_next_like", [1, 4, 8192], sample=6)


# ---------------------------------------------------------------- edge cases and errors
@pytest.fixture(scope="module")
def small():
    wl = synth.custom_workload(256, 128, 8, 2, n_slots=4)
    lw = synth.make_layer(wl, seed=9)
    layer = G.make_layer(lw, n_slots=4, max_tokens=40)
    yield lw, layer
    layer.close()


def test_zero_tokens_is_noop_and_bounds(small):
    F = G.library()
    lw, layer = small
    t = G.torch()
    x = t.zeros((0, 256), dtype=t.bfloat16, device="cuda")
    y = layer.forward(x)
    assert y.shape == (0, 256)
    x41 = t.zeros((41, 256), dtype=t.bfloat16, device="cuda")
    with pytest.raises(F.MoEError) as ei:
        layer.forward(x41)
    assert ei.value.status == 1


def test_slot_table_validation_keeps_previous_table(small):
    F = G.library()
    lw, layer = small
    x = synth.make_tokens(lw.wl, 40, seed=9)
    y0, _ = G.run(layer, x)
    for bad in ([0, 1, 2, 3, 4, -1, -1, -1],      # slot 4 out of range (S = 4)
                [0, 0, -1, -1, -1, -1, -1, -1],    # duplicate slot
                [-2, -1, -1, -1, -1, -1, -1, -1]):
        with pytest.raises(F.MoEError) as ei:
            layer.set_slot_table(np.array(bad, dtype=np.int32))
        assert ei.value.status == 3
    y1, _ = G.run(layer, x)
    assert np.array_equal(y0, y1)
    # a different valid table gives the same output bit for bit
    layer.set_slot_table(np.array([-1, -1, -1, -1, 3, 2, 1, 0], dtype=np.int32))
    y2, _ = G.run(layer, x)
    assert np.array_equal(y0, y2)
    layer.set_slot_table(np.full(8, -1, dtype=np.int32))
    y3, _ = G.run(layer, x)
    assert np.array_equal(y0, y3)


def test_injected_staging_failure_returns_error_and_recovers(small):
    F = G.library()
    lw, layer = small
    layer.set_slot_table(np.full(8, -1, dtype=np.int32))
    x = synth.make_tokens(lw.wl, 40, seed=11)
    y0, _ = G.run(layer, x)
    layer.inject(1)
    with pytest.raises(F.MoEError) as ei:
        G.run(layer, x)
    assert ei.value.status == 5
    G.torch().cuda.synchronize()
    y1, _ = G.run(layer, x)
    assert np.array_equal(y0, y1)


def test_injected_allocation_failure_at_create():
    F = G.library()
    wl = synth.custom_workload(256, 128, 4, 2)
    lw = synth.make_layer(wl, seed=1)
    F.lib().moe_debug_inject(None, 2)
    with pytest.raises(F.MoEError) as ei:
        F.MoELayer.from_weights(lw, max_tokens=4)
    assert ei.value.status == 4
    layer = G.make_layer(lw, max_tokens=4)     # the next create works
    x = synth.make_tokens(wl, 4, seed=1)
    y, _ = G.run(layer, x)
    assert np.all(np.isfinite(y))
    layer.close()


@pytest.mark.parametrize("fmt, numerics, T", [("mxfp4", "exact", 8), ("mxfp4", "exact", 300),
                                              ("nvfp4", "exact", 3), ("nvfp4", "exact", 300),
                                              ("mxfp4", "a4", 130)])
def test_bounded_waits_give_up_and_the_context_recovers(fmt, numerics, T):
    """The device error word is set before a forward's kernels run (test hook
    3), so every bounded wait of theirs that has to wait gives up at once: the
    kernels run out without hanging (well under their 2 s time limit), the next
    forward reports MOE_ERR_CUDA and clears the word, and the forward after
    that is bit-identical to a clean one.  Shapes cover the MXFP4 tensor-core
    path (8- and 56-token tiles), the NVFP4 register and tensor-core paths,
    both shared-expert kernels, and A4."""
    import time
    t = G.torch()
    F = G.library()
    wl = synth.custom_workload(512, 256, 8, 2, shared_inter=256, fmt=fmt)
    lw = synth.make_layer(wl, seed=71)
    x = synth.make_tokens(wl, T, seed=71)
    layer = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T, numerics=numerics)
    try:
        y0, _ = G.run(layer, x)
        xd = G.to_device(x)
        layer.inject(3)
        t0 = time.perf_counter()
        layer.forward(xd)
        t.cuda.synchronize()
        assert time.perf_counter() - t0 < 1.5, "a wait ran to its time limit"
        assert layer.stats()["device_error"] != 0
        with pytest.raises(F.MoEError) as ei:
            layer.forward(xd)
        assert ei.value.status == 5
        assert layer.stats()["device_error"] == 0
        y1, _ = G.run(layer, x)
        assert np.array_equal(y0, y1)
    finally:
        layer.close()
