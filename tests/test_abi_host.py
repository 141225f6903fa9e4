"""Host-side checks of the C ABI: no GPU needed, no compute call made."""
import ctypes as C
import os
import re

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def F():
    import fp4_expert_layer_b200 as F
    from fp4_expert_layer_b200 import build
    build.build()
    return F


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ \*]*?\b(moe_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(F):
    decl = _declared_functions()
    assert "moe_forward" in decl and "moe_layer_create" in decl
    L = C.CDLL(F._lib.SO)
    missing = [n for n in decl if not hasattr(L, n)]
    assert not missing, missing
    assert set(F._lib.EXPORTED) <= set(decl)


def test_checked_library_builds_and_exports_every_declared_symbol(F):
    from fp4_expert_layer_b200 import build
    so = build.build(checked=True)
    assert so.endswith("libfp4moe_checked.so")
    assert "-DMOE_DEBUG_CHECKS" not in build.nvcc_cmd("x")
    L = C.CDLL(so)
    missing = [n for n in _declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_plan_sizes(F):
    wl = synth.workload("olmoe_like")
    cfg = F.make_config(wl.hidden, wl.inter, wl.n_experts, wl.top_k, max_tokens=32)
    p = F.plan(cfg)
    # codes + scales of one expert, plus one row-reference byte per row, 256-byte aligned pieces
    assert p["expert_bytes"] >= wl.expert_bytes()
    assert p["expert_bytes"] - wl.expert_bytes() < 3 * (wl.inter + wl.hidden) + 9 * 256
    assert p["slot_bytes"] == 64 * p["expert_bytes"]
    assert p["staging_bytes"] == 0
    assert p["pinned_bytes"] == 64 * p["expert_bytes"]
    wl4 = synth.workload("qwen3_8_flash_next_like")
    cfg4 = F.make_config(wl4.hidden, wl4.inter, wl4.n_experts, wl4.top_k, wl4.shared_inter, "nvfp4",
                         n_slots=46, max_tokens=8192)
    p4 = F.plan(cfg4)
    assert p4["staging_bytes"] == 64 * p4["expert_bytes"]
    assert p4["expert_bytes"] >= wl4.expert_bytes()


@pytest.mark.parametrize("bad, status", [
    (dict(hidden=300), 1), (dict(inter=100), 1), (dict(n_experts=0), 1), (dict(top_k=0), 1),
    (dict(top_k=9, n_experts=8), 1), (dict(shared_inter=64), 1), (dict(fmt=7), 1),
    (dict(renormalize=2), 1), (dict(n_slots=65), 1), (dict(max_tokens=0), 1),
    (dict(n_slots=10, n_staging=1), 1), (dict(scoring=2), 1), (dict(n_sinks=-1), 1),
    (dict(n_sinks=961), 1), (dict(shared_gate=1), 1), (dict(out_dtype=2), 1),
    (dict(top_k=11, n_experts=8, n_sinks=2), 1),
])
def test_config_validation(F, bad, status):
    cfg = F.make_config(2048, 1024, 64, 8, max_tokens=8)
    for k, v in bad.items():
        setattr(cfg, k, v)
    with pytest.raises(F.MoEError) as ei:
        F.plan(cfg)
    assert ei.value.status == status


@pytest.mark.parametrize("variant", [
    dict(renormalize=0), dict(scoring=1), dict(scoring=1, renormalize=0), dict(n_sinks=2, top_k=10),
    dict(n_sinks=960), dict(shared_inter=256, shared_gate=1), dict(out_dtype=1),
])
def test_router_variants_and_output_dtype_are_valid_configurations(F, variant):
    """Routing semantics a checkpoint declares are configuration: each of these
    plans without error, and sink targets and a shared-expert gate row add
    router rows to the resident bytes."""
    cfg = F.make_config(2048, 1024, 64, 8, max_tokens=8)
    base = F.plan(cfg)["resident_bytes"]
    for k, v in variant.items():
        setattr(cfg, k, v)
    p = F.plan(cfg)
    extra_rows = variant.get("n_sinks", 0) + variant.get("shared_gate", 0)
    extra_shared = 3 * variant.get("shared_inter", 0) * 2048 * 2
    assert p["resident_bytes"] == base + extra_rows * (2048 * 4 + 4) + extra_shared


def test_shared_gate_needs_its_weights(F):
    wl = synth.custom_workload(256, 128, 4, 2, shared_inter=128)
    lw = synth.make_layer(wl, seed=1)
    cfg = F.make_config(256, 128, 4, 2, shared_inter=128, max_tokens=4, shared_gate=True)
    with pytest.raises(F.MoEError) as ei:
        F.admit(cfg, F.weights_from_layer(lw))
    assert ei.value.status == 1 and "shared_gate_w" in str(ei.value)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_admission_rejects_bad_scale_codes(F, fmt):
    wl = synth.custom_workload(256, 128, 4, 2, fmt=fmt)
    lw = synth.make_layer(wl, seed=1)
    cfg = F.make_config(256, 128, 4, 2, fmt=fmt, max_tokens=4)
    F.admit(cfg, F.weights_from_layer(lw))
    bad_codes = [0, 255] if fmt == "mxfp4" else [0x7F, 0xFF, 0xB8]
    for code in bad_codes:
        lw2 = synth.make_layer(wl, seed=1)
        lw2.scales[2][3, 5, 1] = code
        with pytest.raises(F.MoEError) as ei:
            F.admit(cfg, F.weights_from_layer(lw2))
        assert ei.value.status == 2
        assert "expert 3 matrix 2" in str(ei.value)
    if fmt == "nvfp4":
        lw3 = synth.make_layer(wl, seed=1)
        lw3.global_scale[1, 0] = -1.0
        with pytest.raises(F.MoEError):
            F.admit(cfg, F.weights_from_layer(lw3))


@pytest.mark.parametrize("fmt", ["int4g128", "fp8b128"])
def test_admission_of_other_formats(F, fmt):
    """INT4: non-finite bf16 scales are rejected; FP8: non-positive or
    non-finite fp32 scales and E4M3 NaN weights are rejected; A4 numerics is
    refused for both (it quantises activations to an FP4 format)."""
    wl = synth.custom_workload(256, 128, 4, 2, fmt=fmt)
    lw = synth.make_layer(wl, seed=2)
    cfg = F.make_config(256, 128, 4, 2, fmt=fmt, max_tokens=4)
    F.admit(cfg, F.weights_from_layer(lw))
    bad = synth.make_layer(wl, seed=2)
    if fmt == "int4g128":
        bad.scales[1][3, 5, 0] = 0x7FC0          # NaN bf16
    else:
        bad.scales[1][3, 0, 1] = -0.5
    with pytest.raises(F.MoEError) as ei:
        F.admit(cfg, F.weights_from_layer(bad))
    assert ei.value.status == 2 and "expert 3 matrix 1" in str(ei.value)
    if fmt == "fp8b128":
        bad = synth.make_layer(wl, seed=2)
        bad.codes[0][1, 2, 3] = 0x7F
        with pytest.raises(F.MoEError) as ei:
            F.admit(cfg, F.weights_from_layer(bad))
        assert ei.value.status == 2 and "NaN" in str(ei.value)
    cfg_a4 = F.make_config(256, 128, 4, 2, fmt=fmt, numerics="a4", max_tokens=4)
    with pytest.raises(F.MoEError) as ei:
        F.plan(cfg_a4)
    assert ei.value.status == 6


@pytest.mark.parametrize("fmt", ["int4g128", "fp8b128"])
def test_plan_sizes_of_other_formats(F, fmt):
    wl = synth.custom_workload(2048, 1024, 8, 2, fmt=fmt)
    p = F.plan(F.make_config(2048, 1024, 8, 2, fmt=fmt, max_tokens=4))
    assert wl.expert_bytes() <= p["expert_bytes"] < wl.expert_bytes() + 6 * 256


def test_a4_not_silently_substituted(F):
    cfg = F.make_config(256, 128, 4, 2, numerics="a4", max_tokens=4)
    try:
        F.plan(cfg)
    except F.MoEError as e:       # a build without the A4 path must refuse, never fall back
        assert e.status == 6


def test_null_handles_are_refused_without_touching_the_gpu(F):
    """Entry points check their arguments before any CUDA call: a NULL layer or
    graph returns MOE_ERR_INVALID_ARG (destroy of NULL is a no-op)."""
    L = F.lib()
    out = C.c_void_p(123)
    assert L.moe_graph_capture(None, None, 1, None, None, C.byref(out)) == 1
    assert L.moe_graph_launch(None, None) == 1
    assert L.moe_graph_destroy(None) == 0
    assert L.moe_forward(None, None, 1, None, None, None) == 1
    assert L.moe_forward_host(None, None, 1, None, None) == 1
    assert L.moe_set_slot_table(None, None, None) == 1
    assert b"NULL" in L.moe_last_error()
