"""Expert formats of at least four bits beyond FP4: INT4 group-128 (W4A16, bf16
scales) and FP8 E4M3 block-128 (fp32 inverse scales), on the dequantising
tensor-core kernels, against the oracle.

The GPU decodes each weight to bf16 (q * s rounded to nearest even; q * s is
not always a bf16 value) before the bf16 MMA, where the oracle keeps q * s
exact in fp64: a relative error of at most 2^-9 per weight, inside the layer
tolerance.  Routing is unchanged (bit-exact ids).
"""
import numpy as np
import pytest

import oracle
import synth
from tests import _cases as cs
from tests import _gpu as G

pytestmark = pytest.mark.gpu

SHAPES = {
    "int4": dict(hidden=512, inter=256, n_experts=8, top_k=2, fmt="int4g128"),
    "int4_shared_zipf": dict(hidden=768, inter=384, n_experts=12, top_k=3, shared_inter=256, fmt="int4g128",
                             zipf_s=1.1),
    "fp8": dict(hidden=512, inter=256, n_experts=8, top_k=2, fmt="fp8b128"),
    "fp8_sinks": dict(hidden=512, inter=384, n_experts=10, top_k=4, fmt="fp8b128", n_sinks=2),
}


@pytest.mark.parametrize("T", [1, 5, 100, 300])
@pytest.mark.parametrize("name", list(SHAPES))
def test_format_parity(name, T):
    wl = synth.custom_workload(**SHAPES[name])
    lw = synth.make_layer(wl, seed=61)
    L = oracle.Layer.from_weights(lw)
    x, _ = cs.tokens_with_margin(L, wl, T, seed=61, stream=T)
    y_ref, lg, ids, g = L.forward(x)
    layer = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T)
    try:
        y, r = G.run(layer, x)
        assert layer.stats()["last_path"] == 3
        G.check_routing(r, lg, ids, g, wl.n_targets)
        G.check_output(y, y_ref)
    finally:
        layer.close()


@pytest.mark.parametrize("fmt", ["int4g128", "fp8b128"])
def test_format_paged_equals_resident(fmt):
    wl = synth.custom_workload(512, 256, 16, 2, fmt=fmt, zipf_s=1.1, n_slots=4)
    lw = synth.make_layer(wl, seed=62)
    T = 64
    x = synth.make_tokens(wl, T, seed=62)
    # the coldest experts resident: most pairs miss, so the forward runs several waves
    paged = G.make_layer(lw, n_slots=4, max_tokens=T, n_staging=2,
                         table=synth.slot_table(lw, 4, policy="coldest"))
    resident = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T)
    try:
        yp, _ = G.run(paged, x)
        yr, _ = G.run(resident, x)
        assert paged.stats()["last_waves"] > 1
        assert np.array_equal(yp, yr)
    finally:
        paged.close()
        resident.close()


def test_format_admission_at_create():
    F = G.library()
    wl = synth.custom_workload(256, 128, 4, 2, fmt="fp8b128")
    lw = synth.make_layer(wl, seed=63)
    lw.codes[1][2, 3, 4] = 0xFF                 # an E4M3 NaN weight
    with pytest.raises(F.MoEError) as ei:
        F.MoELayer.from_weights(lw, max_tokens=4)
    assert ei.value.status == 2
    wl4 = synth.custom_workload(256, 128, 4, 2, fmt="int4g128")
    lw4 = synth.make_layer(wl4, seed=63)
    lw4.scales[2][1, 7, 0] = 0x7F80             # +inf bf16 scale
    with pytest.raises(F.MoEError) as ei:
        F.MoELayer.from_weights(lw4, max_tokens=4)
    assert ei.value.status == 2
