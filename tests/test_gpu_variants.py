"""Router variants a checkpoint may declare, and the bf16 output, on every
kernel path, against the oracle: sigmoid scoring, top-k without
renormalisation, sink targets (chosen like experts, no FFN), a sigmoid-gated
shared expert; y written as bf16 (round to nearest even of the fp32 combine).

Routing acceptance is the default one (ids bit-exact on inputs drawn with a
1e-3 top-(k+1) margin, logits within 1e-5, gates to fp32 rounding); outputs
within the layer tolerance.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import _cases as cs
from tests import _gpu as G

pytestmark = pytest.mark.gpu

VARIANTS = {
    "sigmoid_renorm": dict(scoring="sigmoid"),
    "softmax_no_renorm": dict(renormalize=False),
    "sigmoid_no_renorm_sinks": dict(scoring="sigmoid", renormalize=False, n_sinks=2),
    "sinks_shared_gate": dict(n_sinks=3, shared_inter=128, shared_gate=True, zipf_s=1.1),
}

# (format, numerics, T): decode and prefill sizes of each kernel path --
# NVFP4 register decode / NVFP4 tensor core, MXFP4 tensor core (8- and
# 56-token tiles), A4
PATHS = [("nvfp4", "exact", 3), ("nvfp4", "exact", 300), ("mxfp4", "exact", 5), ("mxfp4", "exact", 300),
         ("mxfp4", "a4", 40)]


def _layer(variant, fmt):
    kw = dict(hidden=512, inter=256, n_experts=12, top_k=4, fmt=fmt)
    kw.update(VARIANTS[variant])
    wl = synth.custom_workload(**kw)
    return wl, synth.make_layer(wl, seed=41)


@pytest.mark.parametrize("fmt, numerics, T", PATHS)
@pytest.mark.parametrize("variant", list(VARIANTS))
def test_router_variant_parity(variant, fmt, numerics, T):
    wl, lw = _layer(variant, fmt)
    L = oracle.Layer.from_weights(lw, numerics=numerics)
    x, _ = cs.tokens_with_margin(L, wl, T, seed=41, stream=T)
    y_ref, lg, ids, g = L.forward(x)
    layer = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T, numerics=numerics)
    try:
        y, r = G.run(layer, x)
        G.check_routing(r, lg, ids, g, wl.n_targets)
        G.check_output(y, y_ref)
        if wl.n_sinks and T >= 16:        # (a few tokens may all pass the sinks by)
            assert (ids >= wl.n_experts).any(), "no token chose a sink"
    finally:
        layer.close()


def test_variant_paged_equals_resident():
    """Sinks and the shared-expert gate on the staged path: paged output is
    bit-identical to the all-resident output."""
    wl, lw = _layer("sinks_shared_gate", "mxfp4")
    T = 64
    x = synth.make_tokens(wl, T, seed=3)
    paged = G.make_layer(lw, n_slots=4, max_tokens=T, n_staging=2)
    resident = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T)
    try:
        yp, _ = G.run(paged, x)
        yr, _ = G.run(resident, x)
        assert paged.stats()["last_misses"] > 0
        assert np.array_equal(yp, yr)
    finally:
        paged.close()
        resident.close()


@pytest.mark.parametrize("fmt, numerics, T", PATHS)
def test_bf16_output_is_the_rounded_fp32_output(fmt, numerics, T):
    """out_dtype bf16: y is the fp32 combine rounded to nearest even, bit for bit."""
    t = G.torch()
    F = G.library()
    wl = synth.custom_workload(512, 256, 12, 4, shared_inter=128, fmt=fmt)
    lw = synth.make_layer(wl, seed=43)
    x = G.to_device(synth.make_tokens(wl, T, seed=43))
    l32 = F.MoELayer.from_weights(lw, max_tokens=T, numerics=numerics)
    l16 = F.MoELayer.from_weights(lw, max_tokens=T, numerics=numerics, out_dtype="bf16")
    try:
        for lay in (l32, l16):
            lay.set_slot_table(synth.slot_table(lw, wl.n_experts))
        y32 = l32.forward(x)
        y16 = l16.forward(x)
        t.cuda.synchronize()
        assert y16.dtype == t.bfloat16
        assert t.equal(y16, y32.to(t.bfloat16))
        # the host-buffer call returns the same bf16 bits
        yh = l16.forward_host(synth.make_tokens(wl, T, seed=43))
        assert np.array_equal(yh, y16.cpu().view(t.int16).numpy().view(np.uint16))
    finally:
        l32.close()
        l16.close()
