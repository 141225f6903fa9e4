"""CUDA-graph capture of one all-resident forward (moe_graph_capture / launch /
destroy): a replay writes the same y, bit for bit, as the eager forward it was
captured from, on each kernel path; capture is refused while experts are not
all resident, and a replay is refused after the slot table changed."""
import numpy as np
import pytest

import oracle
import synth
from tests import _cases as cs
from tests import _gpu as G

pytestmark = pytest.mark.gpu


def _graph_vs_eager(lw, T, numerics="exact", seed=3):
    t = G.torch()
    wl = lw.wl
    x_bits, _ = cs.tokens_with_margin(oracle.Layer.from_weights(lw), wl, T, seed=seed, stream=T)
    layer = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T, numerics=numerics)
    try:
        x = G.to_device(x_bits)
        y_eager = t.empty((T, wl.hidden), dtype=t.float32, device="cuda")
        y_graph = t.full((T, wl.hidden), float("nan"), dtype=t.float32, device="cuda")
        s = t.cuda.Stream()
        with t.cuda.stream(s):
            layer.forward_ptr(x.data_ptr(), T, y_eager.data_ptr(), s.cuda_stream)
            g = layer.capture_graph(x.data_ptr(), T, y_graph.data_ptr(), s.cuda_stream)
        s.synchronize()
        # capture runs nothing
        assert bool(t.isnan(y_graph).all()), "capture wrote y"
        f0 = layer.stats()["forwards"]
        try:
            g.launch(s.cuda_stream)
            s.synchronize()
            assert np.array_equal(y_graph.cpu().numpy(), y_eager.cpu().numpy()), "graph replay differs from eager"
            y_graph.fill_(float("nan"))
            g.launch(s.cuda_stream)
            s.synchronize()
            assert np.array_equal(y_graph.cpu().numpy(), y_eager.cpu().numpy()), "second replay differs"
            st = layer.stats()
            assert st["forwards"] == f0 + 2 and st["device_error"] == 0
        finally:
            g.close()
    finally:
        layer.close()
    return y_eager


@pytest.mark.parametrize("T", [1, 32])
def test_graph_tensor_core_path(T):
    lw = synth.make_layer(synth.workload("olmoe_like"))
    _graph_vs_eager(lw, T)


def test_graph_register_path_nvfp4():
    wl = synth.custom_workload(hidden=512, inter=256, n_experts=8, top_k=2, shared_inter=128, fmt="nvfp4")
    lw = synth.make_layer(wl, seed=11)
    y = _graph_vs_eager(lw, 4)
    L = oracle.Layer.from_weights(lw)
    x_bits, _ = cs.tokens_with_margin(L, wl, 4, seed=3, stream=4)
    G.check_output(y.cpu().numpy(), L.forward(x_bits)[0])


def test_graph_a4_path():
    lw = synth.make_layer(synth.workload("tiny"))
    _graph_vs_eager(lw, 16, numerics="a4")


def test_graph_refused_when_paged_and_after_table_change():
    F = G.library()
    t = G.torch()
    wl = synth.workload("tiny")
    lw = synth.make_layer(wl)
    T = 4
    x = G.to_device(synth.make_tokens(wl, T))
    y = t.empty((T, wl.hidden), dtype=t.float32, device="cuda")
    s = t.cuda.Stream()
    paged = G.make_layer(lw, n_slots=wl.n_experts // 2, max_tokens=T, n_staging=2)
    try:
        with pytest.raises(F.MoEError) as ei:
            paged.capture_graph(x.data_ptr(), T, y.data_ptr(), s.cuda_stream)
        assert ei.value.status == 1
    finally:
        paged.close()
    layer = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T)
    try:
        g = layer.capture_graph(x.data_ptr(), T, y.data_ptr(), s.cuda_stream)
        try:
            g.launch(s.cuda_stream)
            s.synchronize()
            # any moe_set_slot_table call invalidates the capture, even the same table
            layer.set_slot_table(synth.slot_table(lw, wl.n_experts, policy="all"))
            with pytest.raises(F.MoEError) as ei:
                g.launch(s.cuda_stream)
            assert ei.value.status == 1
        finally:
            g.close()
    finally:
        layer.close()
