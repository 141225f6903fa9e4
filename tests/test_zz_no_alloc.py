"""The routing entry point that allocates nothing, checked against moe_forward.

Some callers cannot allocate device memory when they call into the library (a
serving loop that plans all of HBM at start-up, or a path that must not pay the
device-wide synchronisation of cudaMalloc/cudaFree); moe_route_topk_noalloc
serves them from a fixed device scratch array.  This file is collected last so
that a failure here leaves every other test already run; it also passes alone
in a fresh process.
"""
import numpy as np
import pytest

import synth
from tests import _gpu as G

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name, T", [("olmoe_like", 32), ("qwen3_8_flash_next_like", 40)])
def test_noalloc_routing_matches_forward_routing(name, T):
    torch = G.torch()
    F = G.library()
    wl = synth.workload(name)
    if wl.n_experts > 64:   # keep host generation small: the router is what is compared
        wl = synth.custom_workload(wl.hidden, 128, wl.n_experts, wl.top_k, zipf_s=wl.zipf_s)
    lw = synth.make_layer(wl, experts=2)
    layer = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T)
    x_bits = synth.make_tokens(wl, T, stream=5)
    x = G.to_device(x_bits)
    _, ref = layer.forward(x, routing=True)
    torch.cuda.synchronize()
    w = torch.from_numpy(lw.router_w).cuda()
    b = None if lw.router_bias is None else torch.from_numpy(lw.router_bias).cuda()
    for call in range(2):                      # two calls in a row share the scratch
        ids = torch.full((T, wl.top_k), -1, dtype=torch.int32, device="cuda")
        gates = torch.zeros((T, wl.top_k), dtype=torch.float32, device="cuda")
        logits = torch.zeros((T, wl.n_experts), dtype=torch.float32, device="cuda")
        F._lib.route_topk_noalloc(x, w, b, wl.top_k, ids, gates, logits)
        torch.cuda.synchronize()
        assert np.array_equal(ids.cpu().numpy(), ref["ids"].cpu().numpy()), f"call {call}: ids differ"
        dl = float((logits - ref["logits"]).abs().max())
        dg = float((gates - ref["gates"]).abs().max())
        assert dl <= 1e-5, f"call {call}: logits differ by {dl}"
        assert dg <= 2e-6, f"call {call}: gates differ by {dg}"
    layer.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    torch = G.torch()
    F = G.library()
    T, H, E, k = 2048, 256, 1024, 4          # T * E = 2^21 > 2^20 logits
    x = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((E, H), dtype=torch.float32, device="cuda")
    ids = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    gates = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    with pytest.raises(F.MoEError) as ei:
        F._lib.route_topk_noalloc(x, w, None, k, ids, gates)
    assert ei.value.status == 1 and "scratch" in str(ei.value)
