"""The routing entry point that allocates nothing, checked against the oracle
and against moe_forward's routing.

Some callers cannot allocate device memory when they call into the library (a
serving loop that plans all of HBM at start-up, or a path that must not pay the
device-wide synchronisation of cudaMalloc/cudaFree); moe_route_topk_noalloc
serves them from a fixed device scratch array.  This file is collected last so
that a failure here leaves every other test already run; it also passes alone
in a fresh process.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import _cases as cs
from tests import _gpu as G

pytestmark = pytest.mark.gpu

# (workload, T): full T tiles and ragged ones (T % 4 != 0), E a multiple of 8 and
# not (60: the last expert block has idle warps), H above the 48 KiB default
# shared-memory tile (H = 4096 takes the opt-in attribute path), with and
# without a router bias
CASES = [
    ("olmoe_like", 32),
    ("olmoe_like", 1),
    ("qwen3_8_flash_next_like", 40),
    ("qwen3_8_flash_next_like", 33),
    ("e60_h4096_bias", 33),
    ("e60_h4096_bias", 1),
]


def _workload(name):
    if name == "e60_h4096_bias":
        return synth.custom_workload(4096, 128, 60, 6, zipf_s=1.1)
    wl = synth.workload(name)
    if wl.n_experts > 64:   # keep host generation small: the router is what is compared
        wl = synth.custom_workload(wl.hidden, 128, wl.n_experts, wl.top_k, zipf_s=wl.zipf_s)
    return wl


@pytest.mark.parametrize("name, T", CASES)
def test_noalloc_routing_matches_oracle_and_forward_routing(name, T):
    torch = G.torch()
    F = G.library()
    wl = _workload(name)
    lw = synth.make_layer(wl, experts=2)
    L = oracle.Layer.from_weights(lw)
    x_bits, _ = cs.tokens_with_margin(L, wl, T, stream=5)
    lg_ref, ids_ref, g_ref = L.route_all(x_bits)
    layer = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T)
    x = G.to_device(x_bits)
    _, fwd = layer.forward(x, routing=True)
    torch.cuda.synchronize()
    w = torch.from_numpy(lw.router_w).cuda()
    b = None if lw.router_bias is None else torch.from_numpy(lw.router_bias).cuda()
    for call in range(2):                      # two calls in a row share the scratch
        ids = torch.full((T, wl.top_k), -1, dtype=torch.int32, device="cuda")
        gates = torch.zeros((T, wl.top_k), dtype=torch.float32, device="cuda")
        logits = torch.zeros((T, wl.n_experts), dtype=torch.float32, device="cuda")
        F._lib.route_topk_noalloc(x, w, b, wl.top_k, ids, gates, logits)
        torch.cuda.synchronize()
        r = {"ids": ids.cpu().numpy(), "logits": logits.cpu().numpy(), "gates": gates.cpu().numpy()}
        # the oracle: ids bit-exact, logits within 1e-5, gates to fp32 rounding
        assert np.array_equal(r["ids"], ids_ref), f"call {call}: ids differ from the oracle"
        dl = float(np.abs(r["logits"].astype(np.float64) - lg_ref).max())
        dg = float(np.abs(r["gates"].astype(np.float64) - g_ref).max())
        assert dl <= 1e-5, f"call {call}: logits differ from the oracle by {dl}"
        assert dg <= 2e-6, f"call {call}: gates differ from the oracle by {dg}"
        # and moe_forward's own routing of the same tokens
        assert np.array_equal(r["ids"], fwd["ids"].cpu().numpy()), f"call {call}: ids differ from moe_forward"
        assert float(np.abs(r["gates"] - fwd["gates"].cpu().numpy()).max()) <= 2e-6
    layer.close()


def test_noalloc_rejects_misaligned_router_weights():
    torch = G.torch()
    F = G.library()
    T, H, E, k = 4, 256, 8, 2
    x = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    wbuf = torch.zeros((E * H + 1,), dtype=torch.float32, device="cuda")
    w = wbuf[1:].view(E, H)                   # an offset view: 4 bytes past a 16-byte boundary
    ids = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    gates = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    with pytest.raises(F.MoEError) as ei:
        F._lib.route_topk_noalloc(x, w, None, k, ids, gates)
    assert ei.value.status == 1 and "aligned" in str(ei.value)


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
