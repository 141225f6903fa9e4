"""GPU-test helpers: build a layer through the C ABI, run it, compare with the oracle."""
from __future__ import annotations

import numpy as np

import oracle
import synth
from tests import _cases as cs


def torch():
    import torch as t
    return t


def library():
    """The built CUDA library; a missing build is an error on a GPU machine, never a skip."""
    import fp4_expert_layer_b200 as F
    from fp4_expert_layer_b200 import build
    build.build(checked=F._lib.SO.endswith("_checked.so"))
    F.lib()
    return F


def make_layer(lw, n_slots=None, max_tokens=1, n_staging=0, table=None, numerics="exact"):
    F = library()
    wl = lw.wl
    S = wl.n_slots if n_slots is None else n_slots
    layer = F.MoELayer.from_weights(lw, n_slots=S, max_tokens=max_tokens, numerics=numerics,
                                    n_staging=n_staging)
    if table is None:
        table = synth.slot_table(lw, S, policy="all" if S >= wl.n_experts else None)
    layer.set_slot_table(table)
    return layer


def to_device(x_bits: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda().view(t.bfloat16)


def run(layer, x_bits):
    t = torch()
    y, r = layer.forward(to_device(x_bits), routing=True)
    t.cuda.synchronize()
    assert layer.stats()["device_error"] == 0, "a device-side wait gave up"
    return y.cpu().numpy(), {k: v.cpu().numpy() for k, v in r.items()}


def check_routing(r, lg, ids, gates, E, rows=None):
    """Bit-exact ids / counts / offsets / perm / inv; logits within 1e-5; gates to fp32 rounding."""
    T = r["ids"].shape[0]
    sel = np.arange(T) if rows is None else np.asarray(rows)
    assert np.array_equal(r["ids"][sel], ids), "expert ids differ from the oracle"
    dl = np.abs(r["logits"][sel].astype(np.float64) - lg.astype(np.float64)).max()
    assert dl <= 1e-5, f"router logits differ by {dl}"
    dg = np.abs(r["gates"][sel].astype(np.float64) - gates.astype(np.float64)).max()
    assert dg <= 2e-6, f"gates differ by {dg}"
    if rows is None:
        counts, offsets, perm, inv = oracle.permute(r["ids"], E)
        assert np.array_equal(r["counts"], counts)
        assert np.array_equal(r["offsets"], offsets)
        assert np.array_equal(r["perm"], perm)
        assert np.array_equal(r["inv"], inv)
    return dl


def check_output(y, ref):
    tol = cs.output_tolerance(ref)
    err = np.abs(y.astype(np.float64) - ref.astype(np.float64))
    worst = float(err.max())
    assert np.all(np.isfinite(y)), "non-finite output"
    assert worst <= tol, f"max |gpu - oracle| = {worst} > {tol}"
    return worst / max(float(np.abs(ref).max()), 1e-30)


def check_routing_invariants(r, T, k, E):
    """Routing tensors that hold at any size (used where the oracle would be too slow)."""
    ids = r["ids"]
    assert ids.min() >= 0 and ids.max() < E
    assert all(len(set(row)) == k for row in ids.tolist())
    lg = r["logits"]
    sel = np.take_along_axis(lg, ids.astype(np.int64), axis=1)
    assert np.all(np.diff(sel, axis=1) <= 0)
    assert np.all(lg.max(axis=1) == sel[:, 0])
    assert np.allclose(r["gates"].sum(axis=1), 1.0, atol=1e-6)
    counts, offsets, perm, inv = oracle.permute(ids, E)
    assert np.array_equal(r["counts"], counts) and np.array_equal(r["offsets"], offsets)
    assert np.array_equal(r["perm"], perm) and np.array_equal(r["inv"], inv)



def tile_list(layer):
    """The last forward's tile list: rows (expert, first padded row, rows, first sorted position)."""
    n = int(layer.debug_read(17, np.int32, 1)[0])
    return layer.debug_read(16, np.int32, 4 * n).reshape(n, 4)


def boundary_rows(layer, r, k, rng=None, extra=0, max_tiles=6):
    """Token rows that exercise the tile scheduler of the last forward: the first
    and last row of every tile of the hottest expert (at most max_tiles of them),
    of the coldest active expert's tile, and of a few ragged tails (tiles
    shorter than the longest tile, the last one of an expert that has several),
    token 0 and the last token, plus `extra` random tokens."""
    tiles = tile_list(layer)
    perm = np.asarray(r["perm"])
    counts = np.asarray(r["counts"])
    T = np.asarray(r["ids"]).shape[0]
    active = np.nonzero(counts > 0)[0]
    hot = int(np.argmax(counts))
    cold = int(active[np.argmin(counts[active])])
    pick = list(np.nonzero(tiles[:, 0] == hot)[0][:max_tiles]) + list(np.nonzero(tiles[:, 0] == cold)[0][:1])
    longest = int(tiles[:, 2].max())
    multi = np.nonzero(np.bincount(tiles[:, 0], minlength=counts.size) > 1)[0]
    tails = [i for i in range(len(tiles)) if tiles[i, 2] < longest and tiles[i, 0] in multi]
    pick += tails[:: max(1, len(tails) // 3)][:3]
    pos = set()
    for i in pick:
        _, _, n, s0 = (int(v) for v in tiles[i])
        pos.update({s0, s0 + n - 1})
    rows = {int(perm[p]) // k for p in pos} | {0, T - 1}
    if extra and rng is not None:
        rows |= set(int(v) for v in rng.integers(0, T, extra))
    return np.array(sorted(rows), dtype=np.int32)
