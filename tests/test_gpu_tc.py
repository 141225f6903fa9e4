"""EXACT numerics of MXFP4 layers on the tensor core: E2M1 weights (with their
E8M0 block scales) against activations written as two E4M3 pieces with UE8M0
block scales each, tcgen05 kind::mxf8f6f4.

Checks the pieces themselves (x exactly within 13 binades of each block
maximum, h to the two-piece precision against an fp64 SwiGLU of the
dequantised weights), the tile list, and the whole layer against the oracle.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import _cases as cs
from tests import _gpu as G

pytestmark = pytest.mark.gpu

SLOT_ROWS = 128   # activation rows reserved per tile (two pieces per token)


def _sf_offset(nsf, r, c):
    """Byte offset of scale (row r, column c) in 512-byte blocks of 128 rows x 4 columns."""
    return ((r // 128) * (nsf // 4) + c // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + c % 4


def _e4m3_values():
    t = G.torch()
    codes = t.arange(256, dtype=t.uint8).view(t.float8_e4m3fn)
    return codes.to(t.float64).numpy()


def _decode_row(q, sf, row, K, tab):
    nsf = K // 32
    ex = np.array([int(sf[_sf_offset(nsf, row, c)]) for c in range(nsf)], dtype=np.int64)
    assert np.all((ex >= 0) & (ex <= 254)), "scale code outside UE8M0 range"
    return tab[q[row]] * np.repeat(np.ldexp(1.0, ex - 127), 32)


def _tiles(layer):
    n = int(layer.debug_read(17, np.int32, 1)[0])
    t = layer.debug_read(16, np.int32, 4 * n).reshape(n, 4)   # expert, prow0, nrows, sorted0
    return t


def _run_olmoe(T, seed=5):
    wl = synth.workload("olmoe_like")
    lw = synth.make_layer(wl)
    L = oracle.Layer.from_weights(lw)
    x, _ = cs.tokens_with_margin(L, wl, T, seed=seed, stream=T)
    layer = G.make_layer(lw, max_tokens=T)
    y, r = G.run(layer, x)
    return wl, lw, L, x, layer, y, r


def test_tile_list_covers_every_pair_once():
    wl, lw, L, x, layer, y, r = _run_olmoe(32)
    try:
        assert layer.stats()["last_path"] == 2
        tiles = _tiles(layer)
        k = wl.top_k
        counts = np.bincount(r["ids"].ravel(), minlength=wl.n_experts)
        assert tiles[:, 2].sum() == 32 * k
        assert np.all(tiles[:, 2] >= 1) and np.all(tiles[:, 2] <= 8)
        for e in range(wl.n_experts):
            assert tiles[tiles[:, 0] == e, 2].sum() == counts[e]
        prow_pair = layer.debug_read(8, np.int32, int(tiles[:, 1].max() + 16))
        seen = np.concatenate([prow_pair[p0:p0 + n] for _, p0, n, _ in tiles])
        assert np.array_equal(np.sort(seen), np.arange(32 * k))
        for e, p0, n, _ in tiles:
            assert np.all(r["ids"].ravel()[prow_pair[p0:p0 + n]] == e)
    finally:
        layer.close()


@pytest.mark.parametrize("T", [1, 32])
def test_x_pieces_reconstruct_x(T):
    """Exact for every element within 13 binades of its 32-block maximum (the
    remainder of a bf16 value after four bits fits E4M3); below that the second
    piece rounds at its subnormal step, at most 2^-20 of the block maximum."""
    wl, lw, L, x, layer, y, r = _run_olmoe(T)
    try:
        H = wl.hidden
        tiles = _tiles(layer)
        rows = len(tiles) * SLOT_ROWS
        q = layer.debug_read(12, np.uint8, rows * H).reshape(rows, H)
        sf = layer.debug_read(13, np.uint8, rows * H // 32)
        prow_token = layer.debug_read(7, np.int32, int(tiles[:, 1].max() + 16))
        tab = _e4m3_values()
        xf = synth.bf16_bits_to_f32(x).astype(np.float64)
        inexact = total = 0
        for t, (e, p0, n, _) in enumerate(tiles):
            for j in range(n):
                tok = prow_token[p0 + j]
                rec = _decode_row(q, sf, t * SLOT_ROWS + 2 * j, H, tab) + \
                    _decode_row(q, sf, t * SLOT_ROWS + 2 * j + 1, H, tab)
                xv = xf[tok]
                bmax = np.repeat(np.abs(xv).reshape(-1, 32).max(axis=1), 32)
                err = np.abs(rec - xv)
                assert np.all(err <= 2.0 ** -20 * bmax), f"tile {t} token {tok}: piece error above bound"
                wide = np.abs(xv) >= 2.0 ** -13 * bmax
                assert np.array_equal(rec[wide], xv[wide]), f"tile {t} token {tok}: inexact in range"
                inexact += int((err > 0).sum())
                total += err.size
        assert inexact <= 1e-3 * total
    finally:
        layer.close()


def test_h_pieces_match_fp64_swiglu():
    T = 8
    wl, lw, L, x, layer, y, r = _run_olmoe(T)
    try:
        I = wl.inter
        tiles = _tiles(layer)
        rows = len(tiles) * SLOT_ROWS
        q = layer.debug_read(14, np.uint8, rows * I).reshape(rows, I)
        sf = layer.debug_read(15, np.uint8, rows * I // 32)
        prow_token = layer.debug_read(7, np.int32, int(tiles[:, 1].max() + 16))
        tab = _e4m3_values()
        xf = synth.bf16_bits_to_f32(x).astype(np.float64)
        worst = 0.0
        for t, (e, p0, n, _) in enumerate(tiles[:6]):
            wg, wu = L.dequant(0, int(e)), L.dequant(1, int(e))
            for j in range(n):
                tok = prow_token[p0 + j]
                a = wg @ xf[tok]
                u = wu @ xf[tok]
                h = a / (1.0 + np.exp(-a)) * u
                rec = _decode_row(q, sf, t * SLOT_ROWS + 2 * j, I, tab) + \
                    _decode_row(q, sf, t * SLOT_ROWS + 2 * j + 1, I, tab)
                # two E4M3 pieces: |error| <= 2^-8 |h| (+ fp32 accumulation and tiny-value rounding)
                bound = 2.0 ** -8 * np.abs(h) + 1e-5 * np.abs(h).max()
                err = np.abs(rec - h)
                assert np.all(err <= bound), f"tile {t}: h error {err.max()} above the two-piece bound"
                big = np.abs(h) >= 1e-3 * np.abs(h).max()
                worst = max(worst, float((err[big] / np.abs(h[big])).max()))
        assert worst <= 2.0 ** -8 + 1e-6
    finally:
        layer.close()


@pytest.mark.parametrize("T", [1, 8, 32])
def test_tensor_core_path_matches_oracle(T):
    wl, lw, L, x, layer, y, r = _run_olmoe(T, seed=9)
    try:
        y_ref, lg, ids, g = L.forward(x)
        G.check_routing(r, lg, ids, g, wl.n_experts)
        G.check_output(y, y_ref)
        assert layer.stats()["last_path"] == 2
        y2, _ = G.run(layer, x)
        assert np.array_equal(y2, y), "tensor-core path is not deterministic"
    finally:
        layer.close()


@pytest.mark.parametrize("T", [100, 400])
def test_large_tiles_vs_oracle(T):
    """64-token tiles (128 piece rows): several tiles per expert."""
    wl = synth.custom_workload(hidden=512, inter=256, n_experts=8, top_k=2, shared_inter=128)
    lw = synth.make_layer(wl, seed=77)
    L = oracle.Layer.from_weights(lw)
    x, _ = cs.tokens_with_margin(L, wl, T, seed=77, stream=T)
    y_ref, lg, ids, g = L.forward(x)
    layer = G.make_layer(lw, n_slots=wl.n_experts, max_tokens=T)
    try:
        y, r = G.run(layer, x)
        G.check_routing(r, lg, ids, g, wl.n_experts)
        G.check_output(y, y_ref)
        tiles = _tiles(layer)
        assert tiles[:, 2].max() > 8 and tiles[:, 2].max() <= 64
    finally:
        layer.close()
