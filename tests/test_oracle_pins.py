"""Pins of the CPU oracle against things other than itself.

Each test checks one oracle function against a hand-written fixture, a library
routine, a closed form, brute force on tiny inputs, or an invariant, so that a
plausible slip (wrong nibble, wrong bias, dropped bias term, transposed
operand, wrong tie rule) fails at least one of them.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import _cases as cs


# ----------------------------------------------------------------- formats
def test_e2m1_matches_fixture_table():
    tab = cs.e2m1_table()
    got = np.array([oracle.e2m1(c) for c in range(16)])
    assert np.array_equal(got, tab)
    assert np.array_equal(np.signbit(got), np.signbit(tab))


def test_e8m0_bf16_exponent_field_fixture():
    for code, bits, value, admitted in cs.read_golden("e8m0_bf16_field.txt"):
        code = int(code)
        bits = int(bits, 16)
        assert bits == code << 7
        f = synth.bf16_bits_to_f32(np.array([bits], dtype=np.uint16))[0]
        assert float(f) == float(value)
        ok = oracle.admit_scales("mxfp4", np.array([code], dtype=np.uint8)) < 0
        assert ok == (admitted == "yes")
        if ok:
            assert oracle.e8m0(code) == float(value)


def test_e8m0_all_codes_vs_ldexp():
    for c in range(1, 255):
        assert oracle.e8m0(c) == np.ldexp(1.0, c - 127)
    bad = oracle.admit_scales("mxfp4", np.array([5, 0, 7, 255], dtype=np.uint8))
    assert bad == 1


def test_e4m3_all_codes_vs_torch():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # admission: NaN and negative block scales rejected, zero allowed
    assert oracle.admit_scales("nvfp4", np.array([0, 0x38, 0x7E], dtype=np.uint8)) < 0
    assert oracle.admit_scales("nvfp4", np.array([0x38, 0x7F], dtype=np.uint8)) == 1
    assert oracle.admit_scales("nvfp4", np.array([0x38, 0xB8], dtype=np.uint8)) == 1


def _one_row_layer(fmt, codes, scales, gscale=1.0):
    K = codes.size * 2
    z = np.zeros((1, 1, K // 2), dtype=np.uint8)
    G = 32 if fmt == "mxfp4" else 16
    c = [np.zeros((1, K, K // 2), np.uint8), np.zeros((1, K, K // 2), np.uint8),
         np.zeros((1, K, K // 2), np.uint8)]
    s = [np.full((1, K, K // G), 127 if fmt == "mxfp4" else 0x38, np.uint8) for _ in range(3)]
    c[0][0, 0] = codes
    s[0][0, 0] = scales
    gl = np.full((1, 3), gscale, np.float32) if fmt == "nvfp4" else None
    del z
    return oracle.Layer(K, K, 1, 1, fmt, np.zeros((1, K), np.float32), None, c, s, gl)


def test_mxfp4_block_fixture():
    rows = {r[0]: r[1:] for r in cs.read_golden("mxfp4_block.txt")}
    codes = np.array([int(b, 16) for b in rows["bytes"]], dtype=np.uint8)
    want = np.array([float(v) for v in rows["values"]])
    L = _one_row_layer("mxfp4", codes, np.array([int(rows["scale"][0])], np.uint8))
    got = L.dequant(0, 0)[0]
    assert np.array_equal(got, want) and np.array_equal(np.signbit(got), np.signbit(want))


def test_nvfp4_block_fixture():
    rows = {r[0]: r[1:] for r in cs.read_golden("nvfp4_block.txt")}
    codes = np.array([int(b, 16) for b in rows["bytes"]], dtype=np.uint8)
    sc = np.array([int(b, 16) for b in rows["scales"]], dtype=np.uint8)
    want = np.array([float(v) for v in rows["values"]])
    L = _one_row_layer("nvfp4", codes, sc, float(rows["tensor"][0]))
    got = L.dequant(0, 0)[0]
    assert np.array_equal(got, want)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_dequant_matches_numpy_decode(fmt):
    wl = synth.custom_workload(128, 64, 3, 2, fmt=fmt)
    lw = synth.make_layer(wl, seed=7)
    L = oracle.Layer.from_weights(lw)
    for m in range(3):
        for e in range(3):
            gs = 1.0 if lw.global_scale is None else float(lw.global_scale[e, m])
            ref = cs.np_decode(lw.codes[m][e], lw.scales[m][e], fmt, gs)
            assert np.array_equal(L.dequant(m, e), ref)


# ----------------------------------------------------------------- routing
def test_router_logits_vs_numpy_matmul():
    wl = synth.custom_workload(256, 64, 16, 4, zipf_s=1.1)
    lw = synth.make_layer(wl, seed=3)
    L = oracle.Layer.from_weights(lw)
    x = synth.make_tokens(wl, 37, seed=3)
    lg, _, _ = L.route_all(x)
    ref = (synth.bf16_bits_to_f32(x).astype(np.float64) @ lw.router_w.astype(np.float64).T
           + lw.router_bias.astype(np.float64))
    # both round an fp64 sum to fp32: at most one fp32 ulp apart (summation order)
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(lg.astype(np.float64) - ref) <= ulp)


def test_route_vs_argsort_and_full_softmax():
    rng = np.random.default_rng(11)
    E, k = 40, 7
    for _ in range(200):
        l = rng.standard_normal(E).astype(np.float32)
        ids, g = oracle.route_row(l, k)
        ref_ids = np.argsort(-l, kind="stable")[:k]
        assert np.array_equal(ids, ref_ids)
        p = np.exp(l.astype(np.float64) - l.max())
        p /= p.sum()
        ref_g = p[ref_ids] / p[ref_ids].sum()
        assert np.allclose(g, ref_g, rtol=2e-7, atol=0)
        assert abs(float(g.astype(np.float64).sum()) - 1.0) <= 4 * np.finfo(np.float32).eps


@pytest.mark.parametrize("scoring, renorm", [("softmax", False), ("sigmoid", True), ("sigmoid", False)])
def test_route_variants_vs_numpy(scoring, renorm):
    """Selection is by logit (both scorings are monotone); scores are the full
    softmax over all targets or the elementwise logistic; gates are the chosen
    scores, renormalised over the k when asked."""
    rng = np.random.default_rng(12)
    n, k = 40, 6
    for _ in range(200):
        l = (3 * rng.standard_normal(n)).astype(np.float32)
        ids, g = oracle.route_row(l, k, scoring, renorm)
        ref_ids = np.argsort(-l, kind="stable")[:k]
        assert np.array_equal(ids, ref_ids)
        l64 = l.astype(np.float64)
        if scoring == "softmax":
            p = np.exp(l64 - l64.max())
            p /= p.sum()
        else:
            p = 1.0 / (1.0 + np.exp(-l64))
        sel = p[ref_ids]
        ref_g = sel / sel.sum() if renorm else sel
        assert np.allclose(g, ref_g, rtol=2e-7, atol=0)
        if renorm:
            assert abs(float(g.astype(np.float64).sum()) - 1.0) <= 4 * np.finfo(np.float32).eps
        elif scoring == "softmax":
            assert float(g.astype(np.float64).sum()) < 1.0 + 1e-6


def test_sigmoid_gate_closed_form():
    """logistic(0) = 1/2 and logistic(ln 3) = 3/4 exactly representable."""
    ids, g = oracle.route_row(np.array([0.0, np.log(3.0), -50.0], np.float32), 2, "sigmoid", False)
    assert ids.tolist() == [1, 0]
    assert g[1] == np.float32(0.5) and abs(float(g[0]) - 0.75) <= 1e-7


def test_sink_choice_contributes_nothing():
    """A layer whose sink target always wins (a large bias) equals the same
    layer without the sink with its remaining k - 1 experts' gates scaled by
    their share: y = sum over chosen experts only; the sink's gate is lost."""
    wl = synth.custom_workload(64, 32, 4, 3, n_sinks=1)
    lw = synth.make_layer(wl, seed=21)
    lw.router_bias = np.zeros(5, np.float32)
    lw.router_bias[4] = 100.0                       # the sink is always chosen first
    L = oracle.Layer.from_weights(lw)
    x = synth.make_tokens(wl, 4, seed=21)
    y, lg, ids, g = L.forward(x)
    assert np.all(ids[:, 0] == 4)
    assert np.all(g[:, 0] > 0.999)                  # nearly all mass on the sink
    ry, _, rids, _ = cs.dense_layer(lw, x)
    assert np.array_equal(ids, rids)
    assert np.allclose(y, ry, rtol=1e-6, atol=1e-6 * np.abs(ry).max())
    assert np.abs(y).max() < 1e-2 * np.abs(cs.dense_layer(
        synth.make_layer(synth.custom_workload(64, 32, 4, 2), seed=21), x)[0]).max()


def test_int4_matches_fixture_table():
    tab = cs.int4_table()
    assert [oracle.int4(c) for c in range(16)] == tab.tolist()


def test_int4g128_row_hand_built():
    """One row of 256 weights: group 0 scale 2^-3, group 1 scale 1.5 (bf16
    0x3FC0); codes 7 and 8 (= -8) at the group edges."""
    wl = synth.custom_workload(256, 128, 1, 1, fmt="int4g128")
    lw = synth.make_layer(wl, seed=1)
    lw.codes[0][0, 0, :] = 0
    lw.codes[0][0, 0, 0] = 0x87          # element 0 -> 7, element 1 -> -8
    lw.codes[0][0, 0, 63] = 0x10         # element 126 -> 0, element 127 -> 1
    lw.codes[0][0, 0, 64] = 0x0F         # element 128 -> -1, element 129 -> 0
    lw.scales[0][0, 0, :] = [0x3E00, 0x3FC0]   # bf16 0.125, 1.5
    L = oracle.Layer.from_weights(lw)
    row = L.dequant(0, 0)[0]
    want = np.zeros(256)
    want[0], want[1], want[127], want[128] = 7 * 0.125, -8 * 0.125, 0.125, -1.5
    assert np.array_equal(row, want)


def test_fp8b128_blocks_hand_built():
    """Down matrix [256, 128]: rows 0..127 use block scale 0.5, rows 128..255
    scale 3.0; E4M3 codes 0x38 (1.0), 0xC0 (-2.0), 0x7E (448)."""
    wl = synth.custom_workload(256, 128, 1, 1, fmt="fp8b128")
    lw = synth.make_layer(wl, seed=1)
    lw.codes[2][0] = 0
    lw.codes[2][0, 0, 0] = 0x38
    lw.codes[2][0, 127, 5] = 0xC0
    lw.codes[2][0, 128, 127] = 0x7E
    lw.scales[2][0] = np.array([[0.5], [3.0]], np.float32)
    W = oracle.Layer.from_weights(lw).dequant(2, 0)
    want = np.zeros((256, 128))
    want[0, 0], want[127, 5], want[128, 127] = 0.5, -1.0, 1344.0
    assert np.array_equal(W, want)


@pytest.mark.parametrize("fmt", ["int4g128", "fp8b128"])
def test_other_formats_dequant_matches_numpy(fmt):
    wl = synth.custom_workload(256, 128, 2, 1, fmt=fmt)
    lw = synth.make_layer(wl, seed=6)
    L = oracle.Layer.from_weights(lw)
    for m in range(3):
        for e in range(2):
            ref = cs.np_decode(lw.codes[m][e], lw.scales[m][e], fmt)
            assert np.array_equal(L.dequant(m, e), ref)


def test_other_formats_admission():
    s = np.array([0x3F80, 0x7F80, 0x0000, 0xFFC1], np.uint16)        # 1.0, +inf, 0, NaN
    assert oracle.admit_scales("int4g128", s) == 1
    assert oracle.admit_scales("int4g128", s[[0, 2]]) == -1          # a zero bf16 scale is admitted
    f = np.array([1.0, 2.0 ** -20, 0.0, -1.0], np.float32)
    assert oracle.admit_scales("fp8b128", f) == 2
    assert oracle.admit_scales("fp8b128", f[:2]) == -1
    assert oracle.admit_scales("fp8b128", np.array([np.inf], np.float32)) == 0
    assert oracle.admit_fp8_codes(np.array([0x00, 0x7E, 0xFE, 0xFF], np.uint8)) == 3
    assert oracle.admit_fp8_codes(np.array([0x7F], np.uint8)) == 0


def test_route_tie_goes_to_lower_index():
    l = np.array([0.5, 2.0, 1.0, 2.0, 1.0, -3.0], dtype=np.float32)
    ids, g = oracle.route_row(l, 4)
    assert ids.tolist() == [1, 3, 2, 4]
    assert g[0] == g[1] and g[2] == g[3]


def test_permute_vs_stable_argsort():
    rng = np.random.default_rng(5)
    for T, k, E in [(1, 2, 8), (16, 2, 8), (33, 8, 64), (500, 6, 256)]:
        ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
        counts, offsets, perm, inv = oracle.permute(ids, E)
        flat = ids.reshape(-1)
        assert np.array_equal(counts, np.bincount(flat, minlength=E))
        assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
        assert offsets[-1] == T * k
        assert np.array_equal(perm, np.argsort(flat, kind="stable"))
        assert np.array_equal(inv[perm], np.arange(T * k))
        assert np.all(np.diff(flat[perm]) >= 0)


# ----------------------------------------------------------------- expert FFN / layer
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_single_expert_is_dense_swiglu(fmt):
    wl = synth.custom_workload(128, 64, 1, 1, fmt=fmt)
    lw = synth.make_layer(wl, seed=21)
    L = oracle.Layer.from_weights(lw)
    x = synth.make_tokens(wl, 5, seed=21)
    y, _, ids, g = L.forward(x)
    assert np.all(ids == 0) and np.all(g == 1.0)
    gs = (1, 1, 1) if lw.global_scale is None else lw.global_scale[0]
    Wg = cs.np_decode(lw.codes[0][0], lw.scales[0][0], fmt, float(gs[0]))
    Wu = cs.np_decode(lw.codes[1][0], lw.scales[1][0], fmt, float(gs[1]))
    Wd = cs.np_decode(lw.codes[2][0], lw.scales[2][0], fmt, float(gs[2]))
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    a = (xf @ Wg.T).astype(np.float32).astype(np.float64)
    u = (xf @ Wu.T).astype(np.float32).astype(np.float64)
    h = (cs.np_silu(a) * u).astype(np.float32).astype(np.float64)
    ref = h @ Wd.T
    assert np.allclose(y, ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())


@pytest.mark.parametrize("shape", [
    dict(hidden=64, inter=32, n_experts=4, top_k=2),
    dict(hidden=64, inter=32, n_experts=4, top_k=2, fmt="nvfp4"),
    dict(hidden=64, inter=32, n_experts=5, top_k=3, shared_inter=32),
    dict(hidden=128, inter=64, n_experts=6, top_k=2, zipf_s=1.1),
    # router variants: sigmoid scoring, no renormalisation, sink targets,
    # sigmoid-gated shared expert
    dict(hidden=64, inter=32, n_experts=6, top_k=2, scoring="sigmoid"),
    dict(hidden=64, inter=32, n_experts=6, top_k=3, renormalize=False),
    dict(hidden=64, inter=32, n_experts=4, top_k=3, n_sinks=2),
    dict(hidden=128, inter=64, n_experts=5, top_k=3, shared_inter=32, shared_gate=True, n_sinks=2,
         scoring="sigmoid", renormalize=False, zipf_s=1.1, fmt="nvfp4"),
    # other expert formats: INT4 group-128 (bf16 scales), FP8 E4M3 block-128 (fp32 scales)
    dict(hidden=256, inter=128, n_experts=4, top_k=2, fmt="int4g128"),
    dict(hidden=256, inter=128, n_experts=4, top_k=2, fmt="fp8b128", shared_inter=128),
])
def test_bruteforce_dense_tiny(shape):
    wl = synth.custom_workload(**shape)
    lw = synth.make_layer(wl, seed=13)
    L = oracle.Layer.from_weights(lw)
    x, _ = cs.tokens_with_margin(L, wl, 3, seed=13)
    y, lg, ids, g = L.forward(x)
    ry, rlg, rids, rg = cs.dense_layer(lw, x)
    assert np.array_equal(ids, rids)
    ulp = np.spacing(np.abs(rlg)).astype(np.float64)
    assert np.all(np.abs(lg.astype(np.float64) - rlg) <= ulp)
    assert np.allclose(g, rg, rtol=4e-7, atol=0)
    assert np.allclose(y, ry, rtol=1e-6, atol=1e-6 * np.abs(ry).max())


def test_bruteforce_dense_tiny_workload():
    wl = synth.workload("tiny")
    lw = synth.make_layer(wl)
    L = oracle.Layer.from_weights(lw)
    x, _ = cs.tokens_with_margin(L, wl, 16)
    y, lg, ids, g = L.forward(x)
    ry, rlg, rids, rg = cs.dense_layer(lw, x)
    assert np.array_equal(ids, rids)
    assert np.allclose(y, ry, rtol=1e-6, atol=1e-6 * np.abs(ry).max())
    assert np.allclose(g.sum(axis=1), 1.0, atol=4 * np.finfo(np.float32).eps)


def test_token_permutation_equivariance_and_subset():
    wl = synth.custom_workload(128, 64, 8, 3, shared_inter=64)
    lw = synth.make_layer(wl, seed=2)
    L = oracle.Layer.from_weights(lw)
    x = synth.make_tokens(wl, 9, seed=2)
    y, lg, ids, g = L.forward(x)
    pi = np.random.default_rng(0).permutation(9)
    y2, lg2, ids2, g2 = L.forward(x[pi])
    assert np.array_equal(y2, y[pi]) and np.array_equal(ids2, ids[pi]) and np.array_equal(g2, g[pi])
    rows = np.array([4, 0, 8], dtype=np.int32)
    y3, _, ids3, _ = L.forward(x, rows=rows)
    assert np.array_equal(y3, y[rows]) and np.array_equal(ids3, ids[rows])


def test_output_is_linear_in_down_projection_sign():
    """Flipping the sign bit of every down-projection code negates the routed output."""
    wl = synth.custom_workload(64, 32, 4, 2)
    lw = synth.make_layer(wl, seed=4)
    x = synth.make_tokens(wl, 4, seed=4)
    y, *_ = oracle.Layer.from_weights(lw).forward(x)
    lw.codes[2] = lw.codes[2] ^ np.uint8(0x88)
    y2, *_ = oracle.Layer.from_weights(lw).forward(x)
    assert np.array_equal(y2, -y)


# ----------------------------------------------------------------- A4 quantisers
def test_rne_e2m1_properties():
    tab = cs.e2m1_table()
    mags = tab[:8]
    # exact values map to themselves
    for c in range(16):
        if c == 8:
            continue
        assert oracle.rne_e2m1(float(tab[c])) == c
    # ties go to the even mantissa bit (codes 0, 2, 4, 6 are even)
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in ties.items():
        assert tab[oracle.rne_e2m1(v)] == want
        assert tab[oracle.rne_e2m1(-v)] == -want
    # saturation
    assert tab[oracle.rne_e2m1(7.0)] == 6.0 and tab[oracle.rne_e2m1(1e30)] == 6.0
    assert tab[oracle.rne_e2m1(-100.0)] == -6.0
    # nearest: no representable value is strictly closer
    rng = np.random.default_rng(1)
    for v in rng.uniform(-7, 7, 2000).astype(np.float32):
        q = tab[oracle.rne_e2m1(float(v))]
        d = abs(abs(float(v)) - np.abs(mags))
        assert abs(abs(float(v)) - abs(q)) <= d.min() + 0.0
        assert np.sign(q) in (0.0, np.sign(v))


def test_rn_e4m3_vs_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.uniform(0, 448, 3000), np.exp(rng.uniform(-14, 6, 3000)),
                        [0.0, 448.0, 2.0 ** -9, 1.0625, 1.1875, 0.0009765625 * 1.5]]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.rn_e4m3(float(t)) for t in v], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_quant_mx_block_hand_built():
    tab = cs.e2m1_table()
    for n in (-3, 0, 5):
        v = np.zeros(32, np.float32)
        v[3] = 6.0 * 2.0 ** n
        v[7] = -1.5 * 2.0 ** n
        codes, sc = oracle.quant_mx_block(v)
        assert sc == 127 + n
        deq = tab[codes] * 2.0 ** (sc - 127)
        assert np.array_equal(deq, v.astype(np.float64))
        v2 = v.copy()
        v2[3] = 8.0 * 2.0 ** n          # amax 8*2^n: exponent n+1, 8 -> 4
        codes, sc = oracle.quant_mx_block(v2)
        assert sc == 128 + n and tab[codes[3]] == 4.0
        v3 = v.copy()
        v3[3] = 7.0 * 2.0 ** n          # amax 7*2^n: exponent n, 7 saturates to 6
        codes, sc = oracle.quant_mx_block(v3)
        assert sc == 127 + n and tab[codes[3]] == 6.0
    codes, sc = oracle.quant_mx_block(np.zeros(32, np.float32))
    assert sc == 1 and np.all(tab[codes] == 0)


def test_quant_nv_row_hand_built():
    tab = cs.e2m1_table()
    v = np.zeros(32, np.float32)
    v[0] = 2688.0            # amax = 6*448: G = 1, scale 448
    v[16] = 3.0              # block 1: scale RN(0.5) = 0.5, code 6
    codes, sc, G = oracle.quant_nv_row(v)
    assert G == 1.0
    assert oracle.e4m3(int(sc[0])) == 448.0 and tab[codes[0]] == 6.0
    assert oracle.e4m3(int(sc[1])) == 0.5 and tab[codes[16]] == 6.0
    codes, sc, G = oracle.quant_nv_row(v * np.float32(4.0))
    assert G == 4.0
    codes, sc, G = oracle.quant_nv_row(v * np.float32(1.001))
    assert G == 2.0
    codes, sc, G = oracle.quant_nv_row(np.zeros(32, np.float32))
    assert G == 1.0 and np.all(sc == 0) and np.all(codes == 0)


def test_a4_mode_single_expert_matches_quantised_dense():
    wl = synth.custom_workload(128, 64, 1, 1)
    lw = synth.make_layer(wl, seed=8)
    L = oracle.Layer.from_weights(lw, numerics="a4")
    x = synth.make_tokens(wl, 3, seed=8)
    y, *_ = L.forward(x)
    tab = cs.e2m1_table()

    def qdq(row):
        out = np.empty(row.size)
        for b in range(row.size // 32):
            c, s = oracle.quant_mx_block(row[b * 32:(b + 1) * 32].astype(np.float32))
            out[b * 32:(b + 1) * 32] = tab[c] * 2.0 ** (s - 127)
        return out

    Wg = cs.np_decode(lw.codes[0][0], lw.scales[0][0], "mxfp4")
    Wu = cs.np_decode(lw.codes[1][0], lw.scales[1][0], "mxfp4")
    Wd = cs.np_decode(lw.codes[2][0], lw.scales[2][0], "mxfp4")
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(3):
        xq = qdq(xf[t])
        a = np.float32(Wg @ xq).astype(np.float64)
        u = np.float32(Wu @ xq).astype(np.float64)
        h = (cs.np_silu(a) * u).astype(np.float32)
        ref = Wd @ qdq(h)
        assert np.allclose(y[t], ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())


def _np_e4m3(codes):
    import torch
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn) \
        .to(torch.float64).numpy()


def test_a4_qdq_row_nvfp4_hand_built():
    """NVFP4 activation rule on a hand-worked row: per-row G != 1, two different
    block scales, a tie broken to the even code.  Worked by hand:
      amax_row = 168 -> G = 2^ceil(log2(168 / 2688)) = 2^-4;
      block 0: amax 168 -> scale RN_E4M3(168/6/G) = 448; 168 -> code 6, 14 -> 0.5;
      block 1: amax 3 -> scale RN_E4M3(3/6/G) = 8; 3 -> 6, 1 -> 2, 1.25 -> 2.5,
               a tie between 2 and 3 broken to the even code 2."""
    v = np.zeros(32, np.float32)
    v[0], v[1], v[16], v[17], v[18] = 168.0, 14.0, 3.0, 1.0, 1.25
    codes, sc, G = oracle.quant_nv_row(v)
    assert G == 2.0 ** -4
    assert oracle.e4m3(int(sc[0])) == 448.0 and oracle.e4m3(int(sc[1])) == 8.0
    out = oracle.a4_qdq_row("nvfp4", v)
    want = np.zeros(32)
    want[0], want[1], want[16], want[17], want[18] = 168.0, 14.0, 3.0, 1.0, 1.0
    assert np.array_equal(out, want)


def test_a4_qdq_row_mxfp4_hand_built():
    """MXFP4 activation rule on a hand-worked row of two 32-blocks with
    different shared exponents: block 0 amax 6 -> 2^0 (codes exact: 6, 0.5);
    block 1 amax 0.75 -> 2^(floor(log2 .75) - 2) = 2^-3: 0.75 -> 6 * 2^-3,
    0.3 -> 2.4 -> 2 -> 0.25."""
    v = np.zeros(64, np.float32)
    v[0], v[1], v[32], v[33] = 6.0, 0.5, 0.75, 0.3
    out = oracle.a4_qdq_row("mxfp4", v)
    want = np.zeros(64)
    want[0], want[1], want[32], want[33] = 6.0, 0.5, 0.75, 0.25
    assert np.array_equal(out, want)


def test_a4_qdq_row_nvfp4_recomposes_from_its_pieces():
    """The recomposition e2m1(code) * e4m3(scale[i // 16]) * G, written with numpy
    from the pieces quant_nv_row returns, on rows whose 16-blocks all differ."""
    tab = cs.e2m1_table()
    rng = np.random.default_rng(12)
    for K in (64, 256):
        v = (rng.standard_normal(K) * np.repeat(2.0 ** rng.integers(-6, 6, K // 16), 16)).astype(np.float32)
        codes, sc, G = oracle.quant_nv_row(v)
        assert G != 1.0 and len(set(sc.tolist())) > 1
        ref = tab[codes] * np.repeat(_np_e4m3(sc), 16) * G
        assert np.array_equal(oracle.a4_qdq_row("nvfp4", v), ref)


def test_a4_mode_single_expert_matches_quantised_dense_nvfp4():
    """E = k = 1 NVFP4 layer in A4 numerics against numpy: x and h quantised by the
    NVFP4 activation rule (codes, per-16 E4M3 scales and per-row G from
    quant_nv_row, recomposed here as e2m1 * e4m3(scale[i // 16]) * G), weights
    decoded independently (e2m1 * e4m3 * per-tensor scale)."""
    wl = synth.custom_workload(128, 64, 1, 1, fmt="nvfp4")
    lw = synth.make_layer(wl, seed=8)
    L = oracle.Layer.from_weights(lw, numerics="a4")
    x = synth.make_tokens(wl, 3, seed=8)
    y, *_ = L.forward(x)
    tab = cs.e2m1_table()

    def qdq(row):
        codes, sc, G = oracle.quant_nv_row(np.asarray(row, np.float32))
        assert G != 1.0
        return tab[codes] * np.repeat(_np_e4m3(sc), 16) * G

    gs = lw.global_scale[0].astype(np.float64)
    Wg = cs.np_decode(lw.codes[0][0], lw.scales[0][0], "nvfp4", gs[0])
    Wu = cs.np_decode(lw.codes[1][0], lw.scales[1][0], "nvfp4", gs[1])
    Wd = cs.np_decode(lw.codes[2][0], lw.scales[2][0], "nvfp4", gs[2])
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(3):
        xq = qdq(xf[t])
        a = np.float32(Wg @ xq).astype(np.float64)
        u = np.float32(Wu @ xq).astype(np.float64)
        h = (cs.np_silu(a) * u).astype(np.float32)
        ref = Wd @ qdq(h)
        assert np.allclose(y[t], ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())


def test_expert_rows_sample_sums_to_full_expert():
    """The benchmark's row-range timing sample adds up to the full expert output."""
    wl = synth.custom_workload(128, 64, 3, 1)
    lw = synth.make_layer(wl, seed=6)
    L = oracle.Layer.from_weights(lw)
    x = synth.make_tokens(wl, 1, seed=6)
    y, _, ids, g = L.forward(x)
    o = np.zeros(128)
    for i0 in range(0, 64, 16):
        L.expert_rows(int(ids[0, 0]), x[0], i0, 16, o)
    assert np.allclose(o.astype(np.float32), y[0], rtol=1e-6, atol=1e-6 * np.abs(y).max())
