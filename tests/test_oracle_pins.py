"""Pins of the fp64 oracle against facts other than its own code.

Each test checks one oracle stage against a closed form, an invariant, a
special case that reduces to a textbook or library routine, brute force on a
tiny input, or a number the workload definition states -- chosen so that a
dropped term, a wrong sign or index or a transposed operand fails a test.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import svg_workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny(**kw):
    return W.small_workload(**kw)


def bits(x):
    return W.to_bf16_bits(np.asarray(x, np.float32))


def f32(h):
    return W.bf16_bits_to_f32(h).astype(np.float64)


# ------------------------------------------------------------------ bf16 ----

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 20000).astype(np.float32),
        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 2 ** -130, 3 * 2 ** -134, 2 ** -149,
                  3.3e38, 3.4e38, 0.0, -0.0], np.float32),
    ])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f64_to_bf16(x.astype(np.float64))
    assert np.array_equal(got, ref)


# -------------------------------------------------------------- RMSNorm ----

def _norm_rows(wl, x, gamma, rows, eps=None):
    sh = oracle.shape_of(wl)
    pr = oracle.params_of(wl)
    if eps is not None:
        pr.eps = eps
    return oracle.qknorm_rope_f64(sh, pr, x, gamma, rows)


def test_rmsnorm_closed_form_on_text_rows():
    wl = tiny(T=5)
    inp = W.make_inputs(wl)
    text_rows = np.array([wl.Lv + i for i in range(wl.T)], np.int64)
    y = _norm_rows(wl, inp["q"], np.ones(wl.d, np.float32), text_rows, eps=0.0)
    # gamma = 1, eps = 0: every normalised row has mean square exactly 1
    np.testing.assert_allclose((y ** 2).mean(1), 1.0, rtol=1e-13)
    # and is the input divided by its root mean square
    x = f32(inp["q"].reshape(-1, wl.d)[text_rows])
    np.testing.assert_allclose(y, x / np.sqrt((x ** 2).mean(1, keepdims=True)), rtol=1e-13)


def test_rmsnorm_scale_invariance_and_gamma():
    wl = tiny(T=3)
    inp = W.make_inputs(wl)
    rows = np.arange(wl.Lv, wl.L, dtype=np.int64)
    g = inp["gamma_q"]
    y1 = _norm_rows(wl, inp["q"], g, rows, eps=0.0)
    q2 = bits(f32(inp["q"]) * 4.0)           # power of two: exact in bf16
    y2 = _norm_rows(wl, q2, g, rows, eps=0.0)
    np.testing.assert_allclose(y1, y2, rtol=1e-13)
    y_unit = _norm_rows(wl, inp["q"], np.ones(wl.d, np.float32), rows, eps=0.0)
    np.testing.assert_allclose(y1, y_unit * g.astype(np.float64), rtol=1e-13)
    # eps enters under the square root: huge eps shrinks the row by sqrt(eps)
    y_eps = _norm_rows(wl, inp["q"], np.ones(wl.d, np.float32), rows, eps=1e6)
    x = f32(inp["q"].reshape(-1, wl.d)[rows])
    np.testing.assert_allclose(y_eps, x / np.sqrt((x ** 2).mean(1, keepdims=True) + 1e6), rtol=1e-13)


# ----------------------------------------------------------------- RoPE ----

def _rope_complex(wl, xn, f, yy, xx):
    """RoPE as complex multiplication (RoFormer): pair (2j, 2j+1) of section a
    is the complex number u + iv, multiplied by exp(i * p_a * base^(-2j/n_a))."""
    out = xn.copy()
    off = 0
    for n, p in zip(wl.rope_split, (f, yy, xx)):
        z = xn[off:off + n:2] + 1j * xn[off + 1:off + n:2]
        freq = wl.rope_base ** (-np.arange(0, n, 2) / n)
        z = z * np.exp(1j * p * freq)
        out[off:off + n:2] = z.real
        out[off + 1:off + n:2] = z.imag
        off += n
    return out


@pytest.mark.parametrize("d,split", [(64, (16, 24, 24)), (128, (32, 48, 48)), (32, (8, 12, 12))])
def test_rope_equals_complex_rotation(d, split):
    wl = tiny(d=d, rope_split=split, F=5, Hs=3, Ws=7, T=2)
    inp = W.make_inputs(wl)
    rng = np.random.default_rng(1)
    toks = rng.choice(wl.Lv, 30, replace=False)
    y = _norm_rows(wl, inp["k"], inp["gamma_k"], toks.astype(np.int64))
    x = f32(inp["k"].reshape(-1, d)[toks])
    xn = x / np.sqrt((x ** 2).mean(1, keepdims=True) + wl.eps) * inp["gamma_k"].astype(np.float64)
    for i, t in enumerate(toks):
        f, s = divmod(int(t), wl.S)
        ref = _rope_complex(wl, xn[i], f, s // wl.Ws, s % wl.Ws)
        np.testing.assert_allclose(y[i], ref, rtol=0, atol=1e-12)


def test_rope_identity_at_origin_and_text_rows_untouched():
    wl = tiny(T=4)
    inp = W.make_inputs(wl)
    rows = np.array([0] + list(range(wl.Lv, wl.L)), np.int64)   # token 0 is (f, y, x) = (0, 0, 0)
    y = _norm_rows(wl, inp["q"], inp["gamma_q"], rows)
    x = f32(inp["q"].reshape(-1, wl.d)[rows])
    ref = x / np.sqrt((x ** 2).mean(1, keepdims=True) + wl.eps) * inp["gamma_q"].astype(np.float64)
    np.testing.assert_allclose(y, ref, rtol=1e-13)


def test_rope_pair_norms_preserved():
    wl = tiny(F=6)
    inp = W.make_inputs(wl)
    toks = np.arange(wl.Lv, dtype=np.int64)
    y = _norm_rows(wl, inp["q"], inp["gamma_q"], toks)
    x = f32(inp["q"].reshape(-1, wl.d)[toks])
    xn = x / np.sqrt((x ** 2).mean(1, keepdims=True) + wl.eps) * inp["gamma_q"].astype(np.float64)
    np.testing.assert_allclose(y[:, 0::2] ** 2 + y[:, 1::2] ** 2, xn[:, 0::2] ** 2 + xn[:, 1::2] ** 2,
                               rtol=1e-12)


def test_rope_relative_position_property():
    """<R(p) a, R(p') b> depends only on p - p' (per axis)."""
    wl = tiny(F=6, Hs=5, Ws=5)
    d, S = wl.d, wl.S
    rng = np.random.default_rng(3)
    a, b = rng.standard_normal(d), rng.standard_normal(d)
    x = np.zeros((1, 1, wl.L, d), np.float32)
    tok = lambda f, yy, xx: f * S + yy * wl.Ws + xx
    pairs = [((3, 2, 4), (1, 0, 1)), ((2, 2, 3), (0, 0, 0)), ((5, 4, 4), (3, 2, 1))]  # same deltas (2, 2, 3)
    vals = []
    for pa, pb in pairs:
        x[...] = 0
        x[0, 0, tok(*pa)] = a
        x[0, 0, tok(*pb)] = b
        xb = bits(x)
        y = _norm_rows(wl, xb, np.ones(d, np.float32), np.array([tok(*pa), tok(*pb)], np.int64), eps=0.0)
        vals.append(float(y[0] @ y[1]))
    assert abs(vals[0] - vals[1]) < 1e-10 and abs(vals[0] - vals[2]) < 1e-10
    # and a different delta gives a different value
    x[...] = 0
    x[0, 0, tok(3, 2, 4)] = a
    x[0, 0, tok(0, 0, 1)] = b
    y = _norm_rows(wl, bits(x), np.ones(d, np.float32), np.array([tok(3, 2, 4), tok(0, 0, 1)], np.int64), eps=0.0)
    assert abs(float(y[0] @ y[1]) - vals[0]) > 1e-3


def test_bf16_stage_rounds_fp64_stage():
    wl = tiny(T=3)
    inp = W.make_inputs(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    full = oracle.qknorm_rope(sh, pr, inp["q"], inp["gamma_q"])
    y = oracle.qknorm_rope_f64(sh, pr, inp["q"], inp["gamma_q"])
    ref = torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    # fp64 -> bf16 directly equals fp64 -> fp32 -> bf16 except at exact fp32 halfway points
    assert (full.reshape(-1) != ref.reshape(-1)).sum() <= 2


# ---------------------------------------------------------------- masks ----

def _mask_count(wl, kind, **kw):
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl, **kw)
    return int(oracle.mask(sh, pr, kind).sum())


def test_mask_closed_forms_small():
    wl = tiny(F=5, Hs=2, Ws=3, T=2)
    F, S, Lv, L, T = wl.F, wl.S, wl.Lv, wl.L, wl.T
    text = L * L - Lv * Lv                       # pairs with a text query or a text key
    # w = 0: block diagonal of F blocks S x S
    assert _mask_count(wl, W.SPATIAL, w=0) == F * S * S + text
    # w = 1: frames f and f +- 1
    assert _mask_count(wl, W.SPATIAL, w=1) == (F + 2 * (F - 1)) * S * S + text
    # r = 0: same location in every frame
    assert _mask_count(wl, W.TEMPORAL, r=0) == S * F * F + text
    # r = 1 on S = 6 locations: |ds| <= 1 pairs = S + 2(S-1)
    assert _mask_count(wl, W.TEMPORAL, r=1) == (S + 2 * (S - 1)) * F * F + text
    # windows covering everything reduce to dense
    assert _mask_count(wl, W.SPATIAL, w=F - 1) == L * L
    assert _mask_count(wl, W.TEMPORAL, r=S - 1) == L * L
    assert _mask_count(wl, W.DENSE) == L * L


def test_mask_is_symmetric_and_keeps_diagonal():
    wl = tiny(F=4, Hs=3, Ws=3, T=3)
    sh = oracle.shape_of(wl)
    for kind in (W.SPATIAL, W.TEMPORAL):
        m = oracle.mask(sh, oracle.params_of(wl), kind)
        assert np.array_equal(m, m.T)
        assert m.diagonal().all()


def test_hunyuan_spatial_density_golden():
    """The HunyuanVideo 720p workload states about 9 % key density for a
    +-1-frame spatial window; exact counts from the oracle's mask."""
    g = json.load(open(os.path.join(GOLDEN, "density.json")))
    wl = W.HUNYUAN
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    z = np.zeros((1, 1, wl.L, wl.d), np.uint16)
    sh1 = oracle.make_shape(1, 1, wl.d, wl.F, wl.Hs, wl.Ws, wl.T)
    # the spatial mask depends only on the query frame: one oracle row per frame
    rows = np.array([f * wl.S for f in range(wl.F)], np.int64)
    _, kept = oracle.attention_rows(sh1, pr, np.array([W.SPATIAL], np.uint8), z, z, z, rows, want_kept=True)
    total = int(kept.sum()) * wl.S
    density = total / (wl.Lv * wl.L)
    assert abs(density - g["spatial_w1_density"]) < g["tolerance"]
    assert abs(density - 0.09103) < 5e-5
    # the temporal mask (r = 256) depends only on the query location
    rows = np.arange(wl.S, dtype=np.int64)
    _, kept = oracle.attention_rows(sh1, pr, np.array([W.TEMPORAL], np.uint8), z, z, z, rows, want_kept=True)
    assert abs(int(kept.sum()) * wl.F / (wl.Lv * wl.L) - 0.1393) < 5e-4


def test_profile_sample_fraction_golden():
    g = json.load(open(os.path.join(GOLDEN, "profiling_sample.json")))
    wl = W.HUNYUAN
    frac = wl.n_samples / wl.L
    assert wl.n_samples == g["n_queries"]
    assert abs(frac - g["fraction"]) < g["tolerance"]


# ------------------------------------------------------------ attention ----

def _np_attention(q, k, v, scale, m=None):
    s = (q @ k.T) * scale
    if m is not None:
        s = np.where(m, s, -np.inf)
    mx = s.max(1, keepdims=True)
    p = np.exp(s - mx)
    return (p @ v) / p.sum(1, keepdims=True), (mx[:, 0] + np.log(p.sum(1)))


def _head(x, b=0, h=0):
    return f32(x[b, h])


@pytest.mark.parametrize("kind", [W.DENSE, W.SPATIAL, W.TEMPORAL])
def test_attention_matches_numpy_softmax(kind):
    wl = tiny(F=4, Hs=3, Ws=4, T=3, d=64)
    inp = W.make_inputs(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    kinds = np.array([kind, kind], np.uint8)
    rows = np.arange(wl.L, dtype=np.int64) + wl.L          # head 1
    out, lse = oracle.attention_rows(sh, pr, kinds, inp["q"], inp["k"], inp["v"], rows, want_lse=True)
    m = None if kind == W.DENSE else oracle.mask(sh, pr, kind)
    ref, ref_lse = _np_attention(_head(inp["q"], 0, 1), _head(inp["k"], 0, 1), _head(inp["v"], 0, 1),
                                 1 / math.sqrt(wl.d), m)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12)


def test_full_windows_reduce_to_dense():
    wl = tiny(F=4, Hs=3, Ws=4, T=2)
    inp = W.make_inputs(wl)
    sh = oracle.shape_of(wl)
    rows = np.arange(2 * wl.L, dtype=np.int64)
    dense = oracle.attention_rows(sh, oracle.params_of(wl), np.array([2, 2], np.uint8),
                                  inp["q"], inp["k"], inp["v"], rows)
    sp = oracle.attention_rows(sh, oracle.params_of(wl, w=wl.F - 1), np.array([0, 0], np.uint8),
                               inp["q"], inp["k"], inp["v"], rows)
    tp = oracle.attention_rows(sh, oracle.params_of(wl, r=wl.S - 1), np.array([1, 1], np.uint8),
                               inp["q"], inp["k"], inp["v"], rows)
    np.testing.assert_array_equal(sp, dense)
    np.testing.assert_array_equal(tp, dense)


@pytest.mark.parametrize("kind", [W.SPATIAL, W.TEMPORAL])
def test_attention_permutation_equivariance(kind):
    """Attention on the layout-transformed tensors with the transformed mask,
    read back through the inverse layout, equals attention in model order."""
    wl = tiny(F=5, Hs=3, Ws=4, T=3)
    inp = W.make_inputs(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    kinds = np.array([kind, kind], np.uint8)
    qp, kp, vp = (oracle.layout(sh, kinds, inp[t]) for t in ("q", "k", "v"))
    rows = np.arange(2 * wl.L, dtype=np.int64)
    o_model = oracle.attention_rows(sh, pr, kinds, inp["q"], inp["k"], inp["v"], rows)
    o_lay = oracle.attention_rows(sh, pr, kinds, qp, kp, vp, rows, layout_order=True)
    for bh in range(2):
        for p in range(wl.L):
            i = oracle.perm_inv(sh, kind, p)
            # same terms, summed in another key order
            np.testing.assert_allclose(o_lay[bh * wl.L + p], o_model[bh * wl.L + i], rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------- layout ----

def test_layout_hand_values():
    wl = tiny(F=4, Hs=2, Ws=3, T=2)          # S = 6
    sh = oracle.shape_of(wl)
    T_ = W.TEMPORAL
    assert oracle.perm(sh, T_, 0) == 0
    assert oracle.perm(sh, T_, 6) == 1        # frame 1, location 0 -> right after frame 0's copy
    assert oracle.perm(sh, T_, 1) == 4        # frame 0, location 1 -> after the 4 frames of location 0
    assert oracle.perm(sh, T_, 23) == 23      # last video token is a fixed point
    assert oracle.perm(sh, T_, 24) == 24      # text stays
    assert oracle.perm(sh, W.SPATIAL, 7) == 7
    # positions of one location are contiguous in the new order
    locs = [oracle.perm(sh, T_, f * 6 + 2) for f in range(4)]
    assert locs == [8, 9, 10, 11]


def test_layout_roundtrip_and_fixed_points():
    wl = tiny(F=5, Hs=3, Ws=4, T=3, H=3)
    inp = W.make_inputs(wl)
    sh = oracle.shape_of(wl)
    kinds = np.array([W.TEMPORAL, W.SPATIAL, W.DENSE], np.uint8)
    y = oracle.layout(sh, kinds, inp["q"])
    assert np.array_equal(oracle.layout(sh, kinds, y, inverse=True), inp["q"])
    assert np.array_equal(y[0, 1:], inp["q"][0, 1:])        # non-temporal heads unchanged
    assert not np.array_equal(y[0, 0], inp["q"][0, 0])
    for F_, Hs in ((1, 3), (4, 1)):                      # F = 1 or S = 1: identity
        wl1 = tiny(F=F_, Hs=Hs, Ws=1 if Hs == 1 else 4, T=2, H=1, planted=("T",), n_samples=2)
        inp1 = W.make_inputs(wl1)
        sh1 = oracle.shape_of(wl1)
        assert np.array_equal(oracle.layout(sh1, np.array([1], np.uint8), inp1["q"]), inp1["q"])


# ------------------------------------------------------------ profiling ----

def test_profile_brute_force_tiny():
    wl = W.TINY
    inp = W.make_inputs(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    qn = oracle.qknorm_rope(sh, pr, inp["q"], inp["gamma_q"])
    kn = oracle.qknorm_rope(sh, pr, inp["k"], inp["gamma_k"])
    mse, choice = oracle.profile(sh, pr, qn, kn, inp["v"], inp["sample_idx"])
    ms = oracle.mask(sh, pr, W.SPATIAL)
    mt = oracle.mask(sh, pr, W.TEMPORAL)
    idx = inp["sample_idx"]
    for h in range(wl.H):
        q, k, v = _head(qn, 0, h)[idx], _head(kn, 0, h), _head(inp["v"], 0, h)
        od, _ = _np_attention(q, k, v, 1 / math.sqrt(wl.d))
        os_, _ = _np_attention(q, k, v, 1 / math.sqrt(wl.d), ms[idx])
        ot, _ = _np_attention(q, k, v, 1 / math.sqrt(wl.d), mt[idx])
        e = [((os_ - od) ** 2).mean(), ((ot - od) ** 2).mean()]
        np.testing.assert_allclose(mse[h], e, rtol=1e-9)
        assert choice[h] == int(np.argmin(e))          # ties -> spatial (index 0)
    assert list(choice) == list(inp["planted"])         # planted heads come out as planted


def test_profile_classifies_strongly_planted_heads():
    """With a strong planted signal every planted head must be recognised; a
    swapped or mis-indexed mask would flip these."""
    wl = W.small_workload(H=4, d=64, F=8, Hs=6, Ws=8, T=16, w=1, r=4, n_samples=32, sigma=4.0,
                          planted=("S", "T", "T", "S"))
    inp = W.make_inputs(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    qn = oracle.qknorm_rope(sh, pr, inp["q"], inp["gamma_q"])
    kn = oracle.qknorm_rope(sh, pr, inp["k"], inp["gamma_k"])
    mse, choice = oracle.profile(sh, pr, qn, kn, inp["v"], inp["sample_idx"])
    assert list(choice) == [0, 1, 1, 0]


def test_profile_planted_wan():
    wl = W.WAN
    inp = W.make_inputs(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    qn = oracle.qknorm_rope(sh, pr, inp["q"], inp["gamma_q"])
    kn = oracle.qknorm_rope(sh, pr, inp["k"], inp["gamma_k"])
    _, choice = oracle.profile(sh, pr, qn, kn, inp["v"], inp["sample_idx"])
    for h, p in enumerate(inp["planted"]):
        if p != 255:
            assert choice[h] == p


# ----------------------------------------------------------- block list ----

def _closed_form_tiles(wl, kind, w, r):
    """Independent interval reasoning: in the head's layout every video query
    keeps one contiguous run of video keys plus all text keys."""
    F, S, Lv, L, bq, bk = wl.F, wl.S, wl.Lv, wl.L, wl.bq, wl.bk
    lo = np.zeros(L, np.int64)
    hi = np.full(L, L, np.int64)
    p = np.arange(Lv)
    if kind == W.SPATIAL:
        f = p // S
        lo[:Lv], hi[:Lv] = np.maximum(f - w, 0) * S, np.minimum(f + w + 1, F) * S
    elif kind == W.TEMPORAL:
        s = p // F
        lo[:Lv], hi[:Lv] = np.maximum(s - r, 0) * F, np.minimum(s + r + 1, S) * F
    nqb, nkb = -(-L // bq), -(-L // bk)
    listed = np.zeros((nqb, nkb), bool)
    full = np.zeros((nqb, nkb), bool)
    k = np.arange(L)
    for qb in range(nqb):
        rows = np.arange(qb * bq, min(L, qb * bq + bq))
        kept = ((k[None, :] >= lo[rows, None]) & (k[None, :] < hi[rows, None])) | (k[None, :] >= Lv) \
            | (rows[:, None] >= Lv)
        for kb in range(nkb):
            blk = kept[:, kb * bk:min(L, kb * bk + bk)]
            listed[qb, kb] = blk.any()
            full[qb, kb] = blk.all()
    return listed, full


@pytest.mark.parametrize("wl", [W.TINY, W.COGVIDEOX], ids=["tiny", "cogvideox"])
def test_block_list_brute_force_equals_interval_form(wl):
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    kinds = np.array([W.SPATIAL, W.TEMPORAL, W.DENSE] * (wl.H // 2 + 1), np.uint8)[:wl.H]
    row_ptr, col, full = oracle.block_list(sh, pr, kinds)
    nqb, nkb = wl.nqb, wl.nkb
    for h in range(wl.H):
        listed, fl = _closed_form_tiles(wl, int(kinds[h]), wl.w, wl.r)
        for qb in range(nqb):
            a, b = row_ptr[h * nqb + qb], row_ptr[h * nqb + qb + 1]
            assert list(col[a:b]) == list(np.nonzero(listed[qb])[0])
            assert list(full[a:b]) == list(fl[qb, col[a:b]].astype(np.uint8))


def test_block_list_dense_and_ragged_tail():
    wl = tiny(F=3, Hs=5, Ws=7, T=11, bq=64, bk=32)          # L = 116: ragged on both tile sizes
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    row_ptr, col, full = oracle.block_list(sh, pr, np.array([W.DENSE, W.DENSE], np.uint8))
    assert len(col) == 2 * wl.nqb * wl.nkb and full.all()   # columns past L are not part of a tile
    assert list(col[:wl.nkb]) == list(range(wl.nkb))
