"""Parity of AdaSpa's blockified LSE-cached search ("AdaSpa" abstract) with
the oracle, through the C ABI.

Bars:
  * block masses: |gpu - oracle| <= 2e-4 * oracle + 1e-6 * (rows of the tile)
    (fp32 scores on the tensor cores, the hardware 2^x, fp32 sums);
  * selection on the same float masses: bit-exact per query tile, except on
    tiles whose cut lies within the kernel's fixed-point rounding of the goal
    (the kernel sums trunc(mass * 2^32); the oracle sums in double), counted
    and reported;
  * attention over a block list: max-abs 2e-2, mean-abs 2e-3 against fp64;
  * the whole search on the GPU: its selection equals the oracle's on every
    query tile whose decision is clear of the mass tolerance.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_video_qk_b200 as svg
import svg_workloads as W
from gpu_util import assert_attention_close, dev, host_bits

pytestmark = pytest.mark.gpu

CASES = {
    # d = 128, text, ragged last key tile (L = 403 = 6 * 64 + 19), 4 query tiles
    "d128": (W.small_workload(d=128, H=2, F=4, Hs=8, Ws=12, T=19, seed=31), 0.9),
    # d = 64, three heads, an odd number of query tiles (the last pair has one)
    "d64": (W.small_workload(d=64, H=3, F=5, Hs=6, Ws=10, T=7, seed=32), 0.8),
    # no text, Lv not a multiple of 64: the ragged last key tile is a video tile
    "notext": (W.small_workload(d=128, H=2, F=3, Hs=7, Ws=9, T=0, seed=33), 0.95),
    # two batch entries
    "batch2": (W.small_workload(B=2, d=128, H=2, F=3, Hs=8, Ws=8, T=5, seed=34), 0.7),
    # Wan 2.1 1.3B shape (sampled query tiles)
    "wan": (W.WAN, 0.9),
    # d = 64 at the CogVideoX shape (sampled query tiles)
    "cogvideox": (W.COGVIDEOX, 0.8),
}
SMALL = ("d128", "d64", "notext", "batch2")


def pb_of(wl):
    return svg.Problem.from_workload(wl)


def dense_lse(qn, kn, wl, tiles=None):
    """Each row's log-sum-exp over all keys (fp64 numpy, rounded to float):
    the LSE a dense step would cache.  With `tiles`, only the rows of those
    query tiles; the other rows get log(L)."""
    BH, L, d = wl.B * wl.H, wl.L, wl.d
    qh, kh = qn.reshape(BH, L, d), kn.reshape(BH, L, d)
    lse = np.full((BH, L), np.log(L), np.float64)
    todo = range(BH * wl.nqb) if tiles is None else tiles
    kf = {}
    for t in todo:
        bh, qb = divmod(int(t), wl.nqb)
        if bh not in kf:
            kf = {bh: W.bf16_bits_to_f32(kh[bh]).astype(np.float64)}     # one head's keys at a time
        r0, r1 = qb * wl.bq, min(L, (qb + 1) * wl.bq)
        s = W.bf16_bits_to_f32(qh[bh, r0:r1]).astype(np.float64) @ kf[bh].T / np.sqrt(d)
        m = s.max(1, keepdims=True)
        lse[bh, r0:r1] = m[:, 0] + np.log(np.exp(s - m).sum(1))
    return lse.astype(np.float32).reshape(wl.B, wl.H, L)


@functools.lru_cache(maxsize=None)
def case(key):
    wl, p = CASES[key]
    inp = W.make_inputs(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    qn = oracle.qknorm_rope(sh, pr, inp["q"], inp["gamma_q"])
    kn = oracle.qknorm_rope(sh, pr, inp["k"], inp["gamma_k"])
    if key in SMALL:
        tiles = None
    else:
        rng = np.random.Generator(np.random.PCG64(5))
        tiles = np.sort(rng.choice(wl.B * wl.H * wl.nqb, 12, replace=False)).astype(np.int64)
        # the last query tile of head 0 holds the text rows and the ragged tail
        tiles = np.unique(np.concatenate([tiles, [wl.nqb - 1]])).astype(np.int64)
    lse = dense_lse(qn, kn, wl, tiles)
    mass = oracle.block_mass(qn, kn, lse, wl.bq, wl.bk, tiles=tiles)
    return wl, p, inp, qn, kn, lse, tiles, mass


def rows_in_tiles(wl, tiles):
    q = np.arange(wl.nqb * wl.bq)
    out = []
    for t in tiles:
        bh, qb = divmod(int(t), wl.nqb)
        r = q[qb * wl.bq:(qb + 1) * wl.bq]
        out.append(r[r < wl.L])
    return np.concatenate(out), np.repeat(np.arange(len(tiles)), [len(x) for x in out])


@pytest.mark.parametrize("key", list(CASES))
def test_block_mass_against_fp64(key):
    wl, p, inp, qn, kn, lse, tiles, want = case(key)
    got = svg.adaspa_block_mass(pb_of(wl), dev(qn), dev(kn), dev(lse))
    svg.sync_status()
    got = got.cpu().numpy().reshape(-1, wl.nkb).astype(np.float64)
    if tiles is not None:
        got = got[tiles]
    want = want.reshape(-1, wl.nkb)
    err = np.abs(got - want)
    bound = 2e-4 * want + 1e-6 * wl.bq
    assert (err <= bound).all(), f"{key}: worst excess {(err - bound).max():.3e}"
    if tiles is None:
        # with the exact LSE every row's weights sum to 1
        rows = np.minimum(wl.bq, wl.L - np.arange(wl.nqb) * wl.bq)
        assert np.allclose(got.reshape(-1, wl.nqb, wl.nkb).sum(-1), rows[None, :], rtol=1e-3)


def assert_select_matches(rp, col, full, m32, wl, p, what):
    """The GPU's CSR selection against the oracle's on the same float masses.
    The kernel sums the masses as trunc(mass * 2^32), so its running sums and
    its goal are each off by less than (tiles) * 2^-32: a query tile whose
    oracle running sum lies closer than 2 * nkb * 2^-32 to the goal at the cut
    may be cut one tile earlier or later.  Every other tile is bit-exact."""
    rp = rp.cpu().numpy() if hasattr(rp, "cpu") else rp
    n = int(rp[-1])
    col = (col.cpu().numpy() if hasattr(col, "cpu") else col)[:n]
    full = (full.cpu().numpy() if hasattr(full, "cpu") else full)[:n]
    rp_r, col_r, full_r, margin = oracle.adaspa_select(m32, wl.L, wl.Lv, wl.bq, wl.bk, p, want_margin=True)
    band = 2 * wl.nkb * 2.0 ** -32
    tie = margin < band
    differ = 0
    for t in range(len(rp) - 1):
        same = col[rp[t]:rp[t + 1]].tolist() == col_r[rp_r[t]:rp_r[t + 1]].tolist()
        if not same:
            assert tie[t], f"{what}: query tile {t} differs outside the band (margin {margin[t]:.3e})"
            differ += 1
    assert (full == 1).all() and (full_r == 1).all()
    print(f"{what}: {int(tie.sum())} of {len(tie)} query tiles in the band, {differ} differ")
    assert tie.sum() <= 1e-3 * len(tie) + 2, what
    if differ == 0:
        assert np.array_equal(rp, rp_r) and np.array_equal(col, col_r)


@pytest.mark.parametrize("key", SMALL)
def test_select_matches_the_oracle_on_the_same_masses(key):
    wl, p, inp, qn, kn, lse, tiles, mass = case(key)
    m32 = mass.astype(np.float32).reshape(wl.B * wl.H, wl.nqb, wl.nkb)
    rp, col, full = svg.adaspa_select(pb_of(wl), dev(m32), p)
    svg.sync_status()
    assert_select_matches(rp, col, full, m32, wl, p, key)


def test_select_with_a_tight_capacity_matches():
    """Capacity below one flag per tile: the fill pass sorts again instead of
    reading the flags back; the lists are the same."""
    wl, p, inp, qn, kn, lse, tiles, mass = case("d128")
    m32 = dev(mass.astype(np.float32).reshape(wl.B * wl.H, wl.nqb, wl.nkb))
    rp, col, full = svg.adaspa_select(pb_of(wl), m32, p)
    n = int(rp[-1])
    rp2, col2, full2 = svg.adaspa_select(pb_of(wl), m32, p, capacity=n)
    svg.sync_status()
    assert n < wl.B * wl.H * wl.nqb * wl.nkb
    assert torch.equal(rp, rp2)
    assert torch.equal(col[:n], col2[:n]) and torch.equal(full[:n], full2[:n])


@pytest.mark.parametrize("p", [0.3, 0.6, 0.99, 1.0])
def test_select_bit_exact_random_masses_with_ties(p):
    """Masses with exact ties and zeros, over several sort sizes.  Multiples
    of 1/8 are exact in both the kernel's fixed point and the oracle's double
    sums, so every tile is bit-exact, on the band too (a running sum that meets
    the goal exactly is a decision both sides take the same way)."""
    wl = W.small_workload(d=64, H=3, F=6, Hs=10, Ws=13, T=40, seed=2)   # nkb = 13
    rng = np.random.Generator(np.random.PCG64(int(p * 100)))
    m = rng.integers(0, 6, (wl.B * wl.H, wl.nqb, wl.nkb)).astype(np.float32) / 8
    rp, col, full = svg.adaspa_select(pb_of(wl), dev(m), p)
    svg.sync_status()
    rp = rp.cpu().numpy()
    rp_r, col_r, _ = oracle.adaspa_select(m, wl.L, wl.Lv, wl.bq, wl.bk, p)
    assert np.array_equal(rp, rp_r)
    assert np.array_equal(col.cpu().numpy()[:int(rp[-1])], col_r)


def random_blocks(wl, keep=0.4, seed=3):
    rng = np.random.Generator(np.random.PCG64(seed))
    k = rng.random((wl.B * wl.H * wl.nqb, wl.nkb)) < keep
    k[:, 0] = True
    rp = np.concatenate([[0], np.cumsum(k.sum(1))]).astype(np.int32)
    col = np.concatenate([np.nonzero(r)[0] for r in k]).astype(np.int32)
    return rp, col, np.ones(len(col), np.uint8)


@pytest.mark.parametrize("key", list(CASES))
def test_block_attention_parity(key):
    """Attention over an arbitrary block list (every head DENSE, each listed
    block computed whole) against the oracle's block attention."""
    wl, p, inp, qn, kn, lse, tiles, _ = case(key)
    rp, col, full = random_blocks(wl)
    kinds = dev(np.full(wl.B * wl.H, W.DENSE, np.uint8))
    out = svg.block_sparse_attn(pb_of(wl), dev(qn), dev(kn), dev(inp["v"]), kinds, dev(rp), dev(col), dev(full))
    svg.sync_status()
    rows = (np.arange(wl.B * wl.H * wl.L, dtype=np.int64) if key in SMALL
            else W.random_rows(wl, 64, seed=17, boundary=False))
    want = oracle.block_attention_rows(qn, kn, inp["v"], wl.bq, wl.bk, rp, col, rows)
    assert_attention_close(host_bits(out).reshape(-1, wl.d)[rows], want, what=key)


def clear_tiles(mass, wl, p, rel=1e-3):
    """Query tiles whose top-p set is the same for every mass within `rel` of
    the oracle's: no two video tiles near the cut within rel of each other,
    and no running sum within rel of the goal."""
    nv = wl.nkb if wl.L == wl.Lv else min(wl.nkb, wl.Lv // wl.bk)
    ok = []
    for m in mass.reshape(-1, wl.nkb):
        v = np.sort(m[:nv])[::-1]
        cum = np.cumsum(v)
        goal = p * cum[-1]
        cut = int(np.searchsorted(cum, goal * (1 - 1e-12)))
        near = np.abs(cum - goal) < rel * cum[-1]
        lo, hi = max(0, cut - 1), min(nv - 1, cut + 1)
        gaps = np.abs(np.diff(v[lo:hi + 1])) < rel * v[lo:hi + 1].max(initial=0)
        ok.append(not near.any() and not gaps.any())
    return np.array(ok)


def assert_valid_selection(kept, m, wl, qb, p, tol=1e-3):
    """`kept` is a top-p set under masses m within tol: it holds the text tiles
    (all tiles for a text query tile); its video tiles reach p of the video
    mass, dropping the lightest falls below it, and no tile left out is
    heavier than the lightest kept one."""
    nv = wl.nkb if wl.L == wl.Lv else min(wl.nkb, wl.Lv // wl.bk)
    if min(wl.L, (qb + 1) * wl.bq) > wl.Lv:
        assert kept == list(range(wl.nkb))
        return
    assert [k for k in kept if k >= nv] == list(range(nv, wl.nkb))
    kv = [k for k in kept if k < nv]
    tot = m[:nv].sum()
    mk = m[kv].sum()
    assert mk >= p * tot - tol * tot
    assert mk - m[kv].min() < p * tot + tol * tot
    out = np.setdiff1d(np.arange(nv), kv)
    if len(out):
        assert m[out].max() <= m[kv].min() + tol * m[:nv].max()


@pytest.mark.parametrize("key", list(CASES))
def test_search_end_to_end(key):
    """Masses and selection on the GPU.  Every query tile's kept set is a
    valid top-p set under the oracle's masses within the mass tolerance, and
    equals the oracle's own selection wherever that decision is clear of the
    tolerance; the layer's sparse step matches the oracle's block attention."""
    wl, p, inp, qn, kn, lse, tiles, mass = case(key)
    layer = svg.AdaSpaLayer(pb_of(wl), p)
    layer.lse = dev(lse)
    layer.search(dev(qn), dev(kn))
    out = layer.sparse(dev(qn), dev(kn), dev(inp["v"]))
    svg.sync_status()
    rp, col, _ = (t.cpu().numpy() for t in layer.blocks)
    ids = np.arange(wl.B * wl.H * wl.nqb) if tiles is None else tiles
    m_ref = mass.reshape(-1, wl.nkb)
    for i, t in enumerate(ids):
        assert_valid_selection(col[rp[t]:rp[t + 1]].tolist(), m_ref[i], wl, int(t) % wl.nqb, p)
    clear = clear_tiles(m_ref, wl, p)
    assert clear.sum() >= 1, f"{key}: no query tile is clear of the tolerance"
    # the oracle's selection of the checked tiles, from its own masses
    sub = m_ref.astype(np.float32).reshape(len(ids), 1, wl.nkb)
    for i, t in enumerate(ids):
        if not clear[i]:
            continue
        bh, qb = divmod(int(t), wl.nqb)
        # one query tile at a time: a single-tile problem with the same L, Lv
        one = np.zeros((1, wl.nqb, wl.nkb), np.float32)
        one[0, qb] = sub[i, 0]
        rp_r, col_r, _ = oracle.adaspa_select(one, wl.L, wl.Lv, wl.bq, wl.bk, p)
        assert col[rp[t]:rp[t + 1]].tolist() == col_r[rp_r[qb]:rp_r[qb + 1]].tolist(), (key, int(t))
    # attention rows of the clear tiles, over the GPU's (verified) lists
    rows_local, which = rows_in_tiles(wl, ids[clear])
    bhs = ids[clear] // wl.nqb
    rows = bhs[which] * wl.L + rows_local
    want = oracle.block_attention_rows(qn, kn, inp["v"], wl.bq, wl.bk, rp, col, rows)
    assert_attention_close(host_bits(out).reshape(-1, wl.d)[rows], want, what=key)


def test_layer_requires_lse_and_search():
    wl, p, inp, qn, kn, lse, tiles, _ = case("d128")
    layer = svg.AdaSpaLayer(pb_of(wl), p)
    with pytest.raises(RuntimeError):
        layer.search(dev(qn), dev(kn))
    with pytest.raises(RuntimeError):
        layer.sparse(dev(qn), dev(kn), dev(inp["v"]))
    # a dense step caches the LSE; it matches the oracle's dense LSE
    out = layer.dense(dev(qn), dev(kn), dev(inp["v"]))
    svg.sync_status()
    assert np.allclose(layer.lse.cpu().numpy(), lse, atol=2e-3)
    assert out.shape == dev(qn).shape


def test_bad_arguments_are_reported():
    wl, p, inp, qn, kn, lse, tiles, mass = case("d128")
    pb64 = svg.Problem.from_workload(wl, block_q=64)
    with pytest.raises(RuntimeError):
        svg.adaspa_block_mass(pb64, dev(qn), dev(kn), dev(lse),
                              out=torch.empty(wl.B * wl.H * pb64.nqb * pb64.nkb, device="cuda"))
    with pytest.raises(RuntimeError):
        svg.adaspa_select(pb_of(wl), dev(mass.astype(np.float32)), 0.0)
    svg.sync_status()


def test_select_capacity_overflow_is_reported():
    """A capacity below the kept count: the scan records SVG_ERR_CAPACITY and
    nothing is written past the capacity."""
    wl, p, inp, qn, kn, lse, tiles, mass = case("d128")
    m32 = dev(mass.astype(np.float32).reshape(wl.B * wl.H, wl.nqb, wl.nkb))
    rp, col, full = svg.adaspa_select(pb_of(wl), m32, p)
    n = int(rp[-1])
    svg.sync_status()
    cap = n // 2
    col2 = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    full2 = torch.zeros(n, dtype=torch.uint8, device="cuda")
    rp2 = torch.empty_like(rp)
    from sparse_attention_video_qk_b200._lib import check
    import ctypes
    pb = pb_of(wl)
    sh, pr = pb.c_shape(), pb.c_params()
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    check(svg.lib().svg_adaspa_select(ctypes.byref(sh), ctypes.byref(pr), P(m32), float(p), P(rp2), P(col2),
                                      P(full2), cap, None), "svg_adaspa_select")
    with pytest.raises(svg.SVGError) as e:
        svg.sync_status()
    assert e.value.status == 5
    assert (col2[cap:].cpu().numpy() == -7).all()
    svg.sync_status()


def test_search_at_the_hunyuanvideo_shape_on_sampled_tiles():
    """Block masses, selection and the sparse step at the HunyuanVideo 720p
    shape (24 heads, 931 query tiles x 1861 key tiles per head) on sampled
    query tiles, with the oracle's LSE for their rows."""
    wl, p = W.HUNYUAN, 0.9
    inp = W.make_inputs(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    qn = oracle.qknorm_rope(sh, pr, inp["q"], inp["gamma_q"])
    kn = oracle.qknorm_rope(sh, pr, inp["k"], inp["gamma_k"])
    rng = np.random.Generator(np.random.PCG64(9))
    tiles = np.sort(rng.choice(wl.B * wl.H * wl.nqb, 6, replace=False)).astype(np.int64)
    tiles = np.unique(np.concatenate([tiles, [wl.nqb - 1, 2 * wl.nqb - 2]])).astype(np.int64)
    lse = dense_lse(qn, kn, wl, tiles)
    want = oracle.block_mass(qn, kn, lse, wl.bq, wl.bk, tiles=tiles)
    layer = svg.AdaSpaLayer(pb_of(wl), p)
    layer.lse = dev(lse)
    mass = layer.search(dev(qn), dev(kn))
    out = layer.sparse(dev(qn), dev(kn), dev(inp["v"]))
    svg.sync_status()
    got = mass.cpu().numpy().reshape(-1, wl.nkb)[tiles].astype(np.float64)
    assert (np.abs(got - want) <= 2e-4 * want + 1e-6 * wl.bq).all()
    rp, col, _ = (t.cpu().numpy() for t in layer.blocks)
    for i, t in enumerate(tiles):
        assert_valid_selection(col[rp[t]:rp[t + 1]].tolist(), want[i], wl, int(t) % wl.nqb, p)
    rows_local, which = rows_in_tiles(wl, tiles[:3])
    rows_local, which = rows_local[::8], which[::8]               # every 8th row of three tiles
    rows = (tiles[:3] // wl.nqb)[which] * wl.L + rows_local
    ref = oracle.block_attention_rows(qn, kn, inp["v"], wl.bq, wl.bk, rp, col, rows)
    assert_attention_close(host_bits(out).reshape(-1, wl.d)[rows], ref, what="hunyuan")
