"""Parity of the semantic-aware permutation ("Sparse VideoGen2" explainer,
"A. 语义感知排列" and "B. 基于质心的 Top-p 选择") with the oracle, through the C ABI.

Bars:
  * k-means, stage by stage on the same inputs: the initial centroids are
    bit-exact; every assignment equals the oracle's fp64 nearest centroid
    except on rows whose two nearest centroids lie within the tie band
    (relative gap below 1e-5; the kernel takes the decision in fp32), and
    those rows are counted and reported; every update is within one float
    ulp of the fp64 mean;
  * the cluster sort, the permuted tensors and the block index: bit-exact;
  * top-p sets: bit-exact wherever the oracle's weights leave the decision
    clear of a rounding-level near tie (the kernel's exp and the C library's
    may differ in the last bit);
  * attention: max-abs <= 2e-2 and mean-abs <= 2e-3 against fp64.

Every stage is also run on the oracle's own results of the stage before it, so
a mismatch names the stage that caused it.
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

# name -> (workload, Cq, Ck, iters, top_p)
CASES = {
    # d = 128, text, ragged last tile (L = 403), odd key-cluster count
    "d128": (W.small_workload(d=128, H=2, F=4, Hs=8, Ws=12, T=19, seed=21), 8, 11, 2, 0.9),
    # d = 64, three heads, odd counts on both sides
    "d64": (W.small_workload(d=64, H=3, F=5, Hs=6, Ws=10, T=7, seed=22), 7, 9, 3, 0.8),
    # no text tokens; L a multiple of both tiles
    "notext": (W.small_workload(d=128, H=2, F=3, Hs=8, Ws=16, T=0, seed=23), 16, 16, 2, 0.95),
    # two batch entries, every head index runs over b*H + h
    "batch2": (W.small_workload(B=2, d=128, H=2, F=3, Hs=4, Ws=6, T=5, seed=24), 5, 6, 2, 0.7),
    # one cluster each: every pair is kept, i.e. dense attention
    "onecluster": (W.small_workload(d=64, H=2, F=2, Hs=6, Ws=8, T=3, seed=25), 1, 1, 1, 0.5),
    # 64 clusters (a full 64-bit key set) at the Wan 2.1 1.3B shape
    "wan": (W.WAN, 64, 64, 2, 0.9),
    # d = 64 at the CogVideoX shape: 48 heads, 226 text tokens, 32 + 48 clusters
    "cogvideox": (W.COGVIDEOX, 32, 48, 2, 0.9),
}
FULL_ROWS = ("d128", "d64", "notext", "batch2", "onecluster")


@functools.lru_cache(maxsize=None)
def case(key):
    """Seeded inputs (the oracle's QK-Norm + RoPE of Q and K) and the oracle's
    results of every step (cached)."""
    wl, Cq, Ck, iters, top_p = CASES[key]
    inp = W.make_inputs(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    qn = oracle.qknorm_rope(sh, pr, inp["q"], inp["gamma_q"])
    kn = oracle.qknorm_rope(sh, pr, inp["k"], inp["gamma_k"])
    Lv = wl.Lv
    cq, aq, nq = oracle.kmeans(qn, Lv, Cq, iters)
    ck, ak, nk = oracle.kmeans(kn, Lv, Ck, iters)
    pq, qoff = oracle.cluster_permutation(aq, Cq)
    pk, koff = oracle.cluster_permutation(ak, Ck)
    scale = 1.0 / np.sqrt(wl.d)
    sel, weight = oracle.select_top_p(cq, ck, nk, scale, top_p, want_weight=True)
    ref = dict(cq=cq, aq=aq, nq=nq, ck=ck, ak=ak, nk=nk, pq=pq, qoff=qoff, pk=pk, koff=koff, sel=sel,
               clear=clear_decisions(weight, top_p))
    return wl, inp, qn, kn, ref


def clear_decisions(weight, p, rel=1e-9):
    """Query clusters whose top-p set does not hinge on the last bits of a
    weight: no two unequal weights within `rel` of each other, and no running
    sum within `rel` of the threshold p (weights normalised to sum 1)."""
    BH, Cq, Ck = weight.shape
    ok = np.ones((BH, Cq), bool)
    for bh in range(BH):
        for i in range(Cq):
            w = weight[bh, i]
            ws = np.sort(w[w > 0])[::-1]
            if len(ws) > 1:
                gap = -np.diff(ws)
                if ((gap > 0) & (gap < rel * ws[:-1])).any():
                    ok[bh, i] = False
            if (np.abs(np.cumsum(ws) - p) < rel).any():
                ok[bh, i] = False
    return ok


def pb_of(wl):
    return svg.Problem.from_workload(wl)


def f32_bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def host(t):
    return t.cpu().numpy()


# --------------------------------------------------------------- k-means

# The kernel decides the nearest centroid by |c|^2 - 2 x.c in fp32 (d-term
# fused multiply-add chains), whose rounding error stays below about
# d * 2^-24 * (|x|^2 + |c|^2) ~ 8e-6 of the terms' scale at d = 128.  A row
# whose two nearest fp64 distances differ by less than TIE_BAND of
# |x|^2 + |c1|^2 + |c2|^2 may therefore go either way.
TIE_BAND = 1e-5


def ordered_f32(bits):
    """Monotone integer image of float32 bit patterns (adjacent floats differ by 1)."""
    b = bits.astype(np.int64)
    return np.where(b & 0x80000000, -(b & 0x7FFFFFFF), b)


def check_assignment(x, Lv, cent, assign, what):
    """The GPU assignment against the oracle's fp64 argmin under the same
    centroids.  Returns (rows in the tie band, rows that differ)."""
    want, margin = oracle.kmeans_assign(x, Lv, cent, want_margin=True)
    diff = assign != want
    tie = margin < TIE_BAND
    assert not (diff & ~tie).any(), f"{what}: {(diff & ~tie).sum()} rows differ outside the tie band"
    return int(tie.sum()), int(diff.sum())


def check_update(x, Lv, assign_prev, cent_prev, cent, what):
    """The GPU centroids against the oracle's fp64 means of the same assignment."""
    want, _ = oracle.kmeans_update(x, Lv, assign_prev, cent_prev)
    ulps = np.abs(ordered_f32(f32_bits(cent)) - ordered_f32(f32_bits(want)))
    assert ulps.max() <= 1, f"{what}: centroids {ulps.max()} ulps from the fp64 mean"


def kmeans_checked(pb, x, Lv, C, iters, what, cent0=None):
    """The GPU k-means checked stage by stage against the oracle: each round is
    one call warm-started from the previous call's centroids, so every
    assignment and update is compared on the same inputs.  The single call of
    `iters` rounds must equal the chain bit for bit.  Returns that call's
    (cent, assign, counts) as numpy and the tie-band statistics."""
    xd = dev(x)
    stats = {"rows": 0, "tie_band": 0, "differ": 0}

    def tally(t, dif):
        stats["rows"] += int(np.prod(x.shape[:2])) * Lv
        stats["tie_band"] += t
        stats["differ"] += dif

    if cent0 is None:
        c, a, n = svg.svg2_kmeans(pb, xd, C, 0)
        c_prev = oracle.kmeans_init(x, Lv, C)
        assert np.array_equal(f32_bits(host(c)), f32_bits(c_prev)), f"{what}: initial centroids"
    else:
        c_prev = np.array(cent0, np.float32)
        c, a, n = svg.svg2_kmeans(pb, xd, C, 0, cent=dev(c_prev))
    a_prev = host(a)
    tally(*check_assignment(x, Lv, c_prev, a_prev, f"{what} round 0"))
    for t in range(1, iters + 1):
        c, a, n = svg.svg2_kmeans(pb, xd, C, 1, cent=dev(c_prev))
        c_h, a_h = host(c), host(a)
        check_update(x, Lv, a_prev, c_prev, c_h, f"{what} round {t}")
        tally(*check_assignment(x, Lv, c_h, a_h, f"{what} round {t}"))
        c_prev, a_prev = c_h, a_h
    c1, a1, n1 = svg.svg2_kmeans(pb, xd, C, iters, cent=None if cent0 is None else dev(np.array(cent0, np.float32)))
    svg.sync_status()
    c1, a1, n1 = host(c1), host(a1), host(n1)
    assert np.array_equal(f32_bits(c1), f32_bits(c_prev)) and np.array_equal(a1, a_prev), f"{what}: one call != chain"
    assert np.array_equal(n1, np.stack([np.bincount(r, minlength=C) for r in a1])), f"{what}: sizes"
    print(f"{what}: {stats['tie_band']} of {stats['rows']} row decisions in the tie band, {stats['differ']} differ")
    # the band is a worst-case bound, so it holds a few rows per ten thousand; the
    # decisions that actually went the other way must be rarer still
    assert stats["tie_band"] <= 1e-3 * stats["rows"] + 2, f"{what}: {stats}"
    assert stats["differ"] <= 1e-5 * stats["rows"] + 2, f"{what}: {stats}"
    return (c1, a1, n1), stats


@pytest.mark.parametrize("key", list(CASES))
def test_kmeans_matches_the_oracle_outside_the_tie_band(key):
    wl, inp, qn, kn, ref = case(key)
    _, Cq, Ck, iters, _ = CASES[key]
    pb = pb_of(wl)
    for x, C, s in ((qn, Cq, "q"), (kn, Ck, "k")):
        (cent, assign, counts), st = kmeans_checked(pb, x, wl.Lv, C, iters, f"{key}/{s}")
        if st["differ"] == 0:
            # no decision went the other way: the whole run equals the oracle's
            ulps = np.abs(ordered_f32(f32_bits(cent)) - ordered_f32(f32_bits(ref["c" + s])))
            assert ulps.max() <= 1 and np.array_equal(assign, ref["a" + s]), f"{key}/{s}"
            assert np.array_equal(counts, ref["n" + s]), f"{key}/{s}: sizes"


def test_kmeans_warm_start_continues_the_iteration():
    """Two calls of one round each from the previous centroids (the cached
    centroids of the pages) equal one call of two rounds; the rounds are
    checked against the oracle from the given centroids."""
    wl, inp, qn, kn, ref = case("d128")
    pb = pb_of(wl)
    x = dev(kn)
    cent, _, _ = svg.svg2_kmeans(pb, x, 11, 1)
    cent, assign, counts = svg.svg2_kmeans(pb, x, 11, 1, cent=cent)
    c2, a2, n2 = svg.svg2_kmeans(pb, x, 11, 2)
    svg.sync_status()
    assert np.array_equal(f32_bits(host(cent)), f32_bits(host(c2)))
    assert np.array_equal(host(assign), host(a2))
    assert np.array_equal(host(counts), host(n2))
    start = oracle.kmeans(kn, wl.Lv, 11, 1)[0]
    kmeans_checked(pb, kn, wl.Lv, 11, 2, "warm start", cent0=start)


def test_kmeans_zero_iterations_is_the_init_assignment():
    wl, inp, qn, kn, ref = case("d64")
    pb = pb_of(wl)
    cent, assign, counts = svg.svg2_kmeans(pb, dev(qn), 7, 0)
    svg.sync_status()
    c_ref = oracle.kmeans_init(qn, wl.Lv, 7)
    assert np.array_equal(f32_bits(host(cent)), f32_bits(c_ref))
    check_assignment(qn, wl.Lv, c_ref, host(assign), "init")


# ------------------------------------------------------------ cluster sort

@pytest.mark.parametrize("key", list(CASES))
def test_permutation_bit_exact(key):
    wl, inp, qn, kn, ref = case(key)
    _, Cq, Ck, _, _ = CASES[key]
    pb = pb_of(wl)
    for s, C in (("q", Cq), ("k", Ck)):
        perm, off = svg.svg2_permutation(pb, dev(ref["a" + s]), C)
        svg.sync_status()
        assert np.array_equal(host(perm), ref["p" + s]), f"{key}/{s}: perm"
        assert np.array_equal(host(off), ref[s + "off"]), f"{key}/{s}: off"


def test_permutation_with_empty_and_skewed_clusters():
    """Clusters of size 0 and one cluster holding most rows, across several
    1024-row chunks."""
    wl = W.small_workload(d=64, H=3, F=5, Hs=20, Ws=24, T=0)
    pb = pb_of(wl)
    rng = np.random.Generator(np.random.PCG64(4))
    a = np.where(rng.random((3, wl.Lv)) < 0.8, 5, rng.integers(0, 64, (3, wl.Lv))).astype(np.uint8)
    a[:, a[0] == 17] = 18
    a[1] = 0
    perm_r, off_r = oracle.cluster_permutation(a, 64)
    perm, off = svg.svg2_permutation(pb, dev(a), 64)
    svg.sync_status()
    assert np.array_equal(host(perm), perm_r)
    assert np.array_equal(host(off), off_r)


# ------------------------------------------------------------------ top-p

@pytest.mark.parametrize("key", list(CASES))
def test_select_bit_exact_away_from_near_ties(key):
    wl, inp, qn, kn, ref = case(key)
    _, Cq, Ck, _, top_p = CASES[key]
    pb = pb_of(wl)
    sel = host(svg.svg2_select(pb, dev(ref["cq"]), dev(ref["ck"]), dev(ref["nk"]), top_p)).view(np.uint64)
    svg.sync_status()
    clear = ref["clear"]
    assert clear.mean() > 0.99, f"{key}: {(~clear).sum()} near ties"
    assert np.array_equal(sel[clear], ref["sel"][clear])


def test_select_closed_form_cases():
    """Equal scores: weights are the cluster sizes; top_p = 1 keeps every
    non-empty cluster; an empty cluster is never selected."""
    wl = W.small_workload(d=64, H=1, F=1, Hs=2, Ws=4, T=0)
    pb = pb_of(wl)
    cq = np.zeros((1, 2, 64), np.float32)
    ck = np.zeros((1, 4, 64), np.float32)
    nk = np.array([[5, 0, 2, 1]], np.int32)
    # sizes 5, 0, 2, 1 (total 8): goals 4 and 5 are met by cluster 0, 5.6 and 7 need cluster 2 too
    for p, want in ((0.5, 0b0001), (0.625, 0b0001), (0.7, 0b0101), (0.875, 0b0101), (1.0, 0b1101)):
        sel = host(svg.svg2_select(pb, dev(cq), dev(ck), dev(nk), p)).view(np.uint64)
        svg.sync_status()
        assert sel.tolist() == [[want, want]], p
        assert np.array_equal(sel, oracle.select_top_p(cq, ck, nk, 1 / 8, p))


# --------------------------------------------------------------- permute

@pytest.mark.parametrize("key", ["d128", "d64", "batch2", "wan"])
def test_permute_bit_exact(key):
    wl, inp, qn, kn, ref = case(key)
    pb = pb_of(wl)
    qp, kp, vp = svg.svg2_permute(pb, dev(ref["pq"]), dev(ref["pk"]), dev(qn), dev(kn), dev(inp["v"]))
    svg.sync_status()
    assert np.array_equal(host_bits(qp), oracle.permute_rows(qn, wl.Lv, ref["pq"]))
    assert np.array_equal(host_bits(kp), oracle.permute_rows(kn, wl.Lv, ref["pk"]))
    assert np.array_equal(host_bits(vp), oracle.permute_rows(inp["v"], wl.Lv, ref["pk"]))


# ------------------------------------------------------------ block index

def csr(rp, col, full):
    rp = host(rp)
    n = int(rp[-1])
    return rp, host(col)[:n], host(full)[:n]


@pytest.mark.parametrize("key", list(CASES))
def test_block_index_bit_exact(key):
    wl, inp, qn, kn, ref = case(key)
    pb = pb_of(wl)
    rp, col, full = csr(*svg.svg2_block_index(pb, dev(ref["qoff"]), dev(ref["koff"]), dev(ref["sel"].view(np.int64))))
    svg.sync_status()
    rp_r, col_r, full_r = oracle.block_list2(wl.L, wl.Lv, wl.bq, wl.bk, ref["aq"], ref["ak"], ref["pq"], ref["pk"],
                                             ref["sel"])
    assert np.array_equal(rp, rp_r)
    assert np.array_equal(col, col_r)
    assert np.array_equal(full, full_r)


def test_block_index_random_sets():
    """Random key sets (not from top-p) and empty query clusters."""
    wl, inp, qn, kn, ref = case("d128")
    pb = pb_of(wl)
    rng = np.random.Generator(np.random.PCG64(8))
    a_q = rng.integers(0, 9, (2, wl.Lv)).astype(np.uint8)
    a_q[a_q == 3] = 4                                          # cluster 3 empty
    a_k = (np.arange(wl.Lv) * 11 // wl.Lv).astype(np.uint8)[None].repeat(2, 0)
    pq, qoff = oracle.cluster_permutation(a_q, 9)
    pk, koff = oracle.cluster_permutation(a_k, 11)
    sel = rng.integers(0, 1 << 11, (2, 9)).astype(np.uint64)
    sel[0, 2] = 0                                              # a cluster that keeps no video key
    rp, col, full = csr(*svg.svg2_block_index(pb, dev(qoff), dev(koff), dev(sel.view(np.int64))))
    svg.sync_status()
    rp_r, col_r, full_r = oracle.block_list2(wl.L, wl.Lv, wl.bq, wl.bk, a_q, a_k, pq, pk, sel)
    assert np.array_equal(rp, rp_r) and np.array_equal(col, col_r) and np.array_equal(full, full_r)


# -------------------------------------------------------------- attention

def rows_of(key, wl):
    if key in FULL_ROWS:
        return np.arange(wl.B * wl.H * wl.L, dtype=np.int64)
    return W.random_rows(wl, 96, seed=13, boundary=False)


@pytest.mark.parametrize("key", list(CASES))
def test_attention_parity(key):
    """Attention in cluster order, written back in model order, against the
    oracle's masked attention on the oracle's clusters."""
    wl, inp, qn, kn, ref = case(key)
    pb = pb_of(wl)
    qp, kp, vp = (dev(oracle.permute_rows(x, wl.Lv, ref[p])) for x, p in ((qn, "pq"), (kn, "pk"), (inp["v"], "pk")))
    qoff, koff, sel = dev(ref["qoff"]), dev(ref["koff"]), dev(ref["sel"].view(np.int64))
    rp, col, full = svg.svg2_block_index(pb, qoff, koff, sel)
    out, lse = svg.svg2_attention(pb, qp, kp, vp, qoff, koff, sel, dev(ref["pq"]), rp, col, full, want_lse=True)
    svg.sync_status()
    rows = rows_of(key, wl)
    want, want_lse = oracle.attention2_rows(qn, kn, inp["v"], wl.Lv, ref["aq"], ref["ak"], ref["sel"], rows,
                                            want_lse=True)
    got = host_bits(out).reshape(-1, wl.d)[rows]
    assert_attention_close(got, want, what=key)
    assert np.allclose(host(lse).reshape(-1)[rows], want_lse, rtol=0, atol=2e-3)


def test_attention_one_cluster_equals_dense_kernel():
    """With a single cluster on each side every pair is kept: the result equals
    the dense block-sparse kernel on the same tensors, bit for bit."""
    wl, inp, qn, kn, ref = case("onecluster")
    pb = pb_of(wl)
    q, k, v = dev(qn), dev(kn), dev(inp["v"])
    qoff, koff, sel = dev(ref["qoff"]), dev(ref["koff"]), dev(ref["sel"].view(np.int64))
    rp, col, full = svg.svg2_block_index(pb, qoff, koff, sel)
    ident = dev(np.tile(np.arange(wl.Lv, dtype=np.int32), (wl.B * wl.H, 1)))
    out = svg.svg2_attention(pb, q, k, v, qoff, koff, sel, ident, rp, col, full)
    kinds = dev(np.full(wl.B * wl.H, W.DENSE, np.uint8))
    rp2, col2, full2 = svg.build_block_index(pb, kinds)
    dense = svg.block_sparse_attn(pb, q, k, v, kinds, rp2, col2, full2)
    svg.sync_status()
    assert np.array_equal(host_bits(out), host_bits(dense))


# ------------------------------------------------------------ whole step

def oracle_downstream(wl, qn, kn, cq, ck, aq, ak, nk, top_p):
    """The oracle's steps after k-means, on given clusters."""
    pq, qoff = oracle.cluster_permutation(aq, cq.shape[1])
    pk, koff = oracle.cluster_permutation(ak, ck.shape[1])
    sel, weight = oracle.select_top_p(cq, ck, nk, 1.0 / np.sqrt(wl.d), top_p, want_weight=True)
    return dict(pq=pq, qoff=qoff, pk=pk, koff=koff, sel=sel, clear=clear_decisions(weight, top_p))


@pytest.mark.parametrize("key", ["d128", "batch2", "wan"])
def test_layer_end_to_end(key):
    """SVG2Layer (k-means, sort, top-p, permute, block index, attention) on
    the CUDA path alone.  Its k-means equals the stage-checked k-means call;
    every later intermediate equals the oracle's on those clusters."""
    wl, inp, qn, kn, ref = case(key)
    _, Cq, Ck, iters, top_p = CASES[key]
    pb = pb_of(wl)
    (cq, aq, nq), _ = kmeans_checked(pb, qn, wl.Lv, Cq, iters, f"{key}/q")
    (ck, ak, nk), _ = kmeans_checked(pb, kn, wl.Lv, Ck, iters, f"{key}/k")
    down = oracle_downstream(wl, qn, kn, cq, ck, aq, ak, nk, top_p)
    assert down["clear"].all(), "a near tie in this case: pick another seed"
    layer = svg.SVG2Layer(pb, Cq, Ck, iters, top_p)
    out = layer(dev(qn), dev(kn), dev(inp["v"]))
    svg.sync_status()
    last = layer.last
    assert np.array_equal(f32_bits(host(layer.cq)), f32_bits(cq))
    assert np.array_equal(f32_bits(host(layer.ck)), f32_bits(ck))
    assert np.array_equal(host(last["assign_q"]), aq) and np.array_equal(host(last["assign_k"]), ak)
    for name in ("pq", "pk", "qoff", "koff"):
        gname = {"pq": "perm_q", "pk": "perm_k"}.get(name, name)
        assert np.array_equal(host(last[gname]), down[name]), name
    assert np.array_equal(host(last["sel"]).view(np.uint64), down["sel"])
    rows = rows_of(key, wl)
    want = oracle.attention2_rows(qn, kn, inp["v"], wl.Lv, aq, ak, down["sel"], rows)
    assert_attention_close(host_bits(out).reshape(-1, wl.d)[rows], want, what=key)


def test_bad_arguments_are_reported():
    wl, inp, qn, kn, ref = case("d128")
    pb = pb_of(wl)
    with pytest.raises(RuntimeError):
        svg.svg2_kmeans(pb, dev(qn), 65, 1)                       # more than 64 clusters
    with pytest.raises(RuntimeError):
        svg.svg2_select(pb, dev(ref["cq"]), dev(ref["ck"]), dev(ref["nk"]), 0.0)
    pb64 = svg.Problem.from_workload(wl, block_q=64)
    qoff, koff, sel = dev(ref["qoff"]), dev(ref["koff"]), dev(ref["sel"].view(np.int64))
    rp, col, full = svg.svg2_block_index(pb64, qoff, koff, sel)
    with pytest.raises(RuntimeError):
        svg.svg2_attention(pb64, dev(qn), dev(kn), dev(inp["v"]), qoff, koff, sel, dev(ref["pq"]), rp, col, full)
    svg.sync_status()


def test_kmeans_values_outside_the_exact_range_are_reported():
    """A value the fixed-point centroid sums cannot hold exactly (here 1e30,
    and a NaN) is left out and reported as SVG_ERR_INVALID_ARG; the next call
    on clean inputs runs normally."""
    wl, inp, qn, kn, ref = case("d128")
    pb = pb_of(wl)
    for bad in (0x7149, 0x7FC0):                      # bf16 bits of about 1e30, and a NaN
        x = qn.copy()
        x[0, 1, 7, 3] = bad
        svg.svg2_kmeans(pb, dev(x), 8, 1)
        with pytest.raises(svg.SVGError) as e:
            svg.sync_status()
        assert e.value.status == 1
    cent, assign, counts = svg.svg2_kmeans(pb, dev(qn), 8, 0)
    svg.sync_status()


def test_block_index_capacity_overflow_is_reported():
    wl, inp, qn, kn, ref = case("d128")
    pb = pb_of(wl)
    qoff, koff, sel = dev(ref["qoff"]), dev(ref["koff"]), dev(ref["sel"].view(np.int64))
    rp, col, full = svg.svg2_block_index(pb, qoff, koff, sel)
    n = int(rp[-1])
    svg.sync_status()
    cap = n // 2
    rp2, col2, full2 = svg.svg2_block_index(pb, qoff, koff, sel, capacity=cap)
    with pytest.raises(svg.SVGError) as e:
        svg.sync_status()
    assert e.value.status == 5
    svg.sync_status()


def test_layer_at_the_hunyuanvideo_shape_on_two_heads():
    """The whole layer at the HunyuanVideo 720p shape (24 heads, 119,056
    tokens, 64 + 64 clusters), checked on one planted-spatial and one
    planted-temporal head: k-means stage by stage against the oracle (tie band
    as above), sort and top-p bit-exact on the layer's clusters, attention on
    sampled rows (every step is per head, so two heads of the oracle stand for
    the launch)."""
    wl = W.HUNYUAN
    inp = W.make_inputs(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    qn = oracle.qknorm_rope(sh, pr, inp["q"], inp["gamma_q"])
    kn = oracle.qknorm_rope(sh, pr, inp["k"], inp["gamma_k"])
    layer = svg.SVG2Layer(pb_of(wl), 64, 64, 2, 0.9)
    out = layer(dev(qn), dev(kn), dev(inp["v"]))
    svg.sync_status()
    heads = [0, 1]
    q2, k2, v2 = (np.ascontiguousarray(x[:, heads]) for x in (qn, kn, inp["v"]))
    pb2 = svg.Problem.from_workload(wl, H=2)
    (cq, aq, nq), _ = kmeans_checked(pb2, q2, wl.Lv, 64, 2, "hunyuan/q")
    (ck, ak, nk), _ = kmeans_checked(pb2, k2, wl.Lv, 64, 2, "hunyuan/k")
    # the layer's k-means over 24 heads equals the per-head calls
    assert np.array_equal(f32_bits(host(layer.cq)[heads]), f32_bits(cq))
    assert np.array_equal(f32_bits(host(layer.ck)[heads]), f32_bits(ck))
    assert np.array_equal(host(layer.last["assign_q"])[heads], aq)
    down = oracle_downstream(wl, q2, k2, cq, ck, aq, ak, nk, 0.9)
    assert down["clear"].all()
    assert np.array_equal(host(layer.last["perm_q"])[heads], down["pq"])
    assert np.array_equal(host(layer.last["qoff"])[heads], down["qoff"])
    assert np.array_equal(host(layer.last["sel"]).view(np.uint64)[heads], down["sel"])
    rng = np.random.Generator(np.random.PCG64(3))
    toks = np.unique(np.concatenate([rng.choice(wl.L, 40, replace=False), np.arange(wl.L - 8, wl.L)]))
    rows = np.concatenate([h * wl.L + toks for h in range(2)]).astype(np.int64)
    want = oracle.attention2_rows(q2, k2, v2, wl.Lv, aq, ak, down["sel"], rows)
    got = host_bits(out).reshape(wl.H, wl.L, wl.d)[heads].reshape(-1, wl.d)[rows]
    assert_attention_close(got, want, what="hunyuan")


def test_bad_cluster_ids_and_permutation_entries_are_reported():
    """Caller-supplied assignments and permutations out of range are reported
    (SVG_ERR_INVALID_ARG through svg_sync_status), and nothing outside the
    buffers is touched."""
    wl, inp, qn, kn, ref = case("d128")
    pb = pb_of(wl)
    a = ref["aq"].copy()
    a[0, 5] = 200                                         # cluster id >= C
    svg.svg2_permutation(pb, dev(a), 8)
    with pytest.raises(svg.SVGError) as e:
        svg.sync_status()
    assert e.value.status == 1
    pq = ref["pq"].copy()
    pq[1, 3] = wl.Lv + 1000                               # position outside the video rows
    svg.svg2_permute(pb, dev(pq), dev(ref["pk"]), dev(qn), dev(kn), dev(inp["v"]))
    with pytest.raises(svg.SVGError) as e:
        svg.sync_status()
    assert e.value.status == 1
    qp, kp, vp = (dev(oracle.permute_rows(x, wl.Lv, ref[p])) for x, p in ((qn, "pq"), (kn, "pk"), (inp["v"], "pk")))
    qoff, koff, sel = dev(ref["qoff"]), dev(ref["koff"]), dev(ref["sel"].view(np.int64))
    rp, col, full = svg.svg2_block_index(pb, qoff, koff, sel)
    out = torch.zeros_like(qp)
    svg.svg2_attention(pb, qp, kp, vp, qoff, koff, sel, dev(pq), rp, col, full, out=out)
    with pytest.raises(svg.SVGError) as e:
        svg.sync_status()
    assert e.value.status == 1
    svg.sync_status()
