"""Parity of the semantic-aware permutation ("Sparse VideoGen2" explainer,
"A. 语义感知排列" and "B. 基于质心的 Top-p 选择") with the oracle, through the C ABI.

Bars:
  * k-means centroids (float bits), assignments, cluster sizes, the cluster
    sort, the permuted tensors and the block index: bit-exact;
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

@pytest.mark.parametrize("key", list(CASES))
def test_kmeans_bit_exact(key):
    wl, inp, qn, kn, ref = case(key)
    _, Cq, Ck, iters, _ = CASES[key]
    pb = pb_of(wl)
    for x, C, s in ((qn, Cq, "q"), (kn, Ck, "k")):
        cent, assign, counts = svg.svg2_kmeans(pb, dev(x), C, iters)
        svg.sync_status()
        assert np.array_equal(f32_bits(host(cent)), f32_bits(ref["c" + s])), f"{key}/{s}: centroids"
        assert np.array_equal(host(assign), ref["a" + s]), f"{key}/{s}: assignment"
        assert np.array_equal(host(counts), ref["n" + s]), f"{key}/{s}: sizes"


def test_kmeans_warm_start_continues_the_iteration():
    """Two calls of one round each from the previous centroids (the cached
    centroids of the pages) equal one call of two rounds."""
    wl, inp, qn, kn, ref = case("d128")
    pb = pb_of(wl)
    x = dev(kn)
    cent, _, _ = svg.svg2_kmeans(pb, x, 11, 1)
    cent, assign, counts = svg.svg2_kmeans(pb, x, 11, 1, cent=cent)
    svg.sync_status()
    assert np.array_equal(f32_bits(host(cent)), f32_bits(ref["ck"]))
    assert np.array_equal(host(assign), ref["ak"])
    assert np.array_equal(host(counts), ref["nk"])


def test_kmeans_zero_iterations_is_the_init_assignment():
    wl, inp, qn, kn, ref = case("d64")
    pb = pb_of(wl)
    cent, assign, counts = svg.svg2_kmeans(pb, dev(qn), 7, 0)
    svg.sync_status()
    c_ref = oracle.kmeans_init(qn, wl.Lv, 7)
    assert np.array_equal(f32_bits(host(cent)), f32_bits(c_ref))
    assert np.array_equal(host(assign), oracle.kmeans_assign(qn, wl.Lv, c_ref))


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

@pytest.mark.parametrize("key", ["d128", "batch2", "wan"])
def test_layer_end_to_end(key):
    """SVG2Layer (k-means, sort, top-p, permute, block index, attention) on
    the CUDA path alone, every intermediate against the oracle."""
    wl, inp, qn, kn, ref = case(key)
    _, Cq, Ck, iters, top_p = CASES[key]
    assert ref["clear"].all(), "a near tie in this case: pick another seed"
    layer = svg.SVG2Layer(pb_of(wl), Cq, Ck, iters, top_p)
    out = layer(dev(qn), dev(kn), dev(inp["v"]))
    svg.sync_status()
    last = layer.last
    assert np.array_equal(f32_bits(host(layer.cq)), f32_bits(ref["cq"]))
    assert np.array_equal(f32_bits(host(layer.ck)), f32_bits(ref["ck"]))
    for name in ("pq", "pk", "qoff", "koff"):
        gname = {"pq": "perm_q", "pk": "perm_k"}.get(name, name)
        assert np.array_equal(host(last[gname]), ref[name]), name
    assert np.array_equal(host(last["sel"]).view(np.uint64), ref["sel"])
    rows = rows_of(key, wl)
    want = oracle.attention2_rows(qn, kn, inp["v"], wl.Lv, ref["aq"], ref["ak"], ref["sel"], rows)
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
    planted-temporal head: centroids, sort and top-p bit-exact, attention on
    sampled rows (every step is per head, so two heads of the oracle stand
    for the launch)."""
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
    cq, aq, nq = oracle.kmeans(q2, wl.Lv, 64, 2)
    ck, ak, nk = oracle.kmeans(k2, wl.Lv, 64, 2)
    pq, qoff = oracle.cluster_permutation(aq, 64)
    sel, weight = oracle.select_top_p(cq, ck, nk, 1.0 / np.sqrt(wl.d), 0.9, want_weight=True)
    assert clear_decisions(weight, 0.9).all()
    assert np.array_equal(f32_bits(host(layer.cq)[heads]), f32_bits(cq))
    assert np.array_equal(f32_bits(host(layer.ck)[heads]), f32_bits(ck))
    assert np.array_equal(host(layer.last["perm_q"])[heads], pq)
    assert np.array_equal(host(layer.last["qoff"])[heads], qoff)
    assert np.array_equal(host(layer.last["sel"]).view(np.uint64)[heads], sel)
    rng = np.random.Generator(np.random.PCG64(3))
    toks = np.unique(np.concatenate([rng.choice(wl.L, 40, replace=False), np.arange(wl.L - 8, wl.L)]))
    rows = np.concatenate([h * wl.L + toks for h in range(2)]).astype(np.int64)
    want = oracle.attention2_rows(q2, k2, v2, wl.Lv, aq, ak, sel, rows)
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
