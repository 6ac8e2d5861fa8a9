"""Pins of the semantic-aware-permutation oracle ("Sparse VideoGen2"
explainer, "A. 语义感知排列" and "B. 基于质心的 Top-p 选择"): k-means against
planted clusters and brute force, the counting sort's invariants, top-p on
cases with closed-form weights, and the masked attention against numpy."""
import numpy as np
import pytest

import oracle
import svg_workloads as W


def _blobs(C=4, per=24, d=16, H=2, sep=6.0, noise=0.05, seed=3):
    """bf16 [1, H, Lv, d] rows in C contiguous blocks around well separated centres."""
    rng = np.random.Generator(np.random.PCG64(seed))
    Lv = C * per
    x = np.empty((1, H, Lv, d), np.float32)
    labels = np.repeat(np.arange(C), per)
    for h in range(H):
        centres = rng.standard_normal((C, d)).astype(np.float32) * sep
        x[0, h] = centres[labels] + noise * rng.standard_normal((Lv, d)).astype(np.float32)
    return W.to_bf16_bits(x), labels, Lv


def test_kmeans_recovers_planted_clusters():
    xb, labels, Lv = _blobs()
    cent, assign, counts = oracle.kmeans(xb, Lv, C=4, iters=2)
    for h in range(2):
        assert np.array_equal(assign[h], labels)
        assert np.array_equal(counts[h], np.bincount(labels, minlength=4))
        xf = W.bf16_bits_to_f32(xb[0, h]).astype(np.float64)
        for c in range(4):
            mean = xf[labels == c].mean(0)
            assert np.allclose(cent[h, c], mean, rtol=0, atol=1e-6)


def test_assignment_is_the_fp64_argmin_on_every_row():
    """The assignment is numpy's brute-force argmin of the squared Euclidean
    distance on every row (no tie band: both sides are fp64), and the margin is
    the relative gap to the second nearest centroid."""
    rng = np.random.Generator(np.random.PCG64(5))
    x = W.to_bf16_bits(rng.standard_normal((1, 2, 200, 32)).astype(np.float32))
    cent = oracle.kmeans_init(x, 200, 7)
    a, margin = oracle.kmeans_assign(x, 200, cent, want_margin=True)
    xf = W.bf16_bits_to_f32(x[0]).astype(np.float64)
    for h in range(2):
        c64 = cent[h].astype(np.float64)
        dist = ((xf[h][:, None, :] - c64[None]) ** 2).sum(-1)
        assert np.array_equal(a[h], dist.argmin(1))
        order = np.argsort(dist, 1, kind="stable")
        c1, c2 = order[:, 0], order[:, 1]
        scale = (xf[h] ** 2).sum(1) + (c64[c1] ** 2).sum(1) + (c64[c2] ** 2).sum(1)
        gap = (dist[np.arange(200), c2] - dist[np.arange(200), c1]) / scale
        assert np.allclose(margin[h], gap, rtol=1e-9, atol=1e-15)
    # the init rows are rows floor(c*Lv/C); each init row is its own centroid (distance 0)
    for c in range(7):
        assert np.array_equal(cent[1, c], W.bf16_bits_to_f32(x[0, 1, c * 200 // 7]))
        assert a[1, c * 200 // 7] == c


def test_assignment_tie_goes_to_the_lower_index_with_zero_margin():
    """A row exactly halfway between two centroids: distance 1 to each of
    +-e_0; the lower index wins and the margin is 0.  A third, farther
    centroid does not change either."""
    d = 8
    x = np.zeros((1, 1, 3, d), np.float32)
    x[0, 0, 1, 0] = 0.5                                  # nearer to +e_0
    x[0, 0, 2, 1] = 4.0                                  # nearest to the third centroid
    cent = np.zeros((1, 3, d), np.float32)
    cent[0, 0, 0], cent[0, 1, 0], cent[0, 2, 1] = -1.0, 1.0, 3.0
    a, margin = oracle.kmeans_assign(W.to_bf16_bits(x), 3, cent, want_margin=True)
    assert a.tolist() == [[0, 1, 2]]
    assert margin[0, 0] == 0.0
    # row 1: distances 2.25 and 0.25 -> gap 2 over 0.25 + 1 + 1
    assert margin[0, 1] == 2.0 / 2.25
    # row 2: distances 1 (c2) and 17 (c0, c1) -> gap 16 over 16 + 9 + 1
    assert margin[0, 2] == 16.0 / 26.0
    one, m1 = oracle.kmeans_assign(W.to_bf16_bits(x), 3, cent[:, :1], want_margin=True)
    assert one.tolist() == [[0, 0, 0]] and np.isinf(m1).all()


def test_permutation_is_a_stable_cluster_sort():
    rng = np.random.Generator(np.random.PCG64(2))
    a = rng.integers(0, 6, size=(3, 101)).astype(np.uint8)
    perm, off = oracle.cluster_permutation(a, 6)
    for b in range(3):
        assert np.array_equal(np.sort(perm[b]), np.arange(101))
        assert np.array_equal(perm[b], np.argsort(a[b], kind="stable"))
        assert np.array_equal(np.diff(off[b]), np.bincount(a[b], minlength=6))
        assert off[b, 0] == 0 and off[b, -1] == 101


def test_top_p_on_closed_form_weights():
    d = 4
    cq = np.zeros((1, 1, d), np.float32)
    cq[0, 0, 0] = 1.0
    # equal scores, sizes 3 : 1 : 0 -> weights 3/4, 1/4, 0 (the empty cluster never counts)
    ck = np.zeros((1, 3, d), np.float32)
    ck[0, :, 0] = 2.0
    nk = np.array([[3, 1, 0]], np.int32)
    sel, w = oracle.select_top_p(cq, ck, nk, scale=0.5, p=0.7, want_weight=True)
    assert np.allclose(w[0, 0], [0.75, 0.25, 0.0])
    assert int(sel[0, 0]) == 0b001
    assert int(oracle.select_top_p(cq, ck, nk, 0.5, 0.8)[0, 0]) == 0b011
    assert int(oracle.select_top_p(cq, ck, nk, 0.5, 1.0)[0, 0]) == 0b011
    # equal sizes, scores s_j = scale * t_j: weights proportional to exp(scale * t_j)
    ck2 = np.zeros((1, 3, d), np.float32)
    ck2[0, :, 0] = [0.0, 2.0, 1.0]
    nk2 = np.array([[1, 1, 1]], np.int32)
    _, w2 = oracle.select_top_p(cq, ck2, nk2, 1.0, 0.5, want_weight=True)
    e = np.exp([0.0, 2.0, 1.0])
    assert np.allclose(w2[0, 0], e / e.sum())
    # the largest weight alone exceeds 0.5 -> only cluster 1; p just above it adds cluster 2
    assert int(oracle.select_top_p(cq, ck2, nk2, 1.0, 0.5)[0, 0]) == 0b010
    assert int(oracle.select_top_p(cq, ck2, nk2, 1.0, e[1] / e.sum() + 1e-3)[0, 0]) == 0b110


def _small(seed=4, H=2, F=3, S=16, T=5, d=32):
    rng = np.random.Generator(np.random.PCG64(seed))
    Lv = F * S
    L = Lv + T
    q, k, v = (W.to_bf16_bits(rng.standard_normal((1, H, L, d)).astype(np.float32)) for _ in range(3))
    return q, k, v, Lv, L, d


def test_attention2_with_every_cluster_selected_is_dense_attention():
    q, k, v, Lv, L, d = _small()
    _, aq, _ = oracle.kmeans(q, Lv, 4, 2)
    _, ak, nk = oracle.kmeans(k, Lv, 5, 2)
    sel = np.full((2, 4), (1 << 5) - 1, np.uint64)
    rows = np.arange(2 * L, dtype=np.int64)
    got = oracle.attention2_rows(q, k, v, Lv, aq, ak, sel, rows)
    qf, kf, vf = (W.bf16_bits_to_f32(t[0]).astype(np.float64) for t in (q, k, v))
    for h in range(2):
        s = qf[h] @ kf[h].T / np.sqrt(d)
        p = np.exp(s - s.max(1, keepdims=True))
        ref = (p / p.sum(1, keepdims=True)) @ vf[h]
        assert np.allclose(got[h * L:(h + 1) * L], ref, rtol=1e-10, atol=1e-12)


def test_attention2_matches_numpy_with_the_cluster_mask():
    q, k, v, Lv, L, d = _small(seed=8)
    _, aq, _ = oracle.kmeans(q, Lv, 3, 1)
    _, ak, _ = oracle.kmeans(k, Lv, 4, 1)
    sel = np.array([[0b0001, 0b0110, 0b1000], [0b0011, 0b0100, 0b1001]], np.uint64)
    rows = np.arange(2 * L, dtype=np.int64)
    got, lse = oracle.attention2_rows(q, k, v, Lv, aq, ak, sel, rows, want_lse=True)
    qf, kf, vf = (W.bf16_bits_to_f32(t[0]).astype(np.float64) for t in (q, k, v))
    for h in range(2):
        keep = np.ones((L, L), bool)
        for qq in range(Lv):
            for kk in range(Lv):
                keep[qq, kk] = bool((int(sel[h, aq[h, qq]]) >> int(ak[h, kk])) & 1)
        s = np.where(keep, qf[h] @ kf[h].T / np.sqrt(d), -np.inf)
        m = s.max(1, keepdims=True)
        p = np.exp(s - m)
        ref = (p / p.sum(1, keepdims=True)) @ vf[h]
        assert np.allclose(got[h * L:(h + 1) * L], ref, rtol=1e-10, atol=1e-12)
        assert np.allclose(lse[h * L:(h + 1) * L], m[:, 0] + np.log(p.sum(1)), rtol=1e-12)


def test_block_list2_covers_exactly_the_kept_pairs():
    q, k, v, Lv, L, d = _small(seed=6, S=40, F=4, T=9)
    _, aq, _ = oracle.kmeans(q, Lv, 5, 2)
    _, ak, _ = oracle.kmeans(k, Lv, 6, 2)
    pq, _ = oracle.cluster_permutation(aq, 5)
    pk, _ = oracle.cluster_permutation(ak, 6)
    rng = np.random.Generator(np.random.PCG64(1))
    sel = rng.integers(1, 1 << 6, size=(2, 5)).astype(np.uint64)
    bq, bk = 32, 16
    rp, col, full = oracle.block_list2(L, Lv, bq, bk, aq, ak, pq, pk, sel)
    nqb, nkb = -(-L // bq), -(-L // bk)
    for h in range(2):
        # the kept mask in permuted coordinates
        keep = np.ones((L, L), bool)
        for qq in range(Lv):
            for kk in range(Lv):
                keep[qq, kk] = bool((int(sel[h, aq[h, pq[h, qq]]]) >> int(ak[h, pk[h, kk]])) & 1)
        for qb in range(nqb):
            e0, e1 = rp[h * nqb + qb], rp[h * nqb + qb + 1]
            listed = dict(zip(col[e0:e1].tolist(), full[e0:e1].tolist()))
            for kb in range(nkb):
                t = keep[qb * bq:(qb + 1) * bq, kb * bk:(kb + 1) * bk]
                assert (kb in listed) == bool(t.any())
                if kb in listed:
                    assert listed[kb] == int(t.all())


def test_permute_rows_is_a_row_permutation_and_its_inverse_restores():
    """oracle.permute_rows: the identity changes nothing, text rows stay, every
    video row appears once, and the inverse permutation (argsort) restores
    the input bit for bit."""
    q, k, v, Lv, L, d = _small(seed=12, S=10, F=3, T=4)
    ident = np.tile(np.arange(Lv, dtype=np.int32), (2, 1))
    assert np.array_equal(oracle.permute_rows(q, Lv, ident), q)
    rng = np.random.Generator(np.random.PCG64(4))
    perm = np.stack([rng.permutation(Lv) for _ in range(2)]).astype(np.int32)
    p = oracle.permute_rows(q, Lv, perm)
    assert np.array_equal(p[0, :, Lv:], q[0, :, Lv:])
    for h in range(2):
        assert np.array_equal(p[0, h, :Lv], q[0, h, perm[h]])
        assert sorted(map(bytes, p[0, h, :Lv])) == sorted(map(bytes, q[0, h, :Lv]))
    inv = np.argsort(perm, axis=1).astype(np.int32)
    assert np.array_equal(oracle.permute_rows(p, Lv, inv), q)


def test_block_list2_bounds_the_closed_form_kept_pair_count():
    """Independent of the mask: the kept pairs, from the cluster sizes alone
    (a video query of cluster i keeps the keys of its selected clusters and
    the text keys; a text query keeps all L), lie between the area of the
    tiles marked full and the area of the listed tiles.  One cluster with
    its set selected lists every tile as full; empty sets without text list
    nothing."""
    q, k, v, Lv, L, d = _small(seed=14, S=30, F=4, T=7)
    _, aq, nq = oracle.kmeans(q, Lv, 5, 2)
    _, ak, nk = oracle.kmeans(k, Lv, 6, 2)
    pq, _ = oracle.cluster_permutation(aq, 5)
    pk, _ = oracle.cluster_permutation(ak, 6)
    rng = np.random.Generator(np.random.PCG64(6))
    sel = rng.integers(1, 1 << 6, size=(2, 5)).astype(np.uint64)
    bq, bk = 32, 16
    rp, col, full = oracle.block_list2(L, Lv, bq, bk, aq, ak, pq, pk, sel)
    nqb = -(-L // bq)
    for h in range(2):
        kept = sum(int(nq[h, i]) * (sum(int(nk[h, j]) for j in range(6) if (int(sel[h, i]) >> j) & 1) + (L - Lv))
                   for i in range(5)) + (L - Lv) * L
        listed_area = full_area = 0
        for qb in range(nqb):
            rows = min(bq, L - qb * bq)
            for e in range(rp[h * nqb + qb], rp[h * nqb + qb + 1]):
                a = rows * min(bk, L - int(col[e]) * bk)
                listed_area += a
                full_area += a if full[e] else 0
        assert full_area <= kept <= listed_area
    one = np.zeros_like(aq)
    ident = np.tile(np.arange(Lv, dtype=np.int32), (2, 1))
    rp1, col1, full1 = oracle.block_list2(L, Lv, bq, bk, one, one, ident, ident, np.ones((2, 1), np.uint64))
    nkb = -(-L // bk)
    assert len(col1) == 2 * nqb * nkb and full1.all()
    q0, k0, v0, Lv0, L0, _ = _small(seed=15, S=30, F=2, T=0)
    _, a0, _ = oracle.kmeans(q0, Lv0, 3, 1)
    p0, _ = oracle.cluster_permutation(a0, 3)
    rp0, col0, _ = oracle.block_list2(L0, Lv0, bq, bk, a0, a0, p0, p0, np.zeros((2, 3), np.uint64))
    assert len(col0) == 0 and (rp0 == 0).all()
