"""Pins of the AdaSpa oracle ("AdaSpa" abstract: blockified pattern, fused
LSE-cached search, head-adaptive hierarchical block sparse attention): block
masses against closed forms and the softmax normalisation, top-p selection on
exact binary fractions, and block attention against numpy."""
import numpy as np

import oracle
import svg_workloads as W


def _qkv(B=1, H=2, L=70, d=16, seed=0, scale=1.0):
    rng = np.random.Generator(np.random.PCG64(seed))
    return tuple(W.to_bf16_bits((rng.standard_normal((B, H, L, d)) * scale).astype(np.float32)) for _ in range(3))


def _dense_lse(q, k):
    """log-sum-exp of every row over all keys, by numpy (fp64)."""
    qf = W.bf16_bits_to_f32(q).astype(np.float64)
    kf = W.bf16_bits_to_f32(k).astype(np.float64)
    s = np.einsum("bhqd,bhkd->bhqk", qf, kf) / np.sqrt(q.shape[-1])
    m = s.max(-1, keepdims=True)
    return (m[..., 0] + np.log(np.exp(s - m).sum(-1))).astype(np.float32)


def test_mass_of_zero_queries_is_the_key_count_over_L():
    """q = 0: every score is 0, lse = log L, so a block's mass is rows * cols / L."""
    q, k, _ = _qkv(L=70)
    q[:] = 0
    L, bq, bk = 70, 16, 8
    lse = np.full((1, 2, L), np.log(L), np.float32)
    m = oracle.block_mass(q, k, lse, bq, bk)
    rows = np.minimum(bq, L - np.arange(-(-L // bq)) * bq)
    cols = np.minimum(bk, L - np.arange(-(-L // bk)) * bk)
    want = rows[:, None] * cols[None, :] / L * np.exp(np.log(L) - np.float32(np.log(L)))
    assert np.allclose(m[0], want, rtol=1e-12)
    assert np.allclose(m[1], want, rtol=1e-12)


def test_masses_of_a_tile_sum_to_its_rows_with_the_exact_lse():
    """Each row's weights exp(s - lse) sum to 1 when lse is its log-sum-exp."""
    q, k, _ = _qkv(L=83, d=32, seed=3, scale=2.0)
    lse = _dense_lse(q, k)
    bq, bk = 32, 16
    m = oracle.block_mass(q, k, lse, bq, bk)
    rows = np.minimum(bq, 83 - np.arange(-(-83 // bq)) * bq)
    # lse was rounded to float: each row sums to exp(lse64 - lse32) = 1 within ~1e-7
    assert np.allclose(m.sum(-1), rows[None, :], rtol=2e-7)


def test_mass_matches_per_pair_weights_on_a_tiny_case():
    q, k, _ = _qkv(L=12, d=8, seed=5)
    lse = np.zeros((1, 2, 12), np.float32) + np.float32(0.25)
    m = oracle.block_mass(q, k, lse, 4, 3)
    qf = W.bf16_bits_to_f32(q[0]).astype(np.float64)
    kf = W.bf16_bits_to_f32(k[0]).astype(np.float64)
    for h in range(2):
        for qb in range(3):
            for kb in range(4):
                tot = 0.0
                for qq in range(qb * 4, qb * 4 + 4):
                    for kk in range(kb * 3, kb * 3 + 3):
                        tot += np.exp(float(qf[h, qq] @ kf[h, kk]) / np.sqrt(8) - 0.25)
                assert abs(m[h, qb, kb] - tot) <= 1e-12 * tot


def _one_tile(masses, text_cols=0, L=None, bq=8, bk=4):
    """float32 masses [1, nqb, nkb] with the first query tile's video masses given."""
    nkb_v = len(masses)
    Lv = nkb_v * bk
    L = L or Lv + text_cols
    nqb, nkb = -(-L // bq), -(-L // bk)
    m = np.zeros((1, nqb, nkb), np.float32)
    m[0, 0, :nkb_v] = masses
    return m, L, Lv, bq, bk


def _kept(rp, col, t):
    return col[rp[t]:rp[t + 1]].tolist()


def test_select_on_exact_binary_fractions():
    # video tiles 0..3 with masses 1/8, 1/2, 1/4, 1/8 (every running sum exact in double); no text
    m, L, Lv, bq, bk = _one_tile([0.125, 0.5, 0.25, 0.125], bq=16)
    for p, want in ((0.25, [1]), (0.5, [1]), (0.5001, [1, 2]), (0.75, [1, 2]), (0.76, [0, 1, 2]),
                    (0.875, [0, 1, 2]), (0.9, [0, 1, 2, 3]), (1.0, [0, 1, 2, 3])):
        rp, col, full = oracle.adaspa_select(m, L, Lv, bq, bk, p)
        assert _kept(rp, col, 0) == want, p
        assert (full == 1).all()


def test_select_margin_is_the_distance_of_the_cut_from_the_goal():
    """Sorted masses 1/2, 1/4, 1/8, 1/8 (total 1): at p = 0.7 the cut falls
    after 1/2 + 1/4 = 0.75, so the margin is min(0.7 - 0.5, 0.75 - 0.7); at
    p = 0.75 the running sum meets the goal exactly (margin 0); text query
    tiles make no cut (+inf)."""
    m, L, Lv, bq, bk = _one_tile([0.125, 0.5, 0.25, 0.125], text_cols=3, bq=16)
    rp, col, full, margin = oracle.adaspa_select(m, L, Lv, bq, bk, 0.7, want_margin=True)
    assert _kept(rp, col, 0)[:2] == [1, 2]
    assert abs(margin[0] - 0.05) < 1e-15
    assert np.isinf(margin[-1])                          # the last query tile holds the text rows
    _, _, _, m2 = oracle.adaspa_select(m, L, Lv, bq, bk, 0.75, want_margin=True)
    assert m2[0] == 0.0


def test_select_keeps_text_keys_and_text_query_tiles_keep_all():
    # Lv = 16 video keys (4 tiles of 4) + 5 text keys -> key tiles 4 and 5 hold text
    m, L, Lv, bq, bk = _one_tile([0.0, 0.75, 0.25, 0.0], text_cols=5, bq=8)
    nqb, nkb = m.shape[1], m.shape[2]
    rp, col, full = oracle.adaspa_select(m, L, Lv, bq, bk, 0.5)
    assert _kept(rp, col, 0) == [1, 4, 5]
    # query tile 2 holds rows 16..20, text rows: every key tile
    assert _kept(rp, col, nqb - 1) == list(range(nkb))
    # query tile 1 (all masses 0): the heaviest video tile (index 0 on the tie) and the text tiles
    assert _kept(rp, col, 1) == [0, 4, 5]


def test_block_attention_with_every_tile_is_dense_attention():
    q, k, v = _qkv(L=37, d=16, seed=7)
    L, bq, bk = 37, 8, 8
    nqb, nkb = -(-L // bq), -(-L // bk)
    rp = np.arange(0, 2 * nqb * nkb + 1, nkb, dtype=np.int32)
    col = np.tile(np.arange(nkb, dtype=np.int32), 2 * nqb)
    rows = np.arange(2 * L, dtype=np.int64)
    got, lse = oracle.block_attention_rows(q, k, v, bq, bk, rp, col, rows, want_lse=True)
    qf, kf, vf = (W.bf16_bits_to_f32(t[0]).astype(np.float64) for t in (q, k, v))
    for h in range(2):
        s = qf[h] @ kf[h].T / 4.0
        p = np.exp(s - s.max(1, keepdims=True))
        assert np.allclose(got[h * L:(h + 1) * L], (p / p.sum(1, keepdims=True)) @ vf[h], rtol=1e-10, atol=1e-12)
        assert np.allclose(lse[h * L:(h + 1) * L], _dense_lse(q, k)[0, h], rtol=1e-6)


def test_block_attention_matches_a_numpy_block_mask():
    q, k, v = _qkv(L=45, d=16, seed=9)
    L, bq, bk = 45, 16, 8
    nqb, nkb = -(-L // bq), -(-L // bk)
    rng = np.random.Generator(np.random.PCG64(2))
    keep = rng.random((2, nqb, nkb)) < 0.5
    keep[..., 0] = True
    rp = np.concatenate([[0], np.cumsum(keep.reshape(-1, nkb).sum(1))]).astype(np.int32)
    col = np.concatenate([np.nonzero(r)[0] for r in keep.reshape(-1, nkb)]).astype(np.int32)
    rows = np.arange(2 * L, dtype=np.int64)
    got = oracle.block_attention_rows(q, k, v, bq, bk, rp, col, rows)
    qf, kf, vf = (W.bf16_bits_to_f32(t[0]).astype(np.float64) for t in (q, k, v))
    for h in range(2):
        mask = np.repeat(np.repeat(keep[h], bq, 0), bk, 1)[:L, :L]
        s = np.where(mask, qf[h] @ kf[h].T / 4.0, -np.inf)
        p = np.exp(s - s.max(1, keepdims=True))
        assert np.allclose(got[h * L:(h + 1) * L], (p / p.sum(1, keepdims=True)) @ vf[h], rtol=1e-10, atol=1e-12)


def test_search_then_attention_keeps_at_least_p_of_each_tiles_mass():
    """End to end on the oracle: with the exact LSE, the kept video tiles of a
    query tile hold at least p of its video-key mass."""
    q, k, v = _qkv(L=96, d=16, seed=11, scale=1.5)
    L, Lv, bq, bk, p = 96, 96, 16, 8, 0.8
    lse = _dense_lse(q, k)
    m = oracle.block_mass(q, k, lse, bq, bk).astype(np.float32)
    rp, col, _ = oracle.adaspa_select(m, L, Lv, bq, bk, p)
    nqb = m.shape[1]
    for t in range(2 * nqb):
        kept = col[rp[t]:rp[t + 1]]
        mt = m.reshape(-1, m.shape[2])[t].astype(np.float64)
        assert mt[kept].sum() >= p * mt.sum() * (1 - 1e-6)
        # and it is the shortest such set: dropping the lightest kept tile falls below p
        if len(kept) > 1:
            assert mt[kept].sum() - mt[kept].min() < p * mt.sum()


def test_mass_of_chosen_tiles_equals_the_full_computation():
    q, k, _ = _qkv(L=50, d=16, seed=13)
    lse = _dense_lse(q, k)
    full = oracle.block_mass(q, k, lse, 16, 8)
    tiles = np.array([5, 0, 3], np.int64)                 # bh * nqb + qb, nqb = 4
    part = oracle.block_mass(q, k, lse, 16, 8, tiles=tiles)
    assert np.array_equal(part, full.reshape(-1, full.shape[2])[tiles])
