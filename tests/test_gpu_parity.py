"""Parity of every stage of the CUDA path with the fp64 oracle, through the C ABI.

Bars (exactness where the stage is integer/bit work, the attention tolerance
for floating point):
  * QK-Norm + RoPE: within 1 bf16 ulp of the oracle's rounded fp64 result plus
    2^-20 of the RoPE pair's norm (fp32 cancellation), >= 99% bit-equal;
  * layout / inverse layout, block index lists, head choices: bit-exact;
  * attention: max-abs <= 2e-2 and mean-abs <= 2e-3 against fp64, on the
    oracle's own normalised inputs.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_video_qk_b200 as svg
import svg_workloads as W
from gpu_util import assert_attention_close, assert_norm_rope_close, dev, f64, host_bits

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


@functools.lru_cache(maxsize=None)
def case(key):
    """Inputs and oracle stage-1 results of a named case (cached)."""
    wl = CASES[key]
    inp = W.make_inputs(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    qn = oracle.qknorm_rope(sh, pr, inp["q"], inp["gamma_q"])
    kn = oracle.qknorm_rope(sh, pr, inp["k"], inp["gamma_k"])
    return wl, inp, qn, kn


@functools.lru_cache(maxsize=None)
def profile_ref(key):
    """Oracle profiling of a named case: (mse [BH, 2], kinds [BH]) (cached)."""
    wl, inp, qn, kn = case(key)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    return oracle.profile(sh, pr, qn, kn, inp["v"], inp["sample_idx"])


CASES = {
    "tiny": W.TINY,
    "cogvideox": W.COGVIDEOX,
    "wan": W.WAN,
    "hunyuan": W.HUNYUAN,
    # ragged: L = 116 is a multiple of neither tile size; text present; d = 128
    "ragged128": W.small_workload(d=128, H=3, F=3, Hs=5, Ws=7, T=11, w=1, r=6, n_samples=12, bq=128),
    # tiny: L = 11 < one tile
    "tiny64": W.small_workload(d=64, H=2, F=1, Hs=2, Ws=3, T=5, w=0, r=1, n_samples=4, bq=64),
    # several frames per key tile (S = 20), bq = 64
    "smallS": W.small_workload(d=64, H=4, F=9, Hs=4, Ws=5, T=3, w=2, r=4, n_samples=16, bq=64),
    # the same grid with d = 128, and without text (the last key tile's second half is past L)
    "smallS128": W.small_workload(d=128, H=4, F=9, Hs=4, Ws=5, T=3, w=2, r=4, n_samples=16, bq=128),
    "smallS_T0": W.small_workload(d=64, H=4, F=9, Hs=4, Ws=5, T=0, w=2, r=4, n_samples=16, bq=64),
    # one frame: the temporal layout is the identity
    "oneframe": W.small_workload(d=128, H=2, F=1, Hs=12, Ws=20, T=7, w=0, r=30, n_samples=8),
    # wide windows that reduce to dense
    "wide": W.small_workload(d=64, H=2, F=5, Hs=6, Ws=7, T=9, w=4, r=41, n_samples=8),
    # RoPE sections not multiples of 8 wide: a lane's 4 pairs straddle two sections
    "oddsplit": W.small_workload(d=64, H=2, F=4, Hs=5, Ws=6, T=3, w=1, r=4, n_samples=8, rope_split=(18, 22, 24)),
    # two batch entries: every per-head index runs over b*H + h
    "batch2": W.small_workload(B=2, d=128, H=2, F=3, Hs=4, Ws=6, T=5, w=1, r=3, n_samples=8, bq=128),
}
FULL_ROW_CASES = ("tiny", "ragged128", "tiny64", "smallS", "smallS128", "smallS_T0", "oneframe", "wide",
                  "oddsplit", "batch2")


def pb_of(wl):
    return svg.Problem.from_workload(wl)


def mixed_kinds(H):
    return np.array([(W.SPATIAL, W.TEMPORAL, W.DENSE)[h % 3] for h in range(H)], np.uint8)


def rows_for(key, wl):
    if key in FULL_ROW_CASES:
        return np.arange(wl.B * wl.H * wl.L, dtype=np.int64)
    if key == "hunyuan":
        return W.random_rows(wl, 48, seed=11, max_boundary_tiles=1)
    return W.random_rows(wl, 96, seed=11, max_boundary_tiles=3)


# ------------------------------------------------------------ QK-Norm + RoPE

@pytest.mark.parametrize("key", ["tiny", "cogvideox", "wan", "ragged128", "tiny64", "oneframe", "oddsplit", "batch2"])
def test_qknorm_rope_within_one_ulp(key):
    wl, inp, qn_ref, kn_ref = case(key)
    pb = pb_of(wl)
    table = dev(svg.rope_table(pb))
    qn, kn = svg.qknorm_rope(pb, dev(inp["q"]), dev(inp["k"]), dev(inp["gamma_q"]), dev(inp["gamma_k"]), table)
    svg.sync_status()
    for got, ref, name in ((host_bits(qn), qn_ref, "q"), (host_bits(kn), kn_ref, "k")):
        assert_norm_rope_close(got, ref, f"{key}/{name}")


def test_qknorm_rope_hunyuan_sampled_rows():
    wl = W.HUNYUAN
    inp = W.make_inputs(wl)
    pb = pb_of(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    rows = W.random_rows(wl, 256, seed=5, max_boundary_tiles=2)
    qn, kn = svg.qknorm_rope(pb, dev(inp["q"]), dev(inp["k"]), dev(inp["gamma_q"]), dev(inp["gamma_k"]),
                             dev(svg.rope_table(pb)))
    svg.sync_status()
    for got_t, x, gname in ((qn, inp["q"], "gamma_q"), (kn, inp["k"], "gamma_k")):
        got = host_bits(got_t).reshape(-1, wl.d)[rows]
        ref = oracle.f64_to_bf16(oracle.qknorm_rope_f64(sh, pr, x, inp[gname], rows))
        assert_norm_rope_close(got, ref, gname)


# ------------------------------------------------------------------ layout

@pytest.mark.parametrize("key", ["tiny", "cogvideox", "wan", "ragged128", "tiny64", "smallS", "oneframe", "batch2"])
def test_layout_and_inverse_bit_exact(key):
    wl, inp, _, _ = case(key)
    pb = pb_of(wl)
    sh = oracle.shape_of(wl)
    kinds = mixed_kinds(wl.B * wl.H)
    q, k, v = dev(inp["q"]), dev(inp["k"]), dev(inp["v"])
    qp, kp, vp = svg.layout(pb, q, k, v, dev(kinds))
    back = svg.inverse_layout(pb, dev(kinds), qp)
    svg.sync_status()
    for got, name in ((qp, "q"), (kp, "k"), (vp, "v")):
        assert np.array_equal(host_bits(got), oracle.layout(sh, kinds, inp[name])), name
    assert np.array_equal(host_bits(back), inp["q"])
    assert np.array_equal(host_bits(svg.inverse_layout(pb, dev(kinds), vp)),
                          oracle.layout(sh, kinds, oracle.layout(sh, kinds, inp["v"]), inverse=True))


@pytest.mark.parametrize("key", ["tiny", "ragged128", "smallS"])
def test_fused_norm_rope_layout(key):
    """flags = NORM_ROPE | LAYOUT equals the two separate passes bit for bit."""
    wl, inp, _, _ = case(key)
    pb = pb_of(wl)
    kinds = dev(mixed_kinds(wl.B * wl.H))
    args = (dev(inp["q"]), dev(inp["k"]))
    g = (dev(inp["gamma_q"]), dev(inp["gamma_k"]), dev(svg.rope_table(pb)))
    qn, kn = svg.qknorm_rope(pb, *args, *g)
    two = svg.layout(pb, qn, kn, dev(inp["v"]), kinds)
    one = svg.qknorm_rope_layout(pb, *args, dev(inp["v"]), *g, kinds, flags=3)
    svg.sync_status()
    for a, b in zip(one, two):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


# ------------------------------------------------------------- block index

def csr_host(row_ptr, col, full):
    rp = row_ptr.cpu().numpy()
    nnz = int(rp[-1])
    return rp, col[:nnz].cpu().numpy(), full[:nnz].cpu().numpy()


@pytest.mark.parametrize("key,kinds_mode", [("tiny", "mixed"), ("cogvideox", "mixed"), ("wan", "mixed"),
                                            ("ragged128", "mixed"), ("tiny64", "mixed"), ("smallS", "mixed"),
                                            ("oneframe", "mixed"), ("wide", "mixed"), ("batch2", "mixed"),
                                            ("hunyuan", "planted")])
def test_block_index_bit_exact(key, kinds_mode):
    wl = CASES[key]
    pb = pb_of(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    kinds = mixed_kinds(wl.B * wl.H) if kinds_mode == "mixed" else \
        np.array([W.SPATIAL if c == "S" else W.TEMPORAL for c in wl.planted], np.uint8)
    rp, col, full = csr_host(*svg.build_block_index(pb, dev(kinds)))
    svg.sync_status()
    rp_ref, col_ref, full_ref = oracle.block_list(sh, pr, kinds)
    assert np.array_equal(rp, rp_ref)
    assert np.array_equal(col, col_ref)
    assert np.array_equal(full, full_ref)


def test_block_index_capacity_overflow_is_reported():
    wl = CASES["smallS"]
    pb = pb_of(wl)
    kinds = dev(np.full(wl.H, W.DENSE, np.uint8))
    need = wl.H * wl.nqb * wl.nkb
    cap = need // 2
    col = torch.full((need,), -7, dtype=torch.int32, device="cuda")
    full = torch.zeros(need, dtype=torch.uint8, device="cuda")
    row_ptr = torch.empty(wl.H * wl.nqb + 1, dtype=torch.int32, device="cuda")
    svg.build_block_index(pb, kinds, capacity=cap, out=(row_ptr, col, full))
    with pytest.raises(svg.SVGError) as e:
        svg.sync_status()
    assert e.value.status == 5
    assert (col[cap:].cpu().numpy() == -7).all()          # nothing written past capacity
    svg.sync_status()                                     # the error word was cleared


# --------------------------------------------------------------- profiling

@pytest.mark.parametrize("key", ["tiny", "cogvideox", "wan", "smallS", "smallS128", "smallS_T0", "ragged128", "batch2",
                                 "hunyuan"])
def test_profile_choices_bit_exact(key):
    wl, inp, qn, kn = case(key)
    pb = pb_of(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    mse_ref, kinds_ref = profile_ref(key)
    kinds, mse = svg.profile_heads(pb, dev(qn), dev(kn), dev(inp["v"]), dev(inp["sample_idx"]))
    svg.sync_status()
    kinds = kinds.cpu().numpy()
    mse = mse.cpu().numpy().astype(np.float64)
    gap = np.abs(mse_ref[:, 0] - mse_ref[:, 1]) / mse_ref.max(1)
    near_tie = gap < 1e-4
    assert np.array_equal(kinds[~near_tie], kinds_ref[~near_tie]), (kinds, kinds_ref, gap)
    assert near_tie.sum() == 0, f"near-ties: {np.nonzero(near_tie)[0]}"
    rel = np.abs(mse - mse_ref) / mse_ref
    assert rel.max() < 2e-2, rel.max()
    planted = inp["planted"]
    if key in ("tiny", "wan", "hunyuan"):
        sel = planted != 255
        assert np.array_equal(kinds[sel], planted[sel])


def test_profile_bad_sample_index_reported():
    wl, inp, qn, kn = case("tiny")
    pb = pb_of(wl)
    bad = inp["sample_idx"].copy()
    bad[3] = wl.L + 5
    svg.profile_heads(pb, dev(qn), dev(kn), dev(inp["v"]), dev(bad))
    with pytest.raises(svg.SVGError) as e:
        svg.sync_status()
    assert e.value.status == 1


# --------------------------------------------------------------- attention

def run_sparse(wl, qn, kn, v, kinds, want_lse=False, model_order=False):
    """Layout, block index and attention; the output comes back in model
    order either through the inverse-layout pass or (model_order=True) from
    the attention epilogue.  LSE is in the head's layout unless model_order."""
    pb = pb_of(wl)
    kd = dev(kinds)
    qp, kp, vp = svg.layout(pb, dev(qn), dev(kn), dev(v), kd)
    row_ptr, col, full = svg.build_block_index(pb, kd)
    res = svg.block_sparse_attn(pb, qp, kp, vp, kd, row_ptr, col, full, want_lse=want_lse, model_order=model_order)
    op, lse = res if want_lse else (res, None)
    out = op if model_order else svg.inverse_layout(pb, kd, op)
    svg.sync_status()
    return out, lse


@pytest.mark.parametrize("key", ["tiny", "ragged128", "tiny64", "smallS", "smallS128", "smallS_T0", "oneframe", "wide",
                                 "batch2", "cogvideox", "wan"])
@pytest.mark.parametrize("kinds_mode", ["mixed", "spatial", "temporal"])
def test_attention_parity(key, kinds_mode):
    wl, inp, qn, kn = case(key)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    kinds = {"mixed": mixed_kinds(wl.B * wl.H), "spatial": np.zeros(wl.B * wl.H, np.uint8),
             "temporal": np.ones(wl.B * wl.H, np.uint8)}[kinds_mode]
    out, lse = run_sparse(wl, qn, kn, inp["v"], kinds, want_lse=True)
    rows = rows_for(key, wl)
    ref, ref_lse = oracle.attention_rows(sh, pr, kinds, qn, kn, inp["v"], rows, want_lse=True)
    got = host_bits(out).reshape(-1, wl.d)[rows]
    assert_attention_close(got, ref, MAX_ABS, MEAN_ABS, f"{key}/{kinds_mode}")
    # LSE is stored in the head's layout order
    lse_h = lse.cpu().numpy().reshape(wl.B * wl.H, wl.L)
    bh, tok = rows // wl.L, rows % wl.L
    pos = np.array([oracle.perm(sh, int(kinds[b]), int(t)) for b, t in zip(bh, tok)])
    assert np.abs(lse_h[bh, pos] - ref_lse).max() < 5e-3


@pytest.mark.parametrize("key", ["tiny", "ragged128", "smallS128", "wan"])
def test_attention_model_order_equals_inverse_layout_pass(key):
    """The inverse layout fused into the attention epilogue stores exactly
    the bits the separate pass produces, and the LSE at the same positions."""
    wl, inp, qn, kn = case(key)
    sh = oracle.shape_of(wl)
    kinds = mixed_kinds(wl.B * wl.H)
    out_a, lse_a = run_sparse(wl, qn, kn, inp["v"], kinds, want_lse=True)
    out_b, lse_b = run_sparse(wl, qn, kn, inp["v"], kinds, want_lse=True, model_order=True)
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
    lse_a = lse_a.cpu().numpy().reshape(wl.B * wl.H, wl.L)
    lse_b = lse_b.cpu().numpy().reshape(wl.B * wl.H, wl.L)
    for bh in range(wl.B * wl.H):
        pos = np.array([oracle.perm(sh, int(kinds[bh]), t) for t in range(wl.L)])
        assert np.array_equal(lse_b[bh], lse_a[bh, pos])


def test_attention_dense_kinds_equal_dense_attention():
    wl, inp, qn, kn = case("smallS")
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    kinds = np.full(wl.H, W.DENSE, np.uint8)
    out, _ = run_sparse(wl, qn, kn, inp["v"], kinds)
    rows = np.arange(wl.H * wl.L, dtype=np.int64)
    ref = oracle.attention_rows(sh, pr, kinds, qn, kn, inp["v"], rows)
    assert_attention_close(host_bits(out).reshape(-1, wl.d), ref, MAX_ABS, MEAN_ABS, "dense")


def test_attention_hunyuan_sampled_rows():
    wl, inp, qn, kn = case("hunyuan")
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    kinds = np.array([W.SPATIAL if c == "S" else W.TEMPORAL for c in wl.planted], np.uint8)
    out, _ = run_sparse(wl, qn, kn, inp["v"], kinds, model_order=True)     # the launch bench.py times
    rows = rows_for("hunyuan", wl)
    ref = oracle.attention_rows(sh, pr, kinds, qn, kn, inp["v"], rows)
    assert_attention_close(host_bits(out).reshape(-1, wl.d)[rows], ref, MAX_ABS, MEAN_ABS, "hunyuan")


# ----------------------------------------------------------- sparsity sweep

SWEEP = dict(W.sweep_points())


@functools.lru_cache(maxsize=None)
def sweep_case():
    """Inputs of the sparsity sweep (the HunyuanVideo shape) and the oracle's
    QK-Norm + RoPE of them; every sweep point shares them."""
    wl = W.HUNYUAN_SWEEP
    inp = W.make_inputs(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    return inp, oracle.qknorm_rope(sh, pr, inp["q"], inp["gamma_q"]), oracle.qknorm_rope(sh, pr, inp["k"],
                                                                                            inp["gamma_k"])


@pytest.mark.parametrize("point", list(SWEEP))
def test_sparsity_sweep_point(point):
    """Every point of the sparsity sweep at the HunyuanVideo 720p shape (all 24
    heads forced to one kind; spatial windows 0-8 frames, temporal radii
    32-1800): the block index bit-exact against the oracle's brute-force tile
    list, and the attention launch bench.py times (layout, then attention with
    the inverse layout in its epilogue) on sampled rows within 2e-2 / 2e-3."""
    wl = SWEEP[point]
    inp, qn, kn = sweep_case()
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    kinds = np.array(wl.forced_kinds, np.uint8)
    rp, col, full = csr_host(*svg.build_block_index(pb_of(wl), dev(kinds)))
    svg.sync_status()
    rp_ref, col_ref, full_ref = oracle.block_list(sh, pr, kinds)
    assert np.array_equal(rp, rp_ref) and np.array_equal(col, col_ref) and np.array_equal(full, full_ref), point
    out, _ = run_sparse(wl, qn, kn, inp["v"], kinds, model_order=True)
    rows = W.random_rows(wl, 32, seed=19, max_boundary_tiles=1)
    ref = oracle.attention_rows(sh, pr, kinds, qn, kn, inp["v"], rows)
    assert_attention_close(host_bits(out).reshape(-1, wl.d)[rows], ref, MAX_ABS, MEAN_ABS, point)


# ---------------------------------------------------------------- full step

@pytest.mark.parametrize("key,head_layout_out", [("tiny", False), ("smallS", False), ("batch2", False),
                                                  ("cogvideox", False), ("wan", False), ("tiny", True), ("wan", True),
                                                  ("hunyuan", False)])
def test_full_step_end_to_end(key, head_layout_out):
    """The whole five-pass step (the HunyuanVideo shape: the workload and launches bench.py
    times) against the oracle: head kinds bit-exact, sampled output rows."""
    wl, inp, qn, kn = case(key)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    pb = pb_of(wl)
    buf = svg.StepBuffers(pb, wl.n_samples, head_layout_out=head_layout_out)
    out = svg.attention_step(pb, dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["gamma_q"]),
                             dev(inp["gamma_k"]), dev(inp["sample_idx"]), buf)
    svg.sync_status()
    _, kinds_ref = profile_ref(key)
    assert np.array_equal(buf.kinds.cpu().numpy(), kinds_ref)
    rows = rows_for(key, wl)
    ref = oracle.attention_rows(sh, pr, kinds_ref, qn, kn, inp["v"], rows)
    assert_attention_close(host_bits(out).reshape(-1, wl.d)[rows], ref, MAX_ABS, MEAN_ABS, key)


@pytest.mark.parametrize("key,groups", [("wan", 4), ("wan", 5), ("batch2", 3), ("tiny", 1), ("batch2", 4)])
def test_host_step_groups_match_one_shot_step(key, groups):
    """svg_attention_step_host (head groups copied in, computed and copied out
    on the library's three streams) gives the one-shot device step's bits and
    head kinds, for even and uneven groups, one head per group and B > 1, on
    two calls in a row (the second reuses the workspace)."""
    wl, inp, _, _ = case(key)
    pb = pb_of(wl)
    pin = lambda a: torch.from_numpy(a).view(torch.bfloat16).pin_memory()
    step = svg.HostStep(pb, wl.n_samples, groups=groups)
    args = (pin(inp["q"]), pin(inp["k"]), pin(inp["v"]), torch.from_numpy(inp["gamma_q"]).pin_memory(),
            torch.from_numpy(inp["gamma_k"]).pin_memory(), torch.from_numpy(inp["sample_idx"]).pin_memory())
    kinds_h = torch.empty(wl.B * wl.H, dtype=torch.uint8).pin_memory()
    out_h = step(*args, kinds_out=kinds_h)
    out_h2 = step(*args)
    torch.cuda.synchronize()
    buf = svg.StepBuffers(pb, wl.n_samples)
    out_d = svg.attention_step(pb, *(dev(inp[k]) for k in ("q", "k", "v", "gamma_q", "gamma_k", "sample_idx")), buf)
    svg.sync_status()
    ref = out_d.cpu().view(torch.int16)
    assert torch.equal(out_h.view(torch.int16), ref)
    assert torch.equal(out_h2.view(torch.int16), ref)
    assert torch.equal(kinds_h, buf.kinds.cpu())


def test_release_then_host_step_again():
    """svg_release frees the host step's streams, events and pinned staging;
    the next host step creates them again and gives the same bits."""
    wl, inp, _, _ = case("wan")
    pb = pb_of(wl)
    pin = lambda a: torch.from_numpy(a).view(torch.bfloat16).pin_memory()
    args = (pin(inp["q"]), pin(inp["k"]), pin(inp["v"]), torch.from_numpy(inp["gamma_q"]).pin_memory(),
            torch.from_numpy(inp["gamma_k"]).pin_memory(), torch.from_numpy(inp["sample_idx"]).pin_memory())
    first = svg.HostStep(pb, wl.n_samples, groups=3)(*args)
    torch.cuda.synchronize()
    first = first.clone()
    svg.release()
    second = svg.HostStep(pb, wl.n_samples, groups=3)(*args)
    torch.cuda.synchronize()
    assert torch.equal(first.view(torch.int16), second.view(torch.int16))
    svg.release()


def test_host_buffer_api_matches_device_api():
    wl, inp, _, _ = case("tiny")
    pb = pb_of(wl)
    pin = lambda a: torch.from_numpy(a).view(torch.bfloat16).pin_memory()
    out_h = svg.sparse_attention(pb, pin(inp["q"]), pin(inp["k"]), pin(inp["v"]), torch.from_numpy(inp["gamma_q"]),
                                 torch.from_numpy(inp["gamma_k"]), torch.from_numpy(inp["sample_idx"]))
    torch.cuda.synchronize()
    buf = svg.StepBuffers(pb, wl.n_samples)
    out_d = svg.attention_step(pb, dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["gamma_q"]),
                               dev(inp["gamma_k"]), dev(inp["sample_idx"]), buf)
    svg.sync_status()
    assert torch.equal(out_h.view(torch.int16), out_d.cpu().view(torch.int16))


def test_layer_schedule_dense_then_profiled_then_reused():
    """SparseAttentionLayer over 4 denoising steps: step 0 dense, step 1
    profiled, step 2 reuses step 1's kinds, step 3 profiles again."""
    wl, inp, qn, kn = case("tiny")
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    layer = svg.SparseAttentionLayer(pb_of(wl), wl.n_samples, total_steps=4, dense_fraction=0.25, reprofile_every=2)
    args = tuple(dev(inp[k]) for k in ("q", "k", "v", "gamma_q", "gamma_k", "sample_idx"))
    _, kinds_ref = oracle.profile(sh, pr, qn, kn, inp["v"], inp["sample_idx"])
    rows = rows_for("tiny", wl)
    modes = [svg.STEP_DENSE, svg.STEP_PROFILE, svg.STEP_REUSE, svg.STEP_PROFILE]
    for t in range(4):
        out = layer(t, *args)
        svg.sync_status()
        assert layer.last_mode == modes[t]
        kinds = np.full(wl.B * wl.H, W.DENSE, np.uint8) if t == 0 else kinds_ref
        ref = oracle.attention_rows(sh, pr, kinds, qn, kn, inp["v"], rows)
        assert_attention_close(host_bits(out).reshape(-1, wl.d)[rows], ref, MAX_ABS, MEAN_ABS, f"step {t}")
    assert np.array_equal(layer.kinds.cpu().numpy(), kinds_ref)


# ------------------------------------------- five-pass step building blocks

@pytest.mark.parametrize("key", ["tiny", "ragged128", "smallS", "oddsplit", "wan"])
def test_selective_norm_passes_match_the_two_stage_path(key):
    """K alone, and {raw Q normalised + K, V moved} in one pass, give the same
    bits as normalising both and then moving all three."""
    wl, inp, _, _ = case(key)
    pb = pb_of(wl)
    table = torch.from_numpy(svg.rope_table(pb)).cuda()
    q, k, v = dev(inp["q"]), dev(inp["k"]), dev(inp["v"])
    gq, gk = dev(inp["gamma_q"]), dev(inp["gamma_k"])
    kd = dev(mixed_kinds(wl.B * wl.H))
    qn, kn = svg.qknorm_rope(pb, q, k, gq, gk, table)
    ref = svg.layout(pb, qn, kn, v, kd)
    _, kn_only, _ = svg.qknorm_rope_layout(pb, None, k, None, None, gk, table, None, 1)
    fused = svg.qknorm_rope_layout(pb, q, kn_only, v, gq, None, table, kd, 3)
    svg.sync_status()
    assert torch.equal(kn_only.view(torch.int16), kn.view(torch.int16))
    for a, b in zip(fused, ref):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("key", ["tiny", "ragged128", "smallS128", "oddsplit", "wan"])
def test_profile_raw_q_equals_profile_on_normalised_q(key):
    """The sampled rows normalised inside the profiling kernel are the rows the
    norm pass writes, so kinds and MSEs agree bit for bit."""
    wl, inp, _, _ = case(key)
    pb = pb_of(wl)
    table = torch.from_numpy(svg.rope_table(pb)).cuda()
    q, k, v = dev(inp["q"]), dev(inp["k"]), dev(inp["v"])
    gq, gk, si = dev(inp["gamma_q"]), dev(inp["gamma_k"]), dev(inp["sample_idx"])
    qn, kn = svg.qknorm_rope(pb, q, k, gq, gk, table)
    kinds_a, mse_a = svg.profile_heads(pb, qn, kn, v, si)
    kinds_b, mse_b = svg.profile_heads_raw_q(pb, q, gq, table, kn, v, si)
    svg.sync_status()
    assert torch.equal(kinds_a, kinds_b)
    assert torch.equal(mse_a.view(torch.int32), mse_b.view(torch.int32))
