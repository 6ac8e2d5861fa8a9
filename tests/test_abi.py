"""The C-ABI library loads, exports every declared symbol, and its host-side
logic (argument checks, helpers) works without a GPU."""
import ctypes
import json
import os
import re

import numpy as np
import pytest

import svg_workloads as W
from sparse_attention_video_qk_b200 import _lib as C
from sparse_attention_video_qk_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return C.lib()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "svg.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(svg2?_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    syms = declared_symbols()
    assert len(syms) >= 12
    for s in syms:
        assert hasattr(L, s), s
    assert set(syms) == set(C.SIGNATURES), set(syms) ^ set(C.SIGNATURES)


def test_version_and_status_strings(L):
    assert b"sm_100a" in L.svg_version()
    for st in range(8):
        assert L.svg_status_string(st)


def test_sample_queries_matches_generator(L):
    for seed, Lv, n in [(1000, 256, 16), (1003, 118800, 64), (7, 10, 10), (5, 1 << 20, 64)]:
        assert np.array_equal(api.sample_queries(seed, Lv, n), W.sample_queries(seed, Lv, n))
    out = api.sample_queries(3, 50, 50)
    assert sorted(out.tolist()) == list(range(50))          # n = Lv: a permutation
    with pytest.raises(C.SVGError):
        api.sample_queries(1, 10, 11)


def _published_splitmix64():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "splitmix64.json")
    with open(path) as f:
        cases = json.load(f)["cases"]
    out = []
    for c in cases:
        xs = c.get("outputs") or [int(h, 16) for h in c["outputs_hex"]]
        out.append((c["seed"], xs))
    return out


def test_splitmix64_stream_equals_published_outputs():
    """The generator module's SplitMix64 against published output sequences
    (seed 0 of the reference implementation; seed 1234567 of the Rosetta Code
    task): a change to any of its three constants or shifts fails here."""
    for seed, xs in _published_splitmix64():
        gen = W.splitmix64_stream(seed)
        assert [next(gen) for _ in xs] == xs, seed


def test_sample_queries_c_helper_follows_published_outputs(L):
    """The C helper's draws against the published SplitMix64 outputs.  With
    Lv = 2^31 - 1 and n = 5 no slot is touched twice, so slot i receives
    i + (x_(i+1) mod (Lv - i)) from the partial Fisher-Yates shuffle."""
    Lv = (1 << 31) - 1
    for seed, xs in _published_splitmix64():
        want = [i + x % (Lv - i) for i, x in enumerate(xs)]
        assert len(set(want)) == len(want) and min(want) >= len(xs)
        assert api.sample_queries(seed, Lv, len(xs)).tolist() == want, seed
        assert W.sample_queries(seed, Lv, len(xs)).tolist() == want, seed


def test_rope_table_values(L):
    wl = W.TINY
    pb = api.Problem.from_workload(wl)
    tab = api.rope_table(pb)
    n0, n1, n2 = wl.rope_split
    assert tab.size == 2 * (wl.F * n0 // 2 + wl.Hs * n1 // 2 + wl.Ws * n2 // 2)
    cs = tab.reshape(-1, 2)
    # position 0 rows are (1, 0); every entry lies on the unit circle
    assert np.allclose(cs[: n0 // 2], [1.0, 0.0])
    assert np.allclose((cs ** 2).sum(1), 1.0, atol=1e-6)
    # frame 1, pair j: angle base^(-2j/n0)
    j = np.arange(n0 // 2)
    ang = np.arctan2(cs[n0 // 2: n0, 1], cs[n0 // 2: n0, 0])
    assert np.allclose(ang, wl.rope_base ** (-2 * j / n0), atol=1e-6)


def test_capacity_and_workspace(L):
    wl = W.HUNYUAN
    pb = api.Problem.from_workload(wl)
    assert api.block_index_capacity(pb) == wl.H * wl.nqb * wl.nkb
    ws = api.profile_workspace_size(pb, 64)
    assert ws > 0 and ws % 16 == 0


@pytest.mark.parametrize("key", sorted(W.WORKLOADS))
def test_workspace_size_covers_every_sample_count(L, key):
    """svg_workspace_size is the scratch of the workspace-taking calls for any
    n in 1..64, and 0 on invalid arguments."""
    pb = api.Problem.from_workload(W.WORKLOADS[key])
    ws = api.workspace_size(pb)
    assert ws > 0
    assert all(api.profile_workspace_size(pb, n) <= ws for n in (1, 7, 32, 64))
    sh, pr = pb.c_shape(), pb.c_params()
    assert L.svg_workspace_size(None, ctypes.byref(pr)) == 0
    assert L.svg_workspace_size(ctypes.byref(sh), None) == 0
    pr.block_k = 32
    assert L.svg_workspace_size(ctypes.byref(sh), ctypes.byref(pr)) == 0


def test_release_with_nothing_cached_touches_no_gpu(L):
    """With no host-buffer step run in this process nothing is cached, so the
    call returns SVG_OK without any CUDA call (this machine may have no GPU)."""
    assert L.svg_release() == 0
    assert L.svg_release() == 0


def _call_attn(L, sh, pr, ptr=16):
    p = ctypes.c_void_p(ptr)
    return L.svg_block_sparse_attn(ctypes.byref(sh), ctypes.byref(pr), p, p, p, p, p, p, p,
                                   ctypes.c_void_p(ptr + 4096), None, None)


def test_host_side_argument_errors(L):
    """Errors are returned before anything touches the GPU."""
    pb = api.Problem.from_workload(W.TINY)
    sh, pr = pb.c_shape(), pb.c_params()
    bad = C.SvgShape(sh.B, sh.H, sh.L + 1, sh.d, sh.F, sh.Hs, sh.Ws, sh.text_len)
    assert _call_attn(L, bad, pr) == C.SVG_ERR_SHAPE
    d96 = C.SvgShape(sh.B, sh.H, sh.L, 96, sh.F, sh.Hs, sh.Ws, sh.text_len)
    assert _call_attn(L, d96, pr) == C.SVG_ERR_UNSUPPORTED
    pr32 = pb.c_params()
    pr32.block_k = 32
    assert _call_attn(L, sh, pr32) == C.SVG_ERR_UNSUPPORTED
    assert _call_attn(L, sh, pr, ptr=8) == C.SVG_ERR_ALIGNMENT
    neg = pb.c_params()
    neg.spatial_frames = -1
    assert _call_attn(L, sh, neg) == C.SVG_ERR_INVALID_ARG
    p = ctypes.c_void_p(16)
    # missing gamma with NORM_ROPE
    assert L.svg_qknorm_rope_layout(ctypes.byref(sh), ctypes.byref(pr), C.SVG_NORM_ROPE, p, p, None, None, None,
                                    None, None, ctypes.c_void_p(32), ctypes.c_void_p(48), None,
                                    None) == C.SVG_ERR_INVALID_ARG
    # bad rope split
    prs = pb.c_params()
    prs.rope_split[0] += 2
    g = ctypes.c_void_p(64)
    assert L.svg_qknorm_rope_layout(ctypes.byref(sh), ctypes.byref(prs), C.SVG_NORM_ROPE, p, p, None, g, g, g, None,
                                    ctypes.c_void_p(32), ctypes.c_void_p(48), None, None) == C.SVG_ERR_SHAPE
    # profiling: n out of range, workspace too small
    assert L.svg_profile_heads(ctypes.byref(sh), ctypes.byref(pr), p, p, p, p, 65, p, 1 << 30, None, p,
                               None) == C.SVG_ERR_INVALID_ARG
    assert L.svg_profile_heads(ctypes.byref(sh), ctypes.byref(pr), p, p, p, p, 16, p, 16, None, p,
                               None) == C.SVG_ERR_CAPACITY


def test_svg2_attention_rejects_null_pointers(L):
    """A NULL perm_q (or qoff, koff, sel) is an argument error returned before
    any launch, not a device-side fault."""
    pb = api.Problem.from_workload(W.small_workload(d=128, H=2, F=4, Hs=8, Ws=12, T=19))
    sh, pr = pb.c_shape(), pb.c_params()
    p = ctypes.c_void_p(16)
    out = ctypes.c_void_p(16 + 4096)
    for null in range(4):                       # qoff, koff, sel, perm_q
        args = [p, p, p, p]
        args[null] = None
        qoff, koff, sel, perm_q = args
        assert L.svg2_attention(ctypes.byref(sh), ctypes.byref(pr), p, p, p, 8, 11, qoff, koff, sel, perm_q, p, p, p,
                                out, None, None) == C.SVG_ERR_INVALID_ARG, null
    # through the binding too: None for perm_q raises before anything runs
    with pytest.raises(C.SVGError) as e:
        C.check(L.svg2_attention(ctypes.byref(sh), ctypes.byref(pr), p, p, p, 8, 11, p, p, p, None, p, p, p, out, None,
                                 None), "svg2_attention")
    assert e.value.status == C.SVG_ERR_INVALID_ARG


def test_host_step_argument_errors(L):
    """svg_attention_step_host rejects bad group counts and a short workspace
    before any CUDA call; the workspace size grows with nothing but the shape."""
    wl = W.TINY
    pb = api.Problem.from_workload(wl)
    sh, pr = pb.c_shape(), pb.c_params()
    p = ctypes.c_void_p(256)
    size = L.svg_attention_step_host_workspace_size(ctypes.byref(sh), ctypes.byref(pr), 16, 1)
    assert size >= 4 * wl.B * wl.H * wl.L * wl.d * 2
    assert L.svg_attention_step_host_workspace_size(ctypes.byref(sh), ctypes.byref(pr), 16, 0) == 0
    assert L.svg_attention_step_host_workspace_size(ctypes.byref(sh), ctypes.byref(pr), 16, wl.B * wl.H + 1) == 0
    call = lambda groups, ws_bytes, n=16: L.svg_attention_step_host(
        ctypes.byref(sh), ctypes.byref(pr), p, p, p, p, p, p, n, p, None, groups, p, ws_bytes, None)
    assert call(0, size) == C.SVG_ERR_INVALID_ARG
    assert call(wl.B * wl.H + 1, size) == C.SVG_ERR_INVALID_ARG
    assert call(1, size, n=0) == C.SVG_ERR_INVALID_ARG
    assert call(1, size - 1) == C.SVG_ERR_CAPACITY
    assert L.svg_attention_step_host(ctypes.byref(sh), ctypes.byref(pr), p, p, p, p, p, p, 16, p, None, 1,
                                     ctypes.c_void_p(8), size, None) == C.SVG_ERR_ALIGNMENT


def test_noalloc_capacity_limit(L):
    """The no-alloc profiling entry rejects shapes whose one key chunk of
    partials does not fit its 16 MiB scratch, before any CUDA call."""
    p = ctypes.c_void_p(16)
    for wl, heads in ((W.WAN, 126), (W.COGVIDEOX, 247)):   # d = 128: B*H > 125; d = 64: B*H > 246
        pb = api.Problem.from_workload(wl)
        sh, pr = pb.c_shape(), pb.c_params()
        big = C.SvgShape(1, heads, sh.L, sh.d, sh.F, sh.Hs, sh.Ws, sh.text_len)
        per_chunk = heads * 128 * (3 + 2 * sh.d) * 4 + heads * 64 * 2 * 8
        assert per_chunk > 16 << 20
        assert (heads - 1) * 128 * (3 + 2 * sh.d) * 4 + (heads - 1) * 64 * 2 * 8 <= 16 << 20
        assert L.svg_profile_heads_noalloc(ctypes.byref(big), ctypes.byref(pr), p, p, p, p, 64, None, p,
                                           None) == C.SVG_ERR_CAPACITY
        assert L.svg_profile_heads_noalloc(ctypes.byref(sh), ctypes.byref(pr), p, p, p, p, 65, None, p,
                                           None) == C.SVG_ERR_INVALID_ARG


def test_step_policy_schedule(L):
    """First 25% of the steps dense, then profiling every sparse step (or every
    `reprofile_every` sparse steps, reusing the kinds in between)."""
    D, P, R = api.STEP_DENSE, api.STEP_PROFILE, api.STEP_REUSE
    assert [api.step_policy(t, 50) for t in range(50)] == [D] * 13 + [P] * 37   # t < 12.5
    assert [api.step_policy(t, 8) for t in range(8)] == [D, D, P, P, P, P, P, P]
    assert [api.step_policy(t, 8, 0.25, 3) for t in range(8)] == [D, D, P, R, R, P, R, R]
    assert [api.step_policy(t, 4, 0.0) for t in range(4)] == [P] * 4
    assert [api.step_policy(t, 4, 1.0) for t in range(4)] == [D] * 4
    for bad in [(-1, 4, 0.25, 1), (4, 4, 0.25, 1), (0, 0, 0.25, 1), (0, 4, 1.5, 1), (0, 4, -0.1, 1),
                (0, 4, float("nan"), 1), (0, 4, 0.25, 0)]:
        with pytest.raises(C.SVGError):
            api.step_policy(*bad)
