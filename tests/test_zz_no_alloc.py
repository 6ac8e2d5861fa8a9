"""svg_profile_heads_noalloc against svg_profile_heads and the oracle, through
the C ABI.

The no-alloc entry point serves callers that cannot allocate device memory
(a plugin inside a runtime that owns all device memory, a serving process with
a pool reserved at start-up): it keeps its scratch in a fixed array inside the
library instead of taking a workspace.  On two calls in a row (the second call
finds the first call's leftovers in the scratch) it must give:
  * bit-identical kinds and MSEs where it splits the keys into as many chunks
    as the workspace entry point (the tiny shape; 125 heads at d = 128 with a
    single key tile);
  * the same kinds, and MSEs within 1e-2 relative (plus a 1e-10 floor), where
    fewer chunks fit.  The two are not bit-equal there: each chunk rounds its
    softmax weights to bf16 against its own running maximum, so a different
    chunking rounds the weights differently (about 2^-9 each), which moves an
    MSE by up to about 1e-3 relative at these shapes.  A dropped or misplaced
    chunk moves it by far more than 1e-2;
  * MSEs within the profiling tolerance of the oracle (relative 2e-2, with a
    1e-10 floor for an MSE of exactly 0, a mask that keeps every key) and the
    oracle's kinds.

Collected last (file name), so a failure here comes after every other test has
run; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_video_qk_b200 as svg
import svg_workloads as W
from gpu_util import dev

pytestmark = pytest.mark.gpu

MSE_RTOL_ORACLE = 2e-2    # the profiling parity tests' tolerance against fp64
MSE_ATOL_ORACLE = 1e-10   # floor for an MSE of 0 (the mask keeps every key)
MSE_RTOL_CHUNKS = 1e-2    # another chunking: softmax weights rounded to bf16 against other maxima

# 125 heads at d = 128 is the most one 16 MiB scratch takes (one key chunk);
# n = 16 < 64 sampled rows leaves padded rows in the error sums.  With one key
# tile both entry points use one chunk; with five the workspace one uses two.
EDGE125 = W.small_workload(d=128, H=125, F=2, Hs=4, Ws=8, T=9, n_samples=16, seed=41)
EDGE125_LONG = W.small_workload(d=128, H=125, F=4, Hs=8, Ws=16, T=9, n_samples=16, seed=42)
# name -> (workload, same chunk count on both entry points)
CASES = {"tiny": (W.TINY, True), "wan": (W.WAN, False), "edge125": (EDGE125, True),
         "edge125_long": (EDGE125_LONG, False)}


def _chunks(wl, noalloc):
    """Key chunks of each entry point (the rule of the library's headers)."""
    bh, ntiles = wl.B * wl.H, -(-wl.L // 128)
    ws = max(1, min(2 * 148 // bh, (ntiles + 1) // 2))
    if not noalloc:
        return ws
    fit = ((16 << 20) - bh * 64 * 2 * 8) // (bh * 128 * (3 + 2 * wl.d) * 4)
    return min(ws, fit)


def _inputs(wl):
    inp = W.make_inputs(wl)
    pb = svg.Problem.from_workload(wl)
    q, k = dev(inp["q"]), dev(inp["k"])
    qn, kn = svg.qknorm_rope(pb, q, k, dev(inp["gamma_q"]), dev(inp["gamma_k"]), dev(svg.rope_table(pb)))
    return inp, pb, qn, kn, dev(inp["v"]), dev(inp["sample_idx"])


@pytest.mark.parametrize("key", list(CASES))
def test_noalloc_matches_workspace_entry_point_and_oracle_twice(key):
    wl, same_chunks = CASES[key]
    inp, pb, qn, kn, v, si = _inputs(wl)
    kinds_ref, mse_ref = svg.profile_heads(pb, qn, kn, v, si)
    svg.sync_status()
    kinds_ref, mse_ref = kinds_ref.cpu().numpy(), mse_ref.cpu().numpy().astype(np.float64)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    qn_h = qn.view(torch.int16).cpu().numpy().view(np.uint16)
    kn_h = kn.view(torch.int16).cpu().numpy().view(np.uint16)
    mse_ora, kinds_ora = oracle.profile(sh, pr, qn_h, kn_h, inp["v"], inp["sample_idx"])
    assert (_chunks(wl, True) == _chunks(wl, False)) == same_chunks
    if key.startswith("edge125"):
        assert _chunks(wl, True) == 1
    for call in range(2):
        kinds, mse = svg.profile_heads_noalloc(pb, qn, kn, v, si)
        svg.sync_status()
        kinds, mse = kinds.cpu().numpy(), mse.cpu().numpy().astype(np.float64)
        if same_chunks:
            assert np.array_equal(kinds, kinds_ref) and np.array_equal(mse, mse_ref), (key, call)
        else:
            err = np.abs(mse - mse_ref)
            print(f"{key}: call {call}, chunking difference {(err / np.maximum(mse_ref, 1e-30)).max():.2e} relative")
            assert (err <= MSE_RTOL_CHUNKS * mse_ref + MSE_ATOL_ORACLE).all(), (key, call)
            assert np.array_equal(kinds, kinds_ref), (key, call)
        gap = np.abs(mse_ora[:, 0] - mse_ora[:, 1]) / mse_ora.max(1)
        assert (gap >= 1e-4).all(), f"{key}: a near tie in the oracle's MSEs"
        assert np.array_equal(kinds, kinds_ora), (key, call)
        assert (np.abs(mse - mse_ora) <= MSE_RTOL_ORACLE * mse_ora + MSE_ATOL_ORACLE).all(), (key, call)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # one key chunk of partials for 200 heads at d = 128 needs 200*128*259*4 B > 16 MiB
    wl = W.small_workload(d=128, H=200, F=2, Hs=2, Ws=4, T=0, n_samples=4)
    pb = svg.Problem.from_workload(wl)
    x = torch.zeros(1, 200, wl.L, 128, dtype=torch.bfloat16, device="cuda")
    si = torch.zeros(4, dtype=torch.int32, device="cuda")
    with pytest.raises(svg.SVGError) as e:
        svg.profile_heads_noalloc(pb, x, x, x, si)
    assert e.value.status == 5
