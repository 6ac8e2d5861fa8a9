"""svg_profile_heads_noalloc against svg_profile_heads, through the C ABI.

The no-alloc entry point serves callers that cannot allocate device memory
(a plugin inside a runtime that owns all device memory, a serving process with
a pool reserved at start-up): it keeps its scratch in a fixed array inside the
library instead of taking a workspace.  It must give the same head choices as
the workspace entry point and MSEs within the profiling tolerance, on two calls
in a row (the second call finds the first call's leftovers in the scratch).

Collected last (file name), so a failure here comes after every other test has
run; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import sparse_attention_video_qk_b200 as svg
import svg_workloads as W
from gpu_util import dev

pytestmark = pytest.mark.gpu

MSE_RTOL = 2e-2      # the profiling tolerance used by the parity tests


def _inputs(wl):
    inp = W.make_inputs(wl)
    pb = svg.Problem.from_workload(wl)
    q, k = dev(inp["q"]), dev(inp["k"])
    qn, kn = svg.qknorm_rope(pb, q, k, dev(inp["gamma_q"]), dev(inp["gamma_k"]), dev(svg.rope_table(pb)))
    return pb, qn, kn, dev(inp["v"]), dev(inp["sample_idx"])


@pytest.mark.parametrize("wl", [W.TINY, W.WAN], ids=["tiny", "wan"])
def test_noalloc_matches_workspace_entry_point_twice(wl):
    pb, qn, kn, v, si = _inputs(wl)
    kinds_ref, mse_ref = svg.profile_heads(pb, qn, kn, v, si)
    svg.sync_status()
    kinds_ref, mse_ref = kinds_ref.cpu().numpy(), mse_ref.cpu().numpy().astype(np.float64)
    for call in range(2):
        kinds, mse = svg.profile_heads_noalloc(pb, qn, kn, v, si)
        svg.sync_status()
        kinds, mse = kinds.cpu().numpy(), mse.cpu().numpy().astype(np.float64)
        assert np.array_equal(kinds, kinds_ref), (call, kinds, kinds_ref)
        rel = np.abs(mse - mse_ref) / mse_ref
        assert rel.max() < MSE_RTOL, (call, rel.max())


def test_noalloc_rejects_problems_beyond_its_scratch():
    # one key chunk of partials for 200 heads at d = 128 needs 200*128*259*4 B > 16 MiB
    wl = W.small_workload(d=128, H=200, F=2, Hs=2, Ws=4, T=0, n_samples=4)
    pb = svg.Problem.from_workload(wl)
    x = torch.zeros(1, 200, wl.L, 128, dtype=torch.bfloat16, device="cuda")
    si = torch.zeros(4, dtype=torch.int32, device="cuda")
    with pytest.raises(svg.SVGError) as e:
        svg.profile_heads_noalloc(pb, x, x, x, si)
    assert e.value.status == 5
