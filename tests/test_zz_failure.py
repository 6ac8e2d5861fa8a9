"""Failure detection on the GPU without a fault: a wait that nothing
completes gives up after its limit, the host reads SVG_ERR_TIMEOUT, and the
context keeps working.  Collected late (zz) because it spins for about a
second."""
import time

import numpy as np
import pytest

import oracle
import sparse_attention_video_qk_b200 as svg
import svg_workloads as W
from gpu_util import assert_attention_close, dev, host_bits
from sparse_attention_video_qk_b200 import _lib as C

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_survives():
    svg.sync_status()                                   # start from a clear error word
    assert svg.lib().svg_selftest_wait_timeout(None) == C.SVG_OK
    t0 = time.time()
    with pytest.raises(svg.SVGError) as e:
        svg.sync_status()
    assert e.value.status == C.SVG_ERR_TIMEOUT
    assert time.time() - t0 < 30
    svg.sync_status()                                   # the error word was cleared
    # the same context still runs a whole step correctly
    wl = W.TINY
    inp = W.make_inputs(wl)
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    pb = svg.Problem.from_workload(wl)
    buf = svg.StepBuffers(pb, wl.n_samples)
    out = svg.attention_step(pb, *(dev(inp[k]) for k in ("q", "k", "v", "gamma_q", "gamma_k", "sample_idx")), buf)
    svg.sync_status()
    qn = oracle.qknorm_rope(sh, pr, inp["q"], inp["gamma_q"])
    kn = oracle.qknorm_rope(sh, pr, inp["k"], inp["gamma_k"])
    _, kinds = oracle.profile(sh, pr, qn, kn, inp["v"], inp["sample_idx"])
    rows = np.arange(wl.B * wl.H * wl.L, dtype=np.int64)
    ref = oracle.attention_rows(sh, pr, kinds, qn, kn, inp["v"], rows)
    assert_attention_close(host_bits(out).reshape(-1, wl.d), ref, 2e-2, 2e-3, "after timeout")
