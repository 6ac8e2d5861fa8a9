"""Benchmark of the Sparse VideoGen attention step on B200.

Default workload: HunyuanVideo 720p 5 s shape (B=1, H=24, d=128, 33 latent
frames of 45x80 = 118,800 video tokens + 256 text tokens), one full step per
iteration: QK-Norm + 3D RoPE -> online profiling -> block index -> layout
transform -> block-sparse attention with the inverse layout in its epilogue.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--sweep]

Prints one JSON line (rank 0).  `value` is effective TFLOP/s: the FLOPs of
QK^T and PV over the kept 128x64 tiles (4*d*rows*cols per tile) divided by the
whole step's device time.  With N > 1 (torchrun) every rank runs its own
independent layer (weak scaling, no data-path collective); time is the max
over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import svg_workloads as W  # noqa: E402

METRIC = "sparse-attn layer ms and effective TFLOP/s (% bf16 peak) at 118,800 tokens"
SHAPE_LABEL = {W.TINY.name: "tiny test shape", W.COGVIDEOX.name: "CogVideoX shape",
               W.WAN.name: "Wan 2.1-1.3B shape", W.HUNYUAN.name: "HunyuanVideo 720p 5 s shape",
               W.HUNYUAN_SWEEP.name: "HunyuanVideo 720p 5 s shape, sweep seed"}
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 7700.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: d[k] for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK), "fallback"


def clock_basis(clocks, achieved_tflops, pk):
    """The SM clock the kernel ran at next to the clocks the peaks were taken
    at: the burst peak is a short cuBLAS run near the maximum clock; the
    sustained peak was measured at the median clock MEASURED_PEAKS.json
    records.  Also the sustained peak scaled to this run's median clock."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    sus_mhz = None
    if os.path.exists(p):
        sus_mhz = json.load(open(p)).get("clocks_under_load", {}).get("sm_mhz_median")
    med = clocks.get("sm_mhz") if isinstance(clocks, dict) else None
    out = {"run_sm_mhz_median": med, "sustained_peak_sm_mhz": sus_mhz,
           "time_x_mhz_note": "the tensor pipe's rate scales with the SM clock"}
    if med and sus_mhz:
        scaled = pk["bf16_tflops_sustained"] * med / sus_mhz
        out["sustained_peak_scaled_to_run_clock"] = round(scaled, 1)
        out["frac_of_scaled_sustained"] = round(achieved_tflops / scaled, 4)
    return out


def reduce_over_ranks(times, work, device="cpu"):
    """Max over ranks of `times`, sum over ranks of `work` (lists of floats);
    the identity when no process group of more than one rank is up.  Every
    rank must call it, in the same order."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(times, dtype=torch.float64, device=device)
    w = torch.tensor(work, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.cpu()], [float(x) for x in w.cpu()]


def executed_tile_flops(row_ptr: np.ndarray, col: np.ndarray, wl) -> float:
    """FLOPs the attention kernel's tensor cores execute for this block list.
    With 128-row query tiles a CTA walks the union of its two tiles' lists and
    runs S and P.V for both tiles on every block in it (a block listed for one
    tile only is masked for the other), over whole 128x64 tiles; with 64-row
    tiles each listed tile is computed whole."""
    counts = np.diff(row_ptr.astype(np.int64))
    if wl.bq != 128:
        return float(4.0 * wl.d * wl.bq * wl.bk * counts.sum())
    nqb, nkb = wl.nqb, wl.nkb
    t = np.repeat(np.arange(counts.size, dtype=np.int64), counts)      # q-tile of each entry
    pair = (t // nqb) * ((nqb + 1) // 2) + (t % nqb) // 2
    union = np.unique(pair * (nkb + 1) + col.astype(np.int64)).size
    return float(union * 2 * 4.0 * wl.d * wl.bq * wl.bk)


def kept_tile_flops(row_ptr: np.ndarray, col: np.ndarray, wl) -> float:
    """4*d*rows*cols summed over the listed (q-block, k-block) tiles."""
    nqb = wl.nqb
    counts = np.diff(row_ptr.astype(np.int64))
    qb = np.tile(np.arange(nqb), wl.B * wl.H)
    rows = np.minimum(wl.bq, wl.L - qb * wl.bq)
    cols = np.minimum(wl.bk, wl.L - col.astype(np.int64) * wl.bk)
    # every listed tile of one q-block has `rows` query rows
    per_entry_rows = np.repeat(rows, counts)
    return float(4.0 * wl.d * np.sum(per_entry_rows * cols))


def traffic_from_profile(kernel_file: str, summary: str):
    """DRAM bytes per launch recorded in a committed ncu summary, if it was
    taken on the current kernel source (sha256 match); else None."""
    p = os.path.join(ROOT, "profiles", summary)
    src = os.path.join(ROOT, "sparse_attention_video_qk_b200", "csrc", kernel_file)
    if not (os.path.exists(p) and os.path.exists(src)):
        return None
    text = open(p).read()
    m_sha = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text)
    m_b = re.search(r"traffic_bytes_per_launch_full_size:\s*([0-9.eE+]+)", text)
    if not (m_sha and m_b):
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != m_sha.group(1):
        return None
    return float(m_b.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle sampling; only samples whose timestamp falls
    inside [window start, window end] (host clock) are summarised."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None
        self.out = ""

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.5)
        return self

    def start(self):
        self.t0 = time.time()

    def stop(self):
        self.t1 = time.time()

    def __exit__(self, *a):
        time.sleep(0.2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        from datetime import datetime
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                clk, mxc = float(f[1]), float(f[2])
            except ValueError:
                continue
            if self.t0 is not None and not (self.t0 <= ts <= self.t1):
                continue
            sm.append(clk)
            mx = mxc
            try:
                power.append(float(f[3]))
            except ValueError:
                pass
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_median": statistics.median(power) if power else None}


# ---------------------------------------------------------------- GPU arm --

def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import sparse_attention_video_qk_b200 as svg

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    wl = W.WORKLOADS[args.workload]
    pb = svg.Problem.from_workload(wl)
    inp = W.make_inputs(wl, seed=wl.seed + rank)          # each rank: its own layer
    pin = lambda a, bf=True: (torch.from_numpy(a).view(torch.bfloat16) if bf else torch.from_numpy(a)).pin_memory()
    q_h, k_h, v_h = pin(inp["q"]), pin(inp["k"]), pin(inp["v"])
    gq_h, gk_h, si_h = pin(inp["gamma_q"], False), pin(inp["gamma_k"], False), pin(inp["sample_idx"], False)
    q, k, v = (t.to(device) for t in (q_h, k_h, v_h))
    gq, gk, si = gq_h.to(device), gk_h.to(device), si_h.to(device)
    buf = svg.StepBuffers(pb, int(si.numel()), device)
    stream = torch.cuda.current_stream()
    lib = svg.lib()
    sh, pr = pb.c_shape(), pb.c_params()
    cs = ctypes.c_void_p(stream.cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None

    def stage_calls():
        """The step as its five C-ABI calls (the same calls svg_attention_step makes)."""
        b = buf
        return [
            # 1. QK-Norm + RoPE of K
            ("k_norm_rope", lambda: lib.svg_qknorm_rope_layout(ctypes.byref(sh), ctypes.byref(pr), 1, None, P(k),
                                                              None, None, P(gk), P(b.table), None, None, P(b.kn),
                                                              None, cs)),
            # 2. profiling from raw Q (sampled rows normalised in the kernel)
            ("profile", lambda: lib.svg_profile_heads_raw_q(ctypes.byref(sh), ctypes.byref(pr), P(q), P(gq),
                                                            P(b.table), P(b.kn), P(v), P(si), int(si.numel()),
                                                            P(b.workspace), b.workspace.numel(), P(b.mse),
                                                            P(b.kinds), cs)),
            ("block_index", lambda: lib.svg_build_block_index(ctypes.byref(sh), ctypes.byref(pr), P(b.kinds),
                                                              P(b.row_ptr), P(b.col), P(b.full), b.capacity, cs)),
            # 4. QK-Norm + RoPE of Q and the layout transform of Q, K, V in one pass
            ("q_norm_rope_layout", lambda: lib.svg_qknorm_rope_layout(
                ctypes.byref(sh), ctypes.byref(pr), 3, P(q), P(b.kn), P(v), P(gq), None, P(b.table), P(b.kinds),
                P(b.qp), P(b.kp), P(b.vp), cs)),
            # attention with the inverse layout in its epilogue: writes `out` in model order
            ("attention", lambda: lib.svg_block_sparse_attn_model_order(
                ctypes.byref(sh), ctypes.byref(pr), P(b.qp), P(b.kp), P(b.vp), P(b.kinds), P(b.row_ptr),
                P(b.col), P(b.full), P(b.out), None, cs)),
        ]

    calls = stage_calls()
    # kernels per stage: rowmap; profile_tc + merge + choose; count + scan + fill; rowmap; attention
    launches_per_step = 1 + 3 + 3 + 1 + 1

    def one_step(events=None):
        for i, (name, fn) in enumerate(calls):
            st = fn()
            if st != 0:
                raise svg.SVGError(st, name)
            if events is not None:
                events[i + 1].record(stream)

    for _ in range(args.warmup):
        one_step()
    svg.sync_status()
    flops = kept_tile_flops(buf.row_ptr.cpu().numpy(), buf.col[: int(buf.row_ptr[-1])].cpu().numpy(), wl)
    exec_flops = executed_tile_flops(buf.row_ptr.cpu().numpy(), buf.col[: int(buf.row_ptr[-1])].cpu().numpy(), wl)
    kinds = buf.kinds.cpu().numpy()

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        clk.start()
        t_start.record(stream)
        for s in range(args.steps):
            ev[s][0].record(stream)
            one_step(ev[s])
        t_end.record(stream)
        torch.cuda.synchronize()
        clk.stop()
    if world > 1:
        dist.barrier()
    svg.sync_status()
    total_ms = t_start.elapsed_time(t_end)
    stage_ms = {name: statistics.mean(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(args.steps))
                for i, (name, _) in enumerate(calls)}
    clocks = clk.summary()

    # ---- end to end through the public host-buffer API (copies inside the timed region)
    out_h = torch.empty(q_h.shape, dtype=torch.bfloat16, pin_memory=True)
    for _ in range(2):
        svg.sparse_attention(pb, q_h, k_h, v_h, gq_h, gk_h, si_h, out_host=out_h)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 5))
    e0.record(stream)
    for _ in range(e2e_steps):
        svg.sparse_attention(pb, q_h, k_h, v_h, gq_h, gk_h, si_h, out_host=out_h)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h, gq_h, gk_h, si_h))
    d2h = out_h.numel() * out_h.element_size()

    # ---- dense reference point on the same inputs (every head DENSE), outside the timed region
    dense_ms = None
    if not args.no_dense:
        dk = torch.full_like(buf.kinds, svg.DENSE)
        cap_d = svg.block_index_capacity(pb)
        rp_d, col_d, full_d = svg.build_block_index(pb, dk, cap_d)
        out_d = torch.empty_like(buf.qp)
        svg.block_sparse_attn(pb, q, k, v, dk, rp_d, col_d, full_d, out=out_d)
        torch.cuda.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        svg.block_sparse_attn(pb, q, k, v, dk, rp_d, col_d, full_d, out=out_d)
        d1.record(stream)
        torch.cuda.synchronize()
        dense_ms = d0.elapsed_time(d1)
        dense_flops = kept_tile_flops(rp_d.cpu().numpy(), col_d[: int(rp_d[-1])].cpu().numpy(), wl)
        del out_d, rp_d, col_d, full_d
    svg.sync_status()

    # ---- times: max over ranks; work: sum over ranks (each rank runs its own layer)
    (total_ms, e2e_ms, attn_ms_max), (flops_all,) = reduce_over_ranks(
        [total_ms, e2e_ms, stage_ms["attention"]], [flops], device)
    ms_per_step = total_ms / args.steps
    value = flops_all / (ms_per_step * 1e-3) / 1e12
    if rank != 0:
        return None

    pk, pk_src = peaks()
    attn_tflops = flops / (stage_ms["attention"] * 1e-3) / 1e12
    # svg_block_sparse_attn runs the two-query-tile kernel for 128-row tiles
    attn_src, attn_name = (("attention2.cuh", f"attn2_kernel<{wl.d}>") if wl.bq == 128
                           else ("attention.cuh", f"attn_kernel<{wl.d}>"))
    traffic = traffic_from_profile(attn_src, "attention_hunyuanvideo_720p.md") if wl == W.HUNYUAN else None
    d, L, BH = wl.d, wl.L, wl.B * wl.H
    compulsory = 8.0 * BH * L * d          # read Q, K, V and write O once, bf16
    stage_bytes = {"k_norm_rope": 4.0 * BH * L * d, "q_norm_rope_layout": 12.0 * BH * L * d,
                   "profile": 4.0 * BH * L * d}
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q/K/V with planted spatial/temporal heads; no model weights)",
        "config": {
            "workload": f"{wl.name} ({SHAPE_LABEL[wl.name]})",
            "B": wl.B, "H": wl.H, "d": wl.d, "frames": wl.F, "grid": f"{wl.Hs}x{wl.Ws}", "text_tokens": wl.T,
            "video_tokens": wl.Lv, "seq_len": wl.L, "spatial_window": wl.w, "temporal_radius": wl.r,
            "tile": f"{wl.bq}x{wl.bk}", "profiled_rows": wl.n_samples,
            "head_kinds": {"spatial": int((kinds == 0).sum()), "temporal": int((kinds == 1).sum())},
            "kept_tile_tflop": round(flops / 1e12, 4),
            "executed_tile_tflop": round(exec_flops / 1e12, 4),
            "union_walk_overhead": round(exec_flops / flops - 1.0, 4) if flops > 0 else None,
            "l2": "no flush: each step reads > 2 GB of inputs, far above the 126 MB L2",
            "parallelism": f"replicas x{world} (one independent layer per GPU)",
        },
        "layer_ms": round(ms_per_step, 4),
        "pct_bf16_peak": {"measured_sustained": round(100 * value / world / pk["bf16_tflops_sustained"], 2),
                          "measured_burst": round(100 * value / world / pk["bf16_tflops"], 2),
                          "nominal": round(100 * value / world / NOMINAL_BF16_TFLOPS, 2)},
        "stage_ms": {k: round(v, 4) for k, v in stage_ms.items()},
        "stage_gbs": {k: round(stage_bytes[k] / (stage_ms[k] * 1e-3) / 1e9, 1) for k in stage_bytes},
        "roofline": {
            "kernel": f"{attn_name} (svg_block_sparse_attn)",
            "bound": "tensor",
            "achieved": round(attn_tflops, 2),
            "peak": pk["bf16_tflops"],
            "unit": "TFLOP/s",
            "frac": round(attn_tflops / pk["bf16_tflops"], 4),
            "peak_source": f"{pk_src} bf16 burst (cuBLAS 8192^3, best of 10)",
            "clock_basis": clock_basis(clocks, attn_tflops, pk),
            "traffic": traffic,
            "compulsory_bytes": compulsory,
            "traffic_over_compulsory": None if traffic is None else round(traffic / compulsory, 3),
        },
        "dense_attention": None if dense_ms is None else {
            "ms": round(dense_ms, 3), "tflops": round(dense_flops / (dense_ms * 1e-3) / 1e12, 2),
            "speedup_sparse_attn_vs_dense": round(dense_ms / stage_ms["attention"], 3),
            "theoretical_speedup_tiles": round(dense_flops / flops, 3)},
        "e2e": {"value": round(flops_all / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "sparse_attention -> C-ABI svg_attention_step_host (pinned host buffers; the library's three "
                       "streams overlap the copies with the passes over 8 head groups)"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(wl, inp, args.cpu_rows)
    return line


# ------------------------------------- semantic-aware permutation (SVG2) --

def run_svg2(args):
    """The SVG2 step ("Sparse VideoGen2" explainer, "A. 语义感知排列", "B. 基于质心的
    Top-p 选择") on one GPU: QK-Norm + RoPE of Q and K, k-means of Q and K
    (warm-started from the previous step's centroids), cluster sort, top-p key
    clusters, permutation of Q, K, V, block index, attention written back in
    model order.  Prints one JSON line; not the default bench line."""
    import torch

    import sparse_attention_video_qk_b200 as svg

    device = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    wl = W.WORKLOADS[args.workload]
    pb = svg.Problem.from_workload(wl)
    inp = W.make_inputs(wl)
    q, k, v = (torch.from_numpy(inp[n]).view(torch.bfloat16).to(device) for n in ("q", "k", "v"))
    gq, gk = (torch.from_numpy(inp[n]).to(device) for n in ("gamma_q", "gamma_k"))
    table = torch.from_numpy(svg.rope_table(pb)).to(device)
    Cq, Ck, iters, top_p = args.svg2_clusters, args.svg2_clusters, args.svg2_iters, args.svg2_top_p
    stream = torch.cuda.current_stream()
    st = {}

    def step(ev=None):
        mark = (lambda i: ev[i].record(stream)) if ev is not None else (lambda i: None)
        mark(0)
        qn, kn = svg.qknorm_rope(pb, q, k, gq, gk, table)
        mark(1)
        cq, aq, nq = svg.svg2_kmeans(pb, qn, Cq, iters, st.get("cq"))
        ck, ak, nk = svg.svg2_kmeans(pb, kn, Ck, iters, st.get("ck"))
        st["cq"], st["ck"] = cq, ck
        mark(2)
        pq, qoff = svg.svg2_permutation(pb, aq, Cq)
        pk, koff = svg.svg2_permutation(pb, ak, Ck)
        sel = svg.svg2_select(pb, cq, ck, nk, top_p)
        mark(3)
        qp, kp, vp = svg.svg2_permute(pb, pq, pk, qn, kn, v)
        mark(4)
        rp, col, full = svg.svg2_block_index(pb, qoff, koff, sel)
        mark(5)
        out = svg.svg2_attention(pb, qp, kp, vp, qoff, koff, sel, pq, rp, col, full)
        mark(6)
        st.update(rp=rp, col=col, sel=sel, out=out, nq=nq, nk=nk)

    names = ("qk_norm_rope", "kmeans_q_k", "sort_select", "permute", "block_index", "attention")
    for _ in range(args.warmup):
        step()
    svg.sync_status()
    n_ent = int(st["rp"][-1])
    flops = kept_tile_flops(st["rp"].cpu().numpy(), st["col"][:n_ent].cpu().numpy(), wl)
    sel_np = st["sel"].cpu().numpy().view(np.uint64)
    sel_bits = np.array([bin(int(x)).count("1") for x in sel_np.ravel()])
    # kept (query, key) pairs from the cluster sizes: a video query of cluster i keeps
    # the keys of its selected clusters and the text keys; a text query keeps all
    nq_np, nk_np = st["nq"].cpu().numpy().astype(np.int64), st["nk"].cpu().numpy().astype(np.int64)
    bits = ((sel_np[:, :, None] >> np.arange(Ck, dtype=np.uint64)) & np.uint64(1)).astype(np.int64)
    kept_pairs = float(((nq_np * ((bits * nk_np[:, None, :]).sum(-1) + wl.T)).sum()) + wl.B * wl.H * wl.T * wl.L)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        clk.start()
        for s in range(args.steps):
            step(ev[s])
        torch.cuda.synchronize()
        clk.stop()
    svg.sync_status()
    stage_ms = {n: statistics.mean(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(args.steps))
                for i, n in enumerate(names)}
    ms = statistics.mean(ev[s][0].elapsed_time(ev[s][-1]) for s in range(args.steps))
    pk, pk_src = peaks()
    attn_tflops = flops / (stage_ms["attention"] * 1e-3) / 1e12
    BH, Lv, d = wl.B * wl.H, wl.Lv, wl.d
    # element-pairs of the assignments: (iters + 1) passes of Lv*C*d per head, for Q and for K
    assign_pairs = 2.0 * BH * Lv * Cq * d * (iters + 1)
    line = {
        "metric": "SVG2 layer ms and effective TFLOP/s over kept tiles",
        "value": round(flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q/K/V with planted spatial/temporal heads; no model weights)",
        "config": {"workload": f"{wl.name} ({SHAPE_LABEL[wl.name]}), semantic-aware permutation",
                   "clusters_q": Cq, "clusters_k": Ck, "kmeans_iters": iters, "top_p": top_p,
                   "kept_tile_tflop": round(flops / 1e12, 4),
                   "tile_density": round(n_ent / (BH * wl.nqb * wl.nkb), 4),
                   "token_density": round(kept_pairs / (BH * float(wl.L) ** 2), 4),
                   "mean_key_clusters_selected": round(float(sel_bits.mean()), 2)},
        "stage_ms": {n: round(t, 4) for n, t in stage_ms.items()},
        # fp32 ALU bound of the assignment: one FMA per (row, centroid, dimension);
        # 148 SMs x 128 fp32 lanes x 1965 MHz = 37.2 T FMA/s
        "kmeans_roofline": {"bound": "alu", "unit": "G element-pairs/s",
                            "achieved": round(assign_pairs / (stage_ms["kmeans_q_k"] * 1e-3) / 1e9, 1),
                            "peak": round(148 * 128 * 1.965e9 / 1e9, 1),
                            "frac": round(assign_pairs / (stage_ms["kmeans_q_k"] * 1e-3) / (148 * 128 * 1.965e9), 4),
                            "note": "whole k-means stage (assign, sums, means) over the assignment work alone"},
        "roofline": {"kernel": f"attn2_kernel<{d}> (svg2_attention)", "bound": "tensor",
                     "achieved": round(attn_tflops, 2), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(attn_tflops / pk["bf16_tflops"], 4),
                     "peak_source": f"{pk_src} bf16 burst",
                     "traffic": traffic_from_profile("attention2.cuh", "attention_svg2_hunyuanvideo_720p.md")
                     if wl == W.HUNYUAN and (Cq, Ck, iters, top_p) == (64, 64, 2, 0.9) else None},
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------- AdaSpa blockified search --

def run_adaspa(args):
    """AdaSpa's schedule on one GPU ("AdaSpa" abstract): a dense step caches
    every row's LSE (untimed here: it is the last dense step of the schedule);
    a search step computes the exact block masses under that LSE, picks the
    kept tiles (top-p per head and query tile) and runs the block-sparse
    attention; later steps reuse the pattern (attention only).  Prints one
    JSON line; not the default bench line."""
    import torch

    import sparse_attention_video_qk_b200 as svg
    from sparse_attention_video_qk_b200._lib import check

    device = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    wl = W.WORKLOADS[args.workload]
    pb = svg.Problem.from_workload(wl)
    inp = W.make_inputs(wl)
    q, k, v = (torch.from_numpy(inp[n]).view(torch.bfloat16).to(device) for n in ("q", "k", "v"))
    gq, gk = (torch.from_numpy(inp[n]).to(device) for n in ("gamma_q", "gamma_k"))
    table = torch.from_numpy(svg.rope_table(pb)).to(device)
    qn, kn = svg.qknorm_rope(pb, q, k, gq, gk, table)
    stream = torch.cuda.current_stream()
    layer = svg.AdaSpaLayer(pb, args.adaspa_top_p)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    d0, d1 = ev(), ev()
    layer.dense(qn, kn, v)
    d0.record(stream)
    layer.dense(qn, kn, v)                               # the cached LSE comes from this dense step
    d1.record(stream)
    mass = torch.empty(pb.B * pb.H, pb.nqb, pb.nkb, dtype=torch.float32, device=device)
    cap = svg.block_index_capacity(pb)
    rp = torch.empty(pb.B * pb.H * pb.nqb + 1, dtype=torch.int32, device=device)
    col = torch.empty(cap, dtype=torch.int32, device=device)
    full = torch.empty(cap, dtype=torch.uint8, device=device)
    out = torch.empty_like(qn)
    kinds = torch.full((pb.B * pb.H,), svg.DENSE, dtype=torch.uint8, device=device)
    lib, sh, pr = svg.lib(), pb.c_shape(), pb.c_params()
    cs = ctypes.c_void_p(stream.cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())

    def search():
        check(lib.svg_adaspa_block_mass(ctypes.byref(sh), ctypes.byref(pr), P(qn), P(kn), P(layer.lse),
                                            P(mass), cs), "svg_adaspa_block_mass")

    def select():
        check(lib.svg_adaspa_select(ctypes.byref(sh), ctypes.byref(pr), P(mass), float(args.adaspa_top_p),
                                        P(rp), P(col), P(full), cap, cs), "svg_adaspa_select")

    def sparse():
        check(lib.svg_block_sparse_attn(ctypes.byref(sh), ctypes.byref(pr), P(qn), P(kn), P(v), P(kinds),
                                            P(rp), P(col), P(full), P(out), None, cs), "svg_block_sparse_attn")

    for _ in range(args.warmup):
        search()
        select()
        sparse()
    svg.sync_status()
    n_ent = int(rp[-1])
    flops = kept_tile_flops(rp.cpu().numpy(), col[:n_ent].cpu().numpy(), wl)
    evs = [[ev() for _ in range(4)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        clk.start()
        for s_ in range(args.steps):
            evs[s_][0].record(stream)
            search()
            evs[s_][1].record(stream)
            select()
            evs[s_][2].record(stream)
            sparse()
            evs[s_][3].record(stream)
        torch.cuda.synchronize()
        clk.stop()
    svg.sync_status()
    mean = lambda i: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs)
    mass_ms, select_ms, attn_ms = mean(0), mean(1), mean(2)
    dense_ms = d0.elapsed_time(d1)
    BH, L, d = wl.B * wl.H, wl.L, wl.d
    pk, pk_src = peaks()
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    exps = float(BH) * L * L                               # one 2^x per (row, key)
    mufu_peak = 148 * 16 * 1.965e9                         # 16 SFU results per SM per clock at 1965 MHz
    line = {
        "metric": "AdaSpa layer ms: search step (block masses + selection + sparse attention) and reuse step",
        "value": round(mass_ms + select_ms + attn_ms, 3), "unit": "ms", "higher_is_better": False,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q/K/V with planted spatial/temporal heads; no model weights)",
        "config": {"workload": f"{wl.name} ({SHAPE_LABEL[wl.name]}), AdaSpa blockified search",
                   "top_p": args.adaspa_top_p, "tile": f"{wl.bq}x{wl.bk}",
                   "tile_density": round(n_ent / (BH * wl.nqb * wl.nkb), 4),
                   "kept_tile_tflop": round(flops / 1e12, 4)},
        "stage_ms": {"block_mass": round(mass_ms, 3), "select": round(select_ms, 3), "attention": round(attn_ms, 3)},
        "reuse_step_ms": round(attn_ms, 3),
        "dense_attention_ms": round(dense_ms, 3),
        "speedup_reuse_vs_dense": round(dense_ms / attn_ms, 3),
        "roofline": {"kernel": f"attn2_kernel<{d}> (block list, every head dense)", "bound": "tensor",
                     "achieved": round(attn_tflops, 2), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(attn_tflops / pk["bf16_tflops"], 4),
                     "peak_source": f"{pk_src} bf16 burst", "traffic": None},
        "mass_roofline": {"kernel": f"mass_kernel<{d}>", "bound": "alu", "unit": "G exp2/s",
                          "achieved": round(exps / (mass_ms * 1e-3) / 1e9, 1), "peak": round(mufu_peak / 1e9, 1),
                          "frac": round(exps / (mass_ms * 1e-3) / mufu_peak, 4),
                          "tensor_tflops": round(2.0 * BH * L * L * d / (mass_ms * 1e-3) / 1e12, 1)},
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------ sparsity sweep --

def token_density(wl, kind):
    """Kept (query, key) pairs over video query rows against all L keys, from
    the masks' closed forms (text keys always kept)."""
    F, S, T, L = wl.F, wl.S, wl.T, wl.L
    if kind == W.SPATIAL:
        f = np.arange(F)
        frames = np.minimum(f + wl.w, F - 1) - np.maximum(f - wl.w, 0) + 1
        kept = float(np.sum(frames * S + T)) * S
    else:
        s = np.arange(S)
        locs = np.minimum(s + wl.r, S - 1) - np.maximum(s - wl.r, 0) + 1
        kept = float(np.sum(locs * F + T)) * F
    return kept / (float(wl.Lv) * L)


def run_sweep(args):
    """Forced-kind sweep at the HunyuanVideo shape: every head spatial with
    w in {0,1,2,4,8}, then every head temporal (layout applied) with r in
    {32,...,1800}; attention time against dense on the same inputs."""
    import torch

    import sparse_attention_video_qk_b200 as svg

    device = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    base = W.HUNYUAN_SWEEP
    pb0 = svg.Problem.from_workload(base)
    g = torch.Generator(device=device).manual_seed(base.seed)
    shp = (base.B, base.H, base.L, base.d)
    q, k, v = (torch.randn(shp, generator=g, device=device).to(torch.bfloat16) for _ in range(3))
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()

    def time_attn(pb, qq, kk, vv, kinds, rp, col, full, reps):
        for _ in range(args.warmup):
            svg.block_sparse_attn(pb, qq, kk, vv, kinds, rp, col, full, out=out)
        torch.cuda.synchronize()
        ms = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            svg.block_sparse_attn(pb, qq, kk, vv, kinds, rp, col, full, out=out)
            e1.record(stream)
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        svg.sync_status()
        return statistics.median(ms)

    dk = torch.full((base.B * base.H,), svg.DENSE, dtype=torch.uint8, device=device)
    rp, col, full = svg.build_block_index(pb0, dk, svg.block_index_capacity(pb0))
    dense_ms = time_attn(pb0, q, k, v, dk, rp, col, full, max(3, args.steps // 4))
    dense_flops = kept_tile_flops(rp.cpu().numpy(), col[: int(rp[-1])].cpu().numpy(), base)
    points = []
    with ClockSampler(0) as clk:
        clk.start()
        for label, wl in W.sweep_points():
            pb = svg.Problem.from_workload(wl)
            kind = wl.forced_kinds[0]
            kinds = torch.full((wl.B * wl.H,), kind, dtype=torch.uint8, device=device)
            qq, kk, vv = svg.layout(pb, q, k, v, kinds) if kind == W.TEMPORAL else (q, k, v)
            rp, col, full = svg.build_block_index(pb, kinds, svg.block_index_capacity(pb))
            ms = time_attn(pb, qq, kk, vv, kinds, rp, col, full, args.steps)
            nnz = int(rp[-1])
            flops = kept_tile_flops(rp.cpu().numpy(), col[:nnz].cpu().numpy(), wl)
            td = token_density(wl, kind)
            points.append({
                "point": label, "ms": round(ms, 3), "tflops": round(flops / (ms * 1e-3) / 1e12, 1),
                "kept_tile_tflop": round(flops / 1e12, 3), "token_density": round(td, 4),
                "tile_density": round(flops / dense_flops, 4),
                "speedup_vs_dense": round(dense_ms / ms, 2),
                "theoretical_tiles": round(dense_flops / flops, 2),
                "theoretical_tokens": round(1.0 / td, 2)})
            del qq, kk, vv
        clk.stop()
    pk, pk_src = peaks()
    return {"sweep": "forced-kind sparsity sweep at the HunyuanVideo 720p 5 s shape",
            "steps_per_point": args.steps, "warmup": args.warmup, "statistic": "median CUDA-event ms",
            "dense": {"ms": round(dense_ms, 3), "tflops": round(dense_flops / (dense_ms * 1e-3) / 1e12, 1),
                      "tflop": round(dense_flops / 1e12, 3)},
            "peak_bf16_burst": pk["bf16_tflops"], "peak_source": pk_src,
            "points": [dict(p, frac_of_burst_peak=round(p["tflops"] / pk["bf16_tflops"], 4)) for p in points],
            "clocks": clk.summary(),
            "data": "synthetic N(0,1) bf16 Q/K/V, head kinds forced"}


# ---------------------------------------------------------- oracle (CPU) --

def oracle_sample_rate(wl, inp, n_rows: int, seed: int = 0):
    """Times the fp64 oracle on a bounded sample of the step: QK-Norm+RoPE of
    the sampled rows' Q and of K, and masked attention of `n_rows` query rows
    spread over the heads (planted head kinds).  Returns (TFLOP/s counted like
    the GPU metric, seconds, threads, description)."""
    import oracle
    sh, pr = oracle.shape_of(wl), oracle.params_of(wl)
    kinds = np.array([0 if c == "S" else 1 for c in wl.planted], np.uint8)
    rng = np.random.Generator(np.random.PCG64(seed))
    per_head = max(1, min(wl.L, n_rows // (wl.B * wl.H)))
    rows = np.concatenate([bh * wl.L + rng.choice(wl.L, per_head, replace=False) for bh in range(wl.B * wl.H)])
    # the attention rows need normalised Q rows and every normalised K row of their heads
    t0 = time.perf_counter()
    qn_rows = oracle.qknorm_rope_f64(sh, pr, inp["q"], inp["gamma_q"], rows)
    kn = oracle.qknorm_rope(sh, pr, inp["k"], inp["gamma_k"])
    qn = np.zeros_like(inp["q"]).reshape(-1, wl.d)
    qn[rows] = oracle.f64_to_bf16(qn_rows)
    qn = qn.reshape(inp["q"].shape)
    oracle.attention_rows(sh, pr, kinds, qn, kn, inp["v"], rows)
    secs = time.perf_counter() - t0
    # FLOPs the GPU metric would count for these rows: 4*d per (row, key column) of its kept tiles
    flops = 0.0
    cache = {}
    for r in rows:
        bh, tok = divmod(int(r), wl.L)
        kind = int(kinds[bh])
        qb = oracle.perm(sh, kind, tok) // wl.bq
        if (kind, qb) not in cache:
            cache[(kind, qb)] = kept_cols_closed(wl, kind, qb)
        flops += 4.0 * wl.d * cache[(kind, qb)]
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    desc = (f"fp64 oracle: QK-Norm+RoPE of {len(rows)} Q rows and all K rows, masked attention of "
            f"{len(rows)} query rows ({per_head} per head), FLOPs counted as kept-tile columns x 4d")
    return flops / secs / 1e12, secs, threads, desc


def kept_cols_closed(wl, kind, qb):
    """Key columns of the tiles listed for one query tile (used only to count
    the oracle sample's FLOPs at the largest shape)."""
    L, Lv, S, F, bq, bk = wl.L, wl.Lv, wl.S, wl.F, wl.bq, wl.bk
    r0, r1 = qb * bq, min(L, qb * bq + bq)
    nkb = wl.nkb
    if kind == 2 or r1 > Lv:
        kbs = range(nkb)
    else:
        def iv(p):
            if kind == 0:
                f = p // S
                return max(f - wl.w, 0) * S, min(f + wl.w + 1, F) * S
            s = p // F
            return max(s - wl.r, 0) * F, min(s + wl.r + 1, S) * F
        lo, hi = iv(r0)[0], iv(r1 - 1)[1]
        kbs = set(range(lo // bk, (hi - 1) // bk + 1))
        if wl.T > 0:
            kbs |= set(range(Lv // bk, nkb))
    return int(sum(min(bk, L - kb * bk) for kb in kbs))


def cpu_baseline(wl, inp, n_rows):
    rate, secs, threads, desc = oracle_sample_rate(wl, inp, n_rows)
    return {"value": round(rate, 8), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": desc, "seconds": round(secs, 2)}


def run_reference(args, rank):
    if rank != 0:
        return None
    wl = W.WORKLOADS[args.workload]
    inp = W.make_inputs(wl)
    rates, secs_all = [], []
    for s in range(args.warmup + args.steps):
        rate, secs, threads, desc = oracle_sample_rate(wl, inp, args.ref_rows, seed=s)
        if s >= args.warmup:
            rates.append(rate)
            secs_all.append(secs)
    value = statistics.mean(rates)
    flops_step = value * 1e12 * statistics.mean(secs_all)
    return {
        "metric": METRIC, "value": round(value, 8), "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1000 * statistics.mean(secs_all), 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": f"{wl.name} ({SHAPE_LABEL[wl.name]})", "B": wl.B, "H": wl.H, "d": wl.d,
                   "seq_len": wl.L, "sampled_rows_per_step": args.ref_rows,
                   "kept_tile_gflop_per_step": round(flops_step / 1e9, 3)},
        "cpu_baseline": {"value": round(value, 8), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 8), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------- main --

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=W.HUNYUAN.name, choices=sorted(W.WORKLOADS))
    ap.add_argument("--cpu-rows", type=int, default=14400)
    ap.add_argument("--ref-rows", type=int, default=960)
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--svg2", action="store_true",
                    help="time the semantic-aware permutation step (SVG2) instead of the default step")
    ap.add_argument("--svg2-clusters", type=int, default=64)
    ap.add_argument("--svg2-iters", type=int, default=2)
    ap.add_argument("--svg2-top-p", type=float, default=0.9)
    ap.add_argument("--adaspa", action="store_true",
                    help="time AdaSpa's search step and reuse step instead of the default step")
    ap.add_argument("--adaspa-top-p", type=float, default=0.9)
    ap.add_argument("--sweep", action="store_true",
                    help="forced-kind sparsity sweep (one GPU); prints one JSON line with every point")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if world != args.gpus:
        world = max(world, 1)
    if args.svg2:
        if rank == 0:
            run_svg2(args)
        return
    if args.adaspa:
        if rank == 0:
            run_adaspa(args)
        return
    if args.sweep:
        if rank == 0:
            print(json.dumps(run_sweep(args)), flush=True)
        return
    if args.impl == "reference":
        line = run_reference(args, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local_rank))
    try:
        line = run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
