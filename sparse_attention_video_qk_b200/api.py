"""Python binding of the C ABI (include/svg.h).

Argument marshalling only: torch tensors are passed to the library as raw
device pointers on the current CUDA stream; every stage runs in the library's
sm_100a kernels.  PyTorch provides device memory and streams.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np
import torch

from . import _lib as C
from ._lib import check, lib

SPATIAL, TEMPORAL, DENSE = C.SVG_HEAD_SPATIAL, C.SVG_HEAD_TEMPORAL, C.SVG_HEAD_DENSE


@dataclass(frozen=True)
class Problem:
    """Shape and mask parameters of one attention layer (see svg_shape / svg_params)."""
    B: int
    H: int
    d: int
    F: int
    Hs: int
    Ws: int
    text_len: int
    spatial_frames: int
    temporal_radius: int
    block_q: int = 128
    block_k: int = 64
    eps: float = 1e-6
    rope_base: float = 10000.0
    rope_split: tuple = None
    softmax_scale: float = 0.0

    @property
    def S(self):
        return self.Hs * self.Ws

    @property
    def Lv(self):
        return self.F * self.S

    @property
    def L(self):
        return self.Lv + self.text_len

    @property
    def nqb(self):
        return -(-self.L // self.block_q)

    @property
    def nkb(self):
        return -(-self.L // self.block_k)

    @classmethod
    def from_workload(cls, wl, **over):
        kw = dict(B=wl.B, H=wl.H, d=wl.d, F=wl.F, Hs=wl.Hs, Ws=wl.Ws, text_len=wl.T,
                  spatial_frames=wl.w, temporal_radius=wl.r, block_q=wl.bq, block_k=wl.bk,
                  eps=wl.eps, rope_base=wl.rope_base, rope_split=tuple(wl.rope_split))
        kw.update(over)
        return cls(**kw)

    def c_shape(self) -> C.SvgShape:
        return C.SvgShape(self.B, self.H, self.L, self.d, self.F, self.Hs, self.Ws, self.text_len)

    def c_params(self) -> C.SvgParams:
        split = self.rope_split or (self.d // 4, 3 * self.d // 8, 3 * self.d // 8)
        return C.SvgParams(self.spatial_frames, self.temporal_radius, self.block_q, self.block_k,
                           self.eps, self.rope_base, (ctypes.c_int * 3)(*split), self.softmax_scale)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _empty_like_bf16(x):
    return torch.empty_like(x)


# ------------------------------------------------------------ host helpers --

def sample_queries(seed: int, Lv: int, n: int) -> np.ndarray:
    out = np.empty(n, np.int32)
    check(lib().svg_sample_queries(seed, Lv, n, out.ctypes.data), "svg_sample_queries")
    return out


def rope_table(pb: Problem) -> np.ndarray:
    sh, pr = pb.c_shape(), pb.c_params()
    n = lib().svg_rope_table_size(ctypes.byref(sh), ctypes.byref(pr))
    out = np.empty(n, np.float32)
    check(lib().svg_rope_table_fill(ctypes.byref(sh), ctypes.byref(pr), out.ctypes.data), "svg_rope_table_fill")
    return out


def block_index_capacity(pb: Problem) -> int:
    sh, pr = pb.c_shape(), pb.c_params()
    return int(lib().svg_block_index_capacity(ctypes.byref(sh), ctypes.byref(pr)))


def profile_workspace_size(pb: Problem, n: int) -> int:
    sh = pb.c_shape()
    return int(lib().svg_profile_workspace_size(ctypes.byref(sh), n))


def workspace_size(pb: Problem) -> int:
    """svg_workspace_size: device scratch bytes of the workspace-taking calls."""
    sh, pr = pb.c_shape(), pb.c_params()
    return int(lib().svg_workspace_size(ctypes.byref(sh), ctypes.byref(pr)))


def release():
    """svg_release: waits for and frees the library's cached streams, events and
    pinned staging (the host-buffer step's).  Also drops this module's cached
    HostStep workspaces."""
    _HOST_STEPS.clear()
    check(lib().svg_release(), "svg_release")


def sync_status(stream=None):
    """Synchronise the stream and raise if a kernel reported an error."""
    check(lib().svg_sync_status(_stream(stream)), "svg_sync_status")


# ------------------------------------------------------------------ stages --

def qknorm_rope_layout(pb: Problem, q, k, v=None, gamma_q=None, gamma_k=None, table=None, kinds=None,
                       flags=C.SVG_NORM_ROPE, out=None, stream=None):
    """Stage 1 (flags has NORM_ROPE) and/or stage 3 (flags has LAYOUT).
    Returns (q_out, k_out, v_out or None)."""
    sh, pr = pb.c_shape(), pb.c_params()
    if out is None:
        like = lambda t: torch.empty_like(t) if t is not None else None
        out = (like(q), like(k), like(v) if (flags & C.SVG_LAYOUT) else None)
    qo, ko, vo = out
    st = lib().svg_qknorm_rope_layout(ctypes.byref(sh), ctypes.byref(pr), flags, _p(q), _p(k), _p(v),
                                      _p(gamma_q), _p(gamma_k), _p(table), _p(kinds), _p(qo), _p(ko), _p(vo),
                                      _stream(stream))
    check(st, "svg_qknorm_rope_layout")
    return qo, ko, vo


def qknorm_rope(pb: Problem, q, k, gamma_q, gamma_k, table, out=None, stream=None):
    qo, ko, _ = qknorm_rope_layout(pb, q, k, None, gamma_q, gamma_k, table, None, C.SVG_NORM_ROPE,
                                   None if out is None else (out[0], out[1], None), stream)
    return qo, ko


def layout(pb: Problem, q, k, v, kinds, out=None, stream=None):
    return qknorm_rope_layout(pb, q, k, v, None, None, None, kinds, C.SVG_LAYOUT, out, stream)


def profile_heads(pb: Problem, qn, kn, v, sample_idx, workspace=None, kinds_out=None, mse_out=None, stream=None):
    """Returns (kinds uint8 [B*H], mse fp32 [B*H, 2])."""
    sh, pr = pb.c_shape(), pb.c_params()
    n = int(sample_idx.numel())
    need = profile_workspace_size(pb, n)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=qn.device)
    if kinds_out is None:
        kinds_out = torch.empty(pb.B * pb.H, dtype=torch.uint8, device=qn.device)
    if mse_out is None:
        mse_out = torch.empty(pb.B * pb.H, 2, dtype=torch.float32, device=qn.device)
    st = lib().svg_profile_heads(ctypes.byref(sh), ctypes.byref(pr), _p(qn), _p(kn), _p(v), _p(sample_idx), n,
                                 _p(workspace), workspace.numel() * workspace.element_size(), _p(mse_out),
                                 _p(kinds_out), _stream(stream))
    check(st, "svg_profile_heads")
    return kinds_out, mse_out


def profile_heads_raw_q(pb: Problem, q, gamma_q, table, kn, v, sample_idx, workspace=None, kinds_out=None,
                        mse_out=None, stream=None):
    """svg_profile_heads_raw_q: profiling from raw Q (the sampled rows are
    normalised in the kernel).  Returns (kinds uint8 [B*H], mse fp32 [B*H, 2])."""
    sh, pr = pb.c_shape(), pb.c_params()
    n = int(sample_idx.numel())
    if workspace is None:
        workspace = torch.empty(profile_workspace_size(pb, n), dtype=torch.uint8, device=q.device)
    if kinds_out is None:
        kinds_out = torch.empty(pb.B * pb.H, dtype=torch.uint8, device=q.device)
    if mse_out is None:
        mse_out = torch.empty(pb.B * pb.H, 2, dtype=torch.float32, device=q.device)
    st = lib().svg_profile_heads_raw_q(ctypes.byref(sh), ctypes.byref(pr), _p(q), _p(gamma_q), _p(table), _p(kn),
                                       _p(v), _p(sample_idx), n, _p(workspace),
                                       workspace.numel() * workspace.element_size(), _p(mse_out), _p(kinds_out),
                                       _stream(stream))
    check(st, "svg_profile_heads_raw_q")
    return kinds_out, mse_out


def profile_heads_noalloc(pb: Problem, qn, kn, v, sample_idx, kinds_out=None, mse_out=None, stream=None):
    """svg_profile_heads_noalloc: profiling with the library's fixed scratch
    (no workspace argument).  Returns (kinds uint8 [B*H], mse fp32 [B*H, 2])."""
    sh, pr = pb.c_shape(), pb.c_params()
    n = int(sample_idx.numel())
    if kinds_out is None:
        kinds_out = torch.empty(pb.B * pb.H, dtype=torch.uint8, device=qn.device)
    if mse_out is None:
        mse_out = torch.empty(pb.B * pb.H, 2, dtype=torch.float32, device=qn.device)
    st = lib().svg_profile_heads_noalloc(ctypes.byref(sh), ctypes.byref(pr), _p(qn), _p(kn), _p(v), _p(sample_idx),
                                         n, _p(mse_out), _p(kinds_out), _stream(stream))
    check(st, "svg_profile_heads_noalloc")
    return kinds_out, mse_out


def build_block_index(pb: Problem, kinds, capacity=None, out=None, stream=None):
    """Returns (row_ptr int32 [B*H*nqb+1], col int32 [capacity], full uint8 [capacity]).
    Only the first row_ptr[-1] entries of col/full are meaningful."""
    sh, pr = pb.c_shape(), pb.c_params()
    if capacity is None:
        capacity = block_index_capacity(pb)
    dev = kinds.device
    if out is None:
        out = (torch.empty(pb.B * pb.H * pb.nqb + 1, dtype=torch.int32, device=dev),
               torch.empty(capacity, dtype=torch.int32, device=dev),
               torch.empty(capacity, dtype=torch.uint8, device=dev))
    row_ptr, col, full = out
    st = lib().svg_build_block_index(ctypes.byref(sh), ctypes.byref(pr), _p(kinds), _p(row_ptr), _p(col), _p(full),
                                     capacity, _stream(stream))
    check(st, "svg_build_block_index")
    return row_ptr, col, full


def block_sparse_attn(pb: Problem, q, k, v, kinds, row_ptr, col, full, out=None, want_lse=False, stream=None,
                      model_order=False):
    """Stage 4.  out (and lse) in the head's layout, or with model_order=True
    in model order (stage 5 fused into the epilogue)."""
    sh, pr = pb.c_shape(), pb.c_params()
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty(pb.B, pb.H, pb.L, dtype=torch.float32, device=q.device) if want_lse else None
    name = "svg_block_sparse_attn_model_order" if model_order else "svg_block_sparse_attn"
    st = getattr(lib(), name)(ctypes.byref(sh), ctypes.byref(pr), _p(q), _p(k), _p(v), _p(kinds),
                              _p(row_ptr), _p(col), _p(full), _p(out), _p(lse), _stream(stream))
    check(st, name)
    return (out, lse) if want_lse else out


def inverse_layout(pb: Problem, kinds, src, out=None, stream=None):
    sh = pb.c_shape()
    if out is None:
        out = torch.empty_like(src)
    st = lib().svg_inverse_layout(ctypes.byref(sh), _p(kinds), _p(src), _p(out), _stream(stream))
    check(st, "svg_inverse_layout")
    return out


# --------------------------------------------------------------- full step --

class StepBuffers:
    """Device buffers of one step, allocated once for a Problem and reused.
    With head_layout_out=True the step also keeps the attention output in the
    head's layout (`op`) and runs the inverse layout as a pass of its own;
    otherwise (default) the attention writes `out` in model order directly."""

    def __init__(self, pb: Problem, n_samples: int, device="cuda", head_layout_out=False):
        shp = (pb.B, pb.H, pb.L, pb.d)
        mk = lambda: torch.empty(shp, dtype=torch.bfloat16, device=device)
        self.pb = pb
        self.n = n_samples
        self.kn, self.qp, self.kp, self.vp, self.out = (mk() for _ in range(5))
        self.op = mk() if head_layout_out else None
        self.kinds = torch.empty(pb.B * pb.H, dtype=torch.uint8, device=device)
        self.mse = torch.empty(pb.B * pb.H, 2, dtype=torch.float32, device=device)
        self.capacity = block_index_capacity(pb)
        self.row_ptr = torch.empty(pb.B * pb.H * pb.nqb + 1, dtype=torch.int32, device=device)
        self.col = torch.empty(self.capacity, dtype=torch.int32, device=device)
        self.full = torch.empty(self.capacity, dtype=torch.uint8, device=device)
        self.workspace = torch.empty(max(profile_workspace_size(pb, n_samples), 16), dtype=torch.uint8,
                                     device=device)
        self.table = torch.from_numpy(rope_table(pb)).to(device)


def attention_step(pb: Problem, q, k, v, gamma_q, gamma_k, sample_idx, buffers: StepBuffers,
                   kinds_in=None, stream=None):
    """All five stages on device tensors through svg_attention_step; returns
    buffers.out (model order).  With kinds_in the profiling stage is skipped."""
    b = buffers
    sh, pr = pb.c_shape(), pb.c_params()
    st = lib().svg_attention_step(
        ctypes.byref(sh), ctypes.byref(pr), _p(q), _p(k), _p(v), _p(gamma_q), _p(gamma_k), _p(b.table),
        _p(sample_idx), int(sample_idx.numel()), _p(kinds_in), _p(b.kn), _p(b.qp), _p(b.kp), _p(b.vp),
        _p(b.op), _p(b.out), _p(b.kinds), _p(b.mse), _p(b.row_ptr), _p(b.col), _p(b.full), b.capacity,
        _p(b.workspace), b.workspace.numel(), _stream(stream))
    check(st, "svg_attention_step")
    return b.out


class HostStep:
    """svg_attention_step_host for one Problem: the step on host tensors, the
    host<->device copies overlapped with the passes over `groups` head groups
    inside the library.  Holds the device workspace the call needs (allocated
    once, reused by every call; calls are ordered on one stream)."""

    def __init__(self, pb: Problem, n_samples: int, groups: int = 8, device="cuda"):
        self.pb, self.n = pb, int(n_samples)
        self.groups = max(1, min(int(groups), pb.B * pb.H))
        sh, pr = pb.c_shape(), pb.c_params()
        size = lib().svg_attention_step_host_workspace_size(ctypes.byref(sh), ctypes.byref(pr), self.n, self.groups)
        if size == 0:
            raise ValueError("svg_attention_step_host_workspace_size: invalid shape, parameters or group count")
        self.workspace = torch.empty(size, dtype=torch.uint8, device=device)

    def __call__(self, q_host, k_host, v_host, gamma_q, gamma_k, sample_idx, out_host=None, kinds_out=None,
                 stream=None):
        """q/k/v_host: bf16 [B,H,L,d] on the host (pinned for overlap); gamma: fp32 [d];
        sample_idx: int32 [n] (host tensors).  Returns out_host (bf16 [B,H,L,d], pinned
        if allocated here); kinds_out, if given, receives the uint8 [B*H] head kinds.
        The current stream (or `stream`) waits for the last copy."""
        pb = self.pb
        if out_host is None:
            out_host = torch.empty(q_host.shape, dtype=torch.bfloat16, pin_memory=True)
        for t in (q_host, k_host, v_host, gamma_q, gamma_k, sample_idx, out_host):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError("host tensors must be contiguous CPU tensors")
        gq = gamma_q.to(torch.float32).contiguous()
        gk = gamma_k.to(torch.float32).contiguous()
        si = sample_idx.to(torch.int32).contiguous()
        if int(si.numel()) != self.n:
            raise ValueError(f"{si.numel()} sampled rows; this HostStep was made for {self.n}")
        sh, pr = pb.c_shape(), pb.c_params()
        cs = torch.cuda.current_stream(self.workspace.device) if stream is None else stream
        check(lib().svg_attention_step_host(ctypes.byref(sh), ctypes.byref(pr), _p(q_host), _p(k_host), _p(v_host),
                                            _p(gq), _p(gk), _p(si), self.n, _p(out_host), _p(kinds_out), self.groups,
                                            _p(self.workspace), self.workspace.numel(), _stream(cs)),
              "svg_attention_step_host")
        return out_host


_HOST_STEPS = {}


def sparse_attention(pb: Problem, q_host, k_host, v_host, gamma_q, gamma_k, sample_idx, out_host=None,
                     device="cuda", groups: int = 8, host_step: HostStep = None):
    """End-to-end call on host tensors: Q/K/V (bf16 [B,H,L,d], pinned so the
    copies are asynchronous), gamma and the sample go in, O comes back in
    `out_host` (allocated pinned if None), through svg_attention_step_host with
    `groups` head groups (its workspace created once per shape and cached, or
    passed in as `host_step`).  Work is ordered after the current stream, and
    the current stream waits for the last copy.  Returns out_host."""
    if host_step is None:
        key = (pb, int(sample_idx.numel()), int(groups), str(device))
        host_step = _HOST_STEPS.get(key)
        if host_step is None:
            host_step = _HOST_STEPS[key] = HostStep(pb, int(sample_idx.numel()), groups, device)
    return host_step(q_host, k_host, v_host, gamma_q, gamma_k, sample_idx, out_host)


# ------------------------------------------- semantic-aware permutation --

def svg2_kmeans(pb: Problem, x, C: int, iters: int, cent=None, stream=None):
    """k-means of the video rows of every head of x (bf16 [B,H,L,d]); starts from
    `cent` (float [B*H, C, d], e.g. the previous step's) or from evenly spaced
    rows.  Returns (cent, assign uint8 [B*H, Lv], counts int32 [B*H, C])."""
    sh = pb.c_shape()
    bh, dev = pb.B * pb.H, x.device
    init = cent is None
    if init:
        cent = torch.empty(bh, C, pb.d, dtype=torch.float32, device=dev)
    assign = torch.empty(bh, pb.Lv, dtype=torch.uint8, device=dev)
    counts = torch.empty(bh, C, dtype=torch.int32, device=dev)
    ws = torch.empty(max(lib().svg2_kmeans_workspace_size(ctypes.byref(sh), C), 16), dtype=torch.uint8, device=dev)
    check(lib().svg2_kmeans(ctypes.byref(sh), _p(x), C, iters, int(init), _p(cent), _p(assign), _p(counts), _p(ws),
                            ws.numel(), _stream(stream)), "svg2_kmeans")
    return cent, assign, counts


def svg2_permutation(pb: Problem, assign, C: int, stream=None):
    """Stable cluster sort: (perm int32 [B*H, Lv], off int32 [B*H, C+1])."""
    sh = pb.c_shape()
    bh = pb.B * pb.H
    perm = torch.empty(bh, pb.Lv, dtype=torch.int32, device=assign.device)
    off = torch.empty(bh, C + 1, dtype=torch.int32, device=assign.device)
    check(lib().svg2_permutation(ctypes.byref(sh), _p(assign), C, _p(perm), _p(off), _stream(stream)),
          "svg2_permutation")
    return perm, off


def svg2_select(pb: Problem, cq, ck, counts_k, top_p: float, stream=None):
    """Top-p key clusters per query cluster: uint64 masks [B*H, Cq] (as int64)."""
    sh, pr = pb.c_shape(), pb.c_params()
    bh, Cq, Ck = pb.B * pb.H, cq.shape[1], ck.shape[1]
    sel = torch.empty(bh, Cq, dtype=torch.int64, device=cq.device)
    check(lib().svg2_select(ctypes.byref(sh), ctypes.byref(pr), _p(cq), _p(ck), _p(counts_k), Cq, Ck, float(top_p),
                            _p(sel), _stream(stream)), "svg2_select")
    return sel


def svg2_permute(pb: Problem, perm_q, perm_k, q, k, v, stream=None):
    sh = pb.c_shape()
    qo, ko, vo = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    check(lib().svg2_permute(ctypes.byref(sh), _p(perm_q), _p(perm_k), _p(q), _p(k), _p(v), _p(qo), _p(ko), _p(vo),
                             _stream(stream)), "svg2_permute")
    return qo, ko, vo


def svg2_block_index(pb: Problem, qoff, koff, sel, capacity=None, stream=None):
    sh, pr = pb.c_shape(), pb.c_params()
    Cq, Ck = qoff.shape[1] - 1, koff.shape[1] - 1
    if capacity is None:
        capacity = block_index_capacity(pb)
    dev = qoff.device
    row_ptr = torch.empty(pb.B * pb.H * pb.nqb + 1, dtype=torch.int32, device=dev)
    col = torch.empty(capacity, dtype=torch.int32, device=dev)
    full = torch.empty(capacity, dtype=torch.uint8, device=dev)
    check(lib().svg2_build_block_index(ctypes.byref(sh), ctypes.byref(pr), Cq, Ck, _p(qoff), _p(koff), _p(sel),
                                       _p(row_ptr), _p(col), _p(full), capacity, _stream(stream)),
          "svg2_build_block_index")
    return row_ptr, col, full


def svg2_attention(pb: Problem, q, k, v, qoff, koff, sel, perm_q, row_ptr, col, full, out=None, want_lse=False,
                   stream=None):
    """Attention in cluster order, written back in model order."""
    sh, pr = pb.c_shape(), pb.c_params()
    Cq, Ck = qoff.shape[1] - 1, koff.shape[1] - 1
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty(pb.B, pb.H, pb.L, dtype=torch.float32, device=q.device) if want_lse else None
    check(lib().svg2_attention(ctypes.byref(sh), ctypes.byref(pr), _p(q), _p(k), _p(v), Cq, Ck, _p(qoff), _p(koff),
                               _p(sel), _p(perm_q), _p(row_ptr), _p(col), _p(full), _p(out), _p(lse),
                               _stream(stream)), "svg2_attention")
    return (out, lse) if want_lse else out


class SVG2Layer:
    """The semantic-aware permutation step on normalised Q, K and V: k-means of
    Q and K (warm-started from the previous call's centroids, the pages'
    centroid cache), cluster sort, top-p key clusters, block index, attention
    in cluster order written back in model order."""

    def __init__(self, pb: Problem, Cq: int = 64, Ck: int = 64, iters: int = 2, top_p: float = 0.9):
        self.pb, self.Cq, self.Ck, self.iters, self.top_p = pb, Cq, Ck, iters, top_p
        self.cq = self.ck = None
        self.last = None

    def __call__(self, qn, kn, v, stream=None):
        pb = self.pb
        cq, aq, nq = svg2_kmeans(pb, qn, self.Cq, self.iters, self.cq, stream)
        ck, ak, nk = svg2_kmeans(pb, kn, self.Ck, self.iters, self.ck, stream)
        self.cq, self.ck = cq, ck
        pq, qoff = svg2_permutation(pb, aq, self.Cq, stream)
        pk, koff = svg2_permutation(pb, ak, self.Ck, stream)
        sel = svg2_select(pb, cq, ck, nk, self.top_p, stream)
        qp, kp, vp = svg2_permute(pb, pq, pk, qn, kn, v, stream)
        row_ptr, col, full = svg2_block_index(pb, qoff, koff, sel, stream=stream)
        out = svg2_attention(pb, qp, kp, vp, qoff, koff, sel, pq, row_ptr, col, full, stream=stream)
        self.last = dict(assign_q=aq, assign_k=ak, counts_q=nq, counts_k=nk, perm_q=pq, perm_k=pk, qoff=qoff,
                         koff=koff, sel=sel, row_ptr=row_ptr, col=col, full=full)
        return out


# ---------------------------------------------- AdaSpa blockified search --

def adaspa_block_mass(pb: Problem, q, k, lse, out=None, stream=None):
    """Block attention masses float [B*H, nqb, nkb] from normalised q, k (bf16
    [B,H,L,d]) and each row's cached log-sum-exp (float [B,H,L])."""
    sh, pr = pb.c_shape(), pb.c_params()
    if out is None:
        out = torch.empty(pb.B * pb.H, pb.nqb, pb.nkb, dtype=torch.float32, device=q.device)
    check(lib().svg_adaspa_block_mass(ctypes.byref(sh), ctypes.byref(pr), _p(q), _p(k), _p(lse), _p(out),
                                      _stream(stream)), "svg_adaspa_block_mass")
    return out


def adaspa_select(pb: Problem, mass, top_p: float, capacity=None, stream=None):
    """Kept key tiles (row_ptr, col, full) of every (head, query tile)."""
    sh, pr = pb.c_shape(), pb.c_params()
    if capacity is None:
        capacity = block_index_capacity(pb)
    dev = mass.device
    row_ptr = torch.empty(pb.B * pb.H * pb.nqb + 1, dtype=torch.int32, device=dev)
    col = torch.empty(capacity, dtype=torch.int32, device=dev)
    full = torch.empty(capacity, dtype=torch.uint8, device=dev)
    check(lib().svg_adaspa_select(ctypes.byref(sh), ctypes.byref(pr), _p(mass), float(top_p), _p(row_ptr), _p(col),
                                  _p(full), capacity, _stream(stream)), "svg_adaspa_select")
    return row_ptr, col, full


class AdaSpaLayer:
    """AdaSpa's schedule for one layer: a dense step keeps every row's LSE;
    at a search step the block masses under that cached LSE pick the kept
    tiles (top-p per head and query tile); later steps reuse the pattern
    until the next search.  Works on normalised Q, K (model order)."""

    def __init__(self, pb: Problem, top_p: float = 0.9):
        self.pb, self.top_p = pb, top_p
        self.lse = None
        self.blocks = None
        self._dense_kinds = None

    def _kinds(self, device):
        if self._dense_kinds is None or self._dense_kinds.device != device:
            self._dense_kinds = torch.full((self.pb.B * self.pb.H,), DENSE, dtype=torch.uint8, device=device)
        return self._dense_kinds

    def dense(self, qn, kn, v, stream=None):
        """Dense attention; keeps each row's LSE for the next search."""
        kinds = self._kinds(qn.device)
        rp, col, full = build_block_index(self.pb, kinds, stream=stream)
        out, self.lse = block_sparse_attn(self.pb, qn, kn, v, kinds, rp, col, full, want_lse=True, stream=stream)
        return out

    def search(self, qn, kn, stream=None):
        if self.lse is None:
            raise RuntimeError("AdaSpaLayer.search needs the LSE of an earlier dense step")
        mass = adaspa_block_mass(self.pb, qn, kn, self.lse, stream=stream)
        self.blocks = adaspa_select(self.pb, mass, self.top_p, stream=stream)
        return mass

    def sparse(self, qn, kn, v, stream=None):
        if self.blocks is None:
            raise RuntimeError("AdaSpaLayer.sparse needs a search first")
        rp, col, full = self.blocks
        return block_sparse_attn(self.pb, qn, kn, v, self._kinds(qn.device), rp, col, full, stream=stream)


# ------------------------------------------------------ denoising schedule --

STEP_DENSE, STEP_PROFILE, STEP_REUSE = C.SVG_STEP_DENSE, C.SVG_STEP_PROFILE, C.SVG_STEP_REUSE


def step_policy(step: int, total_steps: int, dense_fraction: float = 0.25, reprofile_every: int = 1) -> int:
    """STEP_DENSE, STEP_PROFILE or STEP_REUSE for one layer at a denoising step
    (svg_step_policy)."""
    mode = ctypes.c_int(-1)
    check(lib().svg_step_policy(int(step), int(total_steps), float(dense_fraction), int(reprofile_every),
                                ctypes.byref(mode)), "svg_step_policy")
    return mode.value


class SparseAttentionLayer:
    """One attention layer over a denoising schedule: all heads dense for the
    first `dense_fraction` of the steps, then sparse with online profiling;
    with reprofile_every > 1 the profiled head kinds are reused in between.
    Each call runs the whole step through svg_attention_step."""

    def __init__(self, pb: Problem, n_samples: int, total_steps: int, dense_fraction: float = 0.25,
                 reprofile_every: int = 1, device="cuda"):
        self.pb = pb
        self.total_steps = total_steps
        self.dense_fraction = dense_fraction
        self.reprofile_every = reprofile_every
        self.buffers = StepBuffers(pb, n_samples, device)
        self.dense_kinds = torch.full((pb.B * pb.H,), DENSE, dtype=torch.uint8, device=device)
        self.kinds = None          # the last profiled head kinds (device)
        self.last_mode = None

    def __call__(self, step: int, q, k, v, gamma_q, gamma_k, sample_idx, stream=None):
        mode = step_policy(step, self.total_steps, self.dense_fraction, self.reprofile_every)
        if mode == STEP_DENSE:
            kinds_in = self.dense_kinds
        elif mode == STEP_PROFILE:
            kinds_in = None
        else:
            if self.kinds is None:
                raise RuntimeError("REUSE step before any profiled step")
            kinds_in = self.kinds
        out = attention_step(self.pb, q, k, v, gamma_q, gamma_k, sample_idx, self.buffers, kinds_in=kinds_in,
                             stream=stream)
        if mode == STEP_PROFILE:
            self.kinds = self.buffers.kinds.clone()
        self.last_mode = mode
        return out

