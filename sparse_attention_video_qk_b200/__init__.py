"""B200-native (sm_100a) Sparse VideoGen attention step.

The library ``libsvg_b200.so`` (C ABI: include/svg.h) holds every kernel;
this package is its Python binding.  Build the library with
``python -m sparse_attention_video_qk_b200.build``.

Typical use, one layer of a video DiT (tensors bf16 [B, H, L, d] on the GPU,
video tokens frame-major and text tokens after them)::

    import sparse_attention_video_qk_b200 as svg
    pb = svg.Problem(B=1, H=24, d=128, F=33, Hs=45, Ws=80, text_len=256,
                     spatial_frames=1, temporal_radius=256)
    buf = svg.StepBuffers(pb, n_samples=64)                 # allocated once, reused
    sample = torch.from_numpy(svg.sample_queries(seed, pb.Lv, 64)).cuda()
    out = svg.attention_step(pb, q, k, v, gamma_q, gamma_k, sample, buf)

``SparseAttentionLayer`` adds the denoising schedule (dense for the first
quarter of the steps, then profiled), and ``sparse_attention`` /
``HostStep`` take pinned host tensors and overlap the copies with the
computation.  Each stage is also callable on its own (``qknorm_rope_layout``,
``profile_heads``, ``build_block_index``, ``block_sparse_attn``, ...).

Two further sparse-attention methods run on the same kernels, on normalised
Q and K (``qknorm_rope``)::

    svg2 = svg.SVG2Layer(pb, Cq=64, Ck=64, iters=2, top_p=0.9)   # semantic-aware permutation
    out = svg2(qn, kn, v)            # k-means (warm-started on later calls), sort, top-p, attention

    ada = svg.AdaSpaLayer(pb, top_p=0.9)                       # blockified LSE-cached search
    out = ada.dense(qn, kn, v)       # a dense step keeps every row's LSE
    ada.search(qn, kn)               # block masses under that LSE -> kept tiles
    out = ada.sparse(qn, kn, v)      # later steps reuse the pattern
"""
from ._lib import SVGError, lib  # noqa: F401
from .api import (DENSE, SPATIAL, TEMPORAL, Problem, StepBuffers, attention_step,  # noqa: F401
                  block_index_capacity, block_sparse_attn, build_block_index, inverse_layout, layout,
                  profile_heads, profile_heads_noalloc, profile_heads_raw_q, profile_workspace_size, qknorm_rope,
                  qknorm_rope_layout, release, rope_table, sample_queries, sparse_attention, sync_status,
                  workspace_size)
from .api import STEP_DENSE, STEP_PROFILE, STEP_REUSE, HostStep, SparseAttentionLayer, step_policy  # noqa: F401
from .api import AdaSpaLayer, adaspa_block_mass, adaspa_select  # noqa: F401
from .api import (SVG2Layer, svg2_attention, svg2_block_index, svg2_kmeans, svg2_permutation,  # noqa: F401
                  svg2_permute, svg2_select)

__all__ = [
    "SVGError", "lib", "Problem", "StepBuffers", "SPATIAL", "TEMPORAL", "DENSE",
    "qknorm_rope", "qknorm_rope_layout", "layout", "profile_heads", "profile_heads_noalloc", "profile_heads_raw_q",
    "build_block_index",
    "block_sparse_attn", "inverse_layout", "attention_step", "sparse_attention",
    "sample_queries", "rope_table", "block_index_capacity", "profile_workspace_size", "workspace_size", "release",
    "sync_status",
    "STEP_DENSE", "STEP_PROFILE", "STEP_REUSE", "step_policy", "SparseAttentionLayer", "HostStep",
    "AdaSpaLayer", "adaspa_block_mass", "adaspa_select",
    "SVG2Layer", "svg2_kmeans", "svg2_permutation", "svg2_select", "svg2_permute", "svg2_block_index",
    "svg2_attention",
]
