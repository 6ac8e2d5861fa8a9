"""Seeded synthetic workloads for the Sparse VideoGen attention step.

This module only *creates inputs*: shapes, parameters and seeded random
tensors.  It holds none of the method's arithmetic (no normalisation, RoPE,
masking, softmax or layout), so both the CUDA path and the fp64 oracle can use
it without sharing method code.

Shapes follow the video-DiT sizes the pages name (CogVideoX, Wan 2.1,
HunyuanVideo 720p 5 s; "Sparse VideoGen" WeChat article, first paragraphs and
"Motivation") and stand in for those models' real activations, whose weights
are not available.  Planted structure makes ground truth for profiling:

* planted spatial head: one N(0, sigma^2 I) vector per latent frame is added to
  Q and K of every video token of that frame;
* planted temporal head: one N(0, sigma^2 I) vector per spatial location is
  added to Q and K of that location in every frame;
* unplanted head: plain N(0, 1).

All values are drawn as float32 from numpy's PCG64 and rounded to bfloat16
(round to nearest even) -- the storage type of Q/K/V.

The profiling sample (``sample_idx``) is part of the input: n distinct video
token indices drawn by a partial Fisher-Yates shuffle driven by SplitMix64
(Steele, Lea, Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014; constants as published by Vigna).  The CUDA library exports an
independent C implementation (``svg_sample_queries``) that tests compare
against this one.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np

SPATIAL, TEMPORAL, DENSE = 0, 1, 2
_MASK64 = (1 << 64) - 1


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    F: int
    Hs: int
    Ws: int
    T: int
    w: int                      # spatial window (frames)
    r: int                      # temporal radius (spatial index)
    n_samples: int              # profiled query rows per head
    bq: int                     # query tile rows
    bk: int                     # key tile columns
    planted: tuple              # per head: "S", "T" or "U"
    rope_split: tuple           # t:h:w widths, sum = d
    eps: float = 1e-6
    rope_base: float = 10000.0
    sigma: float = 2.0
    seed: int = 0
    forced_kinds: tuple | None = None   # sweep points fix the head kinds (no profiling)

    @property
    def S(self) -> int:
        return self.Hs * self.Ws

    @property
    def Lv(self) -> int:
        return self.F * self.S

    @property
    def L(self) -> int:
        return self.Lv + self.T

    @property
    def nqb(self) -> int:
        return -(-self.L // self.bq)

    @property
    def nkb(self) -> int:
        return -(-self.L // self.bk)


def _alt(H, pattern):
    return tuple(pattern[h % len(pattern)] for h in range(H))


# The workloads.  Block size is given only for the tiny and CogVideoX shapes;
# the 128 x 64 tile of the CogVideoX shape is used for the larger shapes as
# well.  The RoPE split is given only for d = 64 (16:24:24); for d = 128 the
# same ratio (32:48:48) is used.
TINY = Workload("tiny-f4-8x8", B=1, H=2, d=64, F=4, Hs=8, Ws=8, T=0, w=1, r=8, n_samples=16,
                bq=64, bk=64, planted=("S", "T"), rope_split=(16, 24, 24), seed=1000)
COGVIDEOX = Workload("cogvideox-f13-30x45", B=1, H=48, d=64, F=13, Hs=30, Ws=45, T=226, w=1, r=64,
                     n_samples=64, bq=128, bk=64, planted=_alt(48, "ST"), rope_split=(16, 24, 24),
                     seed=1001)
WAN = Workload("wan2.1-1.3b-f21-30x52", B=1, H=12, d=128, F=21, Hs=30, Ws=52, T=512, w=1, r=96,
               n_samples=64, bq=128, bk=64, planted=_alt(12, "STU"), rope_split=(32, 48, 48),
               seed=1002)
HUNYUAN = Workload("hunyuanvideo-720p-5s-f33-45x80", B=1, H=24, d=128, F=33, Hs=45, Ws=80, T=256,
                   w=1, r=256, n_samples=64, bq=128, bk=64, planted=_alt(24, "ST"),
                   rope_split=(32, 48, 48), seed=1003)
# the HunyuanVideo shape with the head kinds forced, one density per point
HUNYUAN_SWEEP = replace(HUNYUAN, name="hunyuanvideo-sparsity-sweep", seed=1004)

WORKLOADS = {w.name: w for w in (TINY, COGVIDEOX, WAN, HUNYUAN, HUNYUAN_SWEEP)}

# Sweep points (head kinds forced, so each point has one density).
SWEEP_SPATIAL_W = (0, 1, 2, 4, 8)
SWEEP_TEMPORAL_R = (32, 64, 128, 256, 512, 900, 1800)


def sweep_points():
    """(label, workload) pairs of the sparsity sweep at the HunyuanVideo shape."""
    base = HUNYUAN_SWEEP
    pts = []
    for w in SWEEP_SPATIAL_W:
        pts.append((f"spatial_w{w}", replace(base, w=w, forced_kinds=(SPATIAL,) * base.H)))
    for r in SWEEP_TEMPORAL_R:
        pts.append((f"temporal_r{r}", replace(base, r=r, forced_kinds=(TEMPORAL,) * base.H)))
    return pts


def small_workload(**kw) -> Workload:
    """A custom small workload for edge-case tests."""
    d = kw.get("d", 64)
    H = kw.get("H", 2)
    split = kw.pop("rope_split", (d // 4, 3 * d // 8, 3 * d // 8))
    defaults = dict(name="custom", B=1, H=H, d=d, F=4, Hs=4, Ws=6, T=0, w=1, r=3, n_samples=8,
                    bq=128, bk=64, planted=_alt(H, "ST"), rope_split=split, seed=7)
    defaults.update(kw)
    return Workload(**defaults)


# --------------------------------------------------------------- SplitMix64 --

def splitmix64_stream(seed: int):
    """SplitMix64: state += golden gamma; output = mix(state)."""
    state = seed & _MASK64
    while True:
        state = (state + 0x9E3779B97F4A7C15) & _MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        yield z ^ (z >> 31)


def sample_queries(seed: int, Lv: int, n: int) -> np.ndarray:
    """n distinct indices in [0, Lv): the first n slots of a partial
    Fisher-Yates shuffle of 0..Lv-1, where slot i swaps with
    i + (x mod (Lv - i)), x the next SplitMix64 output."""
    if not 0 < n <= Lv:
        raise ValueError("need 0 < n <= Lv")
    gen = splitmix64_stream(seed)
    moved = {}
    out = np.empty(n, np.int32)
    for i in range(n):
        j = i + next(gen) % (Lv - i)
        vi = moved.get(i, i)
        vj = moved.get(j, j)
        moved[i], moved[j] = vj, vi
        out[i] = vj
    return out


# ------------------------------------------------------------------ inputs --

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    u = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def make_inputs(wl: Workload, seed: int | None = None, with_qkv: bool = True) -> dict:
    """Seeded inputs of one attention layer.

    Returns q, k, v (uint16 bf16 bits, [B, H, L, d]), gamma_q, gamma_k
    (float32 [d], U(0.5, 1.5)), sample_idx (int32 [n]) and planted kinds.
    """
    seed = wl.seed if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    B, H, L, d, F, S, Lv = wl.B, wl.H, wl.L, wl.d, wl.F, wl.S, wl.Lv
    out = {}
    if with_qkv:
        q = rng.standard_normal((B, H, L, d), dtype=np.float32)
        k = rng.standard_normal((B, H, L, d), dtype=np.float32)
        v = rng.standard_normal((B, H, L, d), dtype=np.float32)
        for b in range(B):
            for h in range(H):
                kind = wl.planted[h]
                if kind == "S":
                    u = rng.standard_normal((F, 1, d), dtype=np.float32) * np.float32(wl.sigma)
                elif kind == "T":
                    u = rng.standard_normal((1, S, d), dtype=np.float32) * np.float32(wl.sigma)
                else:
                    continue
                q[b, h, :Lv].reshape(F, S, d)[...] += u
                k[b, h, :Lv].reshape(F, S, d)[...] += u
        out["q"] = to_bf16_bits(q)
        del q
        out["k"] = to_bf16_bits(k)
        del k
        out["v"] = to_bf16_bits(v)
        del v
    out["gamma_q"] = rng.uniform(0.5, 1.5, d).astype(np.float32)
    out["gamma_k"] = rng.uniform(0.5, 1.5, d).astype(np.float32)
    out["sample_idx"] = sample_queries(seed, Lv, wl.n_samples)
    out["planted"] = np.array([{"S": SPATIAL, "T": TEMPORAL, "U": 255}[c] for c in wl.planted],
                              np.uint8)
    return out


def random_rows(wl: Workload, n_per_head: int, seed: int, boundary: bool = True,
                max_boundary_tiles: int | None = None) -> np.ndarray:
    """Global row ids (b*H+h)*L + token for sampled checking: n random tokens per
    head plus, if `boundary`, every token of query tiles that straddle a frame
    boundary, the video/text boundary or the end of the sequence (at most
    `max_boundary_tiles` of the frame-boundary tiles, chosen by the seed)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    toks = set()
    if boundary:
        frame_cuts = [f * wl.S for f in range(1, wl.F)]
        if max_boundary_tiles is not None and len(frame_cuts) > max_boundary_tiles:
            frame_cuts = sorted(rng.choice(frame_cuts, max_boundary_tiles, replace=False).tolist())
        for c in list(frame_cuts) + [wl.Lv, wl.L - 1]:
            qb = min(c, wl.L - 1) // wl.bq
            toks.update(range(qb * wl.bq, min(wl.L, (qb + 1) * wl.bq)))
        toks.update(range((wl.nqb - 1) * wl.bq, wl.L))     # the ragged last tile
    toks = np.array(sorted(toks), np.int64)
    rows = []
    for bh in range(wl.B * wl.H):
        r = rng.choice(wl.L, size=min(n_per_head, wl.L), replace=False).astype(np.int64)
        t = np.unique(np.concatenate([toks, r]))
        rows.append(bh * wl.L + t)
    return np.concatenate(rows)
