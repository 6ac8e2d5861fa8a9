"""Plain fp64 CPU oracle for the Sparse VideoGen attention step.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s ``cpu_baseline`` / ``--impl reference`` leg may import this
package.  It shares no code with the CUDA library (``sparse_attention_video_qk_b200``)
and imports nothing from it; the only module both sides use is the seeded
input generator ``svg_workloads``.

The arithmetic lives in ``svg_oracle.c`` (plain loops in double precision);
this file compiles it with gcc on first use and marshals numpy arrays.
Stages, with the page passages they follow (page title, section):

* ``qknorm_rope``   -- RMSNorm + 3D RoPE ("Sparse VideoGen" WeChat article,
  "其他优化方法"; ICML 2025 report, "Layout Transformation + Kernel 加速").
* ``keep`` / masks  -- spatial and temporal heads (article, "Spatial Head",
  "Temporal Head"; report, "Sparse VideoGen 的核心设计").
* ``profile``       -- online profiling by MSE against dense (article,
  "Online Profiling Strategy"; report, "动态自适应的稀疏策略" steps 1-3).
* ``layout`` / ``perm`` -- frame-major -> token-major transform (article,
  "硬件高效的 Layout Transformation"; report, "Layout Transformation + Kernel 加速").
* ``block_list``    -- tiles with at least one kept pair, by brute force over
  the explicit mask (not on the pages; the block-sparse kernel the report
  describes needs it).
* ``attention_rows`` -- masked softmax attention, the textbook definition.

``svg2_oracle.c`` holds the semantic-aware permutation ("Sparse VideoGen2"
explainer, "A. 语义感知排列", "B. 基于质心的 Top-p 选择"): ``kmeans`` (with
``kmeans_init`` / ``kmeans_assign`` / ``kmeans_update``), ``cluster_permutation``,
``select_top_p``, ``attention2_rows``, ``block_list2`` and ``permute_rows``.

``adaspa_oracle.c`` holds AdaSpa's blockified search ("AdaSpa" abstract):
``block_mass`` (exact block attention mass with a cached LSE),
``adaspa_select`` (head-adaptive top-p over key tiles) and
``block_attention_rows`` (attention over the kept tiles).

Every function is pinned by ``tests/test_oracle_*.py``; none is "parity
unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "svg_oracle.c")
_SRC2 = os.path.join(_HERE, "svg2_oracle.c")
_SRC3 = os.path.join(_HERE, "adaspa_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

SPATIAL, TEMPORAL, DENSE = 0, 1, 2


class OraShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "H", "L", "d", "F", "Hs", "Ws", "T")]


class OraParams(ctypes.Structure):
    _fields_ = [
        ("w", ctypes.c_int), ("r", ctypes.c_int), ("bq", ctypes.c_int), ("bk", ctypes.c_int),
        ("eps", ctypes.c_double), ("base", ctypes.c_double), ("scale", ctypes.c_double),
        ("split", ctypes.c_int * 3),
    ]


def build(force: bool = False) -> str:
    """Compile the oracle's C files into oracle/_build/liboracle.so (gcc, -O2, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC2), os.path.getmtime(_SRC3))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".tmp{os.getpid()}"
        # -std=c11 keeps a*b+c unfused (no contraction), as the oracle's text says
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, _SRC2, _SRC3, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            P = ctypes.POINTER
            sh, pr = P(OraShape), P(OraParams)
            vp, i64 = ctypes.c_void_p, ctypes.c_int64
            L.ora_f64_to_bf16.restype = ctypes.c_uint16
            L.ora_f64_to_bf16.argtypes = [ctypes.c_double]
            L.ora_bf16_to_f64.restype = ctypes.c_double
            L.ora_bf16_to_f64.argtypes = [ctypes.c_uint16]
            L.ora_round_bf16.argtypes = [i64, vp, vp]
            L.ora_perm.restype = i64
            L.ora_perm.argtypes = [sh, ctypes.c_int, i64]
            L.ora_perm_inv.restype = i64
            L.ora_perm_inv.argtypes = [sh, ctypes.c_int, i64]
            L.ora_keep.restype = ctypes.c_int
            L.ora_keep.argtypes = [sh, pr, ctypes.c_int, i64, i64]
            L.ora_qknorm_rope_f64.argtypes = [sh, pr, vp, vp, i64, vp, vp]
            L.ora_qknorm_rope_bf16.argtypes = [sh, pr, vp, vp, vp]
            L.ora_layout.argtypes = [sh, vp, ctypes.c_int, vp, vp]
            L.ora_attention_rows.argtypes = [sh, pr, vp, ctypes.c_int, vp, vp, vp, i64, vp, vp, vp, vp]
            L.ora_profile.argtypes = [sh, pr, vp, vp, vp, ctypes.c_int, vp, vp, vp]
            L.ora_block_list.restype = i64
            L.ora_block_list.argtypes = [sh, pr, vp, vp, vp, vp]
            ci = ctypes.c_int
            L.ora2_kmeans_init.argtypes = [vp, ci, i64, i64, ci, ci, vp]
            L.ora2_assign.argtypes = [vp, ci, i64, i64, ci, ci, vp, vp, vp]
            L.ora2_update.argtypes = [vp, ci, i64, i64, ci, ci, vp, vp, vp]
            L.ora2_kmeans.argtypes = [vp, ci, i64, i64, ci, ci, ci, vp, vp, vp]
            L.ora2_permutation.argtypes = [vp, ci, i64, ci, vp, vp]
            L.ora2_select.argtypes = [vp, vp, vp, ci, ci, ci, ci, ctypes.c_double, ctypes.c_double, vp, vp]
            L.ora2_attention_rows.argtypes = [ci, i64, i64, ci, ci, ci, ctypes.c_double, vp, vp, vp, vp, vp, vp,
                                              i64, vp, vp, vp]
            L.ora2_block_list.restype = i64
            L.ora2_block_list.argtypes = [ci, i64, i64, ci, ci, ci, ci, vp, vp, vp, vp, vp, vp, vp, vp, i64]
            dbl = ctypes.c_double
            L.ora3_block_mass.argtypes = [ci, i64, ci, ci, ci, dbl, vp, vp, vp, i64, vp, vp]
            L.ora3_select.restype = i64
            L.ora3_select.argtypes = [ci, i64, i64, ci, ci, vp, dbl, vp, vp, vp, i64, vp]
            L.ora3_attention_rows.argtypes = [ci, i64, ci, ci, ci, dbl, vp, vp, vp, vp, vp, i64, vp, vp, vp]
            _lib = L
    return _lib


# ----------------------------------------------------------------- helpers --

def _ptr(a: np.ndarray | None):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def make_shape(B, H, d, F, Hs, Ws, T) -> OraShape:
    return OraShape(B, H, F * Hs * Ws + T, d, F, Hs, Ws, T)


def make_params(d, w, r, bq, bk, eps=1e-6, base=10000.0, split=None, scale=None) -> OraParams:
    if split is None:
        raise ValueError("RoPE split must be given")
    return OraParams(w, r, bq, bk, eps, base, (1.0 / np.sqrt(d)) if scale is None else scale,
                     (ctypes.c_int * 3)(*split))


def shape_of(wl) -> OraShape:
    return make_shape(wl.B, wl.H, wl.d, wl.F, wl.Hs, wl.Ws, wl.T)


def params_of(wl, w=None, r=None) -> OraParams:
    return make_params(wl.d, wl.w if w is None else w, wl.r if r is None else r, wl.bq, wl.bk,
                       wl.eps, wl.rope_base, wl.rope_split)


# ------------------------------------------------------------------ stages --

def f64_to_bf16(x) -> np.ndarray:
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().ora_round_bf16(x.size, _ptr(x), _ptr(out))
    return out


def bf16_to_f64(h) -> np.ndarray:
    h = _c(h, np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def qknorm_rope_f64(sh, pr, x, gamma, rows=None) -> np.ndarray:
    """RMSNorm + RoPE of the given global rows (all rows if None), fp64 [n, d]."""
    x = _c(x, np.uint16)
    gamma = _c(gamma, np.float32)
    n = sh.B * sh.H * sh.L if rows is None else len(rows)
    rows_a = None if rows is None else _c(rows, np.int64)
    out = np.empty((n, sh.d), np.float64)
    lib().ora_qknorm_rope_f64(ctypes.byref(sh), ctypes.byref(pr), _ptr(x), _ptr(gamma), n,
                              _ptr(rows_a), _ptr(out))
    return out


def qknorm_rope(sh, pr, x, gamma) -> np.ndarray:
    """RMSNorm + RoPE of a whole [B,H,L,d] bf16 tensor, rounded to bf16."""
    x = _c(x, np.uint16)
    gamma = _c(gamma, np.float32)
    out = np.empty_like(x)
    lib().ora_qknorm_rope_bf16(ctypes.byref(sh), ctypes.byref(pr), _ptr(x), _ptr(gamma), _ptr(out))
    return out


def perm(sh, kind: int, i: int) -> int:
    return lib().ora_perm(ctypes.byref(sh), kind, i)


def perm_inv(sh, kind: int, p: int) -> int:
    return lib().ora_perm_inv(ctypes.byref(sh), kind, p)


def keep(sh, pr, kind: int, q: int, k: int) -> bool:
    return bool(lib().ora_keep(ctypes.byref(sh), ctypes.byref(pr), kind, q, k))


def mask(sh, pr, kind: int) -> np.ndarray:
    """Explicit L x L boolean mask (frame-major order); small shapes only."""
    L = sh.L
    m = np.zeros((L, L), bool)
    for q in range(L):
        for k in range(L):
            m[q, k] = keep(sh, pr, kind, q, k)
    return m


def layout(sh, kinds, x, inverse=False) -> np.ndarray:
    x = _c(x, np.uint16)
    kinds = _c(kinds, np.uint8)
    out = np.empty_like(x)
    lib().ora_layout(ctypes.byref(sh), _ptr(kinds), int(inverse), _ptr(x), _ptr(out))
    return out


def attention_rows(sh, pr, kinds, q, k, v, rows, layout_order=False, want_lse=False, want_kept=False):
    """fp64 masked attention for global rows (b*H+h)*L + token; returns out [n,d] (, lse, kept)."""
    q, k, v = (_c(t, np.uint16) for t in (q, k, v))
    kinds = _c(kinds, np.uint8)
    rows = _c(rows, np.int64)
    n = len(rows)
    out = np.empty((n, sh.d), np.float64)
    lse = np.empty(n, np.float64) if want_lse else None
    kept = np.empty(n, np.int64) if want_kept else None
    lib().ora_attention_rows(ctypes.byref(sh), ctypes.byref(pr), _ptr(kinds), int(layout_order),
                             _ptr(q), _ptr(k), _ptr(v), n, _ptr(rows), _ptr(out), _ptr(lse), _ptr(kept))
    res = [out]
    if want_lse:
        res.append(lse)
    if want_kept:
        res.append(kept)
    return res[0] if len(res) == 1 else tuple(res)


def profile(sh, pr, qn, kn, v, sample):
    """Returns (mse [B*H, 2] fp64, choice [B*H] uint8)."""
    qn, kn, v = (_c(t, np.uint16) for t in (qn, kn, v))
    sample = _c(sample, np.int32)
    nbh = sh.B * sh.H
    mse = np.empty((nbh, 2), np.float64)
    choice = np.empty(nbh, np.uint8)
    lib().ora_profile(ctypes.byref(sh), ctypes.byref(pr), _ptr(qn), _ptr(kn), _ptr(v), len(sample),
                      _ptr(sample), _ptr(mse), _ptr(choice))
    return mse, choice


def block_list(sh, pr, kinds):
    """Brute-force CSR block list: (row_ptr int32 [B*H*nqb+1], col int32 [nnz], full uint8 [nnz])."""
    kinds = _c(kinds, np.uint8)
    nqb = -(-sh.L // pr.bq)
    nkb = -(-sh.L // pr.bk)
    nbh = sh.B * sh.H
    row_ptr = np.zeros(nbh * nqb + 1, np.int32)
    cap = nbh * nqb * nkb
    col = np.empty(cap, np.int32)
    full = np.empty(cap, np.uint8)
    nnz = lib().ora_block_list(ctypes.byref(sh), ctypes.byref(pr), _ptr(kinds), _ptr(row_ptr),
                               _ptr(col), _ptr(full))
    return row_ptr, col[:nnz].copy(), full[:nnz].copy()


def step(wl, inputs, kinds=None):
    """The whole step in the oracle: norm+RoPE, profiling (unless kinds given),
    block list.  Returns a dict of intermediate results (attention is evaluated
    per row by the caller through ``attention_rows``; a full pass at the
    largest shapes is hours of fp64 work)."""
    sh, pr = shape_of(wl), params_of(wl)
    qn = qknorm_rope(sh, pr, inputs["q"], inputs["gamma_q"])
    kn = qknorm_rope(sh, pr, inputs["k"], inputs["gamma_k"])
    mse = None
    if kinds is None:
        mse, kinds = profile(sh, pr, qn, kn, inputs["v"], inputs["sample_idx"])
    return {"qn": qn, "kn": kn, "mse": mse, "kinds": np.asarray(kinds, np.uint8)}


# ------------------------------------------------ semantic-aware permutation --
# "Sparse VideoGen2" explainer, "A. 语义感知排列" and "B. 基于质心的 Top-p 选择";
# the readings are stated at the top of svg2_oracle.c.

def kmeans_init(x, Lv: int, C: int) -> np.ndarray:
    """Centroid c = video row floor(c*Lv/C) of each head; x bf16 [B,H,L,d] -> float32 [BH,C,d]."""
    x = _c(x, np.uint16)
    BH, L, d = x.shape[0] * x.shape[1], x.shape[2], x.shape[3]
    cent = np.empty((BH, C, d), np.float32)
    lib().ora2_kmeans_init(_ptr(x), BH, L, Lv, d, C, _ptr(cent))
    return cent


def kmeans_assign(x, Lv: int, cent, want_margin=False):
    """Nearest centroid (fp64 squared distance) of every video row: uint8 [BH, Lv].
    With want_margin also the per-row relative gap to the second nearest
    centroid, (D2 - D1) / (|x|^2 + |c1|^2 + |c2|^2), float64 [BH, Lv]."""
    x = _c(x, np.uint16)
    cent = _c(cent, np.float32)
    BH, L, d = x.shape[0] * x.shape[1], x.shape[2], x.shape[3]
    out = np.empty((BH, Lv), np.uint8)
    margin = np.empty((BH, Lv), np.float64) if want_margin else None
    lib().ora2_assign(_ptr(x), BH, L, Lv, d, cent.shape[1], _ptr(cent), _ptr(out), _ptr(margin))
    return (out, margin) if want_margin else out


def kmeans_update(x, Lv: int, assign, cent):
    """Returns (new centroids float32 [BH,C,d], counts int32 [BH,C]); `cent` is not modified."""
    x = _c(x, np.uint16)
    cent = np.array(cent, dtype=np.float32, copy=True)
    assign = _c(assign, np.uint8)
    BH, L, d = x.shape[0] * x.shape[1], x.shape[2], x.shape[3]
    counts = np.empty((BH, cent.shape[1]), np.int32)
    lib().ora2_update(_ptr(x), BH, L, Lv, d, cent.shape[1], _ptr(assign), _ptr(cent), _ptr(counts))
    return cent, counts


def kmeans(x, Lv: int, C: int, iters: int, cent=None):
    """`iters` Lloyd rounds from `cent` (default: kmeans_init) and a final
    assignment.  Returns (centroids, assign uint8 [BH,Lv], counts int32 [BH,C])."""
    x = _c(x, np.uint16)
    BH, L, d = x.shape[0] * x.shape[1], x.shape[2], x.shape[3]
    cent = kmeans_init(x, Lv, C) if cent is None else np.array(cent, dtype=np.float32, copy=True)
    assign = np.empty((BH, Lv), np.uint8)
    counts = np.empty((BH, C), np.int32)
    lib().ora2_kmeans(_ptr(x), BH, L, Lv, d, C, iters, _ptr(cent), _ptr(assign), _ptr(counts))
    return cent, assign, counts


def cluster_permutation(assign, C: int):
    """Stable counting sort: (perm int32 [BH,Lv] position -> row, off int32 [BH,C+1])."""
    assign = _c(assign, np.uint8)
    BH, Lv = assign.shape
    perm_ = np.empty((BH, Lv), np.int32)
    off = np.empty((BH, C + 1), np.int32)
    lib().ora2_permutation(_ptr(assign), BH, Lv, C, _ptr(perm_), _ptr(off))
    return perm_, off


def select_top_p(cq, ck, nk, scale: float, p: float, want_weight=False):
    """Top-p key clusters per query cluster: sel uint64 [BH,Cq] (and weights [BH,Cq,Ck])."""
    cq, ck = _c(cq, np.float32), _c(ck, np.float32)
    nk = _c(nk, np.int32)
    BH, Cq, d = cq.shape
    Ck = ck.shape[1]
    sel = np.empty((BH, Cq), np.uint64)
    w = np.empty((BH, Cq, Ck), np.float64) if want_weight else None
    lib().ora2_select(_ptr(cq), _ptr(ck), _ptr(nk), BH, Cq, Ck, d, float(scale), float(p), _ptr(sel), _ptr(w))
    return (sel, w) if want_weight else sel


def attention2_rows(q, k, v, Lv: int, aq, ak, sel, rows, scale=None, want_lse=False):
    """fp64 attention with the cluster mask, model order; rows = bh*L + token."""
    q, k, v = (_c(t, np.uint16) for t in (q, k, v))
    aq, ak = _c(aq, np.uint8), _c(ak, np.uint8)
    sel = _c(sel, np.uint64)
    rows = _c(rows, np.int64)
    BH, L, d = q.shape[0] * q.shape[1], q.shape[2], q.shape[3]
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.empty((len(rows), d), np.float64)
    lse = np.empty(len(rows), np.float64) if want_lse else None
    lib().ora2_attention_rows(BH, L, Lv, d, sel.shape[1], 0, sc, _ptr(q), _ptr(k), _ptr(v), _ptr(aq), _ptr(ak),
                              _ptr(sel), len(rows), _ptr(rows), _ptr(out), _ptr(lse))
    return (out, lse) if want_lse else out


def block_list2(L: int, Lv: int, bq: int, bk: int, aq, ak, perm_q, perm_k, sel):
    """Tile list over the permuted order by brute force: (row_ptr, col, full)."""
    aq, ak = _c(aq, np.uint8), _c(ak, np.uint8)
    perm_q, perm_k = _c(perm_q, np.int32), _c(perm_k, np.int32)
    sel = _c(sel, np.uint64)
    BH = aq.shape[0]
    nqb, nkb = -(-L // bq), -(-L // bk)
    cap = BH * nqb * nkb
    row_ptr = np.empty(BH * nqb + 1, np.int32)
    col = np.empty(cap, np.int32)
    full = np.empty(cap, np.uint8)
    n = lib().ora2_block_list(BH, L, Lv, sel.shape[1], 0, bq, bk, _ptr(aq), _ptr(ak), _ptr(perm_q), _ptr(perm_k),
                              _ptr(sel), _ptr(row_ptr), _ptr(col), _ptr(full), cap)
    return row_ptr, col[:n], full[:n]



def permute_rows(x, Lv: int, perm):
    """Video position p of every head takes row perm[bh, p]; text rows stay
    (the cluster-contiguous order of step 2).  x bf16 [B,H,L,d]."""
    x = _c(x, np.uint16)
    B, H, L, d = x.shape
    perm = _c(perm, np.int32).reshape(B, H, Lv)
    out = x.copy()
    for b in range(B):
        for h in range(H):
            out[b, h, :Lv] = x[b, h, perm[b, h]]
    return out


# ------------------------------------------------- AdaSpa blockified search --
# "AdaSpa" abstract (blockified pattern; fused LSE-cached search; head-adaptive
# hierarchical block sparse attention); the readings are stated at the top of
# adaspa_oracle.c.

def block_mass(q, k, lse, bq: int, bk: int, scale=None, tiles=None):
    """fp64 block masses [BH, nqb, nkb] from bf16 q, k [B,H,L,d] and float lse [B,H,L];
    with `tiles` (ids bh*nqb + qb) only those query tiles, [len(tiles), nkb]."""
    q, k = _c(q, np.uint16), _c(k, np.uint16)
    lse = _c(lse, np.float32)
    BH, L, d = q.shape[0] * q.shape[1], q.shape[2], q.shape[3]
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    nqb, nkb = -(-L // bq), -(-L // bk)
    if tiles is None:
        mass = np.empty((BH, nqb, nkb), np.float64)
        lib().ora3_block_mass(BH, L, d, bq, bk, sc, _ptr(q), _ptr(k), _ptr(lse), 0, None, _ptr(mass))
    else:
        tiles = _c(tiles, np.int64)
        mass = np.empty((len(tiles), nkb), np.float64)
        lib().ora3_block_mass(BH, L, d, bq, bk, sc, _ptr(q), _ptr(k), _ptr(lse), len(tiles), _ptr(tiles),
                              _ptr(mass))
    return mass


def adaspa_select(mass, L: int, Lv: int, bq: int, bk: int, p: float, want_margin=False):
    """Kept key tiles from float32 masses [BH, nqb, nkb]: (row_ptr, col, full).
    With want_margin also each query tile's distance of its running sums from
    the goal at the cut, float64 [BH*nqb] (+inf where nothing is cut)."""
    mass = _c(mass, np.float32)
    BH, nqb, nkb = mass.shape
    cap = BH * nqb * nkb
    row_ptr = np.empty(BH * nqb + 1, np.int32)
    col = np.empty(cap, np.int32)
    full = np.empty(cap, np.uint8)
    margin = np.empty(BH * nqb, np.float64) if want_margin else None
    n = lib().ora3_select(BH, L, Lv, bq, bk, _ptr(mass), float(p), _ptr(row_ptr), _ptr(col), _ptr(full), cap,
                          _ptr(margin))
    res = (row_ptr, col[:n], full[:n])
    return res + (margin,) if want_margin else res


def block_attention_rows(q, k, v, bq: int, bk: int, row_ptr, col, rows, scale=None, want_lse=False):
    """fp64 attention of `rows` (bh*L + token) over the kept key tiles of their query tile."""
    q, k, v = (_c(t, np.uint16) for t in (q, k, v))
    row_ptr, col = _c(row_ptr, np.int32), _c(col, np.int32)
    rows = _c(rows, np.int64)
    BH, L, d = q.shape[0] * q.shape[1], q.shape[2], q.shape[3]
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.empty((len(rows), d), np.float64)
    lse = np.empty(len(rows), np.float64) if want_lse else None
    lib().ora3_attention_rows(BH, L, d, bq, bk, sc, _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr), _ptr(col),
                              len(rows), _ptr(rows), _ptr(out), _ptr(lse))
    return (out, lse) if want_lse else out
