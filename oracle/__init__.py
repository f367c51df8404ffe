"""CPU oracle for the CSA / HCA hot path (fp64, plain definitions).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers. The CUDA library never imports this
module and this module never imports the CUDA library; the two share no code.

The arithmetic lives in ``csa_oracle.c`` (plain C, fp64, OpenMP over
independent outputs). This file only builds that library with gcc and moves
numpy arrays in and out. Every function returns float64 arrays (int32 for
indices); bf16 storage rounding is explicit (:func:`bf16_round`).

Which page passage each function follows is stated beside it in
``csa_oracle.c``; the readings taken where the pages are silent are listed at
the top of that file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)


def build(force: bool = False) -> str:
    """Compile ``csa_oracle.c`` into ``_build/liboracle.so`` (gcc, -O2, OpenMP).

    No fast-math: the oracle needs IEEE exp/log and the written summation order.
    """
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-std=c11", "-Wall", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(_LIB_OVERRIDE or build())
            i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
            lib.orc_bf16_round.restype = dbl
            lib.orc_bf16_round.argtypes = [dbl]
            lib.orc_bf16_round_array.argtypes = [_D, i64, _D]
            lib.orc_project.argtypes = [_D, _D, i64, i64, i64, _D]
            lib.orc_csa_compress.argtypes = [_D, _D, _D, i64, i32, i32, _D, _D]
            lib.orc_hca_compress.argtypes = [_D, _D, i64, i32, i32, _D, _D]
            lib.orc_index_scores.argtypes = [_D, _D, _D, _I32, _I32, i32, i32, i32, i64, i32, _D]
            lib.orc_topk.argtypes = [_D, _I32, i32, i64, i32, _I32]
            lib.orc_sparse_mqa.argtypes = [_D, _D, _I32, _I32, i32, i32, i32, i64, i32, dbl, _D, _D, _D]
            lib.orc_dense_mqa.argtypes = [_D, _D, _I32, _I32, i32, i32, i32, i64, i32, dbl, _D, _D, _D]
            lib.orc_e4m3_round.restype = dbl
            lib.orc_e4m3_round.argtypes = [dbl]
            lib.orc_quantize_rows_e4m3.argtypes = [_D, i64, i64, _D, _D]
            lib.orc_norm_rope.argtypes = [_D, i64, i32, i32, _D, dbl, i32, dbl, _I32, i32, _D]
            lib.orc_window_entries.argtypes = [_I32, i32, i32, i64, i64, _I32]
            lib.orc_num_threads.restype = i32
            lib.orc_set_num_threads.argtypes = [i32]
            _lib = lib
    return _lib


# Test hook: the mutation tests load a build of a deliberately broken copy
# of csa_oracle.c through this variable.
_LIB_OVERRIDE = os.environ.get("CSA_ORACLE_LIB") or None


def _f64(a) -> np.ndarray:
    """Any array-like (numpy or a CPU torch tensor, bf16 included) -> C-contiguous float64."""
    if hasattr(a, "detach"):  # torch tensor: go through float32, which holds bf16 exactly
        a = a.detach().cpu()
        if str(a.dtype) in ("torch.bfloat16", "torch.float16"):
            a = a.float()
        a = a.numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _p(a: np.ndarray | None):
    if a is None:
        return None
    if a.dtype == np.float64:
        return a.ctypes.data_as(_D)
    return a.ctypes.data_as(_I32)


def num_threads() -> int:
    return int(_load().orc_num_threads())


def set_num_threads(n: int) -> None:
    """Threads for the oracle's parallel loops from now on (this thread)."""
    _load().orc_set_num_threads(int(n))


def bf16_round(x) -> np.ndarray:
    """Nearest bf16 value (ties to even) of each element, returned as float64."""
    x = _f64(x)
    y = np.empty_like(x)
    _load().orc_bf16_round_array(_p(x), x.size, _p(y))
    return y


def e4m3_round(x) -> np.ndarray:
    """Nearest e4m3 (FP8) value of each element, ties to even, saturating at
    +-448, returned as float64."""
    x = _f64(x)
    f = _load().orc_e4m3_round
    return np.vectorize(f, otypes=[np.float64])(x) if x.size else x.copy()


def quantize_rows_e4m3(x):
    """Row-wise e4m3 quantisation of x [..., n] with scale max|row| / 448.
    Returns (dequantised values, scales [...])."""
    x = _f64(x)
    n = x.shape[-1]
    rows = x.size // n if n else 0
    y = np.empty_like(x)
    s = np.empty(x.shape[:-1])
    _load().orc_quantize_rows_e4m3(_p(x), rows, n, _p(y), _p(s))
    return y, s


def index_scores_fp8(qI, w, K, pos, m: int, seq=None) -> np.ndarray:
    """The indexer with q^I and K stored in e4m3 (one scale per query head
    row and per key row), the products and sums exact: the definition of
    index_scores applied to the dequantised operands."""
    q8, _ = quantize_rows_e4m3(qI)
    k8, _ = quantize_rows_e4m3(K)
    return index_scores(q8, w, k8, pos, m, seq=seq)


def quantize_kv_fp8(KV, rope_dims: int):
    """FP8 KV storage with bf16 rotary dims [Notes §1.3 and §2.4]: each entry
    row's first c - R values get one scale s = max|x| / 448 (1 for an
    all-zero part) and are stored as the e4m3 values nearest x / s; the last
    R values are kept as they are. Returns (codes [..., c-R] as the e4m3
    values, float64; scales [...]; rope [..., R])."""
    KV = _f64(KV)
    c = KV.shape[-1]
    q = KV[..., :c - rope_dims]
    amax = np.abs(q).max(axis=-1) if q.shape[-1] else np.zeros(q.shape[:-1])
    s = np.where(amax > 0, amax / 448.0, 1.0)
    codes = e4m3_round(q / s[..., None])
    return codes, s, KV[..., c - rope_dims:].copy()


def dequantize_kv_fp8(codes, scales, rope):
    """The entries attention sees: code * s (exact), then the rotary values."""
    return np.concatenate([_f64(codes) * _f64(scales)[..., None], _f64(rope)], axis=-1)


def topk_recall(idx, ref_idx) -> float:
    """Mean over rows of |idx ∩ ref_idx| / |ref_idx| (entries >= 0 only)."""
    idx, ref_idx = _i32(idx), _i32(ref_idx)
    rec = []
    for a, b in zip(idx, ref_idx):
        rb = set(b[b >= 0].tolist())
        if rb:
            rec.append(len(set(a[a >= 0].tolist()) & rb) / len(rb))
    return float(np.mean(rec)) if rec else 1.0


def project(X, W) -> np.ndarray:
    """P = X @ W^T with X [n, d] and W [M, d] (one row per output feature).

    A plain fp64 matrix product (numpy's, used as a library primitive so that
    full-size projections finish on the host); project_loops() is the same
    definition written as loops in C."""
    X, W = _f64(X), _f64(W)
    assert X.shape[1] == W.shape[1]
    return X @ W.T


def project_loops(X, W) -> np.ndarray:
    """P = X @ W^T as the plain triple loop of csa_oracle.c."""
    X, W = _f64(X), _f64(W)
    n, d = X.shape
    M = W.shape[0]
    assert W.shape[1] == d
    P = np.empty((n, M))
    _load().orc_project(_p(X), _p(W), n, d, M, _p(P))
    return P


def csa_compress(proj, bias, m: int, left=None, return_weights: bool = False):
    """Overlapping CSA compression. proj [n, 4c] = Ca|Cb|Za|Zb, bias [2m, c],
    left [m, 4c] or None (sequence start). Returns out [n/m, c] (and the softmax
    weights [n/m, 2m, c] when asked)."""
    proj, bias = _f64(proj), _f64(bias)
    n, c4 = proj.shape
    c = c4 // 4
    assert c4 == 4 * c and n % m == 0 and bias.shape == (2 * m, c)
    lp = None
    if left is not None:
        lp = _f64(left)
        assert lp.shape == (m, 4 * c)
    out = np.empty((n // m, c))
    w = np.empty((n // m, 2 * m, c)) if return_weights else None
    _load().orc_csa_compress(_p(proj), _p(lp), _p(bias), n, c, m, _p(out), _p(w))
    return (out, w) if return_weights else out


def hca_compress(proj, bias, mp: int, return_weights: bool = False):
    """Non-overlapping HCA compression. proj [n, 2c] = C|Z, bias [mp, c]."""
    proj, bias = _f64(proj), _f64(bias)
    n, c2 = proj.shape
    c = c2 // 2
    assert c2 == 2 * c and n % mp == 0 and bias.shape == (mp, c)
    out = np.empty((n // mp, c))
    w = np.empty((n // mp, mp, c)) if return_weights else None
    _load().orc_hca_compress(_p(proj), _p(bias), n, c, mp, _p(out), _p(w))
    return (out, w) if return_weights else out


def index_scores(qI, w, K, pos, m: int, seq=None) -> np.ndarray:
    """Indexer scores [nq, Nmax]; -inf where the entry is not visible.
    qI [nq, HI, cI], w [nq, HI], K [B, Nmax, cI] (or [Nmax, cI]), pos [nq]."""
    qI, w, K = _f64(qI), _f64(w), _f64(K)
    if K.ndim == 2:
        K = K[None]
    nq, HI, cI = qI.shape
    B, Nmax, _ = K.shape
    pos = _i32(pos)
    seq = _i32(np.zeros(nq) if seq is None else seq)
    assert int(seq.max(initial=0)) < B
    S = np.empty((nq, Nmax))
    _load().orc_index_scores(_p(qI), _p(w), _p(K), _p(pos), _p(seq), nq, HI, cI, Nmax, m, _p(S))
    return S


def topk(scores, valid, k: int) -> np.ndarray:
    """Top-k column indices per row among the first valid[t] columns, ordered
    (score desc, index asc), padded with -1."""
    S = _f64(scores)
    nq, ncols = S.shape
    valid = _i32(valid)
    idx = np.empty((nq, k), dtype=np.int32)
    _load().orc_topk(_p(S), _p(valid), nq, ncols, k, _p(idx))
    return idx


def sparse_mqa(q, KV, idx, scale: float, sink=None, seq=None):
    """Shared-KV MQA over the selected entries. q [nq, H, c], KV [B, Nmax, c]
    (or [Nmax, c]), idx [nq, k] (-1 = no entry). Returns (out [nq, H, c], lse [nq, H])."""
    q, KV = _f64(q), _f64(KV)
    if KV.ndim == 2:
        KV = KV[None]
    nq, H, c = q.shape
    B, Nmax, _ = KV.shape
    idx = _i32(idx)
    k = idx.shape[1]
    seq = _i32(np.zeros(nq) if seq is None else seq)
    sk = None if sink is None else _f64(sink)
    out = np.empty((nq, H, c))
    lse = np.empty((nq, H))
    _load().orc_sparse_mqa(_p(q), _p(KV), _p(idx), _p(seq), nq, H, c, Nmax, k, float(scale),
                           _p(sk), _p(out), _p(lse))
    return out, lse


def dense_mqa(q, KV, pos, mp: int, scale: float, sink=None, seq=None):
    """Shared-KV MQA over every visible entry s < floor(pos/mp)."""
    q, KV = _f64(q), _f64(KV)
    if KV.ndim == 2:
        KV = KV[None]
    nq, H, c = q.shape
    B, Nmax, _ = KV.shape
    pos = _i32(pos)
    seq = _i32(np.zeros(nq) if seq is None else seq)
    sk = None if sink is None else _f64(sink)
    out = np.empty((nq, H, c))
    lse = np.empty((nq, H))
    _load().orc_dense_mqa(_p(q), _p(KV), _p(pos), _p(seq), nq, H, c, Nmax, mp, float(scale),
                          _p(sk), _p(out), _p(lse))
    return out, lse


def norm_rope(x, pos, gamma=None, eps: float = 1e-6, rope_dims: int = 64, base: float = 10000.0,
              inverse: bool = False) -> np.ndarray:
    """RMSNorm (when gamma is given) then rotary encoding of the last rope_dims
    channels. x [..., G, c] or [G, c]: the rows of group g share position
    pos[g] (x [nq, H, c] with pos [nq]: every head of query t at pos[t]).
    inverse turns by -pos (the output's back-rotation)."""
    x = _f64(x)
    shape = x.shape
    c = shape[-1]
    pos = _i32(pos).reshape(-1)
    rows = x.size // c
    group = rows // max(pos.size, 1) if pos.size else 1
    assert group * pos.size == rows, "rows must split evenly over the positions"
    g = None if gamma is None else _f64(gamma)
    y = np.empty_like(x)
    _load().orc_norm_rope(_p(x), rows, group, c, _p(g), float(eps), int(rope_dims), float(base), _p(pos),
                          1 if inverse else 0, _p(y))
    return y.reshape(shape)


def window_entries(pos, n_win: int, ring_off: int, ring_len: int) -> np.ndarray:
    """Rows of the n_win most recent tokens (the query's own included) in the
    window ring of each query's sequence; -1 before the sequence start."""
    pos = _i32(pos).reshape(-1)
    ent = np.empty((pos.size, n_win), dtype=np.int32)
    _load().orc_window_entries(_p(pos), pos.size, n_win, ring_off, ring_len, _p(ent))
    return ent


# ---------------------------------------------------------------------------
# Chained steps (each one a composition of the definitions above, in the
# order the method applies them)
# ---------------------------------------------------------------------------

def csa_compress_from_hidden(X, W, bias, m: int, X_left=None) -> np.ndarray:
    """Projections then overlapping compression; W [4c, d] packs the a-KV,
    b-KV, a-weight and b-weight maps (one row per output feature)."""
    proj = project(X, W)
    left = None if X_left is None else project(X_left, W)
    return csa_compress(proj, bias, m, left=left)


def hca_compress_from_hidden(X, W, bias, mp: int) -> np.ndarray:
    return hca_compress(project(X, W), bias, mp)


def index_topk(qI, w, K, pos, m: int, k: int, seq=None):
    """Indexer scores, then top-k over the visible entries. Returns (idx, scores)."""
    S = index_scores(qI, w, K, pos, m, seq=seq)
    valid = np.minimum(_i32(pos) // m, S.shape[1]).astype(np.int32)
    return topk(S, valid, k), S


def attend_decode(qI, w, idx_cache, q, kv_cache, ctx_len, m: int, k: int, n_win: int, ring_len: int,
                  scale: float, q_gamma=None, eps: float = 1e-6, rope_dims: int = 64, base: float = 10000.0,
                  sink=None, sel=None):
    """One decode query per sequence with the complete attention output:
    query RMSNorm + rotary at its position, indexer + top-k over the
    compressed entries, the sliding window of the n_win latest tokens (rows
    Nmax + (tau mod ring_len) of kv_cache [B, Nmax + ring_len, c]) joined to
    the selection in one softmax, then the output turned back by the query's
    position. sel, when given, replaces the oracle's own top-k (to compare an
    attention output against a selection made elsewhere).
    Returns (out, lse, idx, scores)."""
    ctx = _i32(ctx_len)
    B = ctx.size
    Nmax = int(idx_cache.shape[1])
    seq = np.arange(B, dtype=np.int32)
    idx, S = index_topk(qI, w, idx_cache, ctx, m, k, seq=seq)
    chosen = idx if sel is None else _i32(sel)
    ent = np.concatenate([chosen, window_entries(ctx, n_win, Nmax, ring_len)], axis=1)
    qn = norm_rope(q, ctx, gamma=q_gamma, eps=eps, rope_dims=rope_dims, base=base)
    out, lse = sparse_mqa(qn, kv_cache, ent, scale, sink=sink, seq=seq)
    out = norm_rope(out, ctx, gamma=None, rope_dims=rope_dims, base=base, inverse=True)
    return out, lse, idx, S
