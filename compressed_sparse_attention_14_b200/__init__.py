"""Python binding of libcsa, the B200 (sm_100a) CUDA library for the
DeepSeek-V4 compressed attention hot path (CSA and HCA).

Argument marshalling only: every function below checks tensor devices,
dtypes and shapes, allocates outputs and the workspace with torch, and calls
the C entry point of the same name (include/csa.h) on the current CUDA
stream. All arithmetic runs in the library's kernels. There is no CPU path:
importing this package without the built library raises.

dtype: bf16 tensors run the CSA_BF16 mode, fp32 tensors the CSA_FP32 mode
(biases, head weights `w`, sinks, scores and lse are fp32 in both).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

CSA_OK, CSA_ERR_INVALID_ARG, CSA_ERR_UNSUPPORTED, CSA_ERR_WORKSPACE, CSA_ERR_CUDA, CSA_ERR_TIMEOUT = range(6)
CSA_BF16, CSA_FP32 = 0, 1
CSA_SCORES_BF16 = 1
CSA_DEBUG_SKIP_FIRST_TILE = 1
CSA_DEBUG_SCORE_BLOCK = 2
CSA_DEBUG_TOPK_FILTER = 4

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python compressed_sparse_attention_14_b200/build.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float

# name -> (restype, argtypes)
_SIGS = {
    "csa_last_error": (ctypes.c_char_p, []),
    "csa_abi_version": (_I, []),
    "csa_launch_count": (ctypes.c_uint64, []),
    "csa_trace_enable": (None, [_I]),
    "csa_trace_read": (_I, [_I, _P, _P, _P, _P]),
    "csa_poll_status": (_I, [_P, _I]),
    "csa_debug_set": (_I, [ctypes.c_uint32, ctypes.c_uint32]),
    "csa_project": (_I, [_P, _P, _I64, _I, _I, _P, _I, _P]),
    "csa_compress": (_I, [_P, _P, _P, _I64, _I, _I, _P, _I, _P]),
    "hca_compress": (_I, [_P, _P, _I64, _I, _I, _P, _I, _P]),
    "csa_compress_from_hidden_workspace_size": (_SZ, [_I64, _I, _I, _I, _I]),
    "csa_compress_from_hidden": (_I, [_P, _P, _P, _P, _I64, _I, _I, _I, _P, _P, _SZ, _I, _P]),
    "hca_compress_from_hidden_workspace_size": (_SZ, [_I64, _I, _I, _I, _I]),
    "hca_compress_from_hidden": (_I, [_P, _P, _P, _I64, _I, _I, _I, _P, _P, _SZ, _I, _P]),
    "csa_index_scores": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I64, _I, _P, _I, _P]),
    "csa_topk_workspace_size": (_SZ, [_I, _I64, _I]),
    "csa_topk_from_scores": (_I, [_P, _I64, _P, _I, _I, _I64, _I, _P, _P, _P, _SZ, _P]),
    "csa_index_topk_workspace_size": (_SZ, [_I, _I64, _I, _I]),
    "csa_index_topk": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I64, _I, _I, _P, _P, _P, _SZ, _I, _P]),
    "csa_index_topk_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I64, _I, _I, _P, _P, _I, _P]),
    "csa_quantize_e4m3": (_I, [_P, _I64, _I, _P, _P, _P, _P, _I, _P]),
    "csa_index_scores_fp8": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I64, _I, _P, _P]),
    "csa_decode_fp8_workspace_size": (_SZ, [_I, _I64, _I, _I, _I, _I, _I]),
    "csa_decode_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I64, _I, _I, _I, _I, _I, _I, _F, _P, _I, _P, _P, _P,
                            _P, _SZ, _P]),
    "csa_topk_from_scores_bf16": (_I, [_P, _I64, _P, _I, _I, _I64, _I, _P, _P, _P]),
    "csa_sparse_mqa_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "csa_sparse_mqa": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I64, _I, _F, _P, _P, _P, _P, _SZ, _I, _P]),
    "hca_dense_mqa_workspace_size": (_SZ, [_I, _I, _I, _I64, _I]),
    "hca_dense_mqa": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I64, _I, _F, _P, _P, _P, _P, _SZ, _I, _P]),
    "csa_decode_workspace_size": (_SZ, [_I, _I64, _I, _I, _I, _I, _I, _I]),
    "csa_decode": (_I, [_P, _P, _P, _P, _P, _P, _I, _I64, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P,
                        _P, _SZ, _I, _P]),
    "hca_decode_workspace_size": (_SZ, [_I, _I64, _I, _I, _I]),
    "hca_decode": (_I, [_P, _P, _P, _I, _I64, _I, _I, _I, _F, _P, _P, _P, _P, _SZ, _I, _P]),
    "csa_prefill_workspace_size": (_SZ, [_I64, _I64, _I, _I, _I, _I, _I, _I, _I, _I]),
    "csa_prefill": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I, _I, _I, _I, _P, _P, _I64, _P, _P, _P, _P, _P,
                         _I, _I, _I, _F, _P, _P, _P, _P, _P, _SZ, _I, _P]),
    "csa_compress_chunk": (_I, [_P, _P, _P, _I64, _I64, _I, _I, _P, _I64, _I, _P]),
    "hca_compress_chunk": (_I, [_P, _P, _P, _I64, _I64, _I, _I, _P, _I64, _I, _P]),
    "csa_compress_step": (_I, [_P, _P, _P, _P, _I, _I, _I, _I64, _P, _I, _P]),
    "hca_compress_step": (_I, [_P, _P, _P, _P, _I, _I, _I, _I64, _P, _I, _P]),
    "csa_decode_compress_workspace_size": (_SZ, [_I, _I, _I]),
    "csa_decode_compress": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I64, _P, _SZ, _I, _P]),
    "csa_quantize_kv_fp8": (_I, [_P, _I64, _I, _I, _P, _P, _P, _P]),
    "csa_decode_fp8kv_workspace_size": (_SZ, [_I, _I64, _I, _I, _I, _I, _I]),
    "csa_decode_fp8kv": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I64, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P,
                              _P, _P, _SZ, _P]),
    "csa_cache_block_layout": (_I, [_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "csa_decode_blocked": (_I, [_P, _P, _P, _P, _P, _P, _I, _I64, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P,
                                _I, _I64, _P, _SZ, _I, _P]),
    "hca_decode_blocked": (_I, [_P, _P, _P, _I, _I64, _I, _I, _I, _F, _P, _P, _P, _I, _I64, _P, _SZ, _I, _P]),
    "csa_decode_compress_blocked": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I64, _I, _I64,
                                         _P, _SZ, _I, _P]),
    "hca_compress_step_blocked": (_I, [_P, _P, _P, _P, _I, _I, _I, _I64, _P, _I, _I64, _I, _P]),
    "csa_norm_rope": (_I, [_P, _P, _I64, _I, _I, _P, _F, _I, _F, _P, _I64, _I64, _I, _I, _P]),
    "csa_window_entries": (_I, [_P, _I, _P, _I64, _I, _I, _I64, _I64, _P, _P]),
    "csa_attend_decode_workspace_size": (_SZ, [_I, _I64, _I64, _I, _I, _I, _I, _I, _I, _I]),
    "csa_attend_decode": (_I, [_P, _P, _P, _P, _P, _P, _I, _I64, _I64, _I, _I, _I, _I, _I, _I, _I, _F, _P, _F,
                               _I, _F, _P, _P, _P, _P, _P, _SZ, _I, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


class CsaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libcsa error {code}: {msg}")
        self.code = code


def _check(rc: int) -> None:
    if rc != CSA_OK:
        raise CsaError(rc, _lib.csa_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libcsa takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("libcsa takes contiguous tensors only")
    return t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _mode(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return CSA_BF16
    if t.dtype == torch.float32:
        return CSA_FP32
    raise ValueError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _ws(nbytes: int, device, ws: Optional[torch.Tensor] = None) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return None
    if ws is not None and ws.numel() * ws.element_size() >= nbytes:
        return ws
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _nbytes(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _shape(t: Optional[torch.Tensor], want: tuple, name: str) -> None:
    """The C entry points take bare pointers: a buffer of the wrong shape would
    be read or written out of bounds, so shapes are checked here."""
    if t is not None and tuple(t.shape) != tuple(want):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(want)}")


def _dtype(t: Optional[torch.Tensor], want: torch.dtype, name: str) -> None:
    if t is not None and t.dtype != want:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {want}")


def abi_version() -> int:
    return _lib.csa_abi_version()


def launch_count() -> int:
    """Kernels this library has launched so far in this process."""
    return int(_lib.csa_launch_count())


def trace_enable(on: bool = True) -> None:
    """Start (or stop) per-kernel event timing; discards earlier records."""
    _lib.csa_trace_enable(int(on))


def trace_read(max_kernels: int = 64) -> dict:
    """{kernel name: (total device ms, launches)} for the records so far."""
    names = ctypes.create_string_buffer(64 * max_kernels)
    ms = (ctypes.c_double * max_kernels)()
    cnt = (ctypes.c_int * max_kernels)()
    n = ctypes.c_int(0)
    _check(_lib.csa_trace_read(max_kernels, ctypes.addressof(names), ctypes.addressof(ms), ctypes.addressof(cnt),
                               ctypes.addressof(n)))
    out = {}
    for i in range(n.value):
        nm = names.raw[64 * i: 64 * i + 64].split(b"\0", 1)[0].decode()
        out[nm] = (ms[i], cnt[i])
    return out


def poll_status(reset: bool = True) -> None:
    _check(_lib.csa_poll_status(_stream(), int(reset)))


def debug_set(wait_limit: int = 0, flags: int = 0) -> None:
    """Failure-path test hooks (off by default): a shorter bound on the
    indexer's device waits, and CSA_DEBUG_SKIP_FIRST_TILE to withhold its first
    key tile so that a wait runs out."""
    _check(_lib.csa_debug_set(wait_limit, flags))


def workspace_size(name: str, *args) -> int:
    return int(getattr(_lib, name + "_workspace_size")(*args))


# ---------------------------------------------------------------- a1
def csa_project(x: torch.Tensor, W: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    n, d = x.shape
    M = W.shape[0]
    out = torch.empty((n, M), dtype=torch.float32, device=x.device) if out is None else out
    _check(_lib.csa_project(_ptr(x), _ptr(W), n, d, M, _ptr(out), _mode(x), _stream()))
    return out


# ---------------------------------------------------------------- a2 / a3
def csa_compress(proj, bias, m: int, left=None, out=None):
    n, c4 = proj.shape
    c = c4 // 4
    out = torch.empty((n // m, c), dtype=proj.dtype, device=proj.device) if out is None else out
    _check(_lib.csa_compress(_ptr(proj), _ptr(left), _ptr(bias), n, c, m, _ptr(out), _mode(proj), _stream()))
    return out


def hca_compress(proj, bias, mp: int, out=None):
    n, c2 = proj.shape
    c = c2 // 2
    out = torch.empty((n // mp, c), dtype=proj.dtype, device=proj.device) if out is None else out
    _check(_lib.hca_compress(_ptr(proj), _ptr(bias), n, c, mp, _ptr(out), _mode(proj), _stream()))
    return out


def csa_compress_from_hidden(x, W, bias, m: int, x_left=None, out=None, ws=None):
    n, d = x.shape
    c = W.shape[0] // 4
    mode = _mode(x)
    out = torch.empty((n // m, c), dtype=x.dtype, device=x.device) if out is None else out
    nb = _lib.csa_compress_from_hidden_workspace_size(n, d, c, m, mode)
    ws = _ws(nb, x.device, ws)
    _check(_lib.csa_compress_from_hidden(_ptr(x), _ptr(x_left), _ptr(W), _ptr(bias), n, d, c, m, _ptr(out),
                                         _ptr(ws), _nbytes(ws), mode, _stream()))
    return out


def hca_compress_from_hidden(x, W, bias, mp: int, out=None, ws=None):
    n, d = x.shape
    c = W.shape[0] // 2
    mode = _mode(x)
    out = torch.empty((n // mp, c), dtype=x.dtype, device=x.device) if out is None else out
    nb = _lib.hca_compress_from_hidden_workspace_size(n, d, c, mp, mode)
    ws = _ws(nb, x.device, ws)
    _check(_lib.hca_compress_from_hidden(_ptr(x), _ptr(W), _ptr(bias), n, d, c, mp, _ptr(out), _ptr(ws),
                                         _nbytes(ws), mode, _stream()))
    return out


# ---------------------------------------------------------------- decode-time compression
def csa_compress_step(proj_new, state, bias, pos, cache, m: int):
    """Store each sequence's newest projected row (proj_new [B, 4c] fp32) in its
    state ring (state [B, 2m, 4c] fp32, updated in place) and write the entry
    of every block the token at pos[b] closes into cache [B, Nmax, c]."""
    B, c4 = proj_new.shape
    c = c4 // 4
    _shape(state, (B, 2 * m, c4), "state")
    _shape(bias, (2 * m, c), "bias")
    _shape(pos, (B,), "pos")
    if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != c:
        raise ValueError(f"cache has shape {tuple(cache.shape)}, expected ({B}, Nmax, {c})")
    _check(_lib.csa_compress_step(_ptr(proj_new), _ptr(state), _ptr(bias), _ptr(pos), B, c4 // 4, m, cache.shape[1],
                                  _ptr(cache), _mode(cache), _stream()))
    return cache


def hca_compress_step(proj_new, state, bias, pos, cache, mp: int):
    """HCA: proj_new [B, 2c] fp32, state [B, mp, 2c] fp32, cache [B, Nmax, c]."""
    B, c2 = proj_new.shape
    c = c2 // 2
    _shape(state, (B, mp, c2), "state")
    _shape(bias, (mp, c), "bias")
    _shape(pos, (B,), "pos")
    if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != c:
        raise ValueError(f"cache has shape {tuple(cache.shape)}, expected ({B}, Nmax, {c})")
    _check(_lib.hca_compress_step(_ptr(proj_new), _ptr(state), _ptr(bias), _ptr(pos), B, c2 // 2, mp, cache.shape[1],
                                  _ptr(cache), _mode(cache), _stream()))
    return cache


def csa_compress_chunk(proj, state, bias, start: int, cache, m: int):
    """Compress tokens start .. start+n-1 of one sequence (proj [n, 4c] fp32)
    at any start and length: writes the entry of every block ending inside
    the chunk into cache [Nmax, c], earlier window tokens from the state ring
    (state [2m, 4c] fp32, updated in place to the last 2m tokens)."""
    n, c4 = proj.shape
    c = c4 // 4
    _dtype(proj, torch.float32, "proj")
    _dtype(state, torch.float32, "state")
    _shape(state, (2 * m, c4), "state")
    _shape(bias, (2 * m, c), "bias")
    if cache.dim() != 2 or cache.shape[1] != c:
        raise ValueError(f"cache has shape {tuple(cache.shape)}, expected (Nmax, {c})")
    _check(_lib.csa_compress_chunk(_ptr(proj), _ptr(state), _ptr(bias), start, n, c, m, _ptr(cache), cache.shape[0],
                                   _mode(cache), _stream()))
    return cache


def hca_compress_chunk(proj, state, bias, start: int, cache, mp: int):
    """HCA: proj [n, 2c] fp32, state [mp, 2c] fp32, cache [Nmax, c]."""
    n, c2 = proj.shape
    c = c2 // 2
    _dtype(proj, torch.float32, "proj")
    _dtype(state, torch.float32, "state")
    _shape(state, (mp, c2), "state")
    _shape(bias, (mp, c), "bias")
    if cache.dim() != 2 or cache.shape[1] != c:
        raise ValueError(f"cache has shape {tuple(cache.shape)}, expected (Nmax, {c})")
    _check(_lib.hca_compress_chunk(_ptr(proj), _ptr(state), _ptr(bias), start, n, c, mp, _ptr(cache), cache.shape[0],
                                   _mode(cache), _stream()))
    return cache


def csa_decode_compress(x_new, W_kv, B_kv, W_idx, B_idx, pos, state_kv, state_idx, kv_cache, idx_cache, m: int = 4,
                        ws=None):
    """One decode step's compression of both CSA streams from the new tokens'
    hidden states x_new [B, d]; states and caches are updated in place."""
    B, d = x_new.shape
    c = W_kv.shape[0] // 4
    cI = W_idx.shape[0] // 4
    Nmax = kv_cache.shape[1]
    _shape(W_kv, (4 * c, d), "W_kv")
    _shape(W_idx, (4 * cI, d), "W_idx")
    _shape(B_kv, (2 * m, c), "B_kv")
    _shape(B_idx, (2 * m, cI), "B_idx")
    _shape(pos, (B,), "pos")
    _shape(state_kv, (B, 2 * m, 4 * c), "state_kv")
    _shape(state_idx, (B, 2 * m, 4 * cI), "state_idx")
    _shape(kv_cache, (B, Nmax, c), "kv_cache")
    _shape(idx_cache, (B, Nmax, cI), "idx_cache")
    ws = _ws(_lib.csa_decode_compress_workspace_size(B, c, cI), x_new.device, ws)
    _check(_lib.csa_decode_compress(_ptr(x_new), _ptr(W_kv), _ptr(B_kv), _ptr(W_idx), _ptr(B_idx), _ptr(pos), B, d, m,
                                    c, cI, _ptr(state_kv), _ptr(state_idx), _ptr(kv_cache), _ptr(idx_cache),
                                    kv_cache.shape[1], _ptr(ws), _nbytes(ws), _mode(x_new), _stream()))


# ---------------------------------------------------------------- a4 / a5
def _kv3(K):
    return K if K.dim() == 3 else K.unsqueeze(0)


def csa_index_scores(qI, w, K, pos, m: int, seq_of_q=None):
    nq, HI, cI = qI.shape
    K = _kv3(K)
    Nmax = K.shape[1]
    scores = torch.empty((nq, Nmax), dtype=torch.float32, device=qI.device)
    _check(_lib.csa_index_scores(_ptr(qI), _ptr(w), _ptr(K), _ptr(pos), _ptr(seq_of_q), nq, K.shape[0], HI, cI,
                                 Nmax, m, _ptr(scores), _mode(qI), _stream()))
    return scores


def csa_topk_from_scores(scores, k: int, valid=None, valid_div: int = 1, ws=None):
    nq, ncols = scores.shape
    idx = torch.empty((nq, k), dtype=torch.int32, device=scores.device)
    top = torch.empty((nq, k), dtype=torch.float32, device=scores.device)
    ws = _ws(_lib.csa_topk_workspace_size(nq, ncols, k), scores.device, ws)
    _check(_lib.csa_topk_from_scores(_ptr(scores), ncols, _ptr(valid), valid_div, nq, ncols, k, _ptr(idx),
                                     _ptr(top), _ptr(ws), _nbytes(ws), _stream()))
    return idx, top


def csa_topk_from_scores_bf16(scores, k: int, valid=None, valid_div: int = 1):
    """Top-k over bf16 scores [nq, ncols] (same rule as csa_topk_from_scores)."""
    nq, ncols = scores.shape
    _dtype(scores, torch.bfloat16, "scores")
    _dtype(valid, torch.int32, "valid")
    _shape(valid, (nq,), "valid")
    idx = torch.empty((nq, k), dtype=torch.int32, device=scores.device)
    top = torch.empty((nq, k), dtype=torch.float32, device=scores.device)
    _check(_lib.csa_topk_from_scores_bf16(_ptr(scores), ncols, _ptr(valid), valid_div, nq, ncols, k, _ptr(idx),
                                          _ptr(top), _stream()))
    return idx, top


def csa_index_topk(qI, w, K, pos, m: int, k: int, seq_of_q=None, ws=None):
    nq, HI, cI = qI.shape
    K = _kv3(K)
    Nmax = K.shape[1]
    mode = _mode(qI)
    idx = torch.empty((nq, k), dtype=torch.int32, device=qI.device)
    top = torch.empty((nq, k), dtype=torch.float32, device=qI.device)
    ws = _ws(_lib.csa_index_topk_workspace_size(nq, Nmax, k, mode), qI.device, ws)
    _check(_lib.csa_index_topk(_ptr(qI), _ptr(w), _ptr(K), _ptr(pos), _ptr(seq_of_q), nq, K.shape[0], HI, cI,
                               Nmax, m, k,
                               _ptr(idx), _ptr(top), _ptr(ws), _nbytes(ws), mode, _stream()))
    return idx, top


def csa_index_topk_noalloc(qI, w, K, pos, m: int, k: int, seq_of_q=None, idx=None, top_scores=None):
    """csa_index_topk without a workspace, for callers that cannot allocate
    device memory when they select: the score block between the indexer and
    the selection lives in a fixed 16 MiB array inside the library
    (nq * Nmax <= CSA_NOALLOC_MAX_SCORES). Pass preallocated idx [nq, k]
    int32 and top_scores [nq, k] fp32 (or None) to make the call itself
    allocation-free. Calls that overlap on the GPU share that array and race."""
    nq, HI, cI = qI.shape
    K = _kv3(K)
    n_seq, Nmax = K.shape[0], K.shape[1]
    mode = _mode(qI)
    _dtype(K, qI.dtype, "K")
    _shape(K, (n_seq, Nmax, cI), "K")
    _dtype(w, torch.float32, "w")
    _shape(w, (nq, HI), "w")
    _dtype(pos, torch.int32, "pos")
    _shape(pos, (nq,), "pos")
    _dtype(seq_of_q, torch.int32, "seq_of_q")
    _shape(seq_of_q, (nq,), "seq_of_q")
    if idx is None:
        idx = torch.empty((nq, k), dtype=torch.int32, device=qI.device)
    _dtype(idx, torch.int32, "idx")
    _shape(idx, (nq, k), "idx")
    _dtype(top_scores, torch.float32, "top_scores")
    _shape(top_scores, (nq, k), "top_scores")
    _check(_lib.csa_index_topk_noalloc(_ptr(qI), _ptr(w), _ptr(K), _ptr(pos), _ptr(seq_of_q), nq, n_seq, HI, cI,
                                       Nmax, m, k, _ptr(idx), _ptr(top_scores), mode, _stream()))
    return idx, top_scores


# ---------------------------------------------------------------- FP8 indexer
def csa_quantize_e4m3(x, w=None):
    """Row-wise e4m3 storage of x [..., cols] (bf16 or fp32): returns (codes,
    a uint8 tensor of x's shape holding the e4m3 bytes (view it as
    torch.float8_e4m3fn to read values), scales [...] fp32, w * scales or
    None). w, when given, has the shape of the scales."""
    cols = x.shape[-1]
    rows = x.numel() // cols if cols else 0
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scale = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    w_out = None
    if w is not None:
        _dtype(w, torch.float32, "w")
        _shape(w, tuple(x.shape[:-1]), "w")
        w_out = torch.empty_like(w)
    _check(_lib.csa_quantize_e4m3(_ptr(x), rows, cols, _ptr(out), _ptr(scale), _ptr(w), _ptr(w_out), _mode(x),
                                  _stream()))
    return out, scale, w_out


def csa_index_scores_fp8(qI8, wq, K8, k_scale, pos, m: int, seq_of_q=None):
    """Indexer scores from e4m3 operands: qI8 [nq, HI, cI] and K8 [B, Nmax, cI]
    uint8 codes, wq [nq, HI] (head weights times query scales), k_scale
    [B, Nmax]. Returns fp32 [nq, Nmax] (-inf where invisible)."""
    nq, HI, cI = qI8.shape
    K8 = _kv3(K8)
    n_seq, Nmax = K8.shape[0], K8.shape[1]
    for t, nm in ((qI8, "qI8"), (K8, "K8")):
        _dtype(t, torch.uint8, nm)
    _shape(wq, (nq, HI), "wq")
    _shape(k_scale, (n_seq, Nmax), "k_scale")
    _shape(pos, (nq,), "pos")
    scores = torch.empty((nq, Nmax), dtype=torch.float32, device=qI8.device)
    _check(_lib.csa_index_scores_fp8(_ptr(qI8), _ptr(wq), _ptr(K8), _ptr(k_scale), _ptr(pos), _ptr(seq_of_q), nq,
                                     n_seq, HI, cI, Nmax, m, _ptr(scores), _stream()))
    return scores


def csa_decode_fp8(qI, w, idx_cache8, idx_scale, q, kv_cache, ctx_len, m: int, k: int, scale: float = 0.0,
                   sink=None, out=None, lse=None, ws=None, return_topk: bool = False, bf16_scores: bool = False):
    """csa_decode with the FP8 indexer: idx_cache8 [B, Nmax, cI] e4m3 codes
    (uint8) with idx_scale [B, Nmax]; qI [B, HI, cI] bf16 is quantized inside.
    bf16_scores: the index scores are stored and selected as bf16."""
    B, HI, cI = qI.shape
    _, Nmax, _ = idx_cache8.shape
    _, H, c = q.shape
    _dtype(idx_cache8, torch.uint8, "idx_cache8")
    _shape(idx_cache8, (B, Nmax, cI), "idx_cache8")
    _shape(idx_scale, (B, Nmax), "idx_scale")
    _shape(w, (B, HI), "w")
    _shape(kv_cache, (B, Nmax, c), "kv_cache")
    _shape(ctx_len, (B,), "ctx_len")
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device) if lse is None else lse
    topk_idx = torch.empty((B, k), dtype=torch.int32, device=q.device) if return_topk else None
    ws = _ws(_lib.csa_decode_fp8_workspace_size(B, Nmax, H, c, HI, cI, k), q.device, ws)
    _check(_lib.csa_decode_fp8(_ptr(qI), _ptr(w), _ptr(idx_cache8), _ptr(idx_scale), _ptr(q), _ptr(kv_cache),
                               _ptr(ctx_len), B, Nmax, m, H, c, HI, cI, k, scale, _ptr(sink),
                               CSA_SCORES_BF16 if bf16_scores else 0, _ptr(out), _ptr(lse),
                               _ptr(topk_idx), _ptr(ws), _nbytes(ws), _stream()))
    return (out, lse, topk_idx) if return_topk else (out, lse)


# ---------------------------------------------------------------- a6 / a7
def csa_sparse_mqa(q, KV, idx, scale: float = 0.0, sink=None, seq_of_q=None, out=None, ws=None):
    nq, H, c = q.shape
    KV = _kv3(KV)
    Nmax = KV.shape[1]
    k = idx.shape[1]
    mode = _mode(q)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((nq, H), dtype=torch.float32, device=q.device)
    ws = _ws(_lib.csa_sparse_mqa_workspace_size(nq, H, c, k, mode), q.device, ws)
    _check(_lib.csa_sparse_mqa(_ptr(q), _ptr(KV), _ptr(idx), _ptr(seq_of_q), nq, KV.shape[0], H, c, Nmax, k, scale,
                               _ptr(sink), _ptr(out), _ptr(lse), _ptr(ws), _nbytes(ws), mode, _stream()))
    return out, lse


def hca_dense_mqa(q, KV, pos, mp: int, scale: float = 0.0, sink=None, seq_of_q=None, out=None, ws=None):
    nq, H, c = q.shape
    KV = _kv3(KV)
    Nmax = KV.shape[1]
    mode = _mode(q)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((nq, H), dtype=torch.float32, device=q.device)
    ws = _ws(_lib.hca_dense_mqa_workspace_size(nq, H, c, Nmax, mode), q.device, ws)
    _check(_lib.hca_dense_mqa(_ptr(q), _ptr(KV), _ptr(pos), _ptr(seq_of_q), nq, KV.shape[0], H, c, Nmax, mp, scale,
                              _ptr(sink), _ptr(out), _ptr(lse), _ptr(ws), _nbytes(ws), mode, _stream()))
    return out, lse


# ---------------------------------------------------------------- fused
def csa_decode_workspace_size(B, Nmax, H, c, HI, cI, k, mode) -> int:
    return int(_lib.csa_decode_workspace_size(B, Nmax, H, c, HI, cI, k, mode))


def csa_decode(qI, w, idx_cache, q, kv_cache, ctx_len, m: int, k: int, scale: float = 0.0, sink=None,
               out=None, lse=None, topk_idx=None, ws=None, return_topk: bool = False):
    B, HI, cI = qI.shape
    _, H, c = q.shape
    Nmax = kv_cache.shape[1]
    mode = _mode(q)
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if return_topk and topk_idx is None:
        topk_idx = torch.empty((B, k), dtype=torch.int32, device=q.device)
    ws = _ws(csa_decode_workspace_size(B, Nmax, H, c, HI, cI, k, mode), q.device, ws)
    _check(_lib.csa_decode(_ptr(qI), _ptr(w), _ptr(idx_cache), _ptr(q), _ptr(kv_cache), _ptr(ctx_len), B, Nmax,
                           m, H, c, HI, cI, k, scale, _ptr(sink), _ptr(out), _ptr(lse), _ptr(topk_idx),
                           _ptr(ws), _nbytes(ws), mode, _stream()))
    return (out, lse, topk_idx) if return_topk else (out, lse)


def hca_decode(q, kv_cache, ctx_len, mp: int, scale: float = 0.0, sink=None, out=None, lse=None, ws=None):
    B, H, c = q.shape
    Nmax = kv_cache.shape[1]
    mode = _mode(q)
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    ws = _ws(_lib.hca_decode_workspace_size(B, Nmax, H, c, mode), q.device, ws)
    _check(_lib.hca_decode(_ptr(q), _ptr(kv_cache), _ptr(ctx_len), B, Nmax, mp, H, c, scale, _ptr(sink),
                           _ptr(out), _ptr(lse), _ptr(ws), _nbytes(ws), mode, _stream()))
    return out, lse


def csa_prefill(x, x_left, W_kv, B_kv, W_idx, B_idx, start: int, kv_cache, idx_cache, qI, w, q, k: int,
                m: int = 4, scale: float = 0.0, sink=None, out=None, ws=None, return_topk: bool = False,
                state_kv=None, state_idx=None):
    """One prefill chunk of one sequence. Without state rings the chunk starts
    and ends on block boundaries (x_left: the m hidden rows before it). With
    state_kv [2m, 4c] and state_idx [2m, 4cI] (fp32, updated in place) the
    chunk may start and end anywhere; x_left is then ignored. With W_kv and
    W_idx None the caches already hold the chunk's entries and only the
    attention runs (x gives the chunk length)."""
    n, d = x.shape
    c = kv_cache.shape[1] if W_kv is None else W_kv.shape[0] // 4
    cI = idx_cache.shape[1] if W_idx is None else W_idx.shape[0] // 4
    _, H, _ = q.shape
    _, HI, _ = qI.shape
    Nmax = kv_cache.shape[0]
    mode = _mode(x)
    if (state_kv is None) != (state_idx is None):
        raise ValueError("state_kv and state_idx go together")
    _shape(state_kv, (2 * m, 4 * c), "state_kv")
    _shape(state_idx, (2 * m, 4 * cI), "state_idx")
    _dtype(state_kv, torch.float32, "state_kv")
    _dtype(state_idx, torch.float32, "state_idx")
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((n, H), dtype=torch.float32, device=x.device)
    topk_idx = torch.empty((n, k), dtype=torch.int32, device=x.device) if return_topk else None
    nb = _lib.csa_prefill_workspace_size(n, Nmax, d, m, c, cI, H, HI, k, mode)
    ws = _ws(nb, x.device, ws)
    _check(_lib.csa_prefill(_ptr(x), _ptr(x_left), _ptr(W_kv), _ptr(B_kv), _ptr(W_idx), _ptr(B_idx), start, n, d,
                            m, c, cI, _ptr(kv_cache), _ptr(idx_cache), Nmax, _ptr(state_kv), _ptr(state_idx),
                            _ptr(qI), _ptr(w), _ptr(q), H, HI, k,
                            scale, _ptr(sink), _ptr(out), _ptr(lse), _ptr(topk_idx), _ptr(ws), _nbytes(ws), mode,
                            _stream()))
    return (out, lse, topk_idx) if return_topk else (out, lse)


# ---------------------------------------------------------------- attention output completion
def csa_norm_rope(x, pos=None, gamma=None, eps: float = 1e-6, rope_dims: int = 64, rope_base: float = 10000.0,
                  inverse: bool = False, pos0: int = 0, pos_step: int = 1, group: Optional[int] = None, out=None):
    """RMSNorm (when gamma is given) then rotary encoding of the last rope_dims
    channels. x [..., c]: with pos [G] the rows split into G equal groups of
    consecutive rows sharing pos[g] (x [nq, H, c] with pos [nq]: all heads of
    query t at pos[t]); with pos None, group g of `group` rows (default 1)
    sits at pos0 + g * pos_step. out may be x (in place)."""
    c = x.shape[-1]
    rows = x.numel() // c
    _shape(gamma, (c,), "gamma")
    _shape(out, tuple(x.shape), "out")
    if pos is not None:
        G = pos.numel()
        if G == 0 or rows % G:
            raise ValueError(f"{rows} rows do not split into {G} position groups")
        group = rows // G
    elif group is None:
        group = 1
    out = torch.empty_like(x) if out is None else out
    _check(_lib.csa_norm_rope(_ptr(x), _ptr(out), rows, group, c, _ptr(gamma), eps, rope_dims, rope_base, _ptr(pos),
                              pos0, pos_step, int(inverse), _mode(x), _stream()))
    return out


def csa_window_entries(sel, pos, n_win: int, ring_off: int, ring_len: int, pos0: int = 0, nq: Optional[int] = None):
    """[nq, k + n_win] entry lists: the selection sel [nq, k] (or None) followed
    by the rows ring_off + (tau mod ring_len) of tokens p-n_win+1 .. p (-1 before
    the sequence start); p = pos[t], or pos0 + t when pos is None."""
    if sel is not None:
        nq, k = sel.shape
        dev = sel.device
    else:
        k = 0
        if nq is None:
            nq = pos.numel()
        dev = pos.device if pos is not None else torch.device("cuda", torch.cuda.current_device())
    ent = torch.empty((nq, k + n_win), dtype=torch.int32, device=dev)
    _check(_lib.csa_window_entries(_ptr(sel), k, _ptr(pos), pos0, nq, n_win, ring_off, ring_len, _ptr(ent),
                                   _stream()))
    return ent


def csa_attend_decode(qI, w, idx_cache, q, kv_cache, ctx_len, m: int, k: int, n_win: int = 128,
                      ring_len: Optional[int] = None, scale: float = 0.0, q_gamma=None, eps: float = 1e-6,
                      rope_dims: int = 64, rope_base: float = 10000.0, sink=None, out=None, lse=None,
                      topk_idx=None, ws=None, return_topk: bool = False):
    """Decode with the complete attention output: query RMSNorm + rotary,
    indexer, top-k, the sliding window joined to the selection in one softmax,
    and the output turned back by the query position. kv_cache [B, Nmax +
    ring_len, c] (compressed rows, then the window ring); idx_cache [B, Nmax, cI]."""
    B, HI, cI = qI.shape
    _, H, c = q.shape
    Nmax = idx_cache.shape[1]
    if ring_len is None:
        ring_len = kv_cache.shape[1] - Nmax
    if kv_cache.shape[1] != Nmax + ring_len:
        raise ValueError(f"kv_cache has {kv_cache.shape[1]} rows per sequence, Nmax + ring_len = {Nmax + ring_len}")
    _shape(kv_cache, (B, Nmax + ring_len, c), "kv_cache")
    _shape(idx_cache, (B, Nmax, cI), "idx_cache")
    _shape(w, (B, HI), "w")
    _shape(ctx_len, (B,), "ctx_len")
    _shape(q_gamma, (c,), "q_gamma")
    _shape(sink, (H,), "sink")
    mode = _mode(q)
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if return_topk and topk_idx is None:
        topk_idx = torch.empty((B, k), dtype=torch.int32, device=q.device)
    nb = _lib.csa_attend_decode_workspace_size(B, Nmax, ring_len, n_win, H, c, HI, cI, k, mode)
    ws = _ws(nb, q.device, ws)
    _check(_lib.csa_attend_decode(_ptr(qI), _ptr(w), _ptr(idx_cache), _ptr(q), _ptr(kv_cache), _ptr(ctx_len), B,
                                  Nmax, ring_len, n_win, m, H, c, HI, cI, k, scale, _ptr(q_gamma), eps, rope_dims,
                                  rope_base, _ptr(sink), _ptr(out), _ptr(lse), _ptr(topk_idx), _ptr(ws), _nbytes(ws),
                                  mode, _stream()))
    return (out, lse, topk_idx) if return_topk else (out, lse)


# ---------------------------------------------------------------- cache blocks
def csa_cache_block_layout(m: int, mp: int, c: int, cI: int, dtype: int = CSA_BF16) -> dict:
    """The lcm(m, m')-token cache block: rows of each part per block, bytes
    per block and each part's byte offset within a block."""
    r1, r2 = ctypes.c_int(0), ctypes.c_int(0)
    bb, o_kv, o_idx, o_hca = ctypes.c_int64(0), ctypes.c_int64(0), ctypes.c_int64(0), ctypes.c_int64(0)
    _check(_lib.csa_cache_block_layout(m, mp, c, cI, dtype, ctypes.byref(r1), ctypes.byref(r2), ctypes.byref(bb),
                                       ctypes.byref(o_kv), ctypes.byref(o_idx), ctypes.byref(o_hca)))
    return {"csa_rows": r1.value, "hca_rows": r2.value, "block_bytes": bb.value, "kv_offset": o_kv.value,
            "idx_offset": o_idx.value, "hca_offset": o_hca.value, "m": m, "mp": mp, "c": c, "cI": cI}


def _blocks_check(blocks, layout, B):
    if blocks.dtype != torch.uint8 or blocks.dim() != 3 or blocks.shape[0] != B or \
            blocks.shape[2] != layout["block_bytes"] or not blocks.is_contiguous():
        raise ValueError(f"blocks must be a contiguous uint8 tensor [B={B}, nblocks, {layout['block_bytes']}], "
                         f"got {tuple(blocks.shape)} {blocks.dtype}")
    return blocks.shape[1]


def csa_decode_blocked(qI, w, q, blocks, layout, ctx_len, k: int, scale: float = 0.0, sink=None, out=None, lse=None,
                       topk_idx=None, ws=None, return_topk: bool = False):
    """csa_decode over block caches: blocks [B, nblocks, block_bytes] uint8
    in the layout of csa_cache_block_layout (bf16 entries)."""
    B, HI, cI = qI.shape
    _, H, c = q.shape
    nblk = _blocks_check(blocks, layout, B)
    if c != layout["c"] or cI != layout["cI"]:
        raise ValueError(f"layout is for c={layout['c']}, cI={layout['cI']}; q has c={c}, qI has cI={cI}")
    rpb, m = layout["csa_rows"], layout["m"]
    Nmax = nblk * rpb
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if return_topk and topk_idx is None:
        topk_idx = torch.empty((B, k), dtype=torch.int32, device=q.device)
    mode = _mode(q)
    ws = _ws(csa_decode_workspace_size(B, Nmax, H, c, HI, cI, k, mode), q.device, ws)
    base = blocks.data_ptr()
    _check(_lib.csa_decode_blocked(_ptr(qI), _ptr(w), base + layout["idx_offset"], _ptr(q), base + layout["kv_offset"],
                                   _ptr(ctx_len), B, Nmax, m, H, c, HI, cI, k, scale, _ptr(sink), _ptr(out),
                                   _ptr(lse), _ptr(topk_idx), rpb, layout["block_bytes"], _ptr(ws), _nbytes(ws), mode,
                                   _stream()))
    return (out, lse, topk_idx) if return_topk else (out, lse)


def hca_decode_blocked(q, blocks, layout, ctx_len, scale: float = 0.0, sink=None, out=None, lse=None, ws=None):
    """hca_decode over the HCA part of block caches (one entry per block)."""
    B, H, c = q.shape
    nblk = _blocks_check(blocks, layout, B)
    rpb = layout["hca_rows"]
    Nmax = nblk * rpb
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    mode = _mode(q)
    ws = _ws(_lib.hca_decode_workspace_size(B, Nmax, H, c, mode), q.device, ws)
    _check(_lib.hca_decode_blocked(_ptr(q), blocks.data_ptr() + layout["hca_offset"], _ptr(ctx_len), B, Nmax,
                                   layout["mp"], H, c, scale, _ptr(sink), _ptr(out), _ptr(lse), rpb,
                                   layout["block_bytes"], _ptr(ws), _nbytes(ws), mode, _stream()))
    return out, lse


def csa_decode_compress_blocked(x_new, W_kv, B_kv, W_idx, B_idx, pos, state_kv, state_idx, blocks, layout, ws=None):
    """csa_decode_compress writing the entries into block caches."""
    B, d = x_new.shape
    c, cI, m = layout["c"], layout["cI"], layout["m"]
    nblk = _blocks_check(blocks, layout, B)
    rpb = layout["csa_rows"]
    _shape(W_kv, (4 * c, d), "W_kv")
    _shape(W_idx, (4 * cI, d), "W_idx")
    _shape(B_kv, (2 * m, c), "B_kv")
    _shape(B_idx, (2 * m, cI), "B_idx")
    _shape(pos, (B,), "pos")
    _shape(state_kv, (B, 2 * m, 4 * c), "state_kv")
    _shape(state_idx, (B, 2 * m, 4 * cI), "state_idx")
    ws = _ws(_lib.csa_decode_compress_workspace_size(B, c, cI), x_new.device, ws)
    base = blocks.data_ptr()
    _check(_lib.csa_decode_compress_blocked(_ptr(x_new), _ptr(W_kv), _ptr(B_kv), _ptr(W_idx), _ptr(B_idx), _ptr(pos),
                                            B, d, m, c, cI, _ptr(state_kv), _ptr(state_idx),
                                            base + layout["kv_offset"], base + layout["idx_offset"], nblk * rpb, rpb,
                                            layout["block_bytes"], _ptr(ws), _nbytes(ws), _mode(x_new), _stream()))


def hca_compress_step_blocked(proj_new, state, bias, pos, blocks, layout):
    """hca_compress_step writing the entries into the HCA part of block caches."""
    B, c2 = proj_new.shape
    c, mp = layout["c"], layout["mp"]
    nblk = _blocks_check(blocks, layout, B)
    _shape(proj_new, (B, 2 * c), "proj_new")
    _shape(state, (B, mp, 2 * c), "state")
    _shape(bias, (mp, c), "bias")
    _shape(pos, (B,), "pos")
    rpb = layout["hca_rows"]
    _check(_lib.hca_compress_step_blocked(_ptr(proj_new), _ptr(state), _ptr(bias), _ptr(pos), B, c, mp, nblk * rpb,
                                          blocks.data_ptr() + layout["hca_offset"], rpb, layout["block_bytes"],
                                          CSA_BF16, _stream()))


# ---------------------------------------------------------------- FP8 KV
def csa_quantize_kv_fp8(kv, rope_dims: int = 64):
    """KV entries [..., c] bf16 into FP8 storage: (codes [..., c-R] uint8,
    scales [...] fp32, rope [..., R] bf16)."""
    _dtype(kv, torch.bfloat16, "kv")
    c = kv.shape[-1]
    rows = kv.numel() // c if c else 0
    lead = tuple(kv.shape[:-1])
    codes = torch.empty(lead + (c - rope_dims,), dtype=torch.uint8, device=kv.device)
    scales = torch.empty(lead, dtype=torch.float32, device=kv.device)
    rope = torch.empty(lead + (rope_dims,), dtype=torch.bfloat16, device=kv.device)
    _check(_lib.csa_quantize_kv_fp8(_ptr(kv.contiguous()), rows, c, rope_dims, _ptr(codes), _ptr(scales),
                                    _ptr(rope) if rope_dims else None, _stream()))
    return codes, scales, rope


def csa_decode_fp8kv(qI, w, idx_cache, q, kv_codes, kv_scales, kv_rope, ctx_len, m: int, k: int, scale: float = 0.0,
                     sink=None, out=None, lse=None, topk_idx=None, ws=None, return_topk: bool = False):
    """csa_decode with the KV entries in FP8 storage (csa_quantize_kv_fp8)."""
    B, HI, cI = qI.shape
    _, H, c = q.shape
    Nmax = idx_cache.shape[1]
    R = kv_rope.shape[-1]
    _shape(kv_codes, (B, Nmax, c - R), "kv_codes")
    _shape(kv_scales, (B, Nmax), "kv_scales")
    _shape(kv_rope, (B, Nmax, R), "kv_rope")
    _dtype(kv_codes, torch.uint8, "kv_codes")
    _dtype(kv_scales, torch.float32, "kv_scales")
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if return_topk and topk_idx is None:
        topk_idx = torch.empty((B, k), dtype=torch.int32, device=q.device)
    ws = _ws(_lib.csa_decode_fp8kv_workspace_size(B, Nmax, H, c, HI, cI, k), q.device, ws)
    _check(_lib.csa_decode_fp8kv(_ptr(qI), _ptr(w), _ptr(idx_cache), _ptr(q), _ptr(kv_codes), _ptr(kv_scales),
                                 _ptr(kv_rope), _ptr(ctx_len), B, Nmax, m, H, c, R, HI, cI, k, scale, _ptr(sink),
                                 _ptr(out), _ptr(lse), _ptr(topk_idx), _ptr(ws), _nbytes(ws), _stream()))
    return (out, lse, topk_idx) if return_topk else (out, lse)
