"""Seeded synthetic inputs for the CSA / HCA hot path.

This module only draws random tensors with the shapes and distributions of the
workloads; it contains none of the method's arithmetic. Both the CUDA path and
the CPU oracle consume what it produces (the oracle through a host copy).

Distributions (one reading, applied to every workload):
  * activations, caches, queries: N(0, 1), rounded to bf16 (nearest-even);
  * projection weights: N(0, 1/d) (variance 1/d), bf16, stored [out, in];
  * positional biases: N(0, 0.1) (variance 0.1), fp32;
  * indexer head weights w: softmax over heads of N(0, 1) logits, fp32;
  * RMSNorm weights: 1 + N(0, 0.01), fp32; sink logits: N(0, 1), fp32;
  * per-query context lengths: integers uniform on [lo, hi], inclusive.

Generation uses torch's seeded generators on the target device. The stream
of every tensor is keyed by (workload seed, tensor tag), so adding a tensor
never changes another one.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Optional

import torch


def _subseed(seed: int, tag: str) -> int:
    h = hashlib.sha256(f"{seed}:{tag}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(seed: int, tag: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_subseed(seed, tag))
    return g


def normal(shape, seed: int, tag: str, std: float = 1.0, dtype=torch.bfloat16, device="cpu"):
    """N(0, std^2) samples, drawn in fp32 and rounded once to ``dtype``."""
    g = _gen(seed, tag, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def head_weights(nq: int, heads: int, seed: int, tag: str = "w", device="cpu"):
    """Indexer head weights: softmax over heads of N(0, 1) logits (fp32)."""
    logits = normal((nq, heads), seed, tag, dtype=torch.float32, device=device)
    return torch.softmax(logits, dim=-1).contiguous()


def uniform_int(n: int, lo: int, hi: int, seed: int, tag: str, device="cpu"):
    g = _gen(seed, tag, "cpu")
    return torch.randint(lo, hi + 1, (n,), generator=g, dtype=torch.int32).to(device)


# ---------------------------------------------------------------------------
# Workload shapes (the five configurations: a tiny end-to-end prefill, the
# Flash-shaped and Pro-shaped decodes, HCA decode + compressor chunk, and the
# long CSA prefill chunk). ``scaled`` variants keep the structure and shrink
# the lengths so the CPU oracle can check them.
# ---------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class DecodeShape:
    name: str
    seed: int
    batch: int          # independent sequences, one query each
    ctx_lo: int         # context length range (tokens), inclusive
    ctx_hi: int
    n_max: int          # compressed-entry capacity per sequence (ctx_hi // m)
    m: int
    c: int              # KV head dim
    heads: int          # MQA query heads
    idx_heads: int
    idx_dim: int
    k: int

    def scale_ctx(self, factor: int) -> "DecodeShape":
        return dataclasses.replace(self, name=f"{self.name}/{factor}", ctx_lo=self.ctx_lo // factor,
                                   ctx_hi=self.ctx_hi // factor, n_max=self.n_max // factor)


@dataclasses.dataclass(frozen=True)
class HcaShape:
    name: str
    seed: int
    batch: int
    ctx: int            # tokens per sequence (decode)
    n_max: int
    mp: int
    c: int
    heads: int
    chunk: int          # compressor chunk length (tokens)
    d: int              # hidden size of the compressor input


@dataclasses.dataclass(frozen=True)
class PrefillShape:
    name: str
    seed: int
    n: int              # new tokens in the chunk
    start: int          # position of the first new token (multiple of m)
    d: int
    m: int
    c: int
    heads: int
    idx_heads: int
    idx_dim: int
    k: int


TINY = PrefillShape("tiny_csa_prefill_seq1024_d512", seed=0, n=1024, start=0, d=512, m=4, c=128,
                    heads=8, idx_heads=4, idx_dim=64, k=16)
FLASH_DECODE = DecodeShape("csa_decode_flash_b64_ctx64k-128k_k512", seed=1, batch=64, ctx_lo=65536,
                           ctx_hi=131072, n_max=32768, m=4, c=512, heads=64, idx_heads=64,
                           idx_dim=128, k=512)
HCA = HcaShape("hca_decode_b16_ctx1m_plus_compress_chunk131072_d4096", seed=2, batch=16,
               ctx=1048576, n_max=8192, mp=128, c=512, heads=64, chunk=131072, d=4096)
PREFILL = PrefillShape("csa_prefill_n65536_at196608_d4096_k512", seed=3, n=65536, start=196608,
                       d=4096, m=4, c=512, heads=64, idx_heads=64, idx_dim=128, k=512)
PRO_DECODE = DecodeShape("csa_decode_pro_b32_ctx512k-1m_k1024", seed=4, batch=32, ctx_lo=524288,
                         ctx_hi=1048576, n_max=262144, m=4, c=512, heads=128, idx_heads=64,
                         idx_dim=128, k=1024)


# ---------------------------------------------------------------------------
# Input bundles
# ---------------------------------------------------------------------------

def decode_inputs(s: DecodeShape, device="cpu", batch: Optional[int] = None):
    """Caches, queries and context lengths for a CSA decode step."""
    B = s.batch if batch is None else batch
    ctx = uniform_int(s.batch, s.ctx_lo, s.ctx_hi, s.seed, "ctx_len", device)[:B].contiguous()
    return dict(
        kv_cache=normal((B, s.n_max, s.c), s.seed, "kv_cache", device=device),
        idx_cache=normal((B, s.n_max, s.idx_dim), s.seed, "idx_cache", device=device),
        q=normal((B, s.heads, s.c), s.seed, "q", device=device),
        qI=normal((B, s.idx_heads, s.idx_dim), s.seed, "qI", device=device),
        w=head_weights(B, s.idx_heads, s.seed, device=device),
        ctx_len=ctx,
    )


def attend_decode_inputs(s: DecodeShape, device="cpu", batch: Optional[int] = None, n_win: int = 128,
                         ring_len: Optional[int] = None):
    """decode_inputs plus what the complete attention output takes: each
    sequence's KV block extended by its sliding-window ring (ring_len rows of
    uncompressed token KV after the n_max compressed rows), the query RMSNorm
    weight (1 + N(0, 0.01)) and per-head sink logits N(0, 1)."""
    inp = decode_inputs(s, device, batch)
    B = inp["q"].shape[0]
    L = n_win if ring_len is None else ring_len
    ring = normal((B, L, s.c), s.seed, "window_ring", device=device)
    inp["kv_cache"] = torch.cat([inp["kv_cache"], ring], dim=1).contiguous()
    del ring
    inp["q_gamma"] = 1.0 + normal((s.c,), s.seed, "q_gamma", std=0.1, dtype=torch.float32, device=device)
    inp["sink"] = normal((s.heads,), s.seed, "sink", dtype=torch.float32, device=device)
    inp["ring_len"] = L
    return inp


def decode_compress_inputs(s: DecodeShape, d: int, device="cpu", batch: Optional[int] = None, caches: bool = True):
    """One decode step's compression inputs: the new tokens' hidden states
    x [B, d], the compressor weights and biases of both CSA streams, the new
    tokens' positions (the context lengths), zeroed state rings and caches."""
    B = s.batch if batch is None else batch
    m, c, cI = s.m, s.c, s.idx_dim
    inp = dict(
        x=normal((B, d), s.seed, "step_x", device=device),
        W_kv=normal((4 * c, d), s.seed, "step_W_kv", std=1.0 / math.sqrt(d), device=device),
        B_kv=normal((2 * m, c), s.seed, "step_B_kv", std=math.sqrt(0.1), dtype=torch.float32, device=device),
        W_idx=normal((4 * cI, d), s.seed, "step_W_idx", std=1.0 / math.sqrt(d), device=device),
        B_idx=normal((2 * m, cI), s.seed, "step_B_idx", std=math.sqrt(0.1), dtype=torch.float32, device=device),
        pos=uniform_int(s.batch, s.ctx_lo, s.ctx_hi, s.seed, "ctx_len", device)[:B].contiguous()
        if B <= s.batch else uniform_int(B, s.ctx_lo, s.ctx_hi, s.seed, "step_pos", device),
    )
    if caches:
        inp["state_kv"] = torch.zeros((B, 2 * m, 4 * c), dtype=torch.float32, device=device)
        inp["state_idx"] = torch.zeros((B, 2 * m, 4 * cI), dtype=torch.float32, device=device)
        inp["kv_cache"] = torch.zeros((B, s.n_max, c), dtype=torch.bfloat16, device=device)
        inp["idx_cache"] = torch.zeros((B, s.n_max, cI), dtype=torch.bfloat16, device=device)
    return inp


def hca_decode_inputs(s: HcaShape, device="cpu", batch: Optional[int] = None, n_max: Optional[int] = None):
    B = s.batch if batch is None else batch
    N = s.n_max if n_max is None else n_max
    ctx = torch.full((B,), N * s.mp, dtype=torch.int32, device=device)
    return dict(
        kv_cache=normal((B, N, s.c), s.seed, "hca_kv_cache", device=device),
        q=normal((B, s.heads, s.c), s.seed, "hca_q", device=device),
        ctx_len=ctx,
    )


def hca_compress_inputs(s: HcaShape, device="cpu", chunk: Optional[int] = None, d: Optional[int] = None):
    n = s.chunk if chunk is None else chunk
    dd = s.d if d is None else d
    return dict(
        x=normal((n, dd), s.seed, "hca_x", device=device),
        W=normal((2 * s.c, dd), s.seed, "hca_W", std=1.0 / math.sqrt(dd), device=device),
        bias=normal((s.mp, s.c), s.seed, "hca_bias", std=math.sqrt(0.1), dtype=torch.float32,
                    device=device),
    )


def prefill_inputs(s: PrefillShape, device="cpu", n: Optional[int] = None, start: Optional[int] = None):
    """Hidden states, compressor weights/biases, existing caches and queries for
    one CSA prefill chunk. The caches have room for start/m + n/m entries; the
    first start/m are filled (the compressed prefix), the rest are appended by
    the chunk."""
    n = s.n if n is None else n
    start = s.start if start is None else start
    m, d = s.m, s.d
    n_max = (start + n) // m
    kv = torch.zeros((n_max, s.c), dtype=torch.bfloat16, device=device)
    ik = torch.zeros((n_max, s.idx_dim), dtype=torch.bfloat16, device=device)
    if start > 0:
        kv[: start // m] = normal((start // m, s.c), s.seed, "prefix_kv", device=device)
        ik[: start // m] = normal((start // m, s.idx_dim), s.seed, "prefix_idx", device=device)
    return dict(
        x=normal((n, d), s.seed, "x", device=device),
        x_left=(normal((m, d), s.seed, "x_left", device=device) if start > 0 else None),
        W_kv=normal((4 * s.c, d), s.seed, "W_kv", std=1.0 / math.sqrt(d), device=device),
        B_kv=normal((2 * m, s.c), s.seed, "B_kv", std=math.sqrt(0.1), dtype=torch.float32, device=device),
        W_idx=normal((4 * s.idx_dim, d), s.seed, "W_idx", std=1.0 / math.sqrt(d), device=device),
        B_idx=normal((2 * m, s.idx_dim), s.seed, "B_idx", std=math.sqrt(0.1), dtype=torch.float32,
                     device=device),
        kv_cache=kv,
        idx_cache=ik,
        q=normal((n, s.heads, s.c), s.seed, "q", device=device),
        qI=normal((n, s.idx_heads, s.idx_dim), s.seed, "qI", device=device),
        w=head_weights(n, s.idx_heads, s.seed, device=device),
        start=start,
        n=n,
    )
