#!/usr/bin/env python
"""Throughput benchmark of the CSA / HCA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Default workload: CSA decode shaped like V4-Flash (64 concurrent queries, each
against its own compressed cache of a 64K..128K-token context: up to 32768
entries of dim 512, indexer keys 64 heads x 128, top-k 512, 64 query heads).
A step is one pass of the decode hot path over the batch: lightning indexer,
top-k, sparse shared-KV MQA (the csa_decode entry point). Caches and queries
are resident in HBM before timing; the L2 is flushed (256 MiB write) before
every timed step, outside the timed events; each step is timed with CUDA
events on the stream the library launches on.

Other workloads (--workload): pro_decode, hca_decode, hca_compress, prefill,
flash_attend_decode (the Flash decode with the complete attention output:
query RMSNorm + partial rotary, the 128-token sliding window joined to the
selection in one softmax with a sink, the output turned back by position),
flash_decode_compress (one decode step's compression of both CSA streams
through the per-sequence state cache, from the new tokens' hidden states).
On one GPU the default line also carries "extra_workloads": Pro decode, the
long prefill chunk, HCA decode and the HCA compressor, each measured the same
way right after the Flash decode line (--no-extra skips them).

Multi-GPU (under torchrun): every rank runs its own independent batch
(decode queries are independent: no collective on the data path), the step
time is the max over ranks, value = all ranks' queries / that time.

--impl reference times the CPU oracle (fp64, the host's cores) on a bounded
sample of the same workload.

Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import hashlib
import io
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "CSA/HCA decode queries/s at 128K–1M ctx and prefill tok/s; % of HBM/TC roofline"
PROFILES = os.path.join(ROOT, "profiles")
CSRC = os.path.join(ROOT, "compressed_sparse_attention_14_b200", "csrc")

L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------
# process group / ranks
# ----------------------------------------------------------------------------

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        if torch.cuda.is_available():
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, ms_step_max: float) -> float:
    """Whole-job throughput: every rank processes units_per_rank units per
    step and the step takes the slowest rank's time."""
    return world * units_per_rank / (ms_step_max / 1e3)


def dist_done(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for r in csv.reader(f):
                if len(r) >= 9:
                    rows.append([x.strip() for x in r])
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = sorted(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        mx = max((float(r[2]) for r in rows if r[2].replace(".", "").isdigit()), default=None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def source_sha(files) -> str:
    h = hashlib.sha256()
    for f in sorted(files):
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str, files) -> float | None:
    """DRAM bytes per launch from a committed ncu summary, if the kernel's
    sources are unchanged since the capture; None otherwise."""
    p = os.path.join(PROFILES, "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("source_sha") != source_sha(files):
        return None
    return float(e["dram_bytes_per_launch"])


def cpu_oracle_threads() -> int:
    import oracle
    return oracle.num_threads()


class Timer:
    """Per-step CUDA-event timing on the current stream with an L2 flush
    before every step (outside the events): a 256 MiB write evicts the step's
    data, then a 256 MiB read evicts the written lines, so the timed step does
    not pay for the flush's own write-back."""

    def __init__(self):
        self.flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.flush_rd = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")
        self.ms = []

    def step(self, fn):
        self.flush.zero_()
        self.flush_rd.sum()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        self.ms.append((a, b))

    def total_ms(self) -> float:
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in self.ms)


# ----------------------------------------------------------------------------
# workloads (ours)
# ----------------------------------------------------------------------------

def decode_workload(shape, rank, batch=None, fp8=False, fp8kv=False):
    """One csa_decode step over the batch. fp8: the FP8 indexer
    (csa_decode_fp8): the indexer keys are held as e4m3 codes with one fp32
    scale per key (quantized once when the cache is built, outside the timed
    region, as the compressor would store them), q^I is quantized in the call;
    fp32 index scores (bf16 scores tie more often and made this top-k slower).
    fp8kv: the KV entries held in FP8 storage with bf16 rotary dims
    (csa_decode_fp8kv; quantized once outside the timed region)."""
    import dataclasses
    import compressed_sparse_attention_14_b200 as csa
    s = shape if batch is None else dataclasses.replace(shape, batch=batch)
    inp = synth.decode_inputs(dataclass_seed(s, rank), device="cuda")
    B = s.batch
    mode = csa.CSA_BF16
    out = torch.empty_like(inp["q"])
    lse = torch.empty((B, s.heads), dtype=torch.float32, device="cuda")
    if fp8kv:
        kv8, kvs, kvr = csa.csa_quantize_kv_fp8(inp["kv_cache"], rope_dims=ATTEND_ROPE)
        del inp["kv_cache"]
        torch.cuda.synchronize()
        ws = torch.empty(csa._lib.csa_decode_fp8kv_workspace_size(B, s.n_max, s.heads, s.c, s.idx_heads, s.idx_dim,
                                                                  s.k), dtype=torch.uint8, device="cuda")

        def call(qI, w, q, ctx, o=out):
            csa.csa_decode_fp8kv(qI, w, inp["idx_cache"], q, kv8, kvs, kvr, ctx, s.m, s.k, out=o, lse=lse, ws=ws)
    elif fp8:
        k8, ks, _ = csa.csa_quantize_e4m3(inp["idx_cache"])
        del inp["idx_cache"]
        torch.cuda.synchronize()
        ws = torch.empty(csa.workspace_size("csa_decode_fp8", B, s.n_max, s.heads, s.c, s.idx_heads, s.idx_dim, s.k),
                         dtype=torch.uint8, device="cuda")

        def call(qI, w, q, ctx, o=out):
            csa.csa_decode_fp8(qI, w, k8, ks, q, inp["kv_cache"], ctx, s.m, s.k, out=o, lse=lse, ws=ws)
    else:
        ws = torch.empty(csa.csa_decode_workspace_size(B, s.n_max, s.heads, s.c, s.idx_heads, s.idx_dim, s.k, mode),
                         dtype=torch.uint8, device="cuda")

        def call(qI, w, q, ctx, o=out):
            csa.csa_decode(qI, w, inp["idx_cache"], q, inp["kv_cache"], ctx, s.m, s.k, out=o, lse=lse, ws=ws)

    def step():
        call(inp["qI"], inp["w"], inp["q"], inp["ctx_len"])

    ctx = inp["ctx_len"].double()
    vis = torch.floor(ctx / s.m)
    v_sum = float(vis.sum())
    # algorithmic bytes: indexer keys of the visible entries (bf16, or e4m3
    # plus one fp32 scale), q^I and w; the selected KV rows; q and out (bf16)
    key_bytes = (s.idx_dim + 4) if fp8 else s.idx_dim * 2
    idx_bytes = v_sum * key_bytes + B * (s.idx_heads * s.idx_dim * (1 if fp8 else 2) + s.idx_heads * 4)
    # a selected KV row: bf16, or e4m3 codes + fp32 scale + bf16 rotary dims
    row_bytes = (s.c - ATTEND_ROPE) + 4 + 2 * ATTEND_ROPE if fp8kv else s.c * 2
    step_bytes = idx_bytes + B * (s.k * row_bytes + 2 * s.heads * s.c * 2)
    # the indexer kernel also writes one score per visible entry (fp32, or
    # bf16 on the low-precision path)
    score_bytes = 4
    idx_kernel_bytes = idx_bytes + v_sum * score_bytes

    pinned = {k: inp[k].cpu().pin_memory() for k in ("q", "qI", "w", "ctx_len")}
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dev_in = {k: torch.empty_like(inp[k]) for k in pinned}

    def e2e_step():
        for k, v in pinned.items():
            dev_in[k].copy_(v, non_blocking=True)
        call(dev_in["qI"], dev_in["w"], dev_in["q"], dev_in["ctx_len"])
        out_h.copy_(out, non_blocking=True)

    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = out_h.numel() * out_h.element_size()
    mqa_bytes = B * (s.k * s.c * 2 + 2 * s.heads * s.c * 2)
    idx_name = "index_scores_tc_fp8" if fp8 else "index_scores_tc"
    kernels = {
        idx_name: dict(bound="hbm", work=idx_kernel_bytes, files=("indexer_tc.cu", "tc.cuh", "common.cuh")),
        # the indexer with the top-k filter on its epilogue: the same reads, no
        # score block (its candidate lists are a few percent of the scores)
        "index_topk_filter_tc": dict(bound="hbm", work=idx_bytes, files=("indexer_tc.cu", "tc.cuh", "common.cuh")),
        "mqa_tc": dict(bound="hbm", work=mqa_bytes, files=("mqa_tc.cu", "tc.cuh", "common.cuh")),
        # one pass over each row's visible scores, k indices out
        "topk_select": dict(bound="hbm", work=v_sum * score_bytes + B * s.k * 4, files=("topk.cu",)),
    }
    if fp8:
        kernels["quantize_e4m3"] = dict(bound="hbm", work=B * s.idx_heads * (s.idx_dim * 3 + 12), files=("quant.cu",))
    if fp8kv:
        # the selection's FP8 rows in, bf16 rows out (then read by the MQA)
        kernels["gather_kv_fp8"] = dict(bound="hbm", work=B * s.k * (row_bytes + s.c * 2 + 8), files=("quant.cu",))
    pipe = dict(pinned=pinned, out=out, run=lambda d, o: call(d["qI"], d["w"], d["q"], d["ctx_len"], o))
    return dict(step=step, e2e_step=e2e_step, pipe=pipe, units=B, unit="queries/s", h2d=h2d, d2h=d2h,
                kernels=kernels, step_bytes=step_bytes,
                config=dict(workload=s.name + ("_fp8_indexer" if fp8 else "_fp8_kv" if fp8kv else ""), batch=B,
                            ctx_len=f"U[{s.ctx_lo},{s.ctx_hi}]", m=s.m,
                            entries_max=s.n_max, head_dim=s.c, heads=s.heads, index_heads=s.idx_heads,
                            index_dim=s.idx_dim, topk=s.k, visible_entries_total=int(v_sum),
                            index_keys="e4m3 + fp32 scale per key" if fp8 else "bf16",
                            index_scores="fp32",
                            kv_entries="e4m3 + fp32 scale per entry, bf16 rotary dims" if fp8kv else "bf16",
                            l2="flushed before every timed step (256 MiB write + 256 MiB read)"),
                inputs=inp)


ATTEND_WINDOW = 128     # sliding-window tokens per query (V4's n_win)
ATTEND_ROPE = 64        # rotary channels at the end of each head


def attend_decode_workload(shape, rank, batch=None):
    """The decode step with the complete attention output (csa_attend_decode):
    query RMSNorm + partial rotary, indexer, top-k, the 128-token sliding
    window joined to the selection in one softmax with a sink, and the output
    turned back by the query position."""
    import dataclasses
    import compressed_sparse_attention_14_b200 as csa
    s = shape if batch is None else dataclasses.replace(shape, batch=batch)
    inp = synth.attend_decode_inputs(dataclass_seed(s, rank), device="cuda", n_win=ATTEND_WINDOW)
    B, L = s.batch, inp["ring_len"]
    mode = csa.CSA_BF16
    out = torch.empty_like(inp["q"])
    lse = torch.empty((B, s.heads), dtype=torch.float32, device="cuda")
    ws = torch.empty(csa.workspace_size("csa_attend_decode", B, s.n_max, L, ATTEND_WINDOW, s.heads, s.c, s.idx_heads,
                                        s.idx_dim, s.k, mode), dtype=torch.uint8, device="cuda")

    def call(qI, w, q, ctx, o=out):
        csa.csa_attend_decode(qI, w, inp["idx_cache"], q, inp["kv_cache"], ctx, s.m, s.k, n_win=ATTEND_WINDOW,
                              ring_len=L, q_gamma=inp["q_gamma"], rope_dims=ATTEND_ROPE, sink=inp["sink"], out=o,
                              lse=lse, ws=ws)

    def step():
        call(inp["qI"], inp["w"], inp["q"], inp["ctx_len"])

    ctx = inp["ctx_len"].double()
    v_sum = float(torch.floor(ctx / s.m).sum())
    ke = s.k + ATTEND_WINDOW
    qo = B * s.heads * s.c * 2                  # one bf16 pass over q or out
    idx_bytes = v_sum * s.idx_dim * 2 + B * (s.idx_heads * s.idx_dim * 2 + s.idx_heads * 4)
    # indexer, the selected and window rows, q read + normalised q written,
    # the normalised q read by the MQA, out written, out read + written back
    step_bytes = idx_bytes + B * ke * s.c * 2 + 2 * qo + 2 * qo + 2 * qo
    idx_kernel_bytes = idx_bytes + v_sum * 4

    pinned = {k: inp[k].cpu().pin_memory() for k in ("q", "qI", "w", "ctx_len")}
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dev_in = {k: torch.empty_like(inp[k]) for k in pinned}

    def e2e_step():
        for k, v in pinned.items():
            dev_in[k].copy_(v, non_blocking=True)
        call(dev_in["qI"], dev_in["w"], dev_in["q"], dev_in["ctx_len"])
        out_h.copy_(out, non_blocking=True)

    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = out_h.numel() * out_h.element_size()
    kernels = {
        "index_scores_tc": dict(bound="hbm", work=idx_kernel_bytes, files=("indexer_tc.cu", "tc.cuh", "common.cuh")),
        "index_topk_filter_tc": dict(bound="hbm", work=idx_kernel_bytes - v_sum * 4,
                                     files=("indexer_tc.cu", "tc.cuh", "common.cuh")),
        "mqa_tc": dict(bound="hbm", work=B * ke * s.c * 2 + 2 * qo, files=("mqa_tc.cu", "tc.cuh", "common.cuh")),
        "topk_select": dict(bound="hbm", work=v_sum * 4 + B * s.k * 4, files=("topk.cu",)),
        # two launches per step (query in, output back): each one read and one write of [B, H, c]
        "norm_rope": dict(bound="hbm", work=2 * 2 * qo, files=("norm_rope.cu",)),
        "window_entries": dict(bound="hbm", work=B * (s.k + ke) * 4, files=("norm_rope.cu",)),
    }
    pipe = dict(pinned=pinned, out=out, run=lambda d, o: call(d["qI"], d["w"], d["q"], d["ctx_len"], o))
    return dict(step=step, e2e_step=e2e_step, pipe=pipe, units=B, unit="queries/s", h2d=h2d, d2h=d2h,
                kernels=kernels, step_bytes=step_bytes,
                config=dict(workload=ATTEND_NAME, batch=B, ctx_len=f"U[{s.ctx_lo},{s.ctx_hi}]", m=s.m,
                            entries_max=s.n_max, head_dim=s.c, heads=s.heads, index_heads=s.idx_heads,
                            index_dim=s.idx_dim, topk=s.k, window=ATTEND_WINDOW, window_ring=L,
                            rope_dims=ATTEND_ROPE, q_rmsnorm=True, sink=True, visible_entries_total=int(v_sum),
                            l2="flushed before every timed step (256 MiB write + 256 MiB read)"),
                inputs=inp)


ATTEND_NAME = synth.FLASH_DECODE.name + "_win128_rope64_qnorm_sink"

COMPRESS_STEP_D = 4096   # V4-Flash hidden size


def decode_compress_workload(rank, batch=None):
    """One decode step's compression of both CSA streams (csa_decode_compress):
    the new token of each of the Flash batch's sequences is projected from its
    hidden state (d = 4096) into the KV and index-key streams, stored in the
    sequence's state ring, and the sequences whose token closes a block (about
    one in four) get their new entries. Every timed step redoes the same
    tokens at the same positions."""
    import dataclasses
    import compressed_sparse_attention_14_b200 as csa
    s = synth.FLASH_DECODE if batch is None else dataclasses.replace(synth.FLASH_DECODE, batch=batch)
    s = dataclass_seed(s, rank)
    inp = synth.decode_compress_inputs(s, COMPRESS_STEP_D, device="cuda")
    B, d, m, c, cI = s.batch, COMPRESS_STEP_D, s.m, s.c, s.idx_dim
    ws = torch.empty(csa.workspace_size("csa_decode_compress", B, c, cI), dtype=torch.uint8, device="cuda")

    def call(x, pos):
        csa.csa_decode_compress(x, inp["W_kv"], inp["B_kv"], inp["W_idx"], inp["B_idx"], pos, inp["state_kv"],
                                inp["state_idx"], inp["kv_cache"], inp["idx_cache"], m, ws=ws)

    def step():
        call(inp["x"], inp["pos"])

    closing = int(((inp["pos"] + 1) % m == 0).sum())
    w_bytes = (4 * c + 4 * cI) * d * 2
    proj_bytes = B * 4 * (c + cI) * 4
    # weights, hidden states and fp32 projections (written, read back), the
    # ring rows stored, the 2m ring rows read and one entry written per block closed
    step_bytes = (w_bytes + B * d * 2 + 2 * proj_bytes + proj_bytes
                  + closing * (2 * m * 4 * (c + cI) * 4 + (c + cI) * 2))
    pinned = {k: inp[k].cpu().pin_memory() for k in ("x", "pos")}
    dev_in = {k: torch.empty_like(inp[k]) for k in pinned}
    flag_h = torch.empty((1,), dtype=inp["kv_cache"].dtype).pin_memory()

    def e2e_step():
        for k, v in pinned.items():
            dev_in[k].copy_(v, non_blocking=True)
        call(dev_in["x"], dev_in["pos"])
        flag_h.copy_(inp["kv_cache"].view(-1)[:1], non_blocking=True)

    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    kernels = {
        # two launches per step (KV: M = 4c, index keys: M = 4cI); work per step
        "project_tc": dict(bound="hbm", work=w_bytes + 2 * B * d * 2 + proj_bytes,
                           files=("gemm_tc.cu", "tc.cuh", "common.cuh")),
        "csa_compress_step": dict(bound="hbm", work=2 * proj_bytes, files=("compress.cu",)),
    }
    d2h = flag_h.numel() * flag_h.element_size()
    # pipelined: the step's result read back is the same cache element
    flag_d = inp["kv_cache"].view(-1)[:1]
    pipe = dict(pinned=pinned, out=flag_d, outs=[flag_d, flag_d], run=lambda dd, o: call(dd["x"], dd["pos"]))
    return dict(step=step, e2e_step=e2e_step, pipe=pipe, units=B, unit="tokens/s", h2d=h2d, d2h=d2h,
                kernels=kernels, step_bytes=step_bytes,
                config=dict(workload=COMPRESS_STEP_NAME, batch=B, d=d, m=m, head_dim=c, index_dim=cI,
                            positions=f"U[{s.ctx_lo},{s.ctx_hi}]", blocks_closed_per_step=closing,
                            l2="flushed before every timed step (256 MiB write + 256 MiB read)"),
                inputs=inp)


COMPRESS_STEP_NAME = f"csa_decode_compress_flash_b64_d{COMPRESS_STEP_D}_m4"


def dataclass_seed(s, rank):
    import dataclasses
    return dataclasses.replace(s, seed=s.seed + 1000 * rank) if rank else s


def hca_decode_workload(rank):
    import compressed_sparse_attention_14_b200 as csa
    s = dataclass_seed(synth.HCA, rank)
    inp = synth.hca_decode_inputs(s, device="cuda")
    B = s.batch
    out = torch.empty_like(inp["q"])
    lse = torch.empty((B, s.heads), dtype=torch.float32, device="cuda")
    ws = torch.empty(csa.workspace_size("hca_decode", B, s.n_max, s.heads, s.c, csa.CSA_BF16), dtype=torch.uint8,
                     device="cuda")

    def step():
        csa.hca_decode(inp["q"], inp["kv_cache"], inp["ctx_len"], s.mp, out=out, lse=lse, ws=ws)

    pinned = {k: inp[k].cpu().pin_memory() for k in ("q", "ctx_len")}
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dev_in = {k: torch.empty_like(inp[k]) for k in pinned}

    def e2e_step():
        for k, v in pinned.items():
            dev_in[k].copy_(v, non_blocking=True)
        csa.hca_decode(dev_in["q"], inp["kv_cache"], dev_in["ctx_len"], s.mp, out=out, lse=lse, ws=ws)
        out_h.copy_(out, non_blocking=True)

    kv_bytes = B * s.n_max * s.c * 2.0
    step_bytes = kv_bytes + 2 * B * s.heads * s.c * 2
    pipe = dict(pinned=pinned, out=out,
                run=lambda d, o: csa.hca_decode(d["q"], inp["kv_cache"], d["ctx_len"], s.mp, out=o, lse=lse, ws=ws))
    kernels = {"mqa_tc": dict(bound="hbm", work=kv_bytes + B * s.heads * s.c * 2,
                              files=("mqa_tc.cu", "tc.cuh", "common.cuh")),
               "mqa_combine": dict(bound="hbm", work=2 * B * s.heads * s.c * 2, files=("mqa.cu",))}
    return dict(step=step, e2e_step=e2e_step, pipe=pipe, units=B, unit="queries/s",
                h2d=sum(v.numel() * v.element_size() for v in pinned.values()),
                d2h=out_h.numel() * out_h.element_size(), kernels=kernels, step_bytes=step_bytes,
                config=dict(workload=s.name.split("_plus")[0], batch=B, ctx_len=s.ctx, mp=s.mp, entries=s.n_max,
                            head_dim=s.c, heads=s.heads, l2="flushed before every timed step (256 MiB write + 256 MiB read)"))


def hca_compress_workload(rank):
    import compressed_sparse_attention_14_b200 as csa
    s = dataclass_seed(synth.HCA, rank)
    inp = synth.hca_compress_inputs(s, device="cuda")
    n, d = inp["x"].shape
    out = torch.empty((n // s.mp, s.c), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(csa.workspace_size("hca_compress_from_hidden", n, d, s.c, s.mp, csa.CSA_BF16),
                     dtype=torch.uint8, device="cuda")

    def step():
        csa.hca_compress_from_hidden(inp["x"], inp["W"], inp["bias"], s.mp, out=out, ws=ws)

    x_h = inp["x"].cpu().pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    x_d = torch.empty_like(inp["x"])

    def e2e_step():
        x_d.copy_(x_h, non_blocking=True)
        csa.hca_compress_from_hidden(x_d, inp["W"], inp["bias"], s.mp, out=out, ws=ws)
        out_h.copy_(out, non_blocking=True)

    flops = 2.0 * n * d * 2 * s.c
    kernels = {"project_tc": dict(bound="tensor", work=flops, files=("gemm_tc.cu", "tc.cuh", "common.cuh")),
               "hca_compress": dict(bound="hbm", work=n * 2 * s.c * 4 + (n // s.mp) * s.c * 2,
                                    files=("compress.cu", "common.cuh"))}
    return dict(step=step, e2e_step=e2e_step, units=n, unit="tokens/s", h2d=x_h.numel() * 2,
                d2h=out_h.numel() * 2, kernels=kernels, step_bytes=None,
                config=dict(workload=f"hca_compress_chunk{n}_d{d}", tokens=n, d=d, mp=s.mp, head_dim=s.c,
                            l2="inputs larger than L2 and flushed before every timed step"))


def prefill_workload(rank, tokens=None):
    import compressed_sparse_attention_14_b200 as csa
    s = dataclass_seed(synth.PREFILL, rank)
    if tokens is None:
        inp = synth.prefill_inputs(s, device="cuda")
    else:
        # the last `tokens` tokens of the chunk: same positions and context
        # (a small profiling case)
        inp = synth.prefill_inputs(s, device="cuda", n=tokens, start=s.start + s.n - tokens)
    n = inp["n"]
    Nmax = inp["kv_cache"].shape[0]
    out = torch.empty_like(inp["q"])
    ws = torch.empty(csa.workspace_size("csa_prefill", n, Nmax, s.d, s.m, s.c, s.idx_dim, s.heads, s.idx_heads,
                                        s.k, csa.CSA_BF16), dtype=torch.uint8, device="cuda")

    def step():
        csa.csa_prefill(inp["x"], inp["x_left"], inp["W_kv"], inp["B_kv"], inp["W_idx"], inp["B_idx"], inp["start"],
                        inp["kv_cache"], inp["idx_cache"], inp["qI"], inp["w"], inp["q"], s.k, m=s.m, out=out, ws=ws)

    pos = torch.arange(inp["start"], inp["start"] + n, dtype=torch.float64)
    pairs = float(torch.floor(pos / s.m).sum())
    idx_flops = 2.0 * pairs * s.idx_heads * s.idx_dim
    names = ("x", "qI", "w", "q")
    pinned = {k: inp[k].cpu().pin_memory() for k in names}
    dev_in = {k: torch.empty_like(inp[k]) for k in names}
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def e2e_step():
        for k, v in pinned.items():
            dev_in[k].copy_(v, non_blocking=True)
        csa.csa_prefill(dev_in["x"], inp["x_left"], inp["W_kv"], inp["B_kv"], inp["W_idx"], inp["B_idx"],
                        inp["start"], inp["kv_cache"], inp["idx_cache"], dev_in["qI"], dev_in["w"], dev_in["q"], s.k,
                        m=s.m, out=out, ws=ws)
        out_h.copy_(out, non_blocking=True)

    # the same chunk as a serving loop streams it: 8 sub-chunks (whole blocks
    # of m tokens; chunked prefill equals the one-chunk call), sub-chunk j+1's
    # inputs copied in on one stream and sub-chunk j-1's output copied out on
    # another while sub-chunk j computes; two device input sets. A sub-chunk
    # after the first takes the m hidden rows before it as its left context
    # (copied with its inputs: m * d * 2 bytes more per sub-chunk).
    n_sub = 8 if n % (8 * s.m) == 0 else 1
    sub = n // n_sub
    ws_sub = torch.empty(csa.workspace_size("csa_prefill", sub, Nmax, s.d, s.m, s.c, s.idx_dim, s.heads, s.idx_heads,
                                            s.k, csa.CSA_BF16), dtype=torch.uint8, device="cuda")
    sets = [{k: torch.empty((sub,) + tuple(inp[k].shape[1:]), dtype=inp[k].dtype, device="cuda") for k in names}
            for _ in range(2)]
    lefts = [torch.empty((s.m, s.d), dtype=inp["x"].dtype, device="cuda") for _ in range(2)]

    def pipelined_ms(steps):
        ms = torch.cuda.current_stream()
        hs, ds = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]

        def h2d(j, i):                 # sub-chunk j into set j % 2 (i: its index in the whole run)
            b = j % 2
            with torch.cuda.stream(hs):
                if i >= 2:
                    hs.wait_event(ev_comp[b])
                for k in names:
                    sets[b][k].copy_(pinned[k][j * sub:(j + 1) * sub], non_blocking=True)
                if j > 0:
                    lefts[b].copy_(pinned["x"][j * sub - s.m:j * sub], non_blocking=True)
                ev_in[b].record(hs)

        def run(nsteps):
            total = nsteps * n_sub
            h2d(0, 0)
            for i in range(total):
                j, b = i % n_sub, i % 2
                ms.wait_event(ev_in[b])
                d = sets[b]
                o = out[j * sub:(j + 1) * sub]
                csa.csa_prefill(d["x"], inp["x_left"] if j == 0 else lefts[b], inp["W_kv"], inp["B_kv"],
                                inp["W_idx"], inp["B_idx"], inp["start"] + j * sub, inp["kv_cache"],
                                inp["idx_cache"], d["qI"], d["w"], d["q"], s.k, m=s.m, out=o, ws=ws_sub)
                ev_comp[b].record(ms)
                if i + 1 < total:
                    h2d((i + 1) % n_sub, i + 1)
                with torch.cuda.stream(ds):
                    ds.wait_event(ev_comp[b])
                    out_h[j * sub:(j + 1) * sub].copy_(o, non_blocking=True)
            ms.wait_stream(hs)
            ms.wait_stream(ds)

        run(1)
        torch.cuda.synchronize()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(ms)
        hs.wait_event(a)
        ds.wait_event(a)
        run(steps)
        z.record(ms)
        torch.cuda.synchronize()
        return a.elapsed_time(z) / steps

    mqa_flops = 4.0 * n * s.heads * s.k * s.c
    proj_flops = 2.0 * (n + s.m) * s.d * 4 * (s.c + s.idx_dim)
    kernels = {"index_scores_tc": dict(bound="tensor", work=idx_flops, files=("indexer_tc.cu", "tc.cuh", "common.cuh")),
               "index_topk_filter_tc": dict(bound="tensor", work=idx_flops,
                                            files=("indexer_tc.cu", "tc.cuh", "common.cuh")),
               "mqa_tc": dict(bound="tensor", work=mqa_flops, files=("mqa_tc.cu", "tc.cuh", "common.cuh")),
               "project_tc": dict(bound="tensor", work=proj_flops, files=("gemm_tc.cu", "tc.cuh", "common.cuh"))}
    return dict(step=step, e2e_step=e2e_step, units=n, unit="tokens/s",
                h2d=sum(v.numel() * v.element_size() for v in pinned.values()), d2h=out_h.numel() * 2,
                e2e_pipelined=pipelined_ms if n_sub > 1 else None,
                e2e_pipelined_mode=(f"pipelined in {n_sub} sub-chunks of {sub} tokens: sub-chunk j+1's inputs copied "
                                    f"in on one copy stream and sub-chunk j-1's output copied out on another while "
                                    f"sub-chunk j computes (each later sub-chunk also copies the {s.m} hidden rows "
                                    f"before it, {(n_sub - 1) * s.m * s.d * 2} bytes per step)"),
                kernels=kernels, step_bytes=None,
                config=dict(workload=s.name, tokens=n, start=inp["start"], d=s.d, m=s.m, head_dim=s.c,
                            heads=s.heads, index_heads=s.idx_heads, index_dim=s.idx_dim, topk=s.k,
                            causal_pairs=int(pairs), l2="inputs larger than L2"))


WORKLOADS = {
    "flash_decode": lambda r, b=None: decode_workload(synth.FLASH_DECODE, r, b),
    "pro_decode": lambda r, b=None: decode_workload(synth.PRO_DECODE, r, b),
    "flash_decode_fp8": lambda r, b=None: decode_workload(synth.FLASH_DECODE, r, b, fp8=True),
    "pro_decode_fp8": lambda r, b=None: decode_workload(synth.PRO_DECODE, r, b, fp8=True),
    "flash_decode_fp8kv": lambda r, b=None: decode_workload(synth.FLASH_DECODE, r, b, fp8kv=True),
    "hca_decode": lambda r, b=None: hca_decode_workload(r),
    "hca_compress": lambda r, b=None: hca_compress_workload(r),
    "prefill": lambda r, b=None: prefill_workload(r, b),
    "flash_attend_decode": lambda r, b=None: attend_decode_workload(synth.FLASH_DECODE, r, b),
    "flash_decode_compress": lambda r, b=None: decode_compress_workload(r, b),
}


# ----------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline object)
# ----------------------------------------------------------------------------

def oracle_decode_sample(shape, n_queries: int, seed_rank: int = 0, fp8=False):
    """Time the oracle (indexer + top-k + sparse MQA, fp64; fp8 True: the
    indexer on e4m3-quantized q^I and keys; fp8 "kv": the attention over the
    selected entries in FP8 storage, quantized and dequantized per selected
    row) on the first n_queries of the decode batch. Returns (seconds,
    queries)."""
    import oracle
    s = dataclass_seed(shape, seed_rank)
    inp = synth.decode_inputs(s, device="cpu", batch=n_queries)
    t0 = time.perf_counter()
    if fp8 is True:
        S = oracle.index_scores_fp8(inp["qI"], inp["w"], inp["idx_cache"], inp["ctx_len"], s.m,
                                    seq=torch.arange(n_queries))
        idx = oracle.topk(S, (inp["ctx_len"].numpy() // s.m).astype("int32"), s.k)
    else:
        idx, _ = oracle.index_topk(inp["qI"], inp["w"], inp["idx_cache"], inp["ctx_len"], s.m, s.k,
                                   seq=torch.arange(n_queries))
    if fp8 == "kv":
        rows = np.stack([inp["kv_cache"][t].double().numpy()[np.maximum(idx[t], 0)] for t in range(n_queries)])
        kv_sel = oracle.dequantize_kv_fp8(*oracle.quantize_kv_fp8(rows, ATTEND_ROPE))
        sel = np.where(idx >= 0, np.arange(idx.shape[1])[None, :], -1).astype("int32")
        oracle.sparse_mqa(inp["q"], kv_sel, sel, 1 / math.sqrt(s.c), seq=np.arange(n_queries))
    else:
        oracle.sparse_mqa(inp["q"], inp["kv_cache"], idx, 1 / math.sqrt(s.c), seq=torch.arange(n_queries))
    return time.perf_counter() - t0, n_queries


def oracle_attend_sample(shape, n_queries: int, seed_rank: int = 0):
    """Time the oracle's complete decode step (query norm + rotary, indexer,
    top-k, window joined in one softmax with the sink, back-rotation) on the
    first n_queries of the batch. Returns (seconds, queries)."""
    import oracle
    s = dataclass_seed(shape, seed_rank)
    inp = synth.attend_decode_inputs(s, device="cpu", batch=n_queries, n_win=ATTEND_WINDOW)
    t0 = time.perf_counter()
    oracle.attend_decode(inp["qI"], inp["w"], inp["idx_cache"], inp["q"], inp["kv_cache"], inp["ctx_len"], s.m, s.k,
                         ATTEND_WINDOW, inp["ring_len"], 1 / math.sqrt(s.c), q_gamma=inp["q_gamma"],
                         rope_dims=ATTEND_ROPE, sink=inp["sink"])
    return time.perf_counter() - t0, n_queries


def oracle_decode_compress_sample(n_tokens: int):
    """The oracle's decode-time compression work for n_tokens new tokens: the
    projections of their hidden states into both streams (plain C loops) and
    the compression of one block per m tokens. Returns (seconds, tokens)."""
    import oracle
    s = synth.FLASH_DECODE
    inp = synth.decode_compress_inputs(dataclass_seed(s, 0), COMPRESS_STEP_D, device="cpu", batch=n_tokens,
                                       caches=False)
    n = n_tokens - n_tokens % s.m
    t0 = time.perf_counter()
    pk = oracle.project_loops(inp["x"], inp["W_kv"])
    pi = oracle.project_loops(inp["x"], inp["W_idx"])
    if n:
        oracle.csa_compress(pk[:n], inp["B_kv"], s.m)
        oracle.csa_compress(pi[:n], inp["B_idx"], s.m)
    return time.perf_counter() - t0, n_tokens


def oracle_hca_sample(n_queries: int):
    import oracle
    s = synth.HCA
    inp = synth.hca_decode_inputs(s, batch=n_queries)
    t0 = time.perf_counter()
    oracle.dense_mqa(inp["q"], inp["kv_cache"], inp["ctx_len"], s.mp, 1 / math.sqrt(s.c), seq=torch.arange(n_queries))
    return time.perf_counter() - t0, n_queries


def oracle_hca_compress_sample(n_blocks: int):
    import oracle
    s = synth.HCA
    inp = synth.hca_compress_inputs(s, chunk=n_blocks * s.mp)
    t0 = time.perf_counter()
    oracle.hca_compress(oracle.project_loops(inp["x"], inp["W"]), inp["bias"], s.mp)
    return time.perf_counter() - t0, n_blocks * s.mp


def oracle_prefill_sample(n_tokens: int):
    """Indexer + top-k + MQA of the last n_tokens of the chunk against a cache
    of the chunk's full size (the dominant per-token work; the projection and
    compression of those tokens' blocks are included)."""
    import oracle
    s = synth.PREFILL
    m = s.m
    Nmax = (s.start + s.n) // m
    kv = synth.normal((Nmax, s.c), s.seed, "oracle_kv", dtype=torch.bfloat16)
    ik = synth.normal((Nmax, s.idx_dim), s.seed, "oracle_ik", dtype=torch.bfloat16)
    q = synth.normal((n_tokens, s.heads, s.c), s.seed, "q")
    qI = synth.normal((n_tokens, s.idx_heads, s.idx_dim), s.seed, "qI")
    w = synth.head_weights(n_tokens, s.idx_heads, s.seed)
    x = synth.normal((n_tokens, s.d), s.seed, "x")
    Wkv = synth.normal((4 * s.c, s.d), s.seed, "W_kv", std=1 / math.sqrt(s.d))
    Bkv = synth.normal((2 * m, s.c), s.seed, "B_kv", dtype=torch.float32)
    pos = torch.arange(s.start + s.n - n_tokens, s.start + s.n, dtype=torch.int32)
    t0 = time.perf_counter()
    oracle.csa_compress(oracle.project_loops(x, Wkv), Bkv, m)
    idx, _ = oracle.index_topk(qI, w, ik, pos, m, s.k)
    oracle.sparse_mqa(q, kv, idx, 1 / math.sqrt(s.c))
    return time.perf_counter() - t0, n_tokens


def oracle_measure(workload: str, budget_s: float = 15.0):
    """Grow the sample until it takes about budget_s seconds; return
    (units per second, description, units)."""
    threads = cpu_oracle_threads()
    if workload in DECODE_SHAPES:
        shape, fp8 = DECODE_SHAPES[workload]
        n = max(1, threads // 2)
        while True:
            sec, units = oracle_decode_sample(shape, min(n, shape.batch), fp8=fp8)
            if sec >= budget_s / 3 or n >= shape.batch:
                break
            n *= 2
        desc = (f"first {units} of the {shape.batch} decode queries (indexer{' on e4m3 operands' if fp8 is True else ''} "
                f"+ top-k + sparse MQA{' on FP8-stored entries' if fp8 == 'kv' else ''}, fp64)")
    elif workload == "flash_attend_decode":
        shape = synth.FLASH_DECODE
        n = max(1, threads // 2)
        while True:
            sec, units = oracle_attend_sample(shape, min(n, shape.batch))
            if sec >= budget_s / 3 or n >= shape.batch:
                break
            n *= 2
        desc = (f"first {units} of the {shape.batch} decode queries (query norm + rotary, indexer, top-k, window "
                f"+ selection MQA with sink, back-rotation; fp64)")
    elif workload == "flash_decode_compress":
        n = 4
        while True:
            sec, units = oracle_decode_compress_sample(n)
            if sec >= budget_s / 3 or n >= 1024:
                break
            n *= 2
        desc = (f"{units} new tokens (projection of their hidden states into both CSA streams, compression of one "
                f"block per {synth.FLASH_DECODE.m} tokens; fp64)")
    elif workload == "hca_decode":
        n = max(1, threads // 4)
        while True:
            sec, units = oracle_hca_sample(min(n, synth.HCA.batch))
            if sec >= budget_s / 3 or n >= synth.HCA.batch:
                break
            n *= 2
        desc = f"first {units} of the {synth.HCA.batch} HCA decode queries (dense MQA, fp64)"
    elif workload == "hca_compress":
        n = 2
        while True:
            sec, units = oracle_hca_compress_sample(n)
            if sec >= budget_s / 3 or n >= 1024:
                break
            n *= 2
        desc = f"{units} tokens ({units // synth.HCA.mp} blocks) of the compressor chunk (projection + compression, fp64)"
    else:
        n = max(1, threads // 2)
        while True:
            sec, units = oracle_prefill_sample(n)
            if sec >= budget_s / 3 or n >= 4096:
                break
            n *= 2
        desc = (f"last {units} tokens of the prefill chunk (projection + compression of their blocks, indexer over "
                f"~65K entries, top-k, sparse MQA; fp64)")
    return units / sec, desc, units, sec


def cpu_baseline_for(workload: str, unit: str) -> dict:
    """The oracle timed on the host at all its threads (the reported value)
    and on one thread (single_core), each on a bounded sample."""
    import oracle
    threads = cpu_oracle_threads()
    cps, desc, _, _ = oracle_measure(workload)
    out = {"value": cps, "unit": unit, "cores": threads, "kind": "oracle", "sample": desc}
    oracle.set_num_threads(1)
    try:
        cps1, desc1, _, _ = oracle_measure(workload, budget_s=6.0)
    finally:
        oracle.set_num_threads(threads)
    out["single_core"] = {"value": cps1, "unit": unit, "cores": 1, "sample": desc1}
    return out


# ----------------------------------------------------------------------------
# main
# ----------------------------------------------------------------------------

def run_reference(args, rank, world):
    if rank != 0:
        dist_done(world)
        return
    threads = cpu_oracle_threads()
    per_step, desc, units, _ = oracle_measure(args.workload, budget_s=6.0)
    # each step: a sample of about the size measured above
    times = []
    for i in range(args.warmup + args.steps):
        if args.workload in DECODE_SHAPES:
            shape, fp8 = DECODE_SHAPES[args.workload]
            sec, u = oracle_decode_sample(shape, units, fp8=fp8)
        elif args.workload == "flash_attend_decode":
            sec, u = oracle_attend_sample(synth.FLASH_DECODE, units)
        elif args.workload == "flash_decode_compress":
            sec, u = oracle_decode_compress_sample(units)
        elif args.workload == "hca_decode":
            sec, u = oracle_hca_sample(units)
        elif args.workload == "hca_compress":
            sec, u = oracle_hca_compress_sample(units // synth.HCA.mp)
        else:
            sec, u = oracle_prefill_sample(units)
        if i >= args.warmup:
            times.append(sec)
    total = sum(times)
    value = units * len(times) / total
    wl = WORKLOADS_CONFIG_NAME.get(args.workload, args.workload)
    unit = "tokens/s" if args.workload in ("hca_compress", "prefill", "flash_decode_compress") else "queries/s"
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": {"workload": wl, "sample_per_step": desc},
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    dist_done(world)


DECODE_SHAPES = {"flash_decode": (synth.FLASH_DECODE, False), "pro_decode": (synth.PRO_DECODE, False),
                 "flash_decode_fp8": (synth.FLASH_DECODE, True), "pro_decode_fp8": (synth.PRO_DECODE, True),
                 "flash_decode_fp8kv": (synth.FLASH_DECODE, "kv")}

WORKLOADS_CONFIG_NAME = {
    "flash_decode_fp8": synth.FLASH_DECODE.name + "_fp8_indexer",
    "flash_decode_fp8kv": synth.FLASH_DECODE.name + "_fp8_kv",
    "pro_decode_fp8": synth.PRO_DECODE.name + "_fp8_indexer",
    "flash_decode": synth.FLASH_DECODE.name,
    "pro_decode": synth.PRO_DECODE.name,
    "hca_decode": synth.HCA.name.split("_plus")[0],
    "hca_compress": "hca_compress_chunk131072_d4096",
    "prefill": synth.PREFILL.name,
    "flash_attend_decode": ATTEND_NAME,
    "flash_decode_compress": COMPRESS_STEP_NAME,
}


def pipelined_e2e_ms(pipe, steps: int, graphs: bool = False) -> float:
    """Device time per step of `steps` steps run through the public call from
    pinned host buffers, as a serving loop runs them: the inputs of step i+1
    go host -> device on one copy stream while step i computes on the current
    stream, and step i's output goes device -> host on a second copy stream
    once it is done (PCIe carries both directions at once, on separate copy
    engines). Two device input sets and outputs: step i+2 overwrites step i's
    inputs only after step i has computed, and its output only after that
    output has been copied out. graphs: each buffer set's library call is
    captured once in a CUDA graph and replayed every step (one host launch
    instead of the call's argument checks and kernel launches), as decode
    serving loops do; the copies stay per step."""
    pinned, run, out0 = pipe["pinned"], pipe["run"], pipe["out"]
    ms = torch.cuda.current_stream()
    hs, ds = torch.cuda.Stream(), torch.cuda.Stream()
    # a step's inputs sit back to back in one pinned staging buffer (as a
    # serving loop's batcher would write them) and cross PCIe as one copy;
    # each device input set is a view of one device buffer of the same layout
    offs, nbytes = {}, 0
    for k, v in pinned.items():
        offs[k] = nbytes
        nbytes += (v.numel() * v.element_size() + 255) // 256 * 256
    stage = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    for k, v in pinned.items():
        stage[offs[k]:offs[k] + v.numel() * v.element_size()].copy_(v.reshape(-1).view(torch.uint8))
    dev_all = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
    dev = [{k: dev_all[b][offs[k]:offs[k] + v.numel() * v.element_size()].view(v.dtype).view(v.shape)
            for k, v in pinned.items()} for b in range(2)]
    outs = pipe.get("outs") or [out0, torch.empty_like(out0)]
    out_h = [torch.empty(out0.shape, dtype=out0.dtype).pin_memory() for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    calls = [lambda b=b: run(dev[b], outs[b]) for b in range(2)]
    if graphs:
        for c in calls:            # one-time library set-up happens outside the capture
            c()
        torch.cuda.synchronize()
        gs = []
        for c in calls:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                c()
            gs.append(g)
        calls = [g.replay for g in gs]

    def h2d(i):
        b = i % 2
        with torch.cuda.stream(hs):
            if i >= 2:
                hs.wait_event(ev_comp[b])          # step i-2 no longer reads this buffer
            dev_all[b].copy_(stage, non_blocking=True)
            ev_in[b].record(hs)

    def loop(n):
        h2d(0)
        for i in range(n):
            b = i % 2
            ms.wait_event(ev_in[b])
            if i >= 2:
                ms.wait_event(ev_out[b])            # step i-2's output has left this buffer
            calls[b]()
            ev_comp[b].record(ms)
            if i + 1 < n:
                h2d(i + 1)
            with torch.cuda.stream(ds):
                ds.wait_event(ev_comp[b])
                out_h[b].copy_(outs[b], non_blocking=True)
                ev_out[b].record(ds)
        ms.wait_stream(hs)
        ms.wait_stream(ds)

    loop(4)                                          # warm-up
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    z = torch.cuda.Event(enable_timing=True)
    a.record(ms)
    hs.wait_event(a)
    ds.wait_event(a)
    loop(steps)
    z.record(ms)
    torch.cuda.synchronize()
    return a.elapsed_time(z) / steps


def measure(name, args, rank, world, local, steps, warmup, batch=None):
    """Time one workload: `warmup` untimed steps, then exactly `steps` steps
    bracketed by barrier + synchronize, each step on the device with CUDA
    events after an L2 flush; per-kernel times from a second, traced pass;
    clocks sampled over the timed region; the end-to-end rate through the
    public call with host buffers. Returns the workload's JSON fields."""
    import compressed_sparse_attention_14_b200 as csa
    wl = WORKLOADS[name](rank, batch)
    step, e2e_step = wl["step"], wl["e2e_step"]

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()

    timer = Timer()
    vis = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    clocks = ClockSampler(vis[local] if local < len(vis) else local)
    l0 = csa.launch_count()
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    for _ in range(steps):
        timer.step(step)
    torch.cuda.synchronize()
    barrier(world)
    t_wall = time.perf_counter() - t_wall0
    launches = csa.launch_count() - l0
    ms_total = timer.total_ms()
    # the timed region runs untraced (events between the library's kernels
    # would stop each from launching while the previous one drains); the
    # per-kernel times come from the same number of steps run again with the
    # library's kernel events on
    csa.trace_enable(True)
    ktimer = Timer()
    for _ in range(steps):
        ktimer.step(step)
    ktimer.total_ms()
    trace = csa.trace_read()
    csa.trace_enable(False)
    # the timed region can be shorter than the sampler's period: keep the GPU
    # on the same step (untimed) until the sampler has covered >= 1.5 s
    soak_steps = 0
    while time.perf_counter() - t_wall0 < 1.5:
        for _ in range(8):
            step()
        soak_steps += 8
        torch.cuda.synchronize()
    clk = clocks.stop()
    clk["window"] = f"timed region plus {soak_steps} untimed steps of the same work"
    ms_total_max = max_over_ranks(ms_total, world)
    ms_step = ms_total_max / steps

    # end to end: host buffers in, host result out, through the public call,
    # one step after the other with an L2 flush between steps (serial) ...
    e2e_timer = Timer()
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    for _ in range(steps):
        e2e_timer.step(e2e_step)
    e2e_serial_ms = max_over_ranks(e2e_timer.total_ms(), world) / steps
    # ... and, for the decode workloads, as a serving loop runs it: the next
    # step's inputs cross PCIe on a copy stream while the current step
    # computes (two input and output buffers), each step's result copied back
    # after it; no flush between steps (each step reads more than the L2 holds)
    e2e_ms, e2e_mode = e2e_serial_ms, "serial: copy in, call, copy out, per step"
    e2e_eager_ms = None
    if wl.get("e2e_pipelined"):
        p_ms = max_over_ranks(wl["e2e_pipelined"](steps), world)
        if p_ms < e2e_ms:
            e2e_ms, e2e_mode = p_ms, wl["e2e_pipelined_mode"]
    if wl.get("pipe"):
        e2e_eager_ms = max_over_ranks(pipelined_e2e_ms(wl["pipe"], steps), world)
        e2e_ms = e2e_eager_ms
        e2e_mode = ("pipelined: step i+1's host inputs copied in on one copy stream and step i-1's result "
                    "copied out on another while step i computes; every step's inputs and result cross PCIe "
                    "inside the timed region")
        # every rank takes the same collective step whether or not its capture worked
        g_err = None
        try:
            g_local = pipelined_e2e_ms(wl["pipe"], steps, graphs=True)
        except RuntimeError as ex:      # capture refused: keep the eager loop's number
            g_local, g_err = float("inf"), str(ex)[:80]
        g_ms = max_over_ranks(g_local, world)
        if g_ms < e2e_ms:
            e2e_ms = g_ms
            e2e_mode = e2e_mode + "; the library call of each step replayed from a CUDA graph captured once"
        elif g_err:
            e2e_mode = e2e_mode + f"; CUDA graph capture unavailable ({g_err})"

    units = wl["units"]
    peaks = measured_peaks()

    def roofline_of(kname):
        info = wl["kernels"][kname]
        k_ms, k_n = trace.get(kname, (float("nan"), 0))
        avg_s = k_ms / max(k_n, 1) / 1e3
        per_launch = info["work"] * steps / max(k_n, 1)   # the work is per step
        if info["bound"] == "hbm":
            achieved = per_launch / avg_s / 1e9
            r = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                 "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"] + " hbm_gbs (copy, burst)"}
        else:
            achieved = per_launch / avg_s / 1e12
            r = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                 "frac": achieved / peaks["bf16_tflops"], "peak_source": peaks["source"] + " bf16_tflops (burst)"}
        r["kernel"] = kname
        r["launches_per_step"] = k_n / steps
        r["ms_per_launch"] = avg_s * 1e3
        r["traffic"] = ncu_traffic(kname, name, info["files"])
        return r

    if "index_topk_filter_tc" in wl["kernels"]:
        wl["config"]["selection"] = ("top-k filter on the indexer epilogue, exact selection over its candidates"
                                     if "index_topk_filter_tc" in trace else "fp32 score block, then top-k")
    timed = [n for n in wl["kernels"] if n in trace]
    dom = max(timed, key=lambda n: trace[n][0]) if timed else next(iter(wl["kernels"]))
    others = {n: roofline_of(n) for n in timed if n != dom}
    out = {"value": job_rate(units, world, ms_step), "unit": wl["unit"], "ms_per_step": ms_step, "steps": steps,
           "warmup": warmup, "config": wl["config"], "roofline": roofline_of(dom),
           "kernels_ms_per_step": {k: v[0] / steps for k, v in sorted(trace.items())},
           "other_kernels_roofline": {n: {k: r[k] for k in ("bound", "achieved", "unit", "frac")}
                                      for n, r in others.items()},
           "e2e": {"value": job_rate(units, world, e2e_ms), "unit": wl["unit"], "h2d_bytes_per_step": wl["h2d"],
                   "d2h_bytes_per_step": wl["d2h"], "mode": e2e_mode,
                   "serial_value": job_rate(units, world, e2e_serial_ms),
                   **({"eager_pipelined_value": job_rate(units, world, e2e_eager_ms)} if e2e_eager_ms else {})},
           "gpu_launches": launches, "clocks": clk, "wall_s_timed": t_wall}
    if wl.get("step_bytes"):
        sb = wl["step_bytes"] / (ms_step / 1e3) / 1e9
        out["step_roofline"] = {"bound": "hbm", "achieved": sb, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                "frac": sb / peaks["hbm_gbs"]}
    del wl, step, e2e_step
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


# Measured after the default (Flash decode) line on one GPU and reported in
# its "extra_workloads": the other workloads the metric names (Pro-shaped
# 1M-context decode, the long prefill chunk, HCA decode, the HCA compressor).
# Each keeps its own step count, at most the headline's.
EXTRA_WORKLOADS = {"pro_decode": 20, "prefill": 5, "hca_decode": 20, "hca_compress": 10, "flash_decode_fp8": 20,
                   "flash_decode_fp8kv": 20, "pro_decode_fp8": 20, "flash_attend_decode": 20,
                   "flash_decode_compress": 20}


def run_ours(args, rank, world, local):
    import compressed_sparse_attention_14_b200 as csa
    if args.topk_filter:
        csa.debug_set(0, csa.CSA_DEBUG_TOPK_FILTER)
    m = measure(args.workload, args, rank, world, local, args.steps, args.warmup, args.batch)
    line = {"metric": METRIC, "value": m["value"], "unit": m["unit"], "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": m["config"],
            "roofline": m["roofline"]}
    for k in ("kernels_ms_per_step", "other_kernels_roofline", "e2e", "gpu_launches", "clocks", "wall_s_timed",
              "step_roofline"):
        if k in m:
            line[k] = m[k]
    line["kernel_times"] = ("per-kernel CUDA events on the library's stream over a second pass of the same steps "
                            "(the timed region itself runs without them)")
    if world == 1 and args.workload == "flash_decode" and args.batch is None and not args.no_extra:
        extra = {}
        for name, cap in EXTRA_WORKLOADS.items():
            extra[name] = measure(name, args, rank, world, local, min(args.steps, cap), min(args.warmup, 3))
        line["extra_workloads"] = extra
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_for(args.workload, line["unit"])
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist_done(world)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="flash_decode", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing (profiling runs)")
    ap.add_argument("--no-extra", action="store_true",
                    help="default workload only: skip the extra_workloads (Pro decode, prefill, HCA) measured after it")
    ap.add_argument("--topk-filter", action="store_true",
                    help="select through the top-k filter on the indexer epilogue instead of the fp32 score block "
                         "(comparison runs)")
    ap.add_argument("--batch", type=int, default=None,
                    help="decode workloads: only the first N queries; prefill: only the last N tokens of the "
                         "chunk, a multiple of m (small profiling cases)")
    args = ap.parse_args()
    rank, world, local = dist_init()
    if world != args.gpus and rank == 0:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
