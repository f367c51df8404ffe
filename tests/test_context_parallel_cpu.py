"""Context-parallel prefill (two-stage exchange: the last m rows of each rank
to the next, then an all-gather of the compressed entries with select-and-pad)
at world sizes 2 and 3 on CPU (gloo). The compute steps are the oracle's, so
the exchange is checked on its own: every rank's caches must hold the
entries of the whole chunk compressed in one piece, and every rank's outputs
must be the whole-chunk prefill's rows for its tokens, bit for bit."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

M, D, C, CI, H, HI, K = 4, 64, 32, 16, 2, 2, 8


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(start, total, seed=21):
    sys.path.insert(0, ROOT)
    import synth
    g = lambda shape, tag, **kw: synth.normal(shape, seed, tag, **kw)   # noqa: E731
    N = (start + total) // M
    inp = dict(
        x=g((total, D), "cp_x"), x_left=g((M, D), "cp_xl") if start > 0 else None,
        W_kv=g((4 * C, D), "cp_Wkv", std=D ** -0.5), B_kv=g((2 * M, C), "cp_Bkv", std=0.3, dtype=torch.float32),
        W_idx=g((4 * CI, D), "cp_Widx", std=D ** -0.5), B_idx=g((2 * M, CI), "cp_Bidx", std=0.3, dtype=torch.float32),
        qI=g((total, HI, CI), "cp_qI"), w=synth.head_weights(total, HI, seed), q=g((total, H, C), "cp_q"),
        sink=g((H,), "cp_sink", dtype=torch.float32),
        kv=torch.zeros((N, C), dtype=torch.bfloat16), ik=torch.zeros((N, CI), dtype=torch.bfloat16),
    )
    if start:
        inp["kv"][:start // M] = g((start // M, C), "cp_prefix_kv")
        inp["ik"][:start // M] = g((start // M, CI), "cp_prefix_ik")
    return inp


def _oracle_ops():
    import oracle
    from compressed_sparse_attention_14_b200.context_parallel import PrefillOps

    def compress(x, W, bias, m, x_left):
        proj = oracle.project_loops(x, W)
        left = None if x_left is None else oracle.project_loops(x_left, W)
        return torch.from_numpy(oracle.bf16_round(oracle.csa_compress(proj, bias, m, left=left))).to(torch.bfloat16)

    def prefill(x, x_left, W_kv, B_kv, W_idx, B_idx, start, kv_cache, idx_cache, qI, w, q, k, m, scale, sink):
        e0, n = start // m, x.shape[0]
        kv_cache[e0:e0 + n // m] = compress(x, W_kv, B_kv, m, x_left)
        idx_cache[e0:e0 + n // m] = compress(x, W_idx, B_idx, m, x_left)
        pos = np.arange(start, start + n, dtype=np.int32)
        idx, _ = oracle.index_topk(qI, w, idx_cache, pos, m, k)
        out, lse = oracle.sparse_mqa(q, kv_cache, idx, scale, sink=sink)
        return torch.from_numpy(out), torch.from_numpy(lse)

    return PrefillOps(compress_from_hidden=compress, prefill=prefill), prefill


def _rank_main(rank, world, port, out_dir, start, sizes):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    from compressed_sparse_attention_14_b200 import context_parallel as cp
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    inp = _inputs(start, sum(sizes))
    lo = sum(sizes[:rank])
    hi = lo + sizes[rank]
    ops, _ = _oracle_ops()
    res = {}
    try:
        out, lse = cp.csa_prefill_context_parallel(
            inp["x"][lo:hi].contiguous(), inp["x_left"] if rank == 0 else None, inp["W_kv"], inp["B_kv"],
            inp["W_idx"], inp["B_idx"], start, inp["kv"], inp["ik"], inp["qI"][lo:hi].contiguous(),
            inp["w"][lo:hi].contiguous(), inp["q"][lo:hi].contiguous(), K, m=M, scale=C ** -0.5, sink=inp["sink"],
            ops=ops)
        torch.save(dict(out=out, lse=lse, kv=inp["kv"], ik=inp["ik"]), os.path.join(out_dir, f"rank{rank}.pt"))
    except ValueError as e:
        res["raised"] = str(e)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)
    dist.destroy_process_group()


def _run(tmp_path, start, sizes):
    world = len(sizes)
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), start, sizes), nprocs=world, join=True,
                       start_method="spawn")
    return [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]


@pytest.mark.parametrize("start,sizes", [(0, [24, 24]), (32, [24, 16]), (32, [8, 16, 12])])
def test_context_parallel_prefill_equals_whole_chunk(tmp_path, start, sizes):
    flags = _run(tmp_path, start, sizes)
    assert not any(f.get("raised") for f in flags), flags
    sys.path.insert(0, ROOT)
    inp = _inputs(start, sum(sizes))
    _, prefill = _oracle_ops()
    ref_o, ref_l = prefill(inp["x"], inp["x_left"], inp["W_kv"], inp["B_kv"], inp["W_idx"], inp["B_idx"], start,
                           inp["kv"], inp["ik"], inp["qI"], inp["w"], inp["q"], K, M, C ** -0.5, inp["sink"])
    lo = 0
    for r, n in enumerate(sizes):
        got = torch.load(tmp_path / f"rank{r}.pt")
        # every rank's caches: the whole chunk's entries (and the untouched prefix)
        assert torch.equal(got["kv"], inp["kv"]) and torch.equal(got["ik"], inp["ik"]), f"rank {r} caches"
        assert torch.equal(got["out"], ref_o[lo:lo + n]), f"rank {r} outputs"
        assert torch.equal(got["lse"], ref_l[lo:lo + n]), f"rank {r} lse"
        lo += n


def test_bad_chunk_raises_on_every_rank(tmp_path):
    # rank 1's chunk is not a multiple of m: both ranks see it in the shape
    # exchange and raise before any data moves (no rank is left waiting)
    flags = _run(tmp_path, 0, [8, 6])
    assert all("multiple of m" in f.get("raised", "") for f in flags), flags


def test_chunk_layout():
    sys.path.insert(0, ROOT)
    from compressed_sparse_attention_14_b200.context_parallel import chunk_layout
    assert chunk_layout(32, [24, 16, 8], 4) == [(32, 8), (56, 14), (72, 18)]


def _subgroup_main(rank, world, port, out_dir, start, sizes):
    # ranks 1 and 2 form the context-parallel group; rank 0 only takes part in
    # creating it (every rank must call new_group)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    from compressed_sparse_attention_14_b200 import context_parallel as cp
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    group = dist.new_group([1, 2])
    if rank > 0:
        inp = _inputs(start, sum(sizes))
        r = rank - 1
        lo = sum(sizes[:r])
        hi = lo + sizes[r]
        ops, _ = _oracle_ops()
        out, lse = cp.csa_prefill_context_parallel(
            inp["x"][lo:hi].contiguous(), inp["x_left"] if r == 0 else None, inp["W_kv"], inp["B_kv"], inp["W_idx"],
            inp["B_idx"], start, inp["kv"], inp["ik"], inp["qI"][lo:hi].contiguous(), inp["w"][lo:hi].contiguous(),
            inp["q"][lo:hi].contiguous(), K, m=M, scale=C ** -0.5, sink=inp["sink"], group=group, ops=ops)
        torch.save(dict(out=out, lse=lse, kv=inp["kv"]), os.path.join(out_dir, f"rank{r}.pt"))
    dist.barrier()
    dist.destroy_process_group()


def test_context_parallel_on_a_subgroup(tmp_path):
    start, sizes = 32, [16, 24]
    mp.start_processes(_subgroup_main, args=(3, _free_port(), str(tmp_path), start, sizes), nprocs=3, join=True,
                       start_method="spawn")
    inp = _inputs(start, sum(sizes))
    _, prefill = _oracle_ops()
    ref_o, ref_l = prefill(inp["x"], inp["x_left"], inp["W_kv"], inp["B_kv"], inp["W_idx"], inp["B_idx"], start,
                           inp["kv"], inp["ik"], inp["qI"], inp["w"], inp["q"], K, M, C ** -0.5, inp["sink"])
    lo = 0
    for r, n in enumerate(sizes):
        got = torch.load(tmp_path / f"rank{r}.pt")
        assert torch.equal(got["kv"], inp["kv"]) and torch.equal(got["out"], ref_o[lo:lo + n])
        lo += n


def _absent_peer_main(rank, world, port, out_dir):
    # rank 1 leaves before the prefill; rank 0's first collective must end
    # with an error (peer gone or the short group timeout), not wait forever
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import time
    import torch.distributed as dist
    from compressed_sparse_attention_14_b200 import context_parallel as cp
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        os._exit(0)
    inp = _inputs(0, 16)
    ops, _ = _oracle_ops()
    t0 = time.time()
    res = {}
    try:
        cp.csa_prefill_context_parallel(inp["x"][:8].contiguous(), None, inp["W_kv"], inp["B_kv"], inp["W_idx"],
                                        inp["B_idx"], 0, inp["kv"], inp["ik"], inp["qI"][:8].contiguous(),
                                        inp["w"][:8].contiguous(), inp["q"][:8].contiguous(), K, m=M, ops=ops)
        res["raised"] = False
    except Exception as e:  # noqa: BLE001 - any error ends the wait; the test checks that one came
        res["raised"] = True
        res["error"] = type(e).__name__
    res["seconds"] = time.time() - t0
    with open(os.path.join(out_dir, "rank0.json"), "w") as f:
        json.dump(res, f)
    os._exit(0)


def test_absent_peer_ends_with_an_error(tmp_path):
    mp.start_processes(_absent_peer_main, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    res = json.load(open(tmp_path / "rank0.json"))
    assert res["raised"], res
    assert res["seconds"] < 60, res
