"""Context-parallel prefill [Walk §4.2; Notes §2.5] through the library's
CUDA kernels.

* World size 1 (NCCL, cuda:0): csa_prefill_context_parallel with its default
  compute steps (cuda_ops) equals csa_prefill on the same chunk, bit for bit.
* World sizes 2 and 3 (gloo ranks on the host, every rank computing on
  cuda:0 through the library: copy in, call, copy out): every rank's caches
  and outputs equal the whole-chunk csa_prefill's, bit for bit.

The ranks' kernels never wait on one another (the exchange is gloo on the
host), so several ranks may share one GPU."""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(start, total):
    sys.path.insert(0, ROOT)
    import synth
    s = synth.TINY
    inp = synth.prefill_inputs(s, n=total, start=start)
    inp["sink"] = synth.normal((s.heads,), 41, "cp_sink", dtype=torch.float32)
    return s, inp


def _whole_chunk(start, total):
    import compressed_sparse_attention_14_b200 as csa
    s, inp = _inputs(start, total)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, lse = csa.csa_prefill(d["x"], d["x_left"], d["W_kv"], d["B_kv"], d["W_idx"], d["B_idx"], start,
                               d["kv_cache"], d["idx_cache"], d["qI"], d["w"], d["q"], s.k, m=s.m, sink=d["sink"])
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu(), d["kv_cache"].cpu(), d["idx_cache"].cpu()


def _library_ops_on_cuda():
    """The library's entry points for host tensors: copy in, call, copy out."""
    import compressed_sparse_attention_14_b200 as csa
    from compressed_sparse_attention_14_b200.context_parallel import PrefillOps

    def g(t):
        return None if t is None else t.cuda()

    def compress(x, W, bias, m, x_left):
        return csa.csa_compress_from_hidden(g(x), g(W), g(bias), m, x_left=g(x_left)).cpu()

    def prefill(x, x_left, W_kv, B_kv, W_idx, B_idx, start, kv_cache, idx_cache, qI, w, q, k, m, scale, sink):
        kv, ik = g(kv_cache), g(idx_cache)
        out, lse = csa.csa_prefill(g(x), None, None, None, None, None, start, kv, ik, g(qI), g(w), g(q), k, m=m,
                                   scale=scale, sink=g(sink))
        kv_cache.copy_(kv.cpu())
        idx_cache.copy_(ik.cpu())
        return out.cpu(), lse.cpu()

    return PrefillOps(compress_from_hidden=compress, prefill=prefill)


def _rank_main(rank, world, port, out_dir, start, sizes):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from compressed_sparse_attention_14_b200 import context_parallel as cp
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    s, inp = _inputs(start, sum(sizes))
    lo = sum(sizes[:rank])
    hi = lo + sizes[rank]
    out, lse = cp.csa_prefill_context_parallel(
        inp["x"][lo:hi].contiguous(), inp["x_left"] if rank == 0 else None, inp["W_kv"], inp["B_kv"], inp["W_idx"],
        inp["B_idx"], start, inp["kv_cache"], inp["idx_cache"], inp["qI"][lo:hi].contiguous(),
        inp["w"][lo:hi].contiguous(), inp["q"][lo:hi].contiguous(), s.k, m=s.m, sink=inp["sink"],
        ops=_library_ops_on_cuda())
    torch.save(dict(out=out, lse=lse, kv=inp["kv_cache"], ik=inp["idx_cache"]), os.path.join(out_dir, f"rank{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("start,sizes", [(0, [512, 512]), (256, [384, 256, 128])])
def test_context_parallel_ranks_through_the_library_equal_whole_chunk(tmp_path, start, sizes):
    mp.start_processes(_rank_main, args=(len(sizes), _free_port(), str(tmp_path), start, sizes), nprocs=len(sizes),
                       join=True, start_method="spawn")
    ref_o, ref_l, ref_kv, ref_ik = _whole_chunk(start, sum(sizes))
    lo = 0
    for r, n in enumerate(sizes):
        got = torch.load(tmp_path / f"rank{r}.pt")
        assert torch.equal(got["kv"], ref_kv) and torch.equal(got["ik"], ref_ik), f"rank {r} caches"
        assert torch.equal(got["out"], ref_o[lo:lo + n]), f"rank {r} outputs"
        assert torch.equal(got["lse"], ref_l[lo:lo + n]), f"rank {r} lse"
        lo += n


def _single_main(rank, world, port, out_dir, start, total):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from compressed_sparse_attention_14_b200 import context_parallel as cp
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=120))
    s, inp = _inputs(start, total)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, lse = cp.csa_prefill_context_parallel(d["x"], d["x_left"], d["W_kv"], d["B_kv"], d["W_idx"], d["B_idx"],
                                               start, d["kv_cache"], d["idx_cache"], d["qI"], d["w"], d["q"], s.k,
                                               m=s.m, sink=d["sink"])
    torch.cuda.synchronize()
    torch.save(dict(out=out.cpu(), lse=lse.cpu(), kv=d["kv_cache"].cpu(), ik=d["idx_cache"].cpu()),
               os.path.join(out_dir, "rank0.pt"))
    dist.destroy_process_group()


@pytest.mark.parametrize("start", [0, 512])
def test_context_parallel_world_one_default_ops_equal_csa_prefill(tmp_path, start):
    total = 512
    mp.start_processes(_single_main, args=(1, _free_port(), str(tmp_path), start, total), nprocs=1, join=True,
                       start_method="spawn")
    ref_o, ref_l, ref_kv, ref_ik = _whole_chunk(start, total)
    got = torch.load(tmp_path / "rank0.pt")
    assert torch.equal(got["kv"], ref_kv) and torch.equal(got["ik"], ref_ik)
    assert torch.equal(got["out"], ref_o) and torch.equal(got["lse"], ref_l)
