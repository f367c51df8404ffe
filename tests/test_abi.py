"""Host-side checks of the C ABI (no GPU needed, no kernel is launched):
the library loads, exports every function include/csa.h declares, rejects
bad arguments before touching the device, and sizes its workspaces."""
import ctypes
import os
import re
import subprocess
import sys

import pytest
import torch

import compressed_sparse_attention_14_b200 as csa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b((?:csa|hca)_\w+)\s*\(", src, flags=re.M)))


def test_header_declarations_are_exported():
    names = _declared()
    assert len(names) >= 20
    lib = ctypes.CDLL(csa.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(csa.EXPORTED) == names


def test_abi_version():
    assert csa.abi_version() == 2


def _lib():
    return csa._lib


def test_invalid_arguments_are_rejected_on_the_host():
    L = _lib()
    fake = 0x10000  # 16-byte aligned, never dereferenced: checks fail first
    # n not a multiple of m
    assert L.csa_compress(fake, None, fake, 6, 8, 4, fake, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    assert b"multiple" in L.csa_last_error()
    # c not a multiple of 8
    assert L.csa_compress(fake, None, fake, 8, 12, 4, fake, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    # null required pointer
    assert L.csa_compress(None, None, fake, 8, 8, 4, fake, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    assert b"NULL" in L.csa_last_error()
    # misaligned pointer
    assert L.hca_compress(fake + 4, fake, 128, 8, 128, fake, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    assert b"aligned" in L.csa_last_error()
    # bad dtype
    assert L.hca_compress(fake, fake, 128, 8, 128, fake, 7, None) == csa.CSA_ERR_INVALID_ARG
    # k out of range
    assert L.csa_topk_from_scores(fake, 16, None, 1, 1, 16, 0, fake, None, None, 0, None) == csa.CSA_ERR_UNSUPPORTED
    assert L.csa_topk_from_scores(fake, 16, None, 1, 1, 16, 4096, fake, None, None, 0, None) == csa.CSA_ERR_UNSUPPORTED
    # attention shapes beyond the kernels
    assert L.csa_sparse_mqa(fake, fake, fake, None, 1, 1, 256, 128, 8, 4, 0.0, None, fake, None, None, 0,
                            csa.CSA_BF16, None) == csa.CSA_ERR_UNSUPPORTED
    assert L.csa_sparse_mqa(fake, fake, fake, None, 1, 1, 8, 1024, 8, 4, 0.0, None, fake, None, None, 0,
                            csa.CSA_BF16, None) == csa.CSA_ERR_UNSUPPORTED
    # identity query->sequence map needs one sequence per query
    assert L.csa_sparse_mqa(fake, fake, fake, None, 4, 2, 8, 128, 8, 4, 0.0, None, fake, None, None, 0,
                            csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    # bf16 indexer runs on tensor cores: cI must be a multiple of 64
    assert L.csa_index_scores(fake, fake, fake, fake, None, 2, 2, 4, 32, 16, 4, fake, csa.CSA_BF16,
                              None) == csa.CSA_ERR_UNSUPPORTED
    # more rows than one launch grid holds
    assert L.csa_topk_from_scores(fake, 16, None, 1, 70000, 16, 4, fake, None, None, 0, None) == csa.CSA_ERR_UNSUPPORTED
    assert b"65535" in L.csa_last_error()
    # the allocation-free indexer + top-k: more scores than its fixed array
    assert L.csa_index_topk_noalloc(fake, fake, fake, fake, None, 64, 64, 64, 128, 65537, 4, 16, fake, None,
                                    csa.CSA_BF16, None) == csa.CSA_ERR_UNSUPPORTED
    assert b"fixed" in L.csa_last_error()
    assert L.csa_index_topk_noalloc(fake, fake, fake, fake, None, 70000, 70000, 64, 128, 8, 4, 16, fake, None,
                                    csa.CSA_BF16, None) == csa.CSA_ERR_UNSUPPORTED
    assert L.csa_index_topk_noalloc(fake, fake, fake, fake + 4, None, 4, 4, 64, 128, 8, 4, 16, fake, None,
                                    csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    # missing / short workspace
    need = L.csa_decode_workspace_size(2, 1024, 8, 128, 4, 64, 16, csa.CSA_BF16)
    assert need > 0
    rc = L.csa_decode(fake, fake, fake, fake, fake, fake, 2, 1024, 4, 8, 128, 4, 64, 16, 0.0, None, fake, None,
                      None, None, 0, csa.CSA_BF16, None)
    assert rc == csa.CSA_ERR_WORKSPACE
    rc = L.csa_decode(fake, fake, fake, fake, fake, fake, 2, 1024, 4, 8, 128, 4, 64, 16, 0.0, None, fake, None,
                      None, fake * 16, need - 1, csa.CSA_BF16, None)
    assert rc == csa.CSA_ERR_WORKSPACE
    # prefill: start not a multiple of m, cache too small, missing left rows
    args = dict(n=8, Nmax=4, start=4)
    rc = L.csa_prefill(fake, fake, fake, fake, fake, fake, 2, 8, 64, 4, 128, 64, fake, fake, 16, None, None, fake, fake, fake,
                       8, 4, 4, 0.0, None, fake, None, None, None, 0, csa.CSA_BF16, None)
    assert rc == csa.CSA_ERR_INVALID_ARG
    rc = L.csa_prefill(fake, fake, fake, fake, fake, fake, 4, 8, 64, 4, 128, 64, fake, fake, 2, None, None, fake, fake, fake,
                       8, 4, 4, 0.0, None, fake, None, None, None, 0, csa.CSA_BF16, None)
    assert rc == csa.CSA_ERR_INVALID_ARG
    rc = L.csa_prefill(fake, None, fake, fake, fake, fake, 4, 8, 64, 4, 128, 64, fake, fake, 16, None, None, fake, fake, fake,
                       8, 4, 4, 0.0, None, fake, None, None, None, 0, csa.CSA_BF16, None)
    assert rc == csa.CSA_ERR_INVALID_ARG
    # FP8 indexer: cI must fill whole 128-byte rows; w and w_out go together
    assert L.csa_index_scores_fp8(fake, fake, fake, fake, fake, None, 2, 2, 4, 64, 16, 4, fake,
                                  None) == csa.CSA_ERR_UNSUPPORTED
    assert L.csa_quantize_e4m3(fake, 4, 12, fake, fake, None, None, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_quantize_e4m3(fake, 4, 16, fake, fake, fake, None, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_decode_fp8(fake, fake, fake, fake, fake, fake, fake, 2, 1024, 4, 8, 128, 4, 128, 16, 0.0, None, 2,
                            fake, None, None, fake * 16, 1 << 30, None) == csa.CSA_ERR_INVALID_ARG
    assert b"flags" in L.csa_last_error()
    assert L.csa_topk_from_scores_bf16(fake, 16, None, 1, 1, 16, 0, fake, None, None) == csa.CSA_ERR_UNSUPPORTED
    assert L.csa_debug_set(0, 8) == csa.CSA_ERR_INVALID_ARG
    # prefill with one state ring but not the other
    rc = L.csa_prefill(fake, None, fake, fake, fake, fake, 6, 9, 64, 4, 128, 64, fake, fake, 16, fake, None, fake,
                       fake, fake, 8, 4, 4, 0.0, None, fake, None, None, None, 0, csa.CSA_BF16, None)
    assert rc == csa.CSA_ERR_INVALID_ARG and b"together" in L.csa_last_error()
    # chunk compression: the cache must hold every block the chunk closes
    assert L.csa_compress_chunk(fake, fake, fake, 6, 11, 64, 4, fake, 3, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    assert L.hca_compress_chunk(fake, None, fake, 0, 8, 64, 4, fake, 2, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    assert L.hca_compress_chunk(fake, fake, fake, -1, 8, 64, 4, fake, 2, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    del args


def test_attention_completion_arguments_are_checked_on_the_host():
    L = _lib()
    fake = 0x10000
    F = ctypes.c_float
    # rotary width not a multiple of 8, wider than c, c not a multiple of 8
    assert L.csa_norm_rope(fake, fake, 64, 1, 128, None, F(1e-6), 12, F(1e4), None, 0, 1, 0, csa.CSA_BF16,
                           None) == csa.CSA_ERR_UNSUPPORTED
    assert L.csa_norm_rope(fake, fake, 64, 1, 128, None, F(1e-6), 136, F(1e4), None, 0, 1, 0, csa.CSA_BF16,
                           None) == csa.CSA_ERR_UNSUPPORTED
    assert L.csa_norm_rope(fake, fake, 64, 1, 100, None, F(1e-6), 8, F(1e4), None, 0, 1, 0, csa.CSA_BF16,
                           None) == csa.CSA_ERR_UNSUPPORTED
    # rows must split into whole position groups; base positive; eps >= 0
    assert L.csa_norm_rope(fake, fake, 65, 8, 128, None, F(1e-6), 64, F(1e4), fake, 0, 1, 0, csa.CSA_BF16,
                           None) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_norm_rope(fake, fake, 64, 8, 128, None, F(1e-6), 64, F(0.0), fake, 0, 1, 0, csa.CSA_BF16,
                           None) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_norm_rope(fake, fake, 64, 8, 128, None, F(-1.0), 64, F(1e4), fake, 0, 1, 0, csa.CSA_BF16,
                           None) == csa.CSA_ERR_INVALID_ARG
    # partial overlap of x and y (in place, y == x, is allowed)
    assert L.csa_norm_rope(fake, fake + 256, 64, 1, 128, None, F(1e-6), 64, F(1e4), None, 0, 1, 0, csa.CSA_BF16,
                           None) == csa.CSA_ERR_INVALID_ARG
    assert b"overlap" in L.csa_last_error()
    # the window must fit its ring; the list must not overwrite the selection
    assert L.csa_window_entries(fake, 16, fake, 0, 4, 128, 1000, 64, fake * 2, None) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_window_entries(fake, 16, fake, 0, 4, 8, 1000, 64, fake, None) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_window_entries(fake, 16, fake, 0, 4, 8, (1 << 31) - 10, 64, fake * 2, None) == csa.CSA_ERR_UNSUPPORTED
    # selection + window beyond the per-query entry limit; window longer than the ring
    assert L.csa_attend_decode(fake, fake, fake, fake, fake, fake, 2, 1024, 128, 128, 4, 8, 128, 4, 64, 2000,
                               F(0.0), None, F(1e-6), 64, F(1e4), None, fake, None, None, None, 0, csa.CSA_BF16,
                               None) == csa.CSA_ERR_UNSUPPORTED
    assert L.csa_attend_decode(fake, fake, fake, fake, fake, fake, 2, 1024, 64, 128, 4, 8, 128, 4, 64, 16,
                               F(0.0), None, F(1e-6), 64, F(1e4), None, fake, None, None, None, 0, csa.CSA_BF16,
                               None) == csa.CSA_ERR_INVALID_ARG
    # missing workspace
    need = L.csa_attend_decode_workspace_size(2, 1024, 128, 128, 8, 128, 4, 64, 16, csa.CSA_BF16)
    assert need > L.csa_decode_workspace_size(2, 1024, 8, 128, 4, 64, 16, csa.CSA_BF16)
    assert L.csa_attend_decode(fake, fake, fake, fake, fake, fake, 2, 1024, 128, 128, 4, 8, 128, 4, 64, 16,
                               F(0.0), None, F(1e-6), 64, F(1e4), None, fake, None, None, None, 0, csa.CSA_BF16,
                               None) == csa.CSA_ERR_WORKSPACE


def test_compress_step_arguments_are_checked_on_the_host():
    L = _lib()
    fake = 0x10000
    # compression rate outside the kernels' range, channels not a multiple of 8
    assert L.csa_compress_step(fake, fake, fake, fake, 4, 64, 0, 16, fake, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_compress_step(fake, fake, fake, fake, 4, 64, 65, 16, fake, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    assert L.hca_compress_step(fake, fake, fake, fake, 4, 60, 128, 16, fake, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    assert L.hca_compress_step(fake, fake, fake, fake, 4, 64, 2048, 16, fake, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    # the state ring is required; misaligned pointers are refused
    assert L.csa_compress_step(fake, None, fake, fake, 4, 64, 4, 16, fake, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    assert b"state" in L.csa_last_error()
    assert L.csa_compress_step(fake + 8, fake, fake, fake, 4, 64, 4, 16, fake, csa.CSA_BF16, None) == csa.CSA_ERR_INVALID_ARG
    # the fused step: workspace for both projections
    need = L.csa_decode_compress_workspace_size(64, 512, 128)
    assert need >= 64 * 4 * (512 + 128) * 4
    rc = L.csa_decode_compress(fake, fake, fake, fake, fake, fake, 64, 4096, 4, 512, 128, fake, fake, fake, fake,
                               32768, None, 0, csa.CSA_BF16, None)
    assert rc == csa.CSA_ERR_WORKSPACE


def test_cache_block_layout_is_the_lcm_block():
    # [Notes §2.6: one block covers lcm(m, m') raw tokens, i.e. lcm/m CSA
    # entries and lcm/m' HCA entries]; parts in the order KV, index keys, HCA
    for m, mp, c, cI in [(4, 128, 512, 128), (4, 6, 64, 32), (3, 5, 16, 8), (8, 8, 128, 64)]:
        lcm = next(L for L in range(max(m, mp), m * mp + 1) if L % m == 0 and L % mp == 0)   # brute force
        lay = csa.csa_cache_block_layout(m, mp, c, cI)
        assert (lay["csa_rows"], lay["hca_rows"]) == (lcm // m, lcm // mp)
        assert lay["kv_offset"] == 0
        assert lay["idx_offset"] == lcm // m * c * 2
        assert lay["hca_offset"] == lay["idx_offset"] + lcm // m * cI * 2
        assert lay["block_bytes"] == lay["hca_offset"] + lcm // mp * c * 2
        assert lay["block_bytes"] % 16 == 0
    assert csa.csa_cache_block_layout(4, 128, 512, 128, csa.CSA_FP32)["block_bytes"] == 4 * (32 * 512 + 32 * 128 + 512)
    L = _lib()
    out = [ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int64(0)]
    assert L.csa_cache_block_layout(0, 128, 512, 128, csa.CSA_BF16, *[ctypes.byref(o) for o in out], None, None,
                                    None) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_cache_block_layout(4, 128, 60, 128, csa.CSA_BF16, *[ctypes.byref(o) for o in out], None, None,
                                    None) == csa.CSA_ERR_INVALID_ARG


def test_blocked_calls_check_the_layout_on_the_host():
    L = _lib()
    fake = 0x10000
    bb = 41984   # lcm block of m = 4, m' = 128, c = 512, cI = 128 (bf16)

    def dec(rpb, block_bytes, Nmax=1024, dtype=csa.CSA_BF16, kv=fake):
        return L.csa_decode_blocked(fake, fake, fake, fake, kv, fake, 4, Nmax, 4, 64, 512, 64, 128, 512, 0.0, None,
                                    fake, None, None, rpb, block_bytes, None, 0, dtype, None)
    assert dec(0, bb) == csa.CSA_ERR_INVALID_ARG                 # no rows per block
    assert dec(32, bb + 8) == csa.CSA_ERR_INVALID_ARG            # block not a multiple of 16 bytes
    assert dec(32, 16 * 1024) == csa.CSA_ERR_INVALID_ARG         # too short for 32 rows of 512 bf16
    assert dec(32, bb, Nmax=1000) == csa.CSA_ERR_INVALID_ARG     # Nmax not a multiple of the block's rows
    assert dec(32, bb, kv=fake + 8) == csa.CSA_ERR_INVALID_ARG   # misaligned cache pointer
    assert dec(32, bb, dtype=csa.CSA_FP32) == csa.CSA_ERR_UNSUPPORTED
    assert dec(24, 24 * 1024 * 2, Nmax=960) == csa.CSA_ERR_UNSUPPORTED   # 24 does not divide the 128-key tile
    assert dec(32, bb) == csa.CSA_ERR_WORKSPACE                  # a consistent layout reaches the workspace check
    rc = L.hca_decode_blocked(fake, fake, fake, 4, 256, 128, 64, 512, 0.0, None, fake, None, 2, bb, None, 0,
                              csa.CSA_BF16, None)
    assert rc == csa.CSA_ERR_UNSUPPORTED                         # one HCA entry per block
    rc = L.csa_decode_compress_blocked(fake, fake, fake, fake, fake, fake, 4, 4096, 4, 512, 128, fake, fake, fake,
                                       fake, 1000, 32, bb, None, 0, csa.CSA_BF16, None)
    assert rc == csa.CSA_ERR_INVALID_ARG
    rc = L.hca_compress_step_blocked(fake, fake, fake, fake, 4, 512, 128, 256, fake, 1, bb + 4, csa.CSA_BF16, None)
    assert rc == csa.CSA_ERR_INVALID_ARG


def test_empty_inputs_are_no_ops():
    L = _lib()
    assert L.csa_compress(None, None, None, 0, 8, 4, None, csa.CSA_BF16, None) == csa.CSA_OK
    assert L.csa_topk_from_scores(None, 0, None, 1, 0, 0, 8, None, None, None, 0, None) == csa.CSA_OK
    assert L.csa_decode(None, None, None, None, None, None, 0, 16, 4, 8, 128, 4, 64, 16, 0.0, None, None, None,
                        None, None, 0, csa.CSA_BF16, None) == csa.CSA_OK
    F = ctypes.c_float
    assert L.csa_norm_rope(None, None, 0, 1, 128, None, F(1e-6), 64, F(1e4), None, 0, 1, 0, csa.CSA_BF16,
                           None) == csa.CSA_OK
    assert L.csa_window_entries(None, 0, None, 0, 0, 128, 0, 128, None, None) == csa.CSA_OK
    assert L.csa_compress_step(None, None, None, None, 0, 64, 4, 16, None, csa.CSA_BF16, None) == csa.CSA_OK
    assert L.csa_decode_compress(None, None, None, None, None, None, 0, 256, 4, 64, 64, None, None, None, None, 16,
                                 None, 0, csa.CSA_BF16, None) == csa.CSA_OK
    assert L.csa_attend_decode(None, None, None, None, None, None, 0, 16, 128, 128, 4, 8, 128, 4, 64, 16, F(0.0),
                               None, F(1e-6), 64, F(1e4), None, None, None, None, None, 0, csa.CSA_BF16,
                               None) == csa.CSA_OK


def test_workspace_sizes():
    L = _lib()
    # the selection keeps its scratch in shared memory at every row length
    assert L.csa_topk_workspace_size(64, 16384, 512) == 0
    assert L.csa_topk_workspace_size(32, 262144, 1024) == 0
    # bf16 MQA: a single split, or two merged on chip, need no workspace;
    # more splits keep fp32 partials (O, max, sum) per split for the combine
    assert L.csa_sparse_mqa_workspace_size(4096, 64, 512, 512, csa.CSA_BF16) == 0      # 1 split
    assert L.csa_sparse_mqa_workspace_size(64, 64, 512, 512, csa.CSA_BF16) == 0        # 2 splits
    three = L.csa_sparse_mqa_workspace_size(40, 64, 512, 384, csa.CSA_BF16)            # 3 splits
    assert three >= 40 * 3 * 64 * 512 * 4 + 40 * 3 * 64 * 2 * 4
    # 148 SMs over 16 queries allow 9 splits; 64 tiles of 128 entries need
    # only 8 splits of 8 tiles
    hca = L.hca_dense_mqa_workspace_size(16, 64, 512, 8192, csa.CSA_BF16)
    assert hca >= 16 * 8 * 64 * 512 * 4
    assert L.csa_decode_workspace_size(64, 32768, 64, 512, 64, 128, 512, csa.CSA_BF16) >= 64 * 32768 * 4
    small = L.csa_prefill_workspace_size(1024, 256, 512, 4, 128, 64, 8, 4, 16, csa.CSA_BF16)
    assert small >= 1024 * 4 * 128 * 4
    # the prefill score block is bounded (query chunking) at long context
    big = L.csa_prefill_workspace_size(65536, 65536, 4096, 4, 512, 128, 64, 64, 512, csa.CSA_BF16)
    assert big < 8 * (1 << 30)


def test_bindings_check_buffer_shapes_before_the_call():
    # buffers the C calls only see as pointers: a wrong shape is refused in
    # the binding before anything reaches the library (CPU tensors suffice)
    B, m, c = 4, 4, 64
    f32 = dict(dtype=torch.float32)
    with pytest.raises(ValueError, match="state"):
        csa.csa_compress_step(torch.zeros(B, 4 * c, **f32), torch.zeros(B, m, 4 * c, **f32),
                              torch.zeros(2 * m, c, **f32), torch.zeros(B, dtype=torch.int32),
                              torch.zeros(B, 8, c, dtype=torch.bfloat16), m)
    with pytest.raises(ValueError, match="cache"):
        csa.hca_compress_step(torch.zeros(B, 2 * c, **f32), torch.zeros(B, 128, 2 * c, **f32),
                              torch.zeros(128, c, **f32), torch.zeros(B, dtype=torch.int32),
                              torch.zeros(B, 8, c + 8, dtype=torch.bfloat16), 128)
    with pytest.raises(ValueError, match="gamma"):
        csa.csa_norm_rope(torch.zeros(3, 2, c, dtype=torch.bfloat16), torch.zeros(3, dtype=torch.int32),
                          gamma=torch.ones(c // 2, **f32))
    with pytest.raises(ValueError, match="q_gamma"):
        csa.csa_attend_decode(torch.zeros(B, 8, 64, dtype=torch.bfloat16), torch.zeros(B, 8, **f32),
                              torch.zeros(B, 16, 64, dtype=torch.bfloat16), torch.zeros(B, 2, 128, dtype=torch.bfloat16),
                              torch.zeros(B, 16 + 8, 128, dtype=torch.bfloat16), torch.zeros(B, dtype=torch.int32), 4, 4,
                              n_win=8, q_gamma=torch.ones(64, **f32))


def test_header_is_plain_c_and_the_library_links_from_c(tmp_path):
    # the boundary is a C ABI: a C program includes csa.h, links libcsa.so
    # and calls into it (host-only calls: no GPU is touched)
    src = tmp_path / "use_csa.c"
    src.write_text(
        '#include <stdio.h>\n#include "csa.h"\n'
        "int main(void) {\n"
        "    int rc = csa_compress(NULL, NULL, NULL, 6, 8, 4, NULL, CSA_BF16, NULL);\n"
        '    printf("%d %d %s\\n", csa_abi_version(), rc, csa_last_error());\n'
        "    return rc == CSA_ERR_INVALID_ARG ? 0 : 1;\n}\n")
    exe = tmp_path / "use_csa"
    libdir = os.path.dirname(csa.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                           "-o", str(exe), "-L", libdir, "-lcsa", "-Wl,-rpath," + libdir])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.startswith(f"{csa.abi_version()} {csa.CSA_ERR_INVALID_ARG} ")


def test_no_cpu_path(tmp_path):
    # without the built library the package refuses to import, and with it
    # every compute call refuses host tensors: there is no CPU fallback
    pkg = os.path.dirname(csa.__file__)
    copy = tmp_path / "compressed_sparse_attention_14_b200"
    copy.mkdir()
    for name in ("__init__.py", "context_parallel.py"):
        (copy / name).write_text(open(os.path.join(pkg, name)).read())
    r = subprocess.run([sys.executable, "-c", "import compressed_sparse_attention_14_b200"], cwd=str(tmp_path),
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "ImportError" in r.stderr and "libcsa.so is missing" in r.stderr
    x = torch.zeros(16, 64, dtype=torch.bfloat16)
    W = torch.zeros(32, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        csa.csa_project(x, W, out=torch.zeros(16, 32))


def test_product_code_does_not_reach_the_oracle():
    # the oracle is test infrastructure: the package and the CUDA sources
    # neither import, include nor load it
    pkg = os.path.dirname(csa.__file__)
    offenders = []
    for dirpath, _, files in os.walk(pkg):
        if "_build" in dirpath:
            continue
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".c")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                if re.search(r"^\s*(import oracle|from oracle)|csa_oracle|liboracle", text, flags=re.M):
                    offenders.append(f)
    assert not offenders, offenders
