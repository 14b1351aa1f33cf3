"""The allocation-free decode entry point, mla_decode_attention_noalloc (GPU).

Some callers cannot allocate device memory when they run a decode step: a serving process
whose device memory is reserved up front by its own allocator, code that must not stall on
the synchronisation cudaMalloc/cudaFree can cause, or a plain C caller without a workspace
allocator. For them the library keeps the split-KV scratch in one static device array. This
test calls that entry point through the C ABI twice in a row and checks each result against
the workspace-taking mla_decode_attention on the same inputs, with the parity tolerance.
It sits in a file of its own, collected last.
"""
import numpy as np
import pytest
import torch

import mla_latent_kv_42_b200 as M
from mla_latent_kv_42_b200 import build, synth
from parity import CacheCase, assert_parity, to64

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode_twice():
    build.build()
    M.load_library()
    M.read_device_status()
    w = synth.workload("production_b4_n131072_bf16")
    d = w.dims
    lens = np.array([20000, 1, 777, 9000])
    assert M.workspace_size(d, M.CALL_DECODE_ATTENTION, len(lens), int(lens.max())) > 0  # scratch is used
    case = CacheCase(w, cached=lens, paging="shuffled", spare_tokens=0)
    seq_lens = torch.from_numpy(lens.astype(np.int32)).cuda()
    for call in range(2):
        q = synth.synthetic_query(w, len(lens), scale=(1.0, 200.0)[call], seed_tag=call).cuda()
        ref_o, ref_l = M.decode_attention(d, q, case.pool, case.block_table, seq_lens, int(lens.max()))
        got_o, got_l = M.decode_attention_noalloc(d, q, case.pool, case.block_table, seq_lens, int(lens.max()))
        assert M.read_device_status() == 0
        assert_parity(to64(got_o), to64(ref_o), f"call {call} o_lat")
        np.testing.assert_allclose(to64(got_l), to64(ref_l), rtol=0, atol=1e-4)


def test_noalloc_small_head_decode_matches_workspace_decode_twice():
    """The running model's eight heads take the CUDA-core attention kernel, whose split-KV
    partials and merge also live in the static array when the caller passes no workspace."""
    build.build()
    M.load_library()
    M.read_device_status()
    w = synth.workload("running_b16_n4096_l12_bf16")
    d = w.dims
    lens = np.array([4097, 1, 300, 4097, 2000])
    assert M.workspace_size(d, M.CALL_DECODE_ATTENTION, len(lens), int(lens.max())) > 0  # scratch is used
    case = CacheCase(w, cached=lens, paging="shuffled", spare_tokens=0)
    seq_lens = torch.from_numpy(lens.astype(np.int32)).cuda()
    for call in range(2):
        q = synth.synthetic_query(w, len(lens), scale=(1.0, 200.0)[call], seed_tag=call).cuda()
        ref_o, ref_l = M.decode_attention(d, q, case.pool, case.block_table, seq_lens, int(lens.max()))
        got_o, got_l = M.decode_attention_noalloc(d, q, case.pool, case.block_table, seq_lens, int(lens.max()))
        assert M.read_device_status() == 0
        assert_parity(to64(got_o), to64(ref_o), f"call {call} o_lat")
        np.testing.assert_allclose(to64(got_l), to64(ref_l), rtol=0, atol=1e-4)
