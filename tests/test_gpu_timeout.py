"""A wait that runs out inside the attention kernel (GPU, fault-injection build).

Every wait in the tensor-core kernels is bounded. The fault-injection build of the library
(libmla_faultinj.so: the same source with MLA_FAULT_INJECT, waits limited to 20 ms) can leave one
cache load of the attention kernel unissued after arming its barrier, so that the matrix-multiply
thread waits for bytes that never come. Its pair of SMs must then give up: record
MLA_ERR_TIMEOUT, wait for the loads it did issue, release its tensor memory and return. The test
checks that status, that the call ends in well under a second, and that the next call on the same
stream, with the injection cleared, matches the oracle. Nothing faults or hangs: the missing load
is a barrier that nothing completes.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import mla_latent_kv_42_b200 as M
import oracle as O
from mla_latent_kv_42_b200 import build, synth
from parity import CacheCase, assert_parity, to64

pytestmark = pytest.mark.gpu


def test_missing_load_times_out_and_the_next_call_is_correct():
    build.build()
    lib = M.load_library(build.LIB_FAULTINJ)
    assert M.load_library().mla_debug_inject_missing_load(0) == -1   # the regular library has no injection
    w = synth.workload("production_b64_n4096_bf16")
    d = w.dims
    lens = np.array([700, 300, 2000])
    B, msl = len(lens), int(lens.max())
    case = CacheCase(w, cached=lens, paging="shuffled", spare_tokens=0)
    q = synth.synthetic_query(w, B, scale=20.0).cuda()
    seq_lens = torch.from_numpy(lens.astype(np.int32)).cuda()
    cd = M.c_dims(d)
    ws_bytes = max(16, int(lib.mla_workspace_size(ctypes.byref(cd), M.CALL_DECODE_ATTENTION, B, msl)))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    o_lat = torch.empty((B, d.n_heads, d.d_c), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, d.n_heads), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())

    def decode():
        r = lib.mla_decode_attention(ctypes.byref(cd), ptr(q), ptr(case.pool), case.num_pages, ptr(case.block_table),
                                     case.block_table.shape[1], ptr(seq_lens), B, msl, ptr(o_lat), ptr(lse), ptr(ws),
                                     ws_bytes, stream)
        assert r == 0

    def status():
        v = ctypes.c_int32(0)
        assert lib.mla_read_device_status(stream, ctypes.byref(v)) == 0
        return v.value

    status()
    assert lib.mla_debug_inject_missing_load(-2) == -1
    assert lib.mla_debug_inject_missing_load(0) == 0
    try:
        t0 = time.perf_counter()
        decode()
        got = status()
        elapsed = time.perf_counter() - t0
    finally:
        assert lib.mla_debug_inject_missing_load(-1) == 0
    assert got == -6, f"device status {got}"             # MLA_ERR_TIMEOUT
    assert elapsed < 1.0, elapsed                          # gave up after the 20 ms limit, not 2 s
    decode()
    assert status() == 0
    for b in range(B):
        ref_o, ref_l = O.latent_attention(O.as64(q[b]), O.as64(case.prefix(b)), d)
        assert_parity(to64(o_lat[b]), ref_o, f"after the timeout, o_lat[b={b}]")
        np.testing.assert_allclose(to64(lse[b]), ref_l, rtol=0, atol=2e-2)
