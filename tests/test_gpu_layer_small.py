"""GPU parity of the fused single-launch layer step for small head counts (mla_layer_step_small)
against the naive and absorbed oracle, and against the four-call path on the same inputs.

Both running-model workloads of the benchmark: B = 1 with 256 cached tokens (fp16) and B = 16 with
4096 cached tokens (bf16, all 12 layers chained by the residual), plus ragged lengths that include
a sequence's first token (nothing cached) and lengths off the 64-token stage grid.
"""
import numpy as np
import pytest
import torch

import mla_latent_kv_42_b200 as M
import oracle as O
from mla_latent_kv_42_b200 import build, harness, synth
from parity import assert_parity, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build()
    M.load_library()
    M.read_device_status()


def check_step(w, cached, layer=0, h=None, label=""):
    d = w.dims
    ix = harness.step_index(cached)
    L = harness.make_layer(w, cached, layer=layer)
    h = synth.hidden(w, batch=len(cached)) if h is None else h
    u, q, o_lat, lse = M.layer_step_small(L.state, h.cuda(), ix.seq_lens, ix.max_seq_len)
    assert M.read_device_status() == 0
    assert M.last_launch_count(M.CALL_LAYER_STEP_SMALL) == 1
    W64 = {k: O.as64(v) for k, v in L.W_host.items()}
    h64 = O.as64(h)
    bt = L.state.block_table.cpu().numpy()
    slots = np.array([O.page_slot(bt, b, int(cached[b]), d.page_size) for b in range(len(cached))])
    rows = to64(L.state.pool.view(-1, d.D)[torch.from_numpy(slots).cuda()])
    ref_rows = O.kv_rows(W64["w_dkv_kr"], h64, cached, d)
    assert_parity(rows[:, :d.d_c], ref_rows[:, :d.d_c], f"{label} appended c^KV")
    assert_parity(rows[:, d.d_c:], ref_rows[:, d.d_c:], f"{label} appended k^R")
    prefix = [O.as64(L.prefix(b)) for b in range(len(cached))]
    naive = O.layer_step_naive(W64, h64, prefix, d)
    absd = O.layer_step_absorbed(W64, h64, prefix, d)
    assert_parity(to64(q), absd["q"], f"{label} q")
    assert_parity(to64(o_lat), absd["o_lat"], f"{label} o_lat")
    assert_parity(to64(u), naive["u"], f"{label} u")
    # the four-call path on a fresh copy of the same layer
    L2 = harness.make_layer(w, cached, layer=layer)
    u4, q4, o4, lse4 = M.layer_step(L2.state, h.cuda(), ix.pos, ix.seq_idx, ix.seq_lens, ix.max_seq_len)
    assert M.read_device_status() == 0
    assert_parity(to64(u), to64(u4), f"{label} u vs four calls")
    assert_parity(to64(o_lat), to64(o4), f"{label} o_lat vs four calls")
    torch.testing.assert_close(lse, lse4, rtol=1e-5, atol=1e-4)
    return u


def test_running_b1_n256_fp16():
    w = synth.workload("running_b1_n256_fp16")
    check_step(w, synth.cached_lengths(w), label="b1 n256")


def test_running_ragged_lengths():
    """First tokens (0 cached), lengths off the stage grid, one long sequence (split over CTAs)."""
    w = synth.workload("running_b16_n4096_l12_bf16")
    check_step(w, np.array([0, 1, 63, 64, 65, 200, 2500], dtype=np.int64), label="ragged")


def test_running_b16_n4096_twelve_layers_bf16():
    """12 layers chained by the residual h <- h + u (fp32 stream on both sides, rounded to bf16
    as each layer's input, as the four-call test does)."""
    w = synth.workload("running_b16_n4096_l12_bf16")
    d = w.dims
    cached = synth.cached_lengths(w)
    ix = harness.step_index(cached)
    h0 = synth.hidden(w)
    h_gpu = h0.float().cuda()
    h_ref = O.as64(h0)
    ws = torch.empty(M.workspace_size(d, M.CALL_LAYER_STEP_SMALL, w.batch, ix.max_seq_len), dtype=torch.uint8,
                     device="cuda")
    for layer in range(w.layers):
        L = harness.make_layer(w, cached, layer=layer)
        u, q, o_lat, lse = M.layer_step_small(L.state, h_gpu.to(torch.bfloat16), ix.seq_lens, ix.max_seq_len, ws=ws)
        assert M.read_device_status() == 0
        W64 = {k: O.as64(v) for k, v in L.W_host.items()}
        h_in64 = O.as64(synth.to_storage(torch.from_numpy(h_ref.astype(np.float32)), d))
        prefix = [O.as64(L.prefix(b)) for b in range(w.batch)]
        naive = O.layer_step_naive(W64, h_in64, prefix, d)
        assert_parity(to64(u), naive["u"], f"layer {layer} u")
        h_gpu = h_gpu + u.float()
        h_ref = h_ref + naive["u"]
    assert_parity(to64(h_gpu), h_ref, "final residual stream")


def test_unsupported_dims_and_bad_length():
    assert not M.layer_step_small_supported(synth.PRODUCTION)
    w = synth.workload("running_b1_n256_fp16")
    d = w.dims
    cached = np.array([10], dtype=np.int64)
    ix = harness.step_index(cached)
    L = harness.make_layer(w, cached)
    bad = torch.tensor([ix.max_seq_len + 5], dtype=torch.int32, device="cuda")  # past max_seq_len
    u, q, o_lat, lse = M.layer_step_small(L.state, synth.hidden(w, batch=1).cuda(), bad, ix.max_seq_len)
    assert M.read_device_status() == -8  # MLA_ERR_BAD_SEQ_LEN
    assert torch.count_nonzero(o_lat) == 0 and torch.isinf(lse).all()
    # the next call on the same stream is unaffected
    check_step(w, np.array([10], dtype=np.int64), label="after a rejected length")
