"""GPU parity of whole layer steps on the five workloads, in the launch configuration the
benchmark times (append -> absorb -> decode -> out_proj through the C ABI).

Small workloads are checked entirely against the naive and absorbed oracle. At full production
sizes the oracle recomputes sampled sequences one by one (all heads): the shortest, the longest
and a seeded random one; q and the appended rows are checked for every sequence.
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


def check_rows_and_q(L, ix, q, W64, h, d):
    bt = L.state.block_table.cpu().numpy()
    slots = np.array([O.page_slot(bt, b, int(ix.cached[b]), d.page_size) for b in range(len(ix.cached))])
    got_rows = to64(L.state.pool.view(-1, d.D)[torch.from_numpy(slots).cuda()])
    ref_rows = O.kv_rows(W64["w_dkv_kr"], O.as64(h), ix.cached, d)
    assert_parity(got_rows[:, :d.d_c], ref_rows[:, :d.d_c], "appended c^KV")
    assert_parity(got_rows[:, d.d_c:], ref_rows[:, d.d_c:], "appended k^R")
    ref_q = O.absorb_query(W64["w_dq"], W64["w_uq_qr"], W64["w_uk"], O.as64(h), ix.cached, d)
    assert_parity(to64(q)[..., :d.d_c], ref_q[..., :d.d_c], "q~")
    assert_parity(to64(q)[..., d.d_c:], ref_q[..., d.d_c:], "q^R")


def test_running_model_twelve_layers_bf16():
    """Running dims, B=16, 4096 cached each, 12 layers chained by the residual h <- h + u.

    The residual stream is carried in fp32 on both sides and rounded to bf16 as each layer's
    input (the oracle rounds its own fp64 stream the same way); the add is harness glue.
    """
    w = synth.workload("running_b16_n4096_l12_bf16")
    d = w.dims
    cached = synth.cached_lengths(w)
    ix = harness.step_index(cached)
    h0 = synth.hidden(w)
    h_gpu = h0.float().cuda()
    h_ref = O.as64(h0)
    ws = torch.empty(M.step_workspace_bytes(d, w.batch, ix.max_seq_len), dtype=torch.uint8, device="cuda")
    for layer in range(w.layers):
        L = harness.make_layer(w, cached, layer=layer)
        h_in = h_gpu.to(torch.bfloat16)
        u, q, o_lat, lse = M.layer_step(L.state, h_in, ix.pos, ix.seq_idx, ix.seq_lens, ix.max_seq_len, ws=ws)
        assert M.read_device_status() == 0
        W64 = {k: O.as64(v) for k, v in L.W_host.items()}
        h_in64 = O.as64(synth.to_storage(torch.from_numpy(h_ref.astype(np.float32)), d))
        prefix = [O.as64(L.prefix(b)) for b in range(w.batch)]
        naive = O.layer_step_naive(W64, h_in64, prefix, d)
        absd = O.layer_step_absorbed(W64, h_in64, prefix, d)
        assert_parity(to64(o_lat), absd["o_lat"], f"layer {layer} o_lat")
        assert_parity(to64(u), naive["u"], f"layer {layer} u")
        assert_parity(to64(q)[..., :d.d_c], absd["q"][..., :d.d_c], f"layer {layer} q~")
        h_gpu = h_gpu + u.float()
        h_ref = h_ref + naive["u"]
    assert_parity(to64(h_gpu), h_ref, "final residual stream")


def sampled(cached, rng_seed=0):
    idx = {int(np.argmin(cached)), int(np.argmax(cached)),
           int(np.random.default_rng([rng_seed, 9]).integers(0, len(cached)))}
    return sorted(idx)


@pytest.mark.parametrize("name", ["production_b64_n4096_bf16", "production_b128_ragged_paged_bf16",
                                  "production_b4_n131072_bf16"])
def test_production_workload_full_size(name):
    w = synth.workload(name)
    d = w.dims
    cached = synth.cached_lengths(w)
    ix = harness.step_index(cached)
    L = harness.make_layer(w, cached)
    h = synth.hidden(w)
    u, q, o_lat, lse = M.layer_step(L.state, h.cuda(), ix.pos, ix.seq_idx, ix.seq_lens, ix.max_seq_len)
    assert M.read_device_status() == 0
    W64 = {k: O.as64(v) for k, v in L.W_host.items()}
    check_rows_and_q(L, ix, q, W64, h, d)
    picks = sampled(cached) if w.batch > 4 else list(range(w.batch))
    for b in picks:
        prefix = [O.as64(L.prefix(b))]
        ref = O.layer_step_absorbed(W64, O.as64(h[b:b + 1]), prefix, d)
        assert_parity(to64(o_lat[b:b + 1]), ref["o_lat"], f"{name} o_lat[{b}]")
        np.testing.assert_allclose(to64(lse[b]), ref["lse"][0], rtol=0, atol=2e-2)
        assert_parity(to64(u[b:b + 1]), ref["u"], f"{name} u[{b}]")
    if name == "production_b64_n4096_bf16":       # one sequence through the naive route as well
        b = picks[0]
        naive = O.layer_step_naive(W64, O.as64(h[b:b + 1]), [O.as64(L.prefix(b))], d)
        assert_parity(to64(u[b:b + 1]), naive["u"], f"{name} u[{b}] naive")
