"""GPU parity of mla_prefill_attention: several new tokens per sequence, each attending to its
sequence's positions up to its own (causal), against the fp64 oracle. Also: every token equals a
decode call at its own length bit for bit, chunks larger than one launch group, rejected tokens,
and a whole multi-token layer step through the C ABI at the running model's dims.

Tolerance as for decode: max and mean absolute error normalised by the reference's largest
magnitude, <= 2e-2 and <= 2e-3. The cache already holds every new token's row, later tokens
included, so a token that looked past its own position would read real rows and fail.
"""
import numpy as np
import pytest
import torch

import mla_latent_kv_42_b200 as M
import oracle as O
from mla_latent_kv_42_b200 import build, harness, synth
from parity import CacheCase, assert_parity, to64

pytestmark = pytest.mark.gpu

W_RUN16 = synth.workload("running_b1_n256_fp16")
W_RUN = synth.workload("running_b16_n4096_l12_bf16")
W_PROD = synth.workload("production_b64_n4096_bf16")
FAMILIES = {"running_fp16": W_RUN16, "running_bf16": W_RUN, "production_bf16": W_PROD}


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build()
    M.load_library()
    assert M.read_device_status() == 0


@pytest.fixture(autouse=True)
def clean_status():
    M.read_device_status()
    yield


def chunk_case(w, prefix_lens, chunk_lens, fill=float("nan")):
    """A shuffled paged cache holding each sequence's prefix and its new tokens' rows, with
    ``fill`` in every slot past a sequence's last token."""
    total = np.asarray(prefix_lens) + np.asarray(chunk_lens)
    case = CacheCase(w, cached=total, paging="shuffled", fill=fill, spare_tokens=0)
    seq_idx, pos = O.chunk_positions(prefix_lens, chunk_lens)
    return case, seq_idx, pos


def dev_i32(a):
    return torch.from_numpy(np.asarray(a, dtype=np.int32)).cuda()


def run_prefill(case, q, seq_idx, pos, max_seq_len=None):
    msl = int(np.max(pos)) + 1 if max_seq_len is None else max_seq_len
    return M.prefill_attention(case.w.dims, q.cuda(), case.pool, case.block_table, dev_i32(seq_idx), dev_i32(pos), msl)


def check_prefill(case, q, seq_idx, pos, o_lat, lse, tokens=None, what=""):
    d = case.w.dims
    q64 = O.as64(q)
    rows = [O.as64(case.prefix(b)) for b in range(len(case.cached))]
    for t in (range(len(pos)) if tokens is None else tokens):
        ref_o, ref_l = O.chunk_latent_attention(q64[t:t + 1], rows, seq_idx[t:t + 1], pos[t:t + 1], d)
        assert_parity(to64(o_lat[t]), ref_o[0], f"{what} o_lat[t={t}]")
        np.testing.assert_allclose(to64(lse[t]), ref_l[0], rtol=0, atol=2e-2, err_msg=f"{what} lse[t={t}]")


@pytest.mark.parametrize("fam", list(FAMILIES))
@pytest.mark.parametrize("scale", [1.0, 300.0], ids=["pages_law", "peaked"])
def test_prefill_causal_chunks(fam, scale):
    """Chunks from an empty prefix, a single token, one crossing two page boundaries, and one
    after a long prefix; tokens of different sequences interleave in the call."""
    w = FAMILIES[fam]
    case, seq_idx, pos = chunk_case(w, [0, 5, 63, 1000], [3, 1, 70, 17])
    perm = np.random.default_rng(31).permutation(len(pos))        # any token order
    seq_idx, pos = seq_idx[perm], pos[perm]
    q = synth.synthetic_query(w, len(pos), scale=scale)
    o_lat, lse = run_prefill(case, q, seq_idx, pos)
    assert M.read_device_status() == 0
    check_prefill(case, q, seq_idx, pos, o_lat, lse, what=fam)


@pytest.mark.parametrize("fam", ["running_bf16", "production_bf16"])
def test_prefill_token_equals_decode_at_its_length(fam):
    """Each new token is one attention item of length pos + 1 over its sequence's pages, so a
    decode call given those lengths and a repeated block-table row gives the same bits."""
    w = FAMILIES[fam]
    case, seq_idx, pos = chunk_case(w, [0, 300, 4000], [40, 64, 9])
    q = synth.synthetic_query(w, len(pos), scale=30.0).cuda()
    msl = int(pos.max()) + 1
    o_lat, lse = run_prefill(case, q, seq_idx, pos, msl)
    bt_rep = case.block_table[torch.from_numpy(seq_idx).cuda()].contiguous()
    o_dec, lse_dec = M.decode_attention(w.dims, q, case.pool, bt_rep, dev_i32(pos + 1), msl)
    assert M.read_device_status() == 0
    assert torch.equal(o_lat, o_dec) and torch.equal(lse, lse_dec)
    o2, l2 = run_prefill(case, q, seq_idx, pos, msl)               # and run to run
    assert torch.equal(o2, o_lat) and torch.equal(l2, lse)


def test_prefill_more_tokens_than_one_launch_group():
    """1100 new tokens run as groups of 1024 and 76: each group is bitwise a decode call over
    its own tokens, and sampled tokens (group edges included) match the oracle."""
    w = W_PROD
    case, seq_idx, pos = chunk_case(w, [10, 40], [550, 550])
    q = synth.synthetic_query(w, len(pos), scale=30.0).cuda()
    msl = int(pos.max()) + 1
    o_lat, lse = run_prefill(case, q, seq_idx, pos, msl)
    assert M.read_device_status() == 0
    bt_rep = case.block_table[torch.from_numpy(seq_idx).cuda()].contiguous()
    for a, b in ((0, 1024), (1024, 1100)):
        o_dec, l_dec = M.decode_attention(w.dims, q[a:b], case.pool, bt_rep[a:b], dev_i32(pos[a:b] + 1), msl)
        assert torch.equal(o_lat[a:b], o_dec) and torch.equal(lse[a:b], l_dec), (a, b)
    check_prefill(case, q, seq_idx, pos, o_lat, lse, tokens=[0, 1, 300, 549, 550, 551, 1022, 1023, 1024, 1025, 1099],
                  what="1100 tokens")


@pytest.mark.parametrize("fam", ["running_bf16", "production_bf16"])
def test_prefill_rejected_tokens_are_zero_and_reported(fam):
    """A token with a sequence index past the block table or a position at max_seq_len gets a
    zero output and -inf log-sum-exp, and the device status reads MLA_ERR_BAD_SEQ_LEN; the
    other tokens are unaffected."""
    w = FAMILIES[fam]
    case, seq_idx, pos = chunk_case(w, [20, 130], [6, 6])
    msl = int(pos.max()) + 1
    seq_idx = seq_idx.copy()
    pos = pos.copy()
    seq_idx[2] = len(case.cached)
    pos[8] = msl
    q = synth.synthetic_query(w, len(pos), scale=10.0)
    o_lat, lse = run_prefill(case, q, seq_idx, pos, msl)
    assert M.read_device_status() == -8
    assert M.read_device_status() == 0
    for t in (2, 8):
        assert torch.count_nonzero(o_lat[t]) == 0
        assert torch.isneginf(lse[t]).all()
    good = [t for t in range(len(pos)) if t not in (2, 8)]
    check_prefill(case, q, seq_idx, pos, o_lat, lse, tokens=good, what=f"{fam} rejected")


def test_prefill_empty_call_is_a_no_op():
    w = W_PROD
    d = w.dims
    case, _, _ = chunk_case(w, [3], [1])
    q = torch.empty((0, d.n_heads, d.D), dtype=synth.storage_dtype(d), device="cuda")
    empty = torch.empty(0, dtype=torch.int32, device="cuda")
    o_lat, lse = M.prefill_attention(d, q, case.pool, case.block_table, empty, empty, 4)
    assert o_lat.shape == (0, d.n_heads, d.d_c) and M.last_launch_count(M.CALL_PREFILL_ATTENTION) == 0


@pytest.mark.parametrize("fam", ["running_fp16", "running_bf16"])
def test_chunked_layer_step_running_model(fam):
    """A layer step that brings 5, 64 and 9 new tokens to sequences holding 0, 7 and 300: append
    every new row, absorb every query, causal prefill attention, then the output projection,
    all through the C ABI, against the naive multi-token step of the oracle."""
    w = FAMILIES[fam]
    d = w.dims
    prefix_lens, chunk_lens = np.array([0, 7, 300]), np.array([5, 64, 9])
    bt, num_pages = synth.page_table(prefix_lens, d.page_size, "shuffled", w.seed, spare_tokens=int(chunk_lens.max()))
    L = harness.make_layer(w, prefix_lens, block_table=bt, num_pages=num_pages, fill=float("nan"))
    seq_idx, pos = O.chunk_positions(prefix_lens, chunk_lens)
    T = len(pos)
    h = synth.hidden(w, batch=T)
    st = L.state
    si, ps = dev_i32(seq_idx), dev_i32(pos)
    M.append_kv(d, h.cuda(), st.w["w_dkv_kr"], si, ps, st.block_table, st.pool)
    q = M.absorb_query(d, h.cuda(), st.w["w_dq"], st.w["w_uq_qr"], st.w["w_uk"], ps)
    o_lat, lse = M.prefill_attention(d, q, st.pool, st.block_table, si, ps, int(pos.max()) + 1)
    u = M.out_proj(d, o_lat, st.w["w_uv"], st.w["w_o"])
    assert M.read_device_status() == 0
    W64 = {k: O.as64(v) for k, v in L.W_host.items()}
    prefix = [O.as64(L.prefix(b)) for b in range(len(prefix_lens))]
    naive = O.chunk_step_naive(W64, O.as64(h), prefix, chunk_lens, d)
    absd = O.chunk_step_absorbed(W64, O.as64(h), prefix, chunk_lens, d)
    slots = np.array([O.page_slot(bt, int(seq_idx[t]), int(pos[t]), d.page_size) for t in range(T)])
    assert_parity(to64(st.pool.view(-1, d.D)[torch.from_numpy(slots).cuda()]), naive["rows"], "new rows")
    assert_parity(to64(q)[..., :d.d_c], absd["q"][..., :d.d_c], "q~")
    assert_parity(to64(q)[..., d.d_c:], absd["q"][..., d.d_c:], "q^R")
    assert_parity(to64(o_lat), absd["o_lat"], "o_lat")
    assert_parity(to64(u), naive["u"], "u")
