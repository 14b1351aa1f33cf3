"""GPU parity of each C-ABI call against the fp64 oracle, with edge cases.

Inputs come from ``synth``; the oracle reads the same host values. Tolerance: max and mean
absolute error normalised by the reference's largest magnitude, <= 2e-2 and <= 2e-3. Paged
placement and status codes are checked exactly.
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


def weights64(w):
    W = synth.weights(w)
    return W, {k: O.as64(v) for k, v in W.items()}


# ---------------------------------------------------------------------------------------- append
@pytest.mark.parametrize("fam", list(FAMILIES))
def test_append_kv_rows_and_exact_placement(fam):
    w = FAMILIES[fam]
    d = w.dims
    W, W64 = weights64(w)
    # several tokens per sequence across page boundaries (pos % 64 in {0, 63}), pages shuffled
    cached = np.array([0, 63, 64, 130])
    bt, num_pages = synth.page_table(cached + 70, d.page_size, "shuffled", seed=3)
    seq_idx = np.repeat(np.arange(4), 3).astype(np.int32)
    pos = np.concatenate([np.arange(c, c + 3) for c in (0, 62, 64, 127)]).astype(np.int32)
    T = len(pos)
    h = synth.hidden(w, step=5, batch=T)
    pool = torch.full((num_pages, d.page_size, d.D), float("nan"), dtype=synth.storage_dtype(d), device="cuda")
    before = pool.clone()
    M.append_kv(d, h.cuda(), W["w_dkv_kr"].cuda(), torch.from_numpy(seq_idx).cuda(), torch.from_numpy(pos).cuda(),
                torch.from_numpy(bt).cuda(), pool)
    assert M.read_device_status() == 0
    flat, flat0 = pool.view(-1, d.D), before.view(-1, d.D)
    changed = (flat.view(torch.int16) != flat0.view(torch.int16)).any(dim=1).nonzero().flatten().cpu().numpy()
    expected = np.array([O.page_slot(bt, s, p, d.page_size) for s, p in zip(seq_idx, pos)])
    assert sorted(changed.tolist()) == sorted(expected.tolist())
    ref = O.kv_rows(W64["w_dkv_kr"], O.as64(h), pos, d)
    got = to64(flat[torch.from_numpy(expected).cuda()])
    assert_parity(got[:, :d.d_c], ref[:, :d.d_c], "c^KV")
    assert_parity(got[:, d.d_c:], ref[:, d.d_c:], "k^R")


def test_append_kv_bad_page_is_reported_and_skipped():
    w = W_RUN
    d = w.dims
    W, _ = weights64(w)
    bt = np.array([[0, -1], [1, 5]], dtype=np.int32)   # page 5 >= num_pages = 2
    pool = torch.zeros((2, d.page_size, d.D), dtype=torch.bfloat16, device="cuda")
    h = synth.hidden(w, batch=3).cuda()
    M.append_kv(d, h, W["w_dkv_kr"].cuda(), torch.tensor([0, 0, 1], dtype=torch.int32, device="cuda"),
                torch.tensor([3, 70, 65], dtype=torch.int32, device="cuda"), torch.from_numpy(bt).cuda(), pool)
    assert M.read_device_status() == -7                     # MLA_ERR_BAD_PAGE
    assert M.read_device_status() == 0                      # reading clears it
    nz = (pool.view(-1, d.D) != 0).any(dim=1).nonzero().flatten().tolist()
    assert nz == [3]                                        # only the valid token was written


# ---------------------------------------------------------------------------------------- absorb
@pytest.mark.parametrize("fam", list(FAMILIES))
def test_absorb_query(fam):
    w = FAMILIES[fam]
    d = w.dims
    W, W64 = weights64(w)
    B = 19
    h = synth.hidden(w, step=1, batch=B)
    pos = np.array([0, 1, 2, 63, 64, 65, 255, 256, 4095, 4096, 4097, 32767, 32768, 65536, 100000, 131071,
                    131072, 7, 12345], dtype=np.int32)
    q = M.absorb_query(d, h.cuda(), W["w_dq"].cuda(), W["w_uq_qr"].cuda(), W["w_uk"].cuda(),
                       torch.from_numpy(pos).cuda())
    ref = O.absorb_query(W64["w_dq"], W64["w_uq_qr"], W64["w_uk"], O.as64(h), pos, d)
    got = to64(q)
    assert_parity(got[..., :d.d_c], ref[..., :d.d_c], "q~")
    assert_parity(got[..., d.d_c:], ref[..., d.d_c:], "q^R")


# ---------------------------------------------------------------------------------------- decode
def run_decode(case, q, max_seq_len=None):
    d = case.w.dims
    seq_lens = torch.from_numpy(case.cached.astype(np.int32)).cuda()
    msl = int(case.cached.max()) if max_seq_len is None else max_seq_len
    return M.decode_attention(d, q.cuda(), case.pool, case.block_table, seq_lens, msl)


def check_decode(case, q, o_lat, lse, what=""):
    d = case.w.dims
    q64 = O.as64(q)
    for b in range(len(case.cached)):
        ref_o, ref_l = O.latent_attention(q64[b], O.as64(case.prefix(b)), d)
        assert_parity(to64(o_lat[b]), ref_o, f"{what} o_lat[b={b}]")
        np.testing.assert_allclose(to64(lse[b]), ref_l, rtol=0, atol=2e-2, err_msg=f"{what} lse[b={b}]")


@pytest.mark.parametrize("fam", list(FAMILIES))
@pytest.mark.parametrize("scale", [1.0, 300.0], ids=["pages_law", "peaked"])
def test_decode_attention_ragged_paged(fam, scale):
    w = FAMILIES[fam]
    lens = np.array([1, 2, 63, 64, 65, 129, 1000, 4097])
    case = CacheCase(w, cached=lens, paging="shuffled", fill=float("nan"), spare_tokens=0)
    q = synth.synthetic_query(w, len(lens), scale=scale)
    o_lat, lse = run_decode(case, q)
    assert M.read_device_status() == 0
    check_decode(case, q, o_lat, lse, fam)


def test_decode_fewer_pages_than_sm_pairs():
    """A handful of pages spread over many SM pairs: most pairs own no page at all."""
    w = W_PROD
    lens = np.array([1, 130, 200, 64])
    case = CacheCase(w, cached=lens, paging="shuffled", fill=float("nan"), spare_tokens=0)
    q = synth.synthetic_query(w, len(lens), scale=40.0)
    o_lat, lse = run_decode(case, q)
    assert M.read_device_status() == 0
    check_decode(case, q, o_lat, lse, "few pages")


def test_decode_split_plans_agree_and_are_deterministic():
    w = W_PROD
    lens = np.array([3000, 17, 4097])
    case = CacheCase(w, cached=lens, paging="shuffled")
    q = synth.synthetic_query(w, 3, scale=50.0)
    a, la = run_decode(case, q)
    b, lb = run_decode(case, q)
    assert torch.equal(a, b) and torch.equal(la, lb)         # bitwise run to run
    c, lc = run_decode(case, q, max_seq_len=int(lens.max()) + 60)   # a different split plan
    assert_parity(to64(c), to64(a), "split plans")


@pytest.mark.parametrize("scale", [1.0, 200.0], ids=["pages_law", "peaked"])
def test_decode_bitwise_repeatable_at_full_load(scale):
    """Every step of decode runs in a fixed order, so repeated calls agree bit for bit. A
    synchronisation slip between pipeline stages (O read or rescaled before an MMA into it has
    finished) shows up here as a run-to-run difference even where it stays inside the parity
    tolerance; full-size ragged batches keep HBM busy so that the producers fall behind."""
    w = W_PROD
    rng = np.random.default_rng(7)
    lens = np.concatenate([rng.integers(1, 9000, size=60), [20000, 1, 777, 64 * 70]])
    case = CacheCase(w, cached=lens, paging="shuffled", fill=float("nan"), spare_tokens=0)
    q = synth.synthetic_query(w, len(lens), scale=scale)
    first, first_l = run_decode(case, q)
    for _ in range(4):
        o, l = run_decode(case, q)
        assert M.read_device_status() == 0
        assert torch.equal(o, first) and torch.equal(l, first_l)


@pytest.mark.parametrize("fam", ["running_bf16", "production_bf16"])
def test_decode_needle_tokens(fam):
    """One planted token per sequence scores ~20 above every other token, for every head. The
    needles sit on page, tile and split boundaries and at the first and last token; the output
    must be the needle's latent, and the split-KV merge must pick the partial that holds it."""
    w = FAMILIES[fam]
    d = w.dims
    lens = np.array([1, 64, 65, 129, 777, 4097, 20000])
    needles = np.array([0, 63, 64, 128, 776, 4096, 11111])
    case = CacheCase(w, cached=lens, paging="shuffled", spare_tokens=0)
    q64 = synth.synthetic_query(w, len(lens)).double()
    target = 20.0 * np.sqrt(d.d_head + d.d_rope)  # raw dot product whose scaled score is 20
    for b, j in enumerate(needles):
        r = case.prefix(b)[int(j)].double().cpu()
        q64[b] += (target / float(r @ r)) * r  # every head gains q.r = target on the needle
    q = q64.to(synth.storage_dtype(d))
    o_lat, lse = run_decode(case, q)
    assert M.read_device_status() == 0
    check_decode(case, q, o_lat, lse, f"{fam} needles")
    for b, j in enumerate(needles):
        want = to64(case.prefix(b)[int(j)][:d.d_c]).reshape(1, -1).repeat(d.n_heads, 0)
        assert_parity(to64(o_lat[b]), want, f"{fam} needle row b={b} j={j}")


def test_decode_timing_hook_brackets_the_attention_kernel():
    w = W_PROD
    lens = np.array([3000, 17, 4097])
    case = CacheCase(w, cached=lens, paging="shuffled")
    q = synth.synthetic_query(w, 3)
    ref_o, ref_l = run_decode(case, q)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in ev:
        e.record()
    M.set_decode_timing_events(ev[1], ev[2])
    try:
        ev[0].record()
        o, l = run_decode(case, q)
        ev[3].record()
    finally:
        M.set_decode_timing_events(None, None)
    torch.cuda.synchronize()
    assert M.read_device_status() == 0
    assert torch.equal(o, ref_o) and torch.equal(l, ref_l)
    kernel_ms, call_ms = ev[1].elapsed_time(ev[2]), ev[0].elapsed_time(ev[3])
    assert 0.0 < kernel_ms <= call_ms


def test_decode_all_equal_rows_and_single_token_are_exact():
    for w in (W_RUN16, W_PROD):
        d = w.dims
        lens = np.array([1, 300])
        case = CacheCase(w, cached=lens)
        row = case.rows[0].clone()
        case.pool.view(-1, d.D)[:] = row               # every slot holds the same row
        q = synth.synthetic_query(w, 2, scale=500.0)
        o_lat, _ = run_decode(case, q)
        expect = row[:d.d_c].expand_as(o_lat)
        assert torch.equal(o_lat, expect)


def test_decode_bad_seq_len_and_bad_page():
    w = W_RUN
    d = w.dims
    lens = np.array([10, 20])
    case = CacheCase(w, cached=lens)
    q = synth.synthetic_query(w, 2).cuda()
    seq_lens = torch.tensor([0, 20], dtype=torch.int32, device="cuda")
    o_lat, _ = M.decode_attention(d, q, case.pool, case.block_table, seq_lens, 20)
    assert M.read_device_status() == -8
    assert torch.count_nonzero(o_lat[0]) == 0
    ref, _ = O.latent_attention(O.as64(q[1]), O.as64(case.prefix(1)), d)
    assert_parity(to64(o_lat[1]), ref, "other sequence")
    bt = case.block_table.clone()
    bt[1, 0] = case.num_pages + 3
    M.decode_attention(d, q, case.pool, bt, torch.tensor([10, 20], dtype=torch.int32, device="cuda"), 20)
    assert M.read_device_status() == -7


# ---------------------------------------------------------------------------------------- out proj
@pytest.mark.parametrize("fam", list(FAMILIES))
def test_out_proj(fam):
    w = FAMILIES[fam]
    d = w.dims
    W, W64 = weights64(w)
    B = 13
    rng = np.random.default_rng(7)
    o_lat = synth.to_storage(rng.standard_normal((B, d.n_heads, d.d_c), dtype=np.float32) * 0.05, d)
    u = M.out_proj(d, o_lat.cuda(), W["w_uv"].cuda(), W["w_o"].cuda())
    ref = O.out_proj_absorbed(W64["w_uv"], W64["w_o"], O.as64(o_lat))
    assert_parity(to64(u), ref, "u")


@pytest.mark.parametrize("fam", ["running_bf16", "production_bf16"])
def test_projections_beyond_one_n_tile(fam):
    """300 tokens: the GEMMs run two n tiles of 256 with no shared-memory RoPE table: the query's
    q^R reads each cos/sin from the global per-token table the W^DQ product fills, the append's
    k^R computes its own, and the append scatters per token."""
    w = FAMILIES[fam]
    d = w.dims
    W, W64 = weights64(w)
    T = 300
    # append: 5 sequences x 60 new tokens, crossing page boundaries, shuffled pages
    seq_idx = np.repeat(np.arange(5), 60).astype(np.int32)
    pos = np.concatenate([np.arange(o, o + 60) for o in (0, 40, 100, 1000, 4090)]).astype(np.int32)
    bt, num_pages = synth.page_table(np.array([60, 100, 160, 1060, 4150]), d.page_size, "shuffled", seed=5)
    h = synth.hidden(w, step=7, batch=T)
    pool = torch.zeros((num_pages, d.page_size, d.D), dtype=synth.storage_dtype(d), device="cuda")
    M.append_kv(d, h.cuda(), W["w_dkv_kr"].cuda(), torch.from_numpy(seq_idx).cuda(), torch.from_numpy(pos).cuda(),
                torch.from_numpy(bt).cuda(), pool)
    assert M.read_device_status() == 0
    slots = np.array([O.page_slot(bt, s_, p_, d.page_size) for s_, p_ in zip(seq_idx, pos)])
    got = to64(pool.view(-1, d.D)[torch.from_numpy(slots).cuda()])
    ref = O.kv_rows(W64["w_dkv_kr"], O.as64(h), pos, d)
    assert_parity(got[:, :d.d_c], ref[:, :d.d_c], "c^KV, 300 tokens")
    assert_parity(got[:, d.d_c:], ref[:, d.d_c:], "k^R, 300 tokens")
    # absorb: 300 queries at positions up to 131072
    qpos = (np.arange(T, dtype=np.int64) * 437) % 131073
    q = M.absorb_query(d, h.cuda(), W["w_dq"].cuda(), W["w_uq_qr"].cuda(), W["w_uk"].cuda(),
                       torch.from_numpy(qpos.astype(np.int32)).cuda())
    refq = O.absorb_query(W64["w_dq"], W64["w_uq_qr"], W64["w_uk"], O.as64(h), qpos.astype(np.int32), d)
    assert_parity(to64(q)[..., :d.d_c], refq[..., :d.d_c], "q~, 300 tokens")
    assert_parity(to64(q)[..., d.d_c:], refq[..., d.d_c:], "q^R, 300 tokens")
    # out_proj of 300 rows
    rng = np.random.default_rng(11)
    o_lat = synth.to_storage(rng.standard_normal((T, d.n_heads, d.d_c), dtype=np.float32) * 0.05, d)
    u = M.out_proj(d, o_lat.cuda(), W["w_uv"].cuda(), W["w_o"].cuda())
    assert_parity(to64(u), O.out_proj_absorbed(W64["w_uv"], W64["w_o"], O.as64(o_lat)), "u, 300 tokens")
    assert M.read_device_status() == 0


# ---------------------------------------------------------------------------------------- one layer step
def test_layer_step_running_model_fp16():
    """The pages' running model, one layer, B=1, 256 cached tokens, fp16 (positions 0..255, new at 256)."""
    w = W_RUN16
    d = w.dims
    cached = synth.cached_lengths(w)
    L = harness.make_layer(w, cached)
    ix = harness.step_index(cached)
    h = synth.hidden(w)
    u, q, o_lat, lse = M.layer_step(L.state, h.cuda(), ix.pos, ix.seq_idx, ix.seq_lens, ix.max_seq_len)
    assert M.read_device_status() == 0
    W64 = {k: O.as64(v) for k, v in L.W_host.items()}
    prefix = [O.as64(L.prefix(b)) for b in range(w.batch)]
    naive = O.layer_step_naive(W64, O.as64(h), prefix, d)
    absd = O.layer_step_absorbed(W64, O.as64(h), prefix, d)
    slot = O.page_slot(L.state.block_table.cpu().numpy(), 0, cached[0], d.page_size)
    assert_parity(to64(L.state.pool.view(-1, d.D)[int(slot)])[None], naive["rows"], "new row")
    assert_parity(to64(q)[..., :d.d_c], absd["q"][..., :d.d_c], "q~")
    assert_parity(to64(q)[..., d.d_c:], absd["q"][..., d.d_c:], "q^R")
    assert_parity(to64(o_lat), absd["o_lat"], "o_lat")
    assert_parity(to64(u), naive["u"], "u")


ODD_DIMS = {
    # 4 heads, 112-wide rows, 16-token pages: attention on the warp-MMA kernel
    "h4_dh40_dc96": synth.Dims(d_model=256, n_heads=4, d_head=40, d_c=96, d_cq=72, d_rope=16, page_size=16),
    # 32 heads, 80-wide rows, 8-token pages: attention on the CUDA-core kernel
    "h32_dh24_dc72": synth.Dims(d_model=256, n_heads=32, d_head=24, d_c=72, d_cq=48, d_rope=8, page_size=8),
}


@pytest.mark.parametrize("name", list(ODD_DIMS))
def test_layer_step_head_widths_off_the_gemm_blocks(name):
    """Dims whose per-head slices are not whole 64-wide blocks (d_h = 40 or 24, d_c = 96 or 72): the
    two per-head products take the CUDA-core kernels (k_absorb_uk for (W^UK_i)^T q^C_i, k_rowdot for
    W^UV_i o_lat_i), the rest the tensor-core GEMM; attention runs on the warp-MMA kernel (4 heads)
    or the CUDA-core kernel (32 heads, rows not a multiple of 16); a whole layer step through the
    C ABI against the naive and absorbed oracle."""
    d = ODD_DIMS[name]
    w = synth.Workload("odd_dims_b3", d, 3, 0, 1, 0.05, "shuffled")
    cached = np.array([0, 17, 300])
    L = harness.make_layer(w, cached)
    ix = harness.step_index(cached)
    h = synth.hidden(w)
    u, q, o_lat, lse = M.layer_step(L.state, h.cuda(), ix.pos, ix.seq_idx, ix.seq_lens, ix.max_seq_len)
    assert M.read_device_status() == 0
    W64 = {k: O.as64(v) for k, v in L.W_host.items()}
    prefix = [O.as64(L.prefix(b)) for b in range(w.batch)]
    naive = O.layer_step_naive(W64, O.as64(h), prefix, d)
    absd = O.layer_step_absorbed(W64, O.as64(h), prefix, d)
    assert_parity(to64(q)[..., :d.d_c], absd["q"][..., :d.d_c], "q~")
    assert_parity(to64(q)[..., d.d_c:], absd["q"][..., d.d_c:], "q^R")
    assert_parity(to64(o_lat), absd["o_lat"], "o_lat")
    assert_parity(to64(u), naive["u"], "u")


@pytest.mark.parametrize("fam", ["running_bf16", "production_bf16"])
def test_caller_rope_table_in_append_and_absorb(fam):
    """A caller-supplied RoPE frequency table (mla_dims.rope_inv_freq; here a YaRN-style
    interpolation for a 40x longer context) replaces base^(-2k/d_R) in the k^R the append writes
    and in the q^R the query path produces, at positions up to 131072 (one n tile and, with 300
    tokens, several)."""
    w0 = FAMILIES[fam]
    d = w0.dims.with_(rope_inv_freq=synth.yarn_inv_freq(w0.dims.d_rope, w0.dims.rope_base))
    W, W64 = weights64(w0)
    for T in (19, 300):
        pos = ((np.arange(T, dtype=np.int64) * 7919) % 131073).astype(np.int32)
        seq_idx = np.arange(T, dtype=np.int32)
        # one physical page per token, at its logical page pos // P (the other entries unused)
        max_pages = int(pos.max()) // d.page_size + 1
        bt = np.full((T, max_pages), -1, dtype=np.int32)
        bt[np.arange(T), pos // d.page_size] = np.random.default_rng(T).permutation(T)
        num_pages = T
        h = synth.hidden(w0, step=3, batch=T)
        pool = torch.zeros((num_pages, d.page_size, d.D), dtype=synth.storage_dtype(d), device="cuda")
        M.append_kv(d, h.cuda(), W["w_dkv_kr"].cuda(), torch.from_numpy(seq_idx).cuda(), torch.from_numpy(pos).cuda(),
                    torch.from_numpy(bt).cuda(), pool)
        q = M.absorb_query(d, h.cuda(), W["w_dq"].cuda(), W["w_uq_qr"].cuda(), W["w_uk"].cuda(),
                           torch.from_numpy(pos).cuda())
        assert M.read_device_status() == 0
        slots = np.array([O.page_slot(bt, s_, p_, d.page_size) for s_, p_ in zip(seq_idx, pos)])
        got = to64(pool.view(-1, d.D)[torch.from_numpy(slots).cuda()])
        ref = O.kv_rows(W64["w_dkv_kr"], O.as64(h), pos, d)
        assert_parity(got[:, d.d_c:], ref[:, d.d_c:], f"k^R with the table, T={T}")
        # the table matters: the base formula's k^R is far from what was written
        plain = O.kv_rows(W64["w_dkv_kr"], O.as64(h), pos, w0.dims)
        assert np.abs(plain[:, d.d_c:] - got[:, d.d_c:]).max() > 10 * np.abs(ref[:, d.d_c:] - got[:, d.d_c:]).max()
        refq = O.absorb_query(W64["w_dq"], W64["w_uq_qr"], W64["w_uk"], O.as64(h), pos, d)
        assert_parity(to64(q)[..., d.d_c:], refq[..., d.d_c:], f"q^R with the table, T={T}")
        assert_parity(to64(q)[..., :d.d_c], refq[..., :d.d_c], f"q~, T={T}")
