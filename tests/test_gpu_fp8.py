"""GPU parity of the FP8 latent cache (mla_append_kv_fp8, mla_decode_attention_fp8) against the
oracle's e4m3 quantisation (quantize_rows_fp8 / dequantize_rows_fp8) and latent attention.

The cache format, the reading of DeepSeek-V2 paper review (velog) §4.2 and the DeepSeek-V2
summary page ("The Model"): e4m3 bytes with two float32 scales per token, max|part| / 448.

- Written bytes and scales are compared bit for bit where the rows the writer quantises are
  exact on both sides: hidden states that are scaled one-hot vectors make c^KV = W^DKV h a column
  of the weight, exact in any summation order, and position 0 makes RoPE the identity.
- With general hidden states, the rows the FP8 cache stands for are compared with the oracle's
  rows at the parity tolerance, and every nonzero part reaches code 448 exactly.
- The decode runs over caches whose bytes the oracle wrote (on the host), shuffled pages, ragged
  lengths and tail pages, against the oracle's attention over the rows the cache stands for as
  the decode forms them: its tensor-core products run in fp16, each e4m3 value (exact in fp16)
  times its token's scale rounded to fp16, the product rounded once to fp16.
"""
import dataclasses

import numpy as np
import pytest
import torch

import mla_latent_kv_42_b200 as M
import oracle as O
from mla_latent_kv_42_b200 import build, synth
from parity import CacheCase, assert_parity, to64

pytestmark = pytest.mark.gpu

W_PROD = synth.workload("production_b64_n4096_bf16")
W_PROD16 = dataclasses.replace(W_PROD, name="production_b64_n4096_fp16", dims=W_PROD.dims.with_(dtype="fp16"))
POS_VALS = O.e4m3_values()[:0x7F]  # codes 0x00 .. 0x7E, increasing


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build()
    M.load_library()
    assert M.read_device_status() == 0


def codes_of(values: np.ndarray) -> np.ndarray:
    """e4m3 byte codes of exact e4m3 values (the sign bit kept for zeros)."""
    a = np.abs(values)
    c = np.searchsorted(POS_VALS, a)
    assert np.array_equal(POS_VALS[c], a), "not e4m3 values"
    return (c | (np.signbit(values).astype(np.int64) << 7)).astype(np.uint8)


def page_views(pool: np.ndarray, d):
    """(rows [pages, P, D] uint8, scales [pages, P, 2] float32) views of FP8 pages."""
    P, D = d.page_size, d.D
    rows = pool[:, :P * D].reshape(-1, P, D)
    scales = pool[:, P * D:].copy().view(np.float32).reshape(-1, P, 2)
    return rows, scales


def fp8_pool_from_rows(rows64: np.ndarray, cached, bt, num_pages, d):
    """FP8 pages holding each sequence's rows (quantised by the oracle), and the rows they stand
    for as the decode forms them (fp16 value times fp16 scale, rounded to fp16); bytes of unused
    slots are the e4m3 NaN code and their scales NaN, so that a read past a sequence shows."""
    vals, sc = O.quantize_rows_fp8(rows64, d.d_c)
    codes = codes_of(vals)
    pool = np.full((num_pages, M.fp8_page_bytes(d)), 0x7F, dtype=np.uint8)
    rows, _ = page_views(pool, d)
    scales = np.full((num_pages, d.page_size, 2), np.nan, dtype=np.float32)
    off = 0
    for b, n in enumerate(cached):
        for j in range(int(n)):
            pg, r = bt[b][j // d.page_size], j % d.page_size
            rows[pg, r] = codes[off + j]
            scales[pg, r] = sc[off + j]
        off += int(n)
    pool[:, d.page_size * d.D:] = scales.view(np.uint8).reshape(num_pages, -1)
    sc16 = sc.astype(np.float16).astype(np.float64)  # the scale rounded to fp16
    return pool, O.dequantize_rows_fp8(vals, sc16, d.d_c).astype(np.float16).astype(np.float64)


def test_page_bytes_and_support():
    d = W_PROD.dims
    assert M.fp8_page_bytes(d) == 64 * (576 + 8)
    assert M.fp8_supported(d)
    assert not M.fp8_supported(synth.RUNNING)


def append_fp8(d, h, w, seq_idx, pos, bt, num_pages):
    pool = torch.full((num_pages, M.fp8_page_bytes(d)), 0x7F, dtype=torch.uint8, device="cuda")
    M.append_kv_fp8(d, h.cuda(), w.cuda(), torch.from_numpy(seq_idx).cuda(), torch.from_numpy(pos).cuda(),
                    torch.from_numpy(bt).cuda(), pool)
    return pool.cpu().numpy()


@pytest.mark.parametrize("w", [W_PROD, W_PROD16], ids=["bf16", "fp16"])
def test_append_fp8_bytes_exact_on_exact_rows(w):
    """Scaled one-hot hidden states: the rows are weight columns times a power of two, exact on
    both sides, so bytes and scales must agree bit for bit (RoPE at position 0 for all parts,
    and the latent part at any position)."""
    d = w.dims
    W = synth.weights(w)
    T = 12
    rng = np.random.default_rng(11)
    ks = rng.choice(d.d_model, size=T, replace=False)
    h = np.zeros((T, d.d_model), dtype=np.float32)
    h[np.arange(T), ks] = 2.0 ** rng.integers(-6, 4, size=T)
    h = synth.to_storage(h, d)
    # tokens 0-5: position 0 of six sequences; tokens 6-11: sequence 6 at positions 0, 1, 63, 64, 65, 200
    seq_idx = np.array([0, 1, 2, 3, 4, 5, 6, 6, 6, 6, 6, 6], dtype=np.int32)
    pos = np.array([0, 0, 0, 0, 0, 0, 0, 1, 63, 64, 65, 200], dtype=np.int32)
    bt, num_pages = synth.page_table(np.array([1, 1, 1, 1, 1, 1, 201]), d.page_size, "shuffled", seed=5,
                                     spare_tokens=0)
    pool = append_fp8(d, h, W["w_dkv_kr"], seq_idx, pos, bt, num_pages)
    assert M.read_device_status() == 0
    ref_rows = O.kv_rows(O.as64(W["w_dkv_kr"]), O.as64(h), pos, d)   # exact for the latent part
    vals, sc = O.quantize_rows_fp8(O.as64(synth.to_storage(ref_rows, d)), d.d_c)
    codes = codes_of(vals)
    rows, scales = page_views(pool, d)
    for t in range(T):
        pg, r = bt[seq_idx[t]][pos[t] // d.page_size], pos[t] % d.page_size
        np.testing.assert_array_equal(rows[pg, r, :d.d_c], codes[t, :d.d_c], err_msg=f"c bytes, token {t}")
        assert scales[pg, r, 0] == sc[t, 0], f"s_c, token {t}"
        if pos[t] == 0:
            np.testing.assert_array_equal(rows[pg, r, d.d_c:], codes[t, d.d_c:], err_msg=f"k^R bytes, token {t}")
            assert scales[pg, r, 1] == sc[t, 1], f"s_r, token {t}"
    # nothing else was written
    written = {(bt[s][p // d.page_size], p % d.page_size) for s, p in zip(seq_idx, pos)}
    for pg in range(num_pages):
        for r in range(d.page_size):
            if (pg, r) not in written:
                assert (rows[pg, r] == 0x7F).all(), (pg, r)


def test_append_fp8_general_rows():
    """Random hidden states across page boundaries: the rows the cache stands for match the
    oracle's rows, and each nonzero part's largest byte is +-448. Tolerance: e4m3 keeps four
    significant bits, so the rounding error is at most half a step, 16 at the top of [-448, 448]:
    3.6% of a part's largest magnitude (max 5e-2 with the element-type rounding before it), and
    about 2^-5 of a typical value on average (mean 1e-2)."""
    w = W_PROD
    d = w.dims
    W = synth.weights(w)
    cached = np.array([0, 63, 64, 130])
    bt, num_pages = synth.page_table(cached + 70, d.page_size, "shuffled", seed=3)
    seq_idx = np.repeat(np.arange(4), 3).astype(np.int32)
    pos = np.concatenate([np.arange(c, c + 3) for c in (0, 62, 64, 127)]).astype(np.int32)
    h = synth.hidden(w, step=5, batch=len(pos))
    pool = append_fp8(d, h, W["w_dkv_kr"], seq_idx, pos, bt, num_pages)
    assert M.read_device_status() == 0
    rows, scales = page_views(pool, d)
    vals = O.e4m3_values()
    slots = [(bt[s][p // d.page_size], p % d.page_size) for s, p in zip(seq_idx, pos)]
    got_codes = np.stack([rows[pg, r] for pg, r in slots])
    got_sc = np.stack([scales[pg, r] for pg, r in slots]).astype(np.float64)
    got = O.dequantize_rows_fp8(vals[got_codes], got_sc, d.d_c)
    ref = O.kv_rows(O.as64(W["w_dkv_kr"]), O.as64(h), pos, d)
    assert_parity(got[:, :d.d_c], ref[:, :d.d_c], "c^KV (fp8)", max_tol=5e-2, mean_tol=1e-2)
    assert_parity(got[:, d.d_c:], ref[:, d.d_c:], "k^R (fp8)", max_tol=5e-2, mean_tol=1e-2)
    for part in (slice(0, d.d_c), slice(d.d_c, d.D)):
        assert (np.abs(vals[got_codes[:, part]]).max(axis=1) == 448.0).all()


def test_append_fp8_bad_page_is_reported_and_skipped():
    w = W_PROD
    d = w.dims
    W = synth.weights(w)
    bt = np.array([[0, -1], [1, 5]], dtype=np.int32)   # page 5 >= num_pages = 2
    h = synth.hidden(w, batch=3)
    pool = append_fp8(d, h, W["w_dkv_kr"], np.array([0, 0, 1], dtype=np.int32), np.array([3, 70, 65], dtype=np.int32),
                      bt, 2)
    assert M.read_device_status() == -7                # MLA_ERR_BAD_PAGE
    rows, _ = page_views(pool, d)
    changed = [(pg, r) for pg in range(2) for r in range(d.page_size) if not (rows[pg, r] == 0x7F).all()]
    assert changed == [(0, 3)]


@pytest.mark.parametrize("w", [W_PROD, W_PROD16], ids=["bf16", "fp16"])
@pytest.mark.parametrize("scale", [1.0, 300.0], ids=["pages_law", "peaked"])
def test_decode_fp8_ragged_paged(w, scale):
    d = w.dims
    lens = np.array([1, 2, 63, 64, 65, 129, 1000, 4097])
    case = CacheCase(w, cached=lens, paging="shuffled", spare_tokens=0, device="cpu")
    pool, deq = fp8_pool_from_rows(O.as64(case.rows), lens, case.bt_np, case.num_pages, d)
    q = synth.synthetic_query(w, len(lens), scale=scale)
    o_lat, lse = M.decode_attention_fp8(d, q.cuda(), torch.from_numpy(pool).cuda(), case.block_table.cuda(),
                                        torch.from_numpy(lens.astype(np.int32)).cuda(), int(lens.max()))
    assert M.read_device_status() == 0
    assert M.last_launch_count(M.CALL_DECODE_ATTENTION_FP8) == 3
    q64 = O.as64(q)
    off = np.concatenate([[0], np.cumsum(lens)])
    for b in range(len(lens)):
        ref_o, ref_l = O.latent_attention(q64[b], deq[off[b]:off[b + 1]], d)
        assert_parity(to64(o_lat[b]), ref_o, f"o_lat[b={b}]")
        np.testing.assert_allclose(to64(lse[b]), ref_l, rtol=0, atol=2e-2, err_msg=f"lse[b={b}]")


def test_decode_fp8_full_load_sampled():
    """Every SM pair busy (64 sequences of 4097 tokens, the benchmark's decode shape): sampled
    sequences against the oracle, and the result bitwise repeatable."""
    w = W_PROD
    d = w.dims
    lens = np.full(64, 4097)
    case = CacheCase(w, cached=lens, paging="contiguous", spare_tokens=0, device="cpu")
    pool, deq = fp8_pool_from_rows(O.as64(case.rows), lens, case.bt_np, case.num_pages, d)
    q = synth.synthetic_query(w, len(lens))
    args = (d, q.cuda(), torch.from_numpy(pool).cuda(), case.block_table.cuda(),
            torch.from_numpy(lens.astype(np.int32)).cuda(), int(lens.max()))
    o1, l1 = M.decode_attention_fp8(*args)
    o2, l2 = M.decode_attention_fp8(*args)
    assert M.read_device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    q64 = O.as64(q)
    for b in (0, 17, 63):
        rows = deq[b * 4097:(b + 1) * 4097]
        ref_o, _ = O.latent_attention(q64[b], rows, d)
        assert_parity(to64(o1[b]), ref_o, f"o_lat[b={b}]")


def test_decode_fp8_matches_bf16_path_on_dequantised_rows():
    """The FP8 decode agrees with the 16-bit decode run over the rows the FP8 cache stands for:
    the one forms them in fp16, the other reads them rounded to bf16, so they differ by that
    rounding (half a bf16 step, 2^-9 relative, per value) and the order of summation."""
    w = W_PROD
    d = w.dims
    lens = np.array([5, 300, 2000])
    case = CacheCase(w, cached=lens, paging="shuffled", spare_tokens=0, device="cpu")
    pool, deq = fp8_pool_from_rows(O.as64(case.rows), lens, case.bt_np, case.num_pages, d)
    q = synth.synthetic_query(w, len(lens)).cuda()
    bt = case.block_table.cuda()
    sl = torch.from_numpy(lens.astype(np.int32)).cuda()
    o8, l8 = M.decode_attention_fp8(d, q, torch.from_numpy(pool).cuda(), bt, sl, int(lens.max()))
    rows16 = synth.to_storage(deq, d)  # already element-type values
    pool16 = synth.paged_pool(rows16.cuda(), lens, case.bt_np, case.num_pages, d.page_size, fill=0.0)
    o16, l16 = M.decode_attention(d, q, pool16, bt, sl, int(lens.max()))
    assert M.read_device_status() == 0
    assert_parity(to64(o8), to64(o16), "fp8 vs bf16 over the same rows", max_tol=1e-2, mean_tol=1e-3)
    torch.testing.assert_close(l8, l16, rtol=0, atol=1e-2)


def test_decode_fp8_bad_seq_len():
    w = W_PROD
    d = w.dims
    lens = np.array([10, 70])
    case = CacheCase(w, cached=lens, paging="shuffled", spare_tokens=0, device="cpu")
    pool, _ = fp8_pool_from_rows(O.as64(case.rows), lens, case.bt_np, case.num_pages, d)
    q = synth.synthetic_query(w, 2).cuda()
    bad = torch.tensor([10, 200], dtype=torch.int32, device="cuda")   # 200 > max_seq_len
    o, l = M.decode_attention_fp8(d, q, torch.from_numpy(pool).cuda(), case.block_table.cuda(), bad, 70)
    assert M.read_device_status() == -8
    assert torch.count_nonzero(o[1]) == 0 and torch.isinf(l[1]).all()
    assert torch.isfinite(l[0]).all()
