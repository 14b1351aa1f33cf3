"""Pins of the fp64 oracle to facts the pages and the mathematics fix (CPU only).

Each test names the passage it checks. None of them re-types the oracle's own formula: they
use printed values, closed forms, invariants, special cases that reduce to a library routine
(torch's scaled_dot_product_attention, complex multiplication), exact identities between
two different computation routes, and brute force with scalar loops on tiny shapes.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from conftest import read_golden
from mla_latent_kv_42_b200 import synth
from mla_latent_kv_42_b200.synth import RUNNING, PRODUCTION, Dims

TINY = Dims(d_model=12, n_heads=3, d_head=4, d_c=6, d_cq=5, d_rope=4, page_size=4, rope_base=100.0)


def rand_weights(dims, rng, scale=0.3):
    n_h, d_h, d_r = dims.n_heads, dims.d_head, dims.d_rope
    return {
        "w_dkv_kr": rng.standard_normal((dims.d_c + d_r, dims.d_model)) * scale,
        "w_dq": rng.standard_normal((dims.d_cq, dims.d_model)) * scale,
        "w_uq_qr": rng.standard_normal((n_h * (d_h + d_r), dims.d_cq)) * scale,
        "w_uk": rng.standard_normal((n_h * d_h, dims.d_c)) * scale,
        "w_uv": rng.standard_normal((n_h * d_h, dims.d_c)) * scale,
        "w_o": rng.standard_normal((dims.d_model, n_h * d_h)) * scale,
    }


# ----------------------------------------------------------------------------- softmax
def test_softmax_worked_example_from_routing_section():
    """DeepSeek-V2 from Scratch, §8.2: the printed exponentials, their sum and the 8 probabilities.

    The page divides its 3-decimal exponentials by the 3-decimal sum and rounds again, so its
    fifth probability reads 0.107 where the exact value is 0.10650 - 1e-6; the probabilities
    are therefore compared to 6e-4 (half a unit in the last printed place plus that slack).
    """
    g = read_golden("softmax_worked_example.txt")
    z = np.array(g["z"])
    assert np.round(np.exp(z), 3).tolist() == pytest.approx(g["exp"], abs=1e-9)
    assert round(float(np.exp(z).sum()), 3) == pytest.approx(g["sum"], abs=1e-9)
    s = O.softmax(z)
    assert s.tolist() == pytest.approx(g["s"], abs=6e-4)
    assert (np.array(g["exp"]) / g["sum"]).round(3).tolist() == pytest.approx(g["s"], abs=1e-9)
    assert float(s.sum()) == pytest.approx(g["s_total"], abs=1e-15)
    assert round(float(np.sum(g["s"])), 3) == pytest.approx(g["s_total"], abs=1e-9)


def test_softmax_rows_sum_to_one_and_shift_invariant():
    """§8.2 states the softmax over all experts sums to 1; softmax is invariant to a shift."""
    rng = np.random.default_rng(1)
    z = rng.standard_normal((7, 33)) * 40.0
    s = O.softmax(z, axis=1)
    np.testing.assert_allclose(s.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    np.testing.assert_allclose(O.softmax(z + 123.0, axis=1), s, rtol=1e-12, atol=0)
    assert (s >= 0).all()


# ----------------------------------------------------------------------------- cache sizes
def test_cache_sizes_match_the_pages():
    """§1, §2, §4.5, §7 of the from-scratch page and the visual explainer's 576 / 32,768."""
    g = read_golden("cache_sizes.txt")
    r, p = RUNNING, PRODUCTION
    assert O.mha_cache_elems(r.n_heads, r.d_head) == g["running.mha_per_layer"]
    assert O.mha_cache_elems(r.n_heads, r.d_head) * 12 == g["running.mha_12_layers"]
    assert O.mha_cache_elems(r.n_heads, r.d_head) * 12 * 2 == g["running.mha_12_layers_fp16_bytes"]
    assert r.d_c == g["running.mla_first_attempt_per_layer"]
    assert O.mla_cache_elems(r.d_c, r.d_rope) == g["running.mla_per_layer"]
    assert O.mla_cache_elems(r.d_c, r.d_rope) * 12 == g["running.mla_12_layers"]
    assert O.mla_cache_elems(r.d_c, r.d_rope) * 12 * 2 == g["running.mla_12_layers_fp16_bytes"]
    assert O.gqa_equivalent_groups(r.d_c, r.d_rope, r.d_head) == g["running.gqa_equivalent_groups"]
    assert O.gqa_cache_elems(2, r.d_head) == g["running.gqa2_per_layer"]
    assert O.gqa_cache_elems(1, r.d_head) == g["running.mqa_per_layer"]
    assert O.mla_cache_elems(p.d_c, p.d_rope) == g["production.mla_per_layer"]
    assert O.mha_cache_elems(p.n_heads, p.d_head) == g["production.mha_per_layer"]
    assert O.gqa_equivalent_groups(p.d_c, p.d_rope, p.d_head) == g["production.gqa_equivalent_groups"]
    assert O.mha_cache_elems(p.n_heads, p.d_head) * 60 == g["production.mha_60_layers"]
    assert O.mla_cache_elems(p.d_c, p.d_rope) * 60 == g["production.mla_60_layers"]
    assert round(g["production.mha_60_layers"] / g["production.mla_60_layers"], 1) == g["production.reduction_factor"]
    # 3.75 KB vs 24 KB and the 1/8 ratio of the first attempt
    assert g["running.mla_12_layers_fp16_bytes"] / 1024 == 3.75
    assert g["running.mla_first_attempt_per_layer"] / g["running.mha_per_layer"] == 1 / 8
    assert 512 * 2 == g["toy.kv_bytes"] and 64 * 2 == g["toy.latent_bytes"]


# ----------------------------------------------------------------------------- RoPE
def test_rope_is_identity_at_position_zero():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 64))
    np.testing.assert_array_equal(O.rope(x, np.zeros(5), 10000.0), x)


def test_rope_preserves_norms_it_is_a_rotation():
    """§3.1: RoPE applies a rotation matrix; rotations preserve lengths."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((50, 64))
    pos = rng.integers(0, 140_000, size=50)
    y = O.rope(x, pos, 10000.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


def test_rope_scores_depend_only_on_relative_position():
    """§3.1: RoPE(q, t) . RoPE(k, j) depends only on t - j."""
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal((2, 32))
    for t, j in [(7, 3), (4096, 17), (131072, 5)]:
        ref = O.rope(q, t, 10000.0) @ O.rope(k, j, 10000.0)
        for delta in (1, 999, 65536):
            got = O.rope(q, t + delta, 10000.0) @ O.rope(k, j + delta, 10000.0)
            assert got == pytest.approx(ref, abs=1e-9)


def test_rope_equals_complex_rotation():
    """The 2x2 rotation of a pair is multiplication of x_2k + i x_2k+1 by e^{i t theta_k}."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((9, 64))
    pos = np.array([0, 1, 2, 63, 64, 4095, 4096, 131071, 131072])
    theta = 10000.0 ** (-np.arange(32) * 2.0 / 64)
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * pos[:, None] * theta)
    y = O.rope(x, pos, 10000.0)
    np.testing.assert_allclose(y[:, 0::2], z.real, atol=1e-12)
    np.testing.assert_allclose(y[:, 1::2], z.imag, atol=1e-12)


def test_rope_frequency_closed_forms():
    th = O.rope_frequencies(64, 10000.0)
    assert th[0] == 1.0 and th[16] == pytest.approx(0.01, rel=1e-15)
    assert th[-1] == pytest.approx(10000.0 ** (-62 / 64), rel=1e-15)
    # a quarter turn of the first pair at position pi/2 of theta_0 = 1 is not an integer, so use
    # the rotation direction on pair 0 at t = 1: (1, 0) -> (cos 1, sin 1)
    e = np.zeros(64)
    e[0] = 1.0
    y = O.rope(e, 1, 10000.0)
    assert y[0] == pytest.approx(math.cos(1.0)) and y[1] == pytest.approx(math.sin(1.0))


def test_rope_with_a_caller_table():
    """A caller-supplied frequency table (reading R9): the default table reproduces the base formula
    exactly; any table is still a rotation whose scores depend only on t - j; pair k turns by
    t * table[k] (checked on unit vectors); and a table that differs changes k^R and q^R."""
    rng = np.random.default_rng(6)
    x = rng.standard_normal((7, 64))
    pos = np.array([0, 1, 63, 4096, 40000, 131071, 131072])
    np.testing.assert_array_equal(O.rope(x, pos, 10000.0, O.rope_frequencies(64, 10000.0)), O.rope(x, pos, 10000.0))
    table = np.asarray(synth.yarn_inv_freq(64, 10000.0))
    y = O.rope(x, pos, 10000.0, table)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    q, k = rng.standard_normal((2, 64))
    ref = O.rope(q, 4100, 10000.0, table) @ O.rope(k, 17, 10000.0, table)
    assert O.rope(q, 4100 + 90000, 10000.0, table) @ O.rope(k, 17 + 90000, 10000.0, table) == pytest.approx(ref,
                                                                                                             abs=1e-9)
    for kk in (0, 13, 31):
        e = np.zeros(64)
        e[2 * kk] = 1.0
        yy = O.rope(e, 1000, 10000.0, table)
        assert yy[2 * kk] == pytest.approx(math.cos(1000 * table[kk]), abs=1e-12)
        assert yy[2 * kk + 1] == pytest.approx(math.sin(1000 * table[kk]), abs=1e-12)
    assert np.abs(y - O.rope(x, pos, 10000.0)).max() > 0.1
    # the example table keeps the fastest pairs and divides the slowest by the factor
    base = O.rope_frequencies(64, 10000.0)
    assert table[0] == base[0] and table[-1] == pytest.approx(base[-1] / 40.0, rel=1e-15)
    # the projections read the table from the dims
    d = synth.RUNNING.with_(rope_inv_freq=tuple(synth.yarn_inv_freq(32, 10000.0)))
    w = rng.standard_normal((d.D, d.d_model)) * 0.02
    h = rng.standard_normal((2, d.d_model))
    rows = O.kv_rows(w, h, [5000, 7], d)
    np.testing.assert_allclose(rows[:, d.d_c:], O.rope(h @ w[d.d_c:].T, np.array([5000, 7]), 10000.0,
                                                       d.rope_inv_freq), atol=1e-12)


# ----------------------------------------------------------------------------- attention
def _sdpa(q, k, v, scale=None):
    """torch's library attention on float64 CPU tensors (one query row per head)."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    return torch.nn.functional.scaled_dot_product_attention(
        t(q)[:, None, :], t(k), t(v), scale=scale)[:, 0, :].numpy()


@pytest.mark.parametrize("dims", [TINY, RUNNING], ids=["tiny", "running"])
def test_naive_attention_equals_library_sdpa(dims):
    """§4.3-§4.4: per-head softmax over [q^C; q^R].[k^C; k^R] with scale 1/sqrt(d_h + d_h^R).

    torch's scaled_dot_product_attention with its default scale 1/sqrt(query width) is the
    textbook routine on the concatenated query/key of width d_h + d_h^R.
    """
    rng = np.random.default_rng(6)
    W = rand_weights(dims, rng, scale=0.5)
    L = 37
    rows = rng.standard_normal((L, dims.D))
    q_c = rng.standard_normal((dims.n_heads, dims.d_head))
    q_r = rng.standard_normal((dims.n_heads, dims.d_rope))
    o = O.attention_naive(q_c, q_r, rows, W["w_uk"], W["w_uv"], dims)
    n_h, d_h = dims.n_heads, dims.d_head
    k_c = (rows[:, :dims.d_c] @ W["w_uk"].T).reshape(L, n_h, d_h).transpose(1, 0, 2)
    v_c = (rows[:, :dims.d_c] @ W["w_uv"].T).reshape(L, n_h, d_h).transpose(1, 0, 2)
    k = np.concatenate([k_c, np.broadcast_to(rows[None, :, dims.d_c:], (n_h, L, dims.d_rope))], -1)
    q = np.concatenate([q_c, q_r], -1)
    np.testing.assert_allclose(o, _sdpa(q, k, v_c), rtol=1e-11, atol=1e-13)


def test_without_rope_branch_it_is_textbook_mha_on_rebuilt_keys():
    """§2.2 / §1: with W^QR = W^KR = 0 the score is q^C . W^UK c only; MHA with K = W^UK c, V = W^UV c.

    The softmax scale stays 1/sqrt(d_h + d_h^R) (§4.4), passed explicitly to the library call.
    """
    dims = RUNNING
    rng = np.random.default_rng(7)
    W = rand_weights(dims, rng, scale=0.05)
    W["w_dkv_kr"][dims.d_c:] = 0.0
    W["w_uq_qr"][dims.n_heads * dims.d_head:] = 0.0
    prefix = [rng.standard_normal((11, dims.D)) * 0.4]
    prefix[0][:, dims.d_c:] = 0.0
    h = rng.standard_normal((1, dims.d_model))
    out = O.layer_step_naive(W, h, prefix, dims)
    rows = np.vstack([prefix[0], out["rows"]])
    L, n_h, d_h = rows.shape[0], dims.n_heads, dims.d_head
    k = (rows[:, :dims.d_c] @ W["w_uk"].T).reshape(L, n_h, d_h).transpose(1, 0, 2)
    v = (rows[:, :dims.d_c] @ W["w_uv"].T).reshape(L, n_h, d_h).transpose(1, 0, 2)
    q = out["q_c"][0]
    o_ref = _sdpa(q, k, v, scale=1.0 / math.sqrt(dims.d_head + dims.d_rope))
    np.testing.assert_allclose(out["o"][0], o_ref, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(out["u"][0], o_ref.reshape(-1) @ W["w_o"].T, rtol=1e-11, atol=1e-12)


def test_identity_head_is_single_head_attention_over_the_latent():
    """One head, d_c = d_h, W^UK = W^UV = I: keys and values are the latent rows themselves."""
    dims = Dims(d_model=8, n_heads=1, d_head=6, d_c=6, d_cq=4, d_rope=2, rope_base=10000.0)
    rng = np.random.default_rng(8)
    rows = rng.standard_normal((9, dims.D))
    q = rng.standard_normal((1, dims.D))
    o_lat, _ = O.latent_attention(q, rows, dims)
    ref = _sdpa(q, rows[None], rows[None, :, :dims.d_c], scale=1 / math.sqrt(dims.d_head + dims.d_rope))
    np.testing.assert_allclose(o_lat, ref, rtol=1e-12)
    o = O.attention_naive(q[:, :6], q[:, 6:], rows, np.eye(6), np.eye(6), dims)
    np.testing.assert_allclose(o, ref, rtol=1e-12)


# ----------------------------------------------------------------------------- absorption (§5)
@pytest.mark.parametrize("dims", [TINY, RUNNING], ids=["tiny", "running"])
def test_absorbed_equals_naive(dims):
    """§5.1-§5.3 and the explainer: absorbing W^UK into the query and W^UV into W^O is exact."""
    rng = np.random.default_rng(9)
    W = rand_weights(dims, rng, scale=0.2)
    prefix = [rng.standard_normal((n, dims.D)) for n in (0, 1, 5, 63, 64, 130)]
    h = rng.standard_normal((len(prefix), dims.d_model))
    naive = O.layer_step_naive(W, h, prefix, dims)
    absd = O.layer_step_absorbed(W, h, prefix, dims)
    np.testing.assert_allclose(absd["rows"], naive["rows"], rtol=1e-14)
    np.testing.assert_allclose(absd["q"][..., dims.d_c:], naive["q_r"], rtol=1e-14)
    # per-head value outputs: o_i = W^UV_i o_lat_i
    w_uv = W["w_uv"].reshape(dims.n_heads, dims.d_head, dims.d_c)
    o_from_lat = np.einsum("irm,bim->bir", w_uv, absd["o_lat"])
    scale_o = np.abs(naive["o"]).max()
    np.testing.assert_allclose(o_from_lat, naive["o"], rtol=0, atol=1e-12 * scale_o)
    scale_u = np.abs(naive["u"]).max()
    np.testing.assert_allclose(absd["u"], naive["u"], rtol=0, atol=1e-12 * scale_u)


def test_content_score_identity_per_head():
    """§5.1: (q^C_i)^T W^UK_i c = ((W^UK_i)^T q^C_i)^T c for every head and cached latent."""
    dims = RUNNING
    rng = np.random.default_rng(10)
    W = rand_weights(dims, rng)
    h = rng.standard_normal((3, dims.d_model))
    pos = np.array([0, 5, 4096])
    q = O.absorb_query(W["w_dq"], W["w_uq_qr"], W["w_uk"], h, pos, dims)
    _, q_c, _ = O.query_path(W["w_dq"], W["w_uq_qr"], h, pos, dims)
    c = rng.standard_normal((17, dims.d_c))
    k_c = (c @ W["w_uk"].T).reshape(17, dims.n_heads, dims.d_head)
    lhs = np.einsum("bik,jik->bij", q_c, k_c)
    rhs = np.einsum("bim,jm->bij", q[..., :dims.d_c], c)
    np.testing.assert_allclose(rhs, lhs, rtol=1e-11, atol=1e-12)


# ----------------------------------------------------------------------------- special cases
def test_single_token_attends_to_itself():
    """N = 0: the only key is the new token's own row, so o_lat = c_t and u = sum_i W^O_i W^UV_i c_t."""
    dims = RUNNING
    rng = np.random.default_rng(11)
    W = rand_weights(dims, rng, scale=0.1)
    h = rng.standard_normal((2, dims.d_model))
    out = O.layer_step_absorbed(W, h, [np.zeros((0, dims.D))] * 2, dims)
    np.testing.assert_allclose(out["o_lat"], np.repeat(out["rows"][:, None, :dims.d_c], dims.n_heads, 1), rtol=1e-15)
    c_t = out["rows"][:, :dims.d_c]
    w_o = W["w_o"].reshape(dims.d_model, dims.n_heads, dims.d_head)
    w_uv = W["w_uv"].reshape(dims.n_heads, dims.d_head, dims.d_c)
    u = sum(w_o[:, i, :] @ w_uv[i] @ c_t.T for i in range(dims.n_heads)).T
    tol = 1e-12 * np.abs(u).max()
    np.testing.assert_allclose(out["u"], u, rtol=0, atol=tol)
    naive = O.layer_step_naive(W, h, [np.zeros((0, dims.D))] * 2, dims)
    np.testing.assert_allclose(naive["u"], u, rtol=0, atol=tol)


def test_zero_query_gives_the_mean_latent():
    """q~ = 0 and q^R = 0: every score is 0, the weights are uniform and o_lat is the mean of c_j."""
    dims = PRODUCTION
    rng = np.random.default_rng(12)
    rows = rng.standard_normal((301, dims.D))
    o_lat, lse = O.latent_attention(np.zeros((dims.n_heads, dims.D)), rows, dims)
    np.testing.assert_allclose(o_lat, np.broadcast_to(rows[:, :dims.d_c].mean(0), o_lat.shape), rtol=1e-12)
    np.testing.assert_allclose(lse, math.log(301), rtol=1e-15)


def test_latent_attention_lse_and_weights_against_scipy():
    """§5.3 steps 2-3 with the §4.4 scale through scipy's logsumexp and softmax: the log-sum-exp
    (natural log, over the scaled scores) and the weighted sum of latents, on scores wide enough
    that a missing max shift would overflow."""
    import scipy.special as sp
    dims = PRODUCTION
    rng = np.random.default_rng(16)
    rows = rng.standard_normal((97, dims.D))
    q = rng.standard_normal((dims.n_heads, dims.D)) * 120.0
    o_lat, lse = O.latent_attention(q, rows, dims)
    s = (q @ rows.T) / math.sqrt(dims.d_head + dims.d_rope)
    assert np.abs(s).max() > 710.0                       # exp would overflow without the shift
    np.testing.assert_allclose(lse, sp.logsumexp(s, axis=1), rtol=1e-14)
    np.testing.assert_allclose(o_lat, sp.softmax(s, axis=1) @ rows[:, :dims.d_c], rtol=1e-10, atol=1e-12)


def test_all_equal_rows_return_that_row():
    dims = RUNNING
    rng = np.random.default_rng(13)
    row = rng.standard_normal(dims.D)
    q = rng.standard_normal((dims.n_heads, dims.D)) * 50
    o_lat, _ = O.latent_attention(q, np.tile(row, (40, 1)), dims)
    np.testing.assert_allclose(o_lat, np.broadcast_to(row[:dims.d_c], o_lat.shape), rtol=1e-13)


def test_heads_are_contiguous_row_blocks():
    """§2.2 / §4.1: [k_1; ...; k_n_h] = k splits W^UK and W^UQ by contiguous row blocks of d_h,
    and u = W^O [o_1; ...; o_n_h] reads column block i for head i (§1)."""
    dims = RUNNING
    rng = np.random.default_rng(14)
    W = rand_weights(dims, rng, scale=0.3)
    n_h, d_h = dims.n_heads, dims.d_head
    keep = 2
    mask = np.zeros(n_h * d_h, bool)
    mask[keep * d_h:(keep + 1) * d_h] = True
    W["w_uk"][~mask] = 0.0                       # only head 2 rebuilds a content key
    W["w_uq_qr"][n_h * d_h:] = 0.0               # no positional query anywhere
    prefix = [rng.standard_normal((20, dims.D))]
    h = rng.standard_normal((1, dims.d_model))
    q = O.absorb_query(W["w_dq"], W["w_uq_qr"], W["w_uk"], h, np.array([20]), dims)
    rows = np.vstack([prefix[0], O.kv_rows(W["w_dkv_kr"], h, [20], dims)])
    o_lat, lse = O.latent_attention(q[0], rows, dims)
    mean = rows[:, :dims.d_c].mean(0)
    for i in range(n_h):
        if i == keep:
            assert np.abs(o_lat[i] - mean).max() > 1e-3
        else:
            np.testing.assert_allclose(o_lat[i], mean, rtol=1e-12)
    # W^O column block i only: u depends on head i alone
    w_o = np.zeros_like(W["w_o"])
    w_o[:, keep * d_h:(keep + 1) * d_h] = W["w_o"][:, keep * d_h:(keep + 1) * d_h]
    o_lat2 = o_lat.copy()
    o_lat2[np.arange(n_h) != keep] = rng.standard_normal((n_h - 1, dims.d_c))
    np.testing.assert_allclose(O.out_proj_absorbed(W["w_uv"], w_o, o_lat[None]),
                               O.out_proj_absorbed(W["w_uv"], w_o, o_lat2[None]), rtol=1e-14)


# ----------------------------------------------------------------------------- split-KV merge
@pytest.mark.parametrize("splits", [1, 2, 3, 7])
def test_split_merge_equals_single_pass(splits):
    """Exact softmax algebra: partials over disjoint token ranges merge to the one-pass result."""
    dims = PRODUCTION
    rng = np.random.default_rng(15 + splits)
    rows = rng.standard_normal((257, dims.D)) * 0.4
    q = rng.standard_normal((dims.n_heads, dims.D)) * 3.0
    o_ref, lse_ref = O.latent_attention(q, rows, dims)
    cuts = np.unique(np.concatenate([[0, 257], rng.choice(np.arange(1, 257), splits - 1, replace=False)]))
    parts = [O.latent_attention(q, rows[a:b], dims) for a, b in zip(cuts[:-1], cuts[1:])]
    o, lse = O.lse_merge([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-13)


# ----------------------------------------------------------------------------- paged layout
def test_page_slot_matches_walking_the_block_table():
    rng = np.random.default_rng(16)
    P = 4
    lens = [1, 4, 5, 17]
    need = [(n + P - 1) // P for n in lens]
    perm = rng.permutation(sum(need))
    bt = np.full((4, max(need)), -1)
    walk = {}
    off = 0
    for b, n in enumerate(need):
        bt[b, :n] = perm[off:off + n]
        off += n
        tok = 0
        for pg in bt[b, :n]:                      # walk pages in logical order
            for s in range(P):
                walk[(b, tok)] = pg * P + s
                tok += 1
    for b, n in enumerate(lens):
        got = O.page_slot(bt, b, np.arange(n), P)
        assert got.tolist() == [walk[(b, t)] for t in range(n)]


# ----------------------------------------------------------------------------- brute force
def _rot(t, theta):
    """Full block-diagonal rotation matrix R(t) built entry by entry."""
    n = 2 * len(theta)
    R = [[0.0] * n for _ in range(n)]
    for k, th in enumerate(theta):
        c, s = math.cos(t * th), math.sin(t * th)
        R[2 * k][2 * k], R[2 * k][2 * k + 1] = c, -s
        R[2 * k + 1][2 * k], R[2 * k + 1][2 * k + 1] = s, c
    return R


def _mv(A, x):
    return [sum(A[r][c] * x[c] for c in range(len(x))) for r in range(len(A))]


def test_brute_force_scalar_loops_on_tiny_shapes():
    """§6 evaluated with scalar Python loops, explicit rotation matrices and math.exp."""
    dims = Dims(d_model=5, n_heads=2, d_head=2, d_c=4, d_cq=3, d_rope=2, rope_base=10.0)
    rng = np.random.default_rng(17)
    W = rand_weights(dims, rng, scale=0.7)
    prefix = [rng.standard_normal((n, dims.D)) for n in (0, 3, 5)]
    h = rng.standard_normal((3, dims.d_model))
    out = O.layer_step_naive(W, h, prefix, dims)
    theta = [dims.rope_base ** (-2 * k / dims.d_rope) for k in range(dims.d_rope // 2)]
    Wl = {k: v.tolist() for k, v in W.items()}
    n_h, d_h, d_c, d_r = dims.n_heads, dims.d_head, dims.d_c, dims.d_rope
    for b in range(3):
        t = len(prefix[b])
        hb = h[b].tolist()
        c_t = _mv(Wl["w_dkv_kr"][:d_c], hb)
        kr_t = _mv(_rot(t, theta), _mv(Wl["w_dkv_kr"][d_c:], hb))
        rows = [list(r) for r in prefix[b].tolist()] + [c_t + kr_t]
        c_q = _mv(Wl["w_dq"], hb)
        q_c = _mv(Wl["w_uq_qr"][:n_h * d_h], c_q)
        q_rh = _mv(Wl["w_uq_qr"][n_h * d_h:], c_q)
        o_all = []
        for i in range(n_h):
            qi = q_c[i * d_h:(i + 1) * d_h] + _mv(_rot(t, theta), q_rh[i * d_r:(i + 1) * d_r])
            scores, vals = [], []
            for r in rows:
                k_c = _mv(Wl["w_uk"][i * d_h:(i + 1) * d_h], r[:d_c])
                v_c = _mv(Wl["w_uv"][i * d_h:(i + 1) * d_h], r[:d_c])
                ki = k_c + r[d_c:]
                scores.append(sum(a * b_ for a, b_ in zip(qi, ki)) / math.sqrt(d_h + d_r))
                vals.append(v_c)
            mx = max(scores)
            ex = [math.exp(s - mx) for s in scores]
            z = sum(ex)
            o_i = [sum(ex[j] * vals[j][e] for j in range(len(rows))) / z for e in range(d_h)]
            np.testing.assert_allclose(out["o"][b, i], o_i, rtol=1e-12, atol=1e-14)
            o_all += o_i
        u = _mv(Wl["w_o"], o_all)
        np.testing.assert_allclose(out["u"][b], u, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(out["rows"][b], c_t + kr_t, rtol=1e-13, atol=1e-15)


def test_pins_catch_planted_mistakes():
    """A pin set that a plausible slip passes is no pin: plant slips in copies of the oracle."""
    dims = RUNNING
    rng = np.random.default_rng(18)
    W = rand_weights(dims, rng, scale=0.2)
    prefix = [rng.standard_normal((9, dims.D))]
    h = rng.standard_normal((1, dims.d_model))
    good = O.layer_step_naive(W, h, prefix, dims)
    # (a) scale 1/sqrt(d_h) instead of 1/sqrt(d_h + d_h^R): SDPA's default scale disagrees
    rows = np.vstack([prefix[0], good["rows"]])
    q = np.concatenate([good["q_c"][0], good["q_r"][0]], -1)
    n_h, d_h, L = dims.n_heads, dims.d_head, rows.shape[0]
    k_c = (rows[:, :dims.d_c] @ W["w_uk"].T).reshape(L, n_h, d_h).transpose(1, 0, 2)
    v_c = (rows[:, :dims.d_c] @ W["w_uv"].T).reshape(L, n_h, d_h).transpose(1, 0, 2)
    k = np.concatenate([k_c, np.broadcast_to(rows[None, :, dims.d_c:], (n_h, L, dims.d_rope))], -1)
    wrong_scale = _sdpa(q, k, v_c, scale=1 / math.sqrt(d_h))
    assert np.abs(wrong_scale - good["o"][0]).max() > 1e-6
    # (b) a sign slip in the rotation breaks the complex-rotation pin
    x = rng.standard_normal((3, 64))
    theta = 10000.0 ** (-np.arange(32) * 2.0 / 64)
    phi = np.array([5, 6, 7])[:, None] * theta
    y_bad = np.empty_like(x)                       # rotation by -phi (sign slip on sin)
    y_bad[:, 0::2] = x[:, 0::2] * np.cos(phi) + x[:, 1::2] * np.sin(phi)
    y_bad[:, 1::2] = -x[:, 0::2] * np.sin(phi) + x[:, 1::2] * np.cos(phi)
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * phi)
    assert np.abs(y_bad[:, 1::2] - z.imag).max() > 1e-3
    assert np.abs(O.rope(x, [5, 6, 7], 10000.0)[:, 1::2] - z.imag).max() < 1e-12
    # (c) a transposed head split (interleaved rows) breaks absorbed == naive
    W2 = {k: v.copy() for k, v in W.items()}
    perm = np.arange(n_h * d_h).reshape(n_h, d_h).T.reshape(-1)
    q_abs = O.absorb_query(W2["w_dq"], W2["w_uq_qr"], W2["w_uk"][perm], h, [9], dims)
    o_lat, _ = O.latent_attention(q_abs[0], rows, dims)
    u_bad = O.out_proj_absorbed(W["w_uv"], W["w_o"], o_lat[None])
    assert np.abs(u_bad - good["u"]).max() > 1e-6 * np.abs(good["u"]).max()


# ----------------------------------------------------------------------------- multi-token step
CHUNK_CASES = [([0, 3, 5], [4, 1, 3]), ([2], [6]), ([0], [1]), ([7, 0], [0, 2])]


@pytest.mark.parametrize("dims", [TINY, RUNNING], ids=["tiny", "running"])
@pytest.mark.parametrize("prefix_lens,chunk_lens", CHUNK_CASES)
def test_chunk_equals_one_token_at_a_time(dims, prefix_lens, chunk_lens):
    """§6 with a general t: a step that brings q tokens of a sequence at once gives each of them
    what q single-token decode steps give, taken in position order, each appending its own row
    before it attends (causal: a token never sees a later one)."""
    rng = np.random.default_rng(21)
    W = rand_weights(dims, rng, scale=0.5)
    prefix = [rng.standard_normal((n, dims.D)) for n in prefix_lens]
    seq_idx, pos = O.chunk_positions(prefix_lens, chunk_lens)
    h = rng.standard_normal((len(pos), dims.d_model))
    got = O.chunk_step_naive(W, h, prefix, chunk_lens, dims)
    grown = [p.copy() for p in prefix]
    for t in range(len(pos)):
        b = int(seq_idx[t])
        assert pos[t] == len(grown[b])
        one = O.layer_step_naive(W, h[t:t + 1], [grown[b]], dims)
        np.testing.assert_allclose(got["rows"][t], one["rows"][0], rtol=1e-12, atol=1e-14)
        # fp64 roundoff only: the two routes multiply matrices of different shapes
        np.testing.assert_allclose(got["o"][t], one["o"][0], rtol=0, atol=1e-10 * np.abs(one["o"]).max())
        np.testing.assert_allclose(got["u"][t], one["u"][0], rtol=0, atol=1e-10 * np.abs(one["u"]).max())
        grown[b] = np.vstack([grown[b], one["rows"]])


@pytest.mark.parametrize("dims", [TINY, RUNNING], ids=["tiny", "running"])
def test_chunk_absorbed_equals_naive(dims):
    """§5.1-§5.3 hold token by token, so the absorbed multi-token step equals the naive one."""
    rng = np.random.default_rng(22)
    W = rand_weights(dims, rng, scale=0.5)
    prefix_lens, chunk_lens = [0, 3, 5], [4, 1, 3]
    prefix = [rng.standard_normal((n, dims.D)) for n in prefix_lens]
    h = rng.standard_normal((sum(chunk_lens), dims.d_model))
    naive = O.chunk_step_naive(W, h, prefix, chunk_lens, dims)
    absorbed = O.chunk_step_absorbed(W, h, prefix, chunk_lens, dims)
    np.testing.assert_array_equal(naive["pos"], absorbed["pos"])
    np.testing.assert_allclose(absorbed["u"], naive["u"], rtol=1e-10, atol=1e-12 * np.abs(naive["u"]).max())


def test_chunk_attention_equals_library_sdpa_with_a_causal_mask():
    """torch's scaled_dot_product_attention with a boolean mask that admits key j for query t
    exactly when j <= pos[t] gives the absorbed chunk attention (values = the latents)."""
    dims = RUNNING
    rng = np.random.default_rng(23)
    L, q_len = 29, 6
    rows = rng.standard_normal((L, dims.D))
    pos = np.arange(L - q_len, L)
    q = rng.standard_normal((q_len, dims.n_heads, dims.D)) * 0.3
    o_lat, _ = O.chunk_latent_attention(q, [rows], np.zeros(q_len, dtype=np.int64), pos, dims)
    mask = torch.from_numpy(np.arange(L)[None, :] <= pos[:, None])
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    ref = torch.nn.functional.scaled_dot_product_attention(
        t(q.transpose(1, 0, 2)), t(rows)[None], t(rows[:, :dims.d_c])[None], attn_mask=mask,
        scale=1.0 / math.sqrt(dims.d_head + dims.d_rope)).numpy().transpose(1, 0, 2)
    np.testing.assert_allclose(o_lat, ref, rtol=1e-11, atol=1e-13)


def test_chunk_first_token_of_an_empty_sequence_sees_only_itself():
    """At position 0 the softmax runs over one row, so o_lat is that token's own latent and the
    log-sum-exp its own scaled score (§4.4 with a single term)."""
    dims = RUNNING
    rng = np.random.default_rng(24)
    W = rand_weights(dims, rng, scale=0.5)
    h = rng.standard_normal((3, dims.d_model))
    out = O.chunk_step_absorbed(W, h, [np.zeros((0, dims.D))], [3], dims)
    np.testing.assert_allclose(out["o_lat"][0], np.broadcast_to(out["rows"][0, :dims.d_c], (dims.n_heads, dims.d_c)),
                               rtol=1e-13, atol=1e-14)
    s0 = out["q"][0] @ out["rows"][0] / math.sqrt(dims.d_head + dims.d_rope)
    np.testing.assert_allclose(out["lse"][0], s0, rtol=1e-12, atol=1e-14)


def test_chunk_pins_catch_a_causal_off_by_one():
    """An attention bound one row short (the token misses itself) or one row long (it sees the
    next token) breaks the token-at-a-time pin; the correct bound passes it."""
    dims = RUNNING
    rng = np.random.default_rng(25)
    W = rand_weights(dims, rng, scale=0.5)
    prefix = [rng.standard_normal((4, dims.D))]
    h = rng.standard_normal((3, dims.d_model))
    good = O.chunk_step_absorbed(W, h, prefix, [3], dims)
    full = np.vstack([prefix[0], good["rows"]])
    seq0 = np.zeros(3, dtype=np.int64)
    step = O.layer_step_absorbed(W, h[1:2], [full[:5]], dims)     # the middle token, decoded alone
    for shift, ok in ((0, True), (-1, False), (1, False)):
        o_lat, _ = O.chunk_latent_attention(good["q"], [full], seq0, good["pos"] + shift, dims)
        err = np.abs(o_lat[1] - step["o_lat"][0]).max()
        assert (err < 1e-12) if ok else (err > 1e-6)


# ----------------------------------------------------------------------------- FP8 latent cache
def _torch_e4m3(y):
    return torch.from_numpy(np.asarray(y, dtype=np.float32)).to(torch.float8_e4m3fn).double().numpy()


def test_e4m3_decoding_matches_the_library_format():
    """The 256 codes decoded from the format's fields equal torch's float8_e4m3fn bytes; closed
    forms: largest 448, smallest normal 2^-6, smallest subnormal 2^-9, NaN only at S.1111.111."""
    v = O.e4m3_values()
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(np.isnan(v), np.isnan(lib))
    np.testing.assert_array_equal(v[~np.isnan(v)], lib[~np.isnan(lib)])
    assert np.flatnonzero(np.isnan(v)).tolist() == [127, 255]
    assert np.nanmax(v) == O.E4M3_MAX == 448.0
    assert v[0b00001000] == 2.0 ** -6 and v[1] == 2.0 ** -9


def test_e4m3_rounding_nearest_even_against_the_library_and_brute_force():
    """Every value, every midpoint between neighbours (ties go to the even fraction) and random
    values across the normal and subnormal range round as torch's conversion does, and as an
    exhaustive nearest-value search with ties to the even code does."""
    v = O.e4m3_values()
    pos = np.unique(v[(~np.isnan(v)) & (v >= 0)])
    mids = (pos[1:] + pos[:-1]) / 2
    rng = np.random.default_rng(40)
    rnd = np.concatenate([rng.uniform(-448, 448, 2000), rng.uniform(-2 ** -5, 2 ** -5, 2000),
                          np.exp2(rng.uniform(-12, 8.8, 2000)) * rng.choice([-1, 1], 2000)])
    rnd = rnd[np.abs(rnd) <= 448]
    for y in (pos, -pos, mids, -mids, rnd):
        y32 = y.astype(np.float32).astype(np.float64)        # the quantiser sees float32 inputs
        np.testing.assert_array_equal(O.quantize_e4m3(y32), _torch_e4m3(y32))
    finite = np.flatnonzero(~np.isnan(v))
    for y in rnd[:300].astype(np.float32).astype(np.float64):
        d = np.abs(v[finite] - y)
        best = finite[d == d.min()]
        code = best[0] if len(best) == 1 else best[(best & 1) == 0][0]
        assert O.quantize_e4m3(y) == v[code], y
    np.testing.assert_array_equal(O.quantize_e4m3(pos), pos)  # representable values are fixed points


def test_fp8_rows_error_bound_scales_and_zero_parts():
    """Per token and part, max|part| maps to 448 and every value is within half an e4m3 spacing:
    2^-4 of its magnitude for normals, 2^-10 of the scale for subnormals (plus float32 division
    rounding). An all-zero part gets scale 1 and zero values."""
    d = PRODUCTION
    rng = np.random.default_rng(41)
    rows = (rng.standard_normal((50, d.D)) * np.exp2(rng.uniform(-6, 6, (50, 1)))).astype(np.float32)
    rows[3, d.d_c:] = 0.0
    rows[4, :d.d_c] = 0.0
    vals, sc = O.quantize_rows_fp8(rows, d.d_c)
    assert sc.dtype == np.float32 and sc.shape == (50, 2)
    assert sc[3, 1] == 1.0 and sc[4, 0] == 1.0
    assert not vals[3, d.d_c:].any() and not vals[4, :d.d_c].any()
    for j, part in enumerate((slice(0, d.d_c), slice(d.d_c, d.D))):
        m = np.abs(vals[:, part]).max(axis=1)
        live = np.abs(rows[:, part]).max(axis=1) > 0
        assert np.all(m[live] == 448.0)
        y = rows[:, part].astype(np.float64) / sc[:, j:j + 1].astype(np.float64)
        err = np.abs(vals[:, part] - y)
        bound = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-6) + np.abs(y) * 2.0 ** -23
        assert np.all(err <= bound)
    back = O.dequantize_rows_fp8(vals, sc, d.d_c)
    rel = np.abs(back - rows) / np.maximum(np.abs(rows), 1e-30)
    assert np.median(rel[rows != 0]) < 2.0 ** -5


def test_fp8_pins_catch_ties_away_from_zero():
    """Rounding halves away from zero (a plausible slip) disagrees with the library at midpoints."""
    v = O.e4m3_values()
    pos = np.unique(v[(~np.isnan(v)) & (v >= 0)])
    mids = (pos[1:] + pos[:-1]) / 2
    a = np.abs(mids)
    step = 2.0 ** (np.maximum(np.floor(np.log2(a)), -6.0) - 3.0)
    away = np.floor(a / step + 0.5) * step
    assert np.any(away != _torch_e4m3(mids))
