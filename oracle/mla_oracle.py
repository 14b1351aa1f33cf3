"""CPU fp64 oracle for Multi-head Latent Attention at decode time (one or several new tokens per sequence).

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or execute this
package: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm
of ``bench.py`` use it. It shares no code with the CUDA library (no kernels, headers,
helpers, tables or pre/post-processing); both sides only receive the same seeded inputs.

It is a plain, slow restatement of the method in float64 with numpy. Library matmuls and
``exp``/``log``/``cos``/``sin`` serve as primitives; nothing is blocked, fused or reordered
beyond what the definitions below state.

Sources (page title, section or equation):
  [S1] "DeepSeek-V2 from Scratch: Multi-head Latent Attention and DeepSeekMoE":
       §1 standard MHA and its cache cost; §2.1 the down-projection c^KV = W^DKV h;
       §2.2 up-projections k^C = W^UK c, v^C = W^UV c, split into heads by contiguous row
       blocks; §3.1 RoPE, a position-dependent rotation whose dot products depend only on
       t - j; §4.1 query compression c^Q = W^DQ h, q^C = W^UQ c^Q, q^R = RoPE(W^QR c^Q);
       §4.2 shared RoPE key k^R = RoPE(W^KR h); §4.3 concatenated per-head q and k;
       §4.4 score split and softmax with scale 1/sqrt(d_h + d_h^R); §4.5 what is cached;
       §5.1 absorbing W^UK into the query; §5.2 absorbing W^UV into W^O; §5.3 the four
       absorbed steps; §6 the complete algorithm; §7 cache comparison table;
       §8.2 the worked softmax example.
  [S2] DeepSeek-V2 paper review (velog): §2.1 latency model; §2.3 decoupled RoPE.
  [S4] DeepSeek-V2 visual explainer: 576 vs 32,768 numbers per token; the toy 512 -> 64.
  [S5] "DeepSeek-V2: A Strong, Economical, and Efficient Mixture-of-Experts Language Model
       (Multi-head Latent Attention)" summary: "The Model: DeepSeek-V2" (a 6-bit KV cache and
       FP8 weights in deployment).

Readings where the pages are silent:
  R1 RoPE rotates adjacent pairs (x_2k, x_2k+1) by the standard 2x2 rotation matrix.
  R2 Angle of pair k at position t is t * base^(-2k/d_h^R), formed in float64.
  R3 Positions are 0-based; cached tokens sit at 0..N-1 and the new token at N.
  R4 The new token attends to itself (the sum runs over j <= t).
  R5 No normalisation of the latent (none is given on [S1]).
  R6 Split-KV partials hold the normalised partial output and the log-sum-exp of the
     scaled scores (natural log); merging them is exact softmax algebra.
  R7 A step may bring several new tokens of one sequence (the attention sum of [S1] §6 for a
     general t): they take the consecutive positions after the prefix, all their rows are
     cached first, and each token attends to the rows up to its own position (causal).
  R8 A quantised latent cache ([S2] §4.2 and [S5] give a KV cache of about 6 bits per element
     without its format): e4m3 bytes with two float32 scales per token, max|part| / 448 for c and for k^R,
     values divided by their scale in float32 and rounded to the nearest e4m3 value, ties to
     even. Attention over it is the attention over the rows it stands for.
  R9 The RoPE frequencies may come from the caller ([S2] §4.1 applies YaRN to the decoupled key
     to reach a 128K context; its constants are not on the pages): theta_k is then the table's
     k-th entry, for the query and the key alike; positions and pairing are unchanged.

Every function has pins in ``tests/test_oracle_pins.py``; none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "rope_frequencies", "rope", "softmax", "softmax_scale",
    "mla_cache_elems", "mha_cache_elems", "gqa_cache_elems", "gqa_equivalent_groups",
    "kv_rows", "query_path", "attention_naive", "output_naive", "layer_step_naive",
    "absorb_query", "latent_attention", "lse_merge", "out_proj_absorbed", "layer_step_absorbed",
    "chunk_positions", "chunk_step_naive", "chunk_latent_attention", "chunk_step_absorbed",
    "E4M3_MAX", "e4m3_values", "quantize_e4m3", "fp8_row_scales", "quantize_rows_fp8", "dequantize_rows_fp8",
    "page_slot", "as64",
]


def as64(x) -> np.ndarray:
    """Exact float64 copy of a host tensor/array (bf16 and fp16 convert exactly)."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        if x.is_floating_point():
            x = x.double()
        return x.numpy()
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------- cache sizes
def mla_cache_elems(d_c: int, d_rope: int) -> int:
    """Elements cached per token per layer by MLA: d_c + d_h^R ([S1] §4.5, boxed)."""
    return d_c + d_rope


def mha_cache_elems(n_h: int, d_h: int) -> int:
    """Elements cached per token per layer by MHA: 2 n_h d_h ([S1] §1)."""
    return 2 * n_h * d_h


def gqa_cache_elems(groups: float, d_h: int) -> float:
    """Elements cached per token per layer by GQA with g groups: 2 g d_h ([S1] §4.5, §7)."""
    return 2 * groups * d_h


def gqa_equivalent_groups(d_c: int, d_rope: int, d_h: int) -> float:
    """g with 2 g d_h = d_c + d_h^R ([S1] §4.5, "Comparison with GQA")."""
    return (d_c + d_rope) / (2 * d_h)


# --------------------------------------------------------------------------- primitives
def rope_frequencies(d_rope: int, base: float) -> np.ndarray:
    """theta_k = base^(-2k/d_h^R), k = 0 .. d_h^R/2 - 1 (reading R2)."""
    k = np.arange(d_rope // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * k / d_rope)


def rope(x, pos, base: float, inv_freq=None) -> np.ndarray:
    """RoPE(x, t): rotate each pair (x_2k, x_2k+1) by the angle t * theta_k ([S1] §3.1; R1, R2).

    ``x`` has shape [..., d_R]; ``pos`` broadcasts against ``x.shape[:-1]``. ``inv_freq`` (d_R/2
    values) replaces the base formula for theta_k when given: a caller-supplied table such as
    YaRN's interpolated frequencies ([S2] §4.1; R9).
    """
    x = np.asarray(x, dtype=np.float64)
    pos = np.asarray(pos, dtype=np.float64)
    theta = rope_frequencies(x.shape[-1], base) if inv_freq is None else np.asarray(inv_freq, dtype=np.float64)
    phi = pos[..., None] * theta
    c, s = np.cos(phi), np.sin(phi)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = np.empty(np.broadcast_shapes(x.shape, phi.shape[:-1] + (x.shape[-1],)), dtype=np.float64)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x0 * s + x1 * c
    return y


def softmax(z, axis: int = -1) -> np.ndarray:
    """Softmax_j(z) = e^{z_j} / sum_k e^{z_k} ([S1] §4.4, §8.2), shifted by the max for range."""
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(z - z.max(axis=axis, keepdims=True))
    return e / e.sum(axis=axis, keepdims=True)


def softmax_scale(d_head: int, d_rope: int) -> float:
    """1 / sqrt(d_h + d_h^R): the dot product lives in the concatenated space ([S1] §4.4)."""
    return 1.0 / np.sqrt(d_head + d_rope)


def page_slot(block_table, b: int, pos, page_size: int):
    """Flat pool row of token ``pos`` of sequence ``b``: bt[b][pos // P] * P + pos % P.

    Paging is not on the pages; this is the definition of the paged cache layout.
    """
    pos = np.asarray(pos, dtype=np.int64)
    return np.asarray(block_table)[b, pos // page_size].astype(np.int64) * page_size + pos % page_size


# --------------------------------------------------------------------------- naive form ([S1] §6)
def kv_rows(w_dkv_kr, h, pos, dims) -> np.ndarray:
    """The cached row [c^KV ‖ k^R] of each new token ([S1] §2.1, §4.2, §4.5).

    c^KV_t = W^DKV h_t and k^R_t = RoPE(W^KR h_t, t); ``w_dkv_kr`` stacks W^DKV's d_c rows
    over W^KR's d_h^R rows. Returns [T, d_c + d_h^R].
    """
    w = as64(w_dkv_kr)
    h = as64(h)
    c = h @ w[:dims.d_c].T
    k_r = rope(h @ w[dims.d_c:].T, np.asarray(pos), dims.rope_base, getattr(dims, "rope_inv_freq", None))
    return np.concatenate([c, k_r], axis=-1)


def query_path(w_dq, w_uq_qr, h, pos, dims):
    """Query pathway of [S1] §4.1 / §6 for each token.

    c^Q = W^DQ h; q^C = W^UQ c^Q split into n_h heads of d_h; q^R = RoPE(W^QR c^Q) split into
    n_h heads of d_h^R, every head rotated at the token's position (reading R3).
    Returns (c^Q [B, d_c'], q^C [B, n_h, d_h], q^R [B, n_h, d_h^R]).
    """
    n_h, d_h, d_r = dims.n_heads, dims.d_head, dims.d_rope
    w_uq_qr = as64(w_uq_qr)
    h = as64(h)
    c_q = h @ as64(w_dq).T
    q_c = (c_q @ w_uq_qr[:n_h * d_h].T).reshape(-1, n_h, d_h)
    q_r_hat = (c_q @ w_uq_qr[n_h * d_h:].T).reshape(-1, n_h, d_r)
    q_r = rope(q_r_hat, np.asarray(pos)[:, None], dims.rope_base, getattr(dims, "rope_inv_freq", None))
    return c_q, q_c, q_r


def attention_naive(q_c, q_r, rows, w_uk, w_uv, dims) -> np.ndarray:
    """Per-head attention of one query token over its cached rows ([S1] §2.2, §4.3, §4.4, §6).

    Keys and values are rebuilt from the latent: k^C_j = W^UK c_j, v^C_j = W^UV c_j, split into
    heads by contiguous row blocks. For head i the key is [k^C_{j,i}; k^R_j] and the query
    [q^C_i; q^R_i]; o_i = sum_j softmax_j(q_i . k_{j,i} / sqrt(d_h + d_h^R)) v^C_{j,i}.
    ``q_c`` [n_h, d_h], ``q_r`` [n_h, d_h^R], ``rows`` [L, d_c + d_h^R]. Returns o [n_h, d_h].
    """
    n_h, d_h, d_c = dims.n_heads, dims.d_head, dims.d_c
    rows = as64(rows)
    c, k_r = rows[:, :d_c], rows[:, d_c:]
    L = rows.shape[0]
    k_c = (c @ as64(w_uk).T).reshape(L, n_h, d_h)
    v_c = (c @ as64(w_uv).T).reshape(L, n_h, d_h)
    scale = softmax_scale(d_h, dims.d_rope)
    o = np.empty((n_h, d_h), dtype=np.float64)
    for i in range(n_h):
        q_i = np.concatenate([q_c[i], q_r[i]])
        k_i = np.concatenate([k_c[:, i, :], k_r], axis=1)
        p = softmax(k_i @ q_i * scale)
        o[i] = p @ v_c[:, i, :]
    return o


def output_naive(w_o, o) -> np.ndarray:
    """u_t = W^O [o_{t,1}; ...; o_{t,n_h}] ([S1] §1, §4.4). ``o`` [B, n_h, d_h] -> [B, d]."""
    o = np.asarray(o, dtype=np.float64)
    return o.reshape(o.shape[0], -1) @ as64(w_o).T


def layer_step_naive(W: dict, h, prefix: list, dims) -> dict:
    """One decode step of one MLA layer in the naive form ([S1] §6).

    ``prefix[b]`` holds the N_b rows already cached for sequence b; the new token sits at
    position N_b (R3), its own row is computed here and appended, and it attends to itself
    (R4). Returns the new rows, q^C, q^R, per-head outputs o and the layer output u.
    """
    pos = np.array([len(p) for p in prefix], dtype=np.int64)
    new_rows = kv_rows(W["w_dkv_kr"], h, pos, dims)
    _, q_c, q_r = query_path(W["w_dq"], W["w_uq_qr"], h, pos, dims)
    o = np.stack([
        attention_naive(q_c[b], q_r[b], np.vstack([as64(prefix[b]), new_rows[b:b + 1]]),
                        W["w_uk"], W["w_uv"], dims)
        for b in range(len(prefix))
    ])
    return {"rows": new_rows, "q_c": q_c, "q_r": q_r, "o": o, "u": output_naive(W["w_o"], o)}


# --------------------------------------------------------------------------- absorbed companion ([S1] §5)
def absorb_query(w_dq, w_uq_qr, w_uk, h, pos, dims) -> np.ndarray:
    """q = [q~ ‖ q^R] per head with q~_i = (W^UK_i)^T q^C_i ([S1] §5.1, §5.3 step 1).

    The layout matches a cache row [c ‖ k^R], so one dot product gives both score terms
    ([S1] §4.4). Returns [B, n_h, d_c + d_h^R].
    """
    n_h, d_h, d_c = dims.n_heads, dims.d_head, dims.d_c
    _, q_c, q_r = query_path(w_dq, w_uq_qr, h, pos, dims)
    w_uk_heads = as64(w_uk).reshape(n_h, d_h, d_c)          # W^UK_i = row block i
    q_t = np.einsum("ikm,bik->bim", w_uk_heads, q_c)         # (W^UK_i)^T q^C_i
    return np.concatenate([q_t, q_r], axis=-1)


def latent_attention(q, rows, dims):
    """Scores against the cached latents and the latent-space weighted sum ([S1] §5.3 steps 2-3).

    s_ij = (q~_i . c_j + q^R_i . k^R_j) / sqrt(d_h + d_h^R); p = softmax_j(s);
    o_lat_i = sum_j p_ij c_j. ``q`` [n_h, D], ``rows`` [L, D] (L >= 1).
    Returns (o_lat [n_h, d_c], lse [n_h]) with lse_i = log sum_j e^{s_ij} (R6).
    """
    q = as64(q)
    rows = as64(rows)
    s = (q @ rows.T) * softmax_scale(dims.d_head, dims.d_rope)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    o_lat = (e @ rows[:, :dims.d_c]) / l
    return o_lat, (m + np.log(l))[:, 0]


def lse_merge(o_parts, lses):
    """Merge split-KV partials (R6): weights e^{lse_s - max lse} renormalised over the splits.

    ``o_parts`` [S, n_h, d_c] normalised per split, ``lses`` [S, n_h].
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lses = np.asarray(lses, dtype=np.float64)
    m = lses.max(axis=0)
    w = np.exp(lses - m)
    z = w.sum(axis=0)
    return (w[..., None] * o_parts).sum(axis=0) / z[..., None], m + np.log(z)


def out_proj_absorbed(w_uv, w_o, o_lat) -> np.ndarray:
    """u = sum_i W^O_i W^UV_i o_lat_i, in two steps ([S1] §5.2, §5.3 step 4).

    o_i = W^UV_i o_lat_i (row block i of W^UV), then u = W^O [o_1; ...; o_n_h].
    ``o_lat`` [B, n_h, d_c] -> u [B, d].
    """
    o_lat = np.asarray(o_lat, dtype=np.float64)
    B, n_h, d_c = o_lat.shape
    w_uv_heads = as64(w_uv).reshape(n_h, -1, d_c)
    o = np.einsum("irm,bim->bir", w_uv_heads, o_lat)
    return o.reshape(B, -1) @ as64(w_o).T


def layer_step_absorbed(W: dict, h, prefix: list, dims) -> dict:
    """The same decode step as ``layer_step_naive`` through the absorbed route ([S1] §5.3)."""
    pos = np.array([len(p) for p in prefix], dtype=np.int64)
    new_rows = kv_rows(W["w_dkv_kr"], h, pos, dims)
    q = absorb_query(W["w_dq"], W["w_uq_qr"], W["w_uk"], h, pos, dims)
    outs = [latent_attention(q[b], np.vstack([as64(prefix[b]), new_rows[b:b + 1]]), dims)
            for b in range(len(prefix))]
    o_lat = np.stack([o for o, _ in outs])
    lse = np.stack([l for _, l in outs])
    return {"rows": new_rows, "q": q, "o_lat": o_lat, "lse": lse,
            "u": out_proj_absorbed(W["w_uv"], W["w_o"], o_lat)}


# --------------------------------------------------------------------------- chunked step ([S1] §6, t general)
def chunk_positions(prefix_lens, chunk_lens):
    """Sequence and position of every new token of a multi-token step (R3, R7).

    Sequence b holds ``prefix_lens[b]`` cached rows and brings ``chunk_lens[b]`` new tokens at
    the positions that follow them. Tokens are listed sequence by sequence. Returns
    (seq_idx [T], pos [T]) as int64.
    """
    seq_idx = np.repeat(np.arange(len(prefix_lens), dtype=np.int64), np.asarray(chunk_lens, dtype=np.int64))
    pos = np.concatenate([n + np.arange(q, dtype=np.int64) for n, q in zip(prefix_lens, chunk_lens)]
                         + [np.zeros(0, dtype=np.int64)])
    return seq_idx, pos


def chunk_step_naive(W: dict, h, prefix: list, chunk_lens, dims) -> dict:
    """One step that brings several new tokens per sequence, in the naive form ([S1] §6).

    ``h`` stacks the new tokens' hidden states in ``chunk_positions`` order. Every new row is
    computed and appended first. The token at position t of sequence b then attends to rows
    0..t of b: the prefix, the new tokens before it and itself (R4, R7), none after it.
    Returns seq_idx, pos, the new rows, q^C, q^R, o and u per new token.
    """
    seq_idx, pos = chunk_positions([len(p) for p in prefix], chunk_lens)
    new_rows = kv_rows(W["w_dkv_kr"], h, pos, dims)
    _, q_c, q_r = query_path(W["w_dq"], W["w_uq_qr"], h, pos, dims)
    full = [np.vstack([as64(prefix[b]).reshape(-1, dims.d_c + dims.d_rope), new_rows[seq_idx == b]])
            for b in range(len(prefix))]
    o = np.stack([attention_naive(q_c[t], q_r[t], full[seq_idx[t]][:pos[t] + 1], W["w_uk"], W["w_uv"], dims)
                  for t in range(len(pos))])
    return {"seq_idx": seq_idx, "pos": pos, "rows": new_rows, "q_c": q_c, "q_r": q_r, "o": o,
            "u": output_naive(W["w_o"], o)}


def chunk_latent_attention(q, seq_rows: list, seq_idx, pos, dims):
    """Absorbed attention for the new tokens of a multi-token step ([S1] §5.3 steps 2-3 for
    every new token of §6): token t attends to rows 0..pos[t] of sequence seq_idx[t] (R7).

    ``q`` [T, n_h, D]; ``seq_rows[b]`` holds at least pos[t] + 1 rows [., D] of sequence b.
    Returns (o_lat [T, n_h, d_c], lse [T, n_h]).
    """
    outs = [latent_attention(q[t], as64(seq_rows[seq_idx[t]])[:pos[t] + 1], dims) for t in range(len(pos))]
    if not outs:
        return np.zeros((0, dims.n_heads, dims.d_c)), np.zeros((0, dims.n_heads))
    return np.stack([o for o, _ in outs]), np.stack([l for _, l in outs])


def chunk_step_absorbed(W: dict, h, prefix: list, chunk_lens, dims) -> dict:
    """The same multi-token step as ``chunk_step_naive`` through the absorbed route ([S1] §5.3)."""
    seq_idx, pos = chunk_positions([len(p) for p in prefix], chunk_lens)
    new_rows = kv_rows(W["w_dkv_kr"], h, pos, dims)
    q = absorb_query(W["w_dq"], W["w_uq_qr"], W["w_uk"], h, pos, dims)
    full = [np.vstack([as64(prefix[b]).reshape(-1, dims.d_c + dims.d_rope), new_rows[seq_idx == b]])
            for b in range(len(prefix))]
    o_lat, lse = chunk_latent_attention(q, full, seq_idx, pos, dims)
    return {"seq_idx": seq_idx, "pos": pos, "rows": new_rows, "q": q, "o_lat": o_lat, "lse": lse,
            "u": out_proj_absorbed(W["w_uv"], W["w_o"], o_lat)}


# --------------------------------------------------------------------------- FP8 latent cache (reading R8)
E4M3_MAX = 448.0


def e4m3_values() -> np.ndarray:
    """The 256 values of the e4m3 ("fn") byte format, indexed by code, decoded from its fields:
    sign bit 7, exponent bits 6-3 with bias 7, fraction bits 2-0. Exponent field 0 holds the
    subnormals f/8 * 2^-6; exponent 15 with fraction 7 is NaN; there are no infinities."""
    v = np.empty(256, dtype=np.float64)
    for code in range(256):
        s, e, f = code >> 7, (code >> 3) & 15, code & 7
        if e == 15 and f == 7:
            v[code] = np.nan
            continue
        mag = (f / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + f / 8.0) * 2.0 ** (e - 7)
        v[code] = -mag if s else mag
    return v


def quantize_e4m3(y) -> np.ndarray:
    """Nearest e4m3 value to each finite y with |y| <= 448, ties to the even fraction (R8).

    The grid spacing is 2^(E-3) for |y| in [2^E, 2^(E+1)), E >= -6, and 2^-9 below 2^-6."""
    y = np.asarray(y, dtype=np.float64)
    assert np.all(np.abs(y) <= E4M3_MAX), "scale the values into range first"
    a = np.abs(y)
    E = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    step = 2.0 ** (np.maximum(E, -6.0) - 3.0)
    return np.sign(y) * np.round(a / step) * step      # np.round rounds halves to even


def fp8_row_scales(rows, d_c: int):
    """Per-token scales of the FP8 latent cache (R8): one for the latent part c (d_c values) and one
    for the RoPE key k^R, each max|part| / 448 computed in float32 (the precision the cache writer
    uses, so that both sides take the same rounding decisions); 1 for an all-zero part.
    Returns float32 [T, 2]."""
    rows = np.asarray(rows, dtype=np.float32)
    out = np.empty((rows.shape[0], 2), dtype=np.float32)
    for j, part in enumerate((rows[:, :d_c], rows[:, d_c:])):
        m = np.abs(part).max(axis=1) if part.shape[1] else np.zeros(rows.shape[0], np.float32)
        out[:, j] = np.where(m > 0, m / np.float32(E4M3_MAX), np.float32(1.0))
    return out


def quantize_rows_fp8(rows, d_c: int):
    """FP8 cache rows (R8): each part divided by its scale in float32, then rounded to e4m3.
    The part's largest value divides to 448 up to one float32 rounding, so the quotient is
    clamped to +-448 first (a saturating conversion). ``rows`` [T, D] (the element-type rows the
    bf16 cache would hold). Returns (values [T, D] as float64, the exact e4m3 values; scales
    float32 [T, 2])."""
    rows32 = np.asarray(rows, dtype=np.float32)
    sc = fp8_row_scales(rows32, d_c)
    y = np.concatenate([rows32[:, :d_c] / sc[:, :1], rows32[:, d_c:] / sc[:, 1:]], axis=1)
    return quantize_e4m3(np.clip(y.astype(np.float64), -E4M3_MAX, E4M3_MAX)), sc


def dequantize_rows_fp8(values, scales, d_c: int) -> np.ndarray:
    """Rows the FP8 cache stands for: each part's e4m3 values times its scale, in float64."""
    values = np.asarray(values, dtype=np.float64)
    sc = np.asarray(scales, dtype=np.float64)
    return np.concatenate([values[:, :d_c] * sc[:, :1], values[:, d_c:] * sc[:, 1:]], axis=1)
