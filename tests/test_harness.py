"""Host logic of the benchmark harness (no GPU): the step index tensors for one or several new
tokens per sequence, and the algorithmic byte and flop counts the roofline divides by, checked
against brute-force enumeration."""
import numpy as np
import pytest
import torch

from mla_latent_kv_42_b200 import harness, synth


@pytest.mark.parametrize("chunk", [1, 3, 128])
def test_step_index_lists_new_tokens_sequence_by_sequence(chunk):
    cached = np.array([0, 5, 4096])
    ix = harness.step_index(cached, device="cpu", chunk=chunk)
    want_seq, want_pos = [], []
    for b, n in enumerate(cached):
        for i in range(chunk):
            want_seq.append(b)
            want_pos.append(int(n) + i)
    assert ix.seq_idx.tolist() == want_seq
    assert ix.pos.tolist() == want_pos
    assert ix.seq_lens.tolist() == [p + 1 for p in want_pos]
    assert ix.max_seq_len == max(want_pos) + 1


def test_decode_step_index_is_the_one_token_case():
    cached = np.array([7, 0, 300])
    ix = harness.step_index(cached, device="cpu")
    assert ix.pos.tolist() == [7, 0, 300] and ix.seq_idx.tolist() == [0, 1, 2]
    assert ix.seq_lens.tolist() == [8, 1, 301] and ix.max_seq_len == 301


@pytest.mark.parametrize("dims", [synth.RUNNING, synth.PRODUCTION], ids=["running", "production"])
@pytest.mark.parametrize("chunk", [1, 2, 128])
def test_attention_work_by_enumeration(dims, chunk):
    """Bytes: each sequence's rows once, q in and o_lat out per new token. Flops: every (new token,
    attended row) pair costs 2 n_h (D + d_c)."""
    cached = np.array([0, 17, 4096])
    byts, flops = harness.attention_work(dims, cached, chunk)
    D = dims.d_c + dims.d_rope
    pairs = sum(int(n) + i + 1 for n in cached for i in range(chunk))
    rows = sum(int(n) + chunk for n in cached)
    T = len(cached) * chunk
    assert flops == pairs * 2 * dims.n_heads * (D + dims.d_c)
    assert byts == 2 * rows * D + 2 * T * dims.n_heads * (D + dims.d_c)


def test_chunk_of_one_matches_the_decode_counts():
    cached = np.array([1, 512, 32768])
    for d in (synth.RUNNING, synth.PRODUCTION):
        assert harness.attention_work(d, cached, 1) == harness.decode_work(d, cached + 1)
        assert harness.layer_work(d, cached, 1) == harness.step_work(d, cached + 1)


def test_layer_work_adds_weights_once_and_projections_per_token():
    d = synth.PRODUCTION
    cached = np.array([4096] * 8)
    ab, af = harness.attention_work(d, cached, 128)
    lb, lf = harness.layer_work(d, cached, 128)
    T = 8 * 128
    assert lb - ab == harness.weight_bytes(d) + 2 * T * (2 * d.d_model + d.d_c + d.d_rope)
    assert lf - af == 2 * T * (harness.weight_bytes(d) // 2)   # 2 flops per weight element per token


def test_fp8_cache_bytes_per_token():
    """The FP8 cache's roofline bytes: D e4m3 bytes and two float32 scales per cached token (584 B at
    production dims, against 1152 for the 16-bit cache); queries, outputs and flops are unchanged."""
    d = synth.PRODUCTION
    cached = np.array([4096] * 64)
    assert harness.cache_row_bytes(d, "fp8") == 584 and harness.cache_row_bytes(d) == 1152
    b16, f16 = harness.attention_work(d, cached, 1)
    b8, f8 = harness.attention_work(d, cached, 1, "fp8")
    rows = int((cached + 1).sum())
    assert f8 == f16 and b16 - b8 == rows * (1152 - 584)
    lb16, _ = harness.layer_work(d, cached, 1)
    lb8, _ = harness.layer_work(d, cached, 1, "fp8")
    assert lb16 - lb8 == (rows + len(cached)) * (1152 - 584)  # the appended rows too
    w = synth.workload("production_b64_n4096_fp8")
    pages = synth.fp8_pages(w, 3)
    assert pages.shape == (3, 64 * 584) and pages.dtype == torch.uint8
    codes = pages[:, :64 * 576]
    assert not ((codes & 0x7F) == 0x7F).any()  # no NaN code
    scales = pages[:, 64 * 576:].contiguous().view(torch.float32)
    assert (scales >= 0.5 / 448).all() and (scales <= 1.5 / 448).all()
