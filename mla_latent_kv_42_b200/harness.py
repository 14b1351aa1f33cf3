"""Workload state for benchmarks, tests and the smoke entry: device-resident weights, paged
latent caches and per-step index tensors built from ``synth``. No method arithmetic here; the
step itself is ``mla_latent_kv_42_b200.layer_step`` (the four C-ABI calls)."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import LayerState, synth


@dataclass
class Layer:
    state: LayerState
    W_host: dict          # weights as drawn (host, storage dtype) — what the oracle reads
    rows: torch.Tensor    # logical prefix rows [sum N_b, D] on the device
    offsets: np.ndarray   # row offsets of each sequence in ``rows``

    def prefix(self, b: int) -> torch.Tensor:
        return self.rows[int(self.offsets[b]):int(self.offsets[b + 1])]


@dataclass
class StepIndex:
    cached: np.ndarray    # N_b
    chunk: int            # new tokens per sequence in the step (1 = decode)
    pos: torch.Tensor     # int32 [T], positions of the new tokens: N_b, N_b + 1, ..., N_b + chunk - 1
    seq_idx: torch.Tensor  # int32 [T], the sequence of each new token
    seq_lens: torch.Tensor  # int32 [T] = pos + 1, the length each new token attends
    max_seq_len: int


def step_index(cached: np.ndarray, device="cuda", chunk: int = 1) -> StepIndex:
    """Index tensors of a step that brings ``chunk`` new tokens to every sequence, listed
    sequence by sequence (T = B * chunk). With chunk = 1 it is a decode step: pos = N_b,
    seq_idx = b, seq_lens = N_b + 1."""
    cached = np.asarray(cached, dtype=np.int64)
    B = len(cached)
    seq = np.repeat(np.arange(B, dtype=np.int64), chunk)
    pos = cached[seq] + np.tile(np.arange(chunk, dtype=np.int64), B)
    i32 = lambda a: torch.from_numpy(a.astype(np.int32)).to(device)
    return StepIndex(cached=cached, chunk=chunk, pos=i32(pos), seq_idx=i32(seq), seq_lens=i32(pos + 1),
                     max_seq_len=int(cached.max()) + chunk)


def make_layer(w: synth.Workload, cached: np.ndarray, layer: int = 0, device="cuda", fill: float = 0.0,
               block_table: np.ndarray | None = None, num_pages: int | None = None, spare_tokens: int = 1) -> Layer:
    d = w.dims
    W = synth.weights(w, layer)
    if block_table is None:
        block_table, num_pages = synth.page_table(cached, d.page_size, w.paging, w.seed, spare_tokens=spare_tokens)
    rows = synth.prefix_rows(w, cached, layer=layer, device=device)
    if w.cache == "fp8":  # random bytes in the FP8 page format (the rows above are not in it)
        pool = synth.fp8_pages(w, num_pages, layer=layer, device=device)
    else:
        pool = synth.paged_pool(rows, cached, block_table, num_pages, d.page_size, fill=fill)
    st = LayerState(dims=d, w={k: v.to(device) for k, v in W.items()}, pool=pool,
                    block_table=torch.from_numpy(block_table).to(device))
    return Layer(state=st, W_host=W, rows=rows, offsets=np.concatenate([[0], np.cumsum(cached)]))


def weight_bytes(d: synth.Dims) -> int:
    n_h = d.n_heads
    elems = ((d.d_c + d.d_rope) * d.d_model + d.d_cq * d.d_model + n_h * (d.d_head + d.d_rope) * d.d_cq
             + 2 * n_h * d.d_head * d.d_c + d.d_model * n_h * d.d_head)
    return 2 * elems


def decode_work(d: synth.Dims, seq_lens: np.ndarray) -> tuple[int, int]:
    """Algorithmic bytes and flops of latent attention over the attended tokens.

    Per attended token: read one cache row of d_c + d_h^R elements; 2 n_h (d_c + d_h^R) flops for
    the scores and 2 n_h d_c for the latent weighted sum. Per sequence: read q, write o_lat.
    """
    L = int(np.sum(seq_lens))
    B = len(seq_lens)
    D = d.d_c + d.d_rope
    byts = 2 * (L * D + B * d.n_heads * D + B * d.n_heads * d.d_c)
    flops = 2 * L * d.n_heads * (D + d.d_c)
    return byts, flops


def step_work(d: synth.Dims, seq_lens: np.ndarray) -> tuple[int, int]:
    """Algorithmic bytes and flops of one whole layer step (weights read once + decode)."""
    B = len(seq_lens)
    db, df = decode_work(d, seq_lens)
    n_h = d.n_heads
    proj_flops = 2 * B * ((d.d_c + d.d_rope) * d.d_model + d.d_cq * d.d_model + n_h * (d.d_head + d.d_rope) * d.d_cq
                          + 2 * n_h * d.d_head * d.d_c + d.d_model * n_h * d.d_head)
    act_bytes = 2 * B * (2 * d.d_model + (d.d_c + d.d_rope))  # h in, u out, the appended row
    return db + weight_bytes(d) + act_bytes, df + proj_flops


def cache_row_bytes(d: synth.Dims, cache: str = "elem") -> int:
    """Bytes of one cached token: D element-type values, or D e4m3 bytes and two float32 scales."""
    D = d.d_c + d.d_rope
    return D + 8 if cache == "fp8" else 2 * D


def attention_work(d: synth.Dims, cached: np.ndarray, chunk: int = 1, cache: str = "elem") -> tuple[int, int]:
    """Algorithmic bytes and flops of the attention call of a step bringing ``chunk`` new tokens
    to every sequence (chunk = 1: decode; equals ``decode_work(d, cached + 1)``).

    Bytes: each sequence's N_b + chunk cache rows read once (the new tokens of a sequence share
    them), q read and o_lat written per new token. Flops: the token at position t attends t + 1
    rows, 2 n_h (d_c + d_h^R) for its scores and 2 n_h d_c for its weighted sum per row.
    """
    cached = np.asarray(cached, dtype=np.int64)
    D = d.d_c + d.d_rope
    T = len(cached) * chunk
    rows = int(np.sum(cached + chunk))
    attended = int(np.sum(chunk * (cached + 1) + chunk * (chunk - 1) // 2))
    byts = rows * cache_row_bytes(d, cache) + 2 * (T * d.n_heads * D + T * d.n_heads * d.d_c)
    flops = 2 * attended * d.n_heads * (D + d.d_c)
    return byts, flops


def layer_work(d: synth.Dims, cached: np.ndarray, chunk: int = 1, cache: str = "elem") -> tuple[int, int]:
    """Algorithmic bytes and flops of a whole layer step bringing ``chunk`` new tokens to every
    sequence: weights read once, the projections of every new token, and the attention call
    (chunk = 1: equals ``step_work(d, cached + 1)``)."""
    T = len(cached) * chunk
    ab, af = attention_work(d, cached, chunk, cache)
    n_h = d.n_heads
    proj_flops = 2 * T * ((d.d_c + d.d_rope) * d.d_model + d.d_cq * d.d_model + n_h * (d.d_head + d.d_rope) * d.d_cq
                          + 2 * n_h * d.d_head * d.d_c + d.d_model * n_h * d.d_head)
    act_bytes = 2 * T * 2 * d.d_model + T * cache_row_bytes(d, cache)  # h in, u out, the appended rows
    return ab + weight_bytes(d) + act_bytes, af + proj_flops
