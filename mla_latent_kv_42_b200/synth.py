"""Seeded synthetic inputs for the MLA absorbed-decode path.

This module only draws random numbers, builds integer layouts (lengths, positions, page
tables) and converts values to the storage dtype. None of the attention arithmetic lives
here: the oracle and the CUDA path both receive what this module produces, and neither
depends on the other.

Notation follows "DeepSeek-V2 from Scratch" (the running model and §6, "The Complete MLA
Algorithm"): d = model dim, n_h heads of d_h, joint KV latent d_c, query latent d_c',
decoupled RoPE dim d_h^R. One cache row is [c^KV (d_c) ‖ k^R (d_h^R)].

Recipes (seed 0 unless stated):
  * weights: iid N(0, sigma_w^2) drawn with numpy ``default_rng([seed, layer, tag])`` in the
    fixed matrix order of ``WEIGHT_ORDER``, rounded to the storage dtype (round to nearest even).
  * new-token hidden states: iid N(0, 1), rounded.
  * cached prefix rows: iid N(0, d * sigma_w^2), the marginal law of one element of
    W^DKV h (or of a rotated W^KR h) for h ~ N(0, I); drawn with a torch generator on the
    requested device so that gigabyte-sized caches are made where they live.
  * ragged lengths: ``rng.integers(lo, hi, endpoint=True)``; shuffled pages: ``rng.permutation``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np
import torch

__all__ = [
    "Dims", "RUNNING", "PRODUCTION", "Workload", "WORKLOADS", "workload",
    "WEIGHT_ORDER", "weights", "hidden", "cached_lengths", "page_table", "prefix_rows",
    "paged_pool", "synthetic_query", "to_storage", "storage_dtype", "yarn_inv_freq", "fp8_pages",
]


@dataclass(frozen=True)
class Dims:
    d_model: int
    n_heads: int
    d_head: int
    d_c: int
    d_cq: int
    d_rope: int
    page_size: int = 64
    dtype: str = "bf16"          # "bf16" or "fp16"
    rope_base: float = 10000.0
    rope_inv_freq: tuple | None = None   # caller-supplied RoPE frequencies theta_k (d_h^R/2 of them)

    @property
    def D(self) -> int:
        """Elements of one cache row, d_c + d_h^R."""
        return self.d_c + self.d_rope

    def with_(self, **kw) -> "Dims":
        return replace(self, **kw)


# The pages' running model (d=512, 8 heads of 64, d_c=128, d_c'=96, d_h^R=32) and the
# DeepSeek-V2 production dims (d=5120, 128 heads of 128, d_c=512, d_c'=1536, d_h^R=64).
RUNNING = Dims(d_model=512, n_heads=8, d_head=64, d_c=128, d_cq=96, d_rope=32)
PRODUCTION = Dims(d_model=5120, n_heads=128, d_head=128, d_c=512, d_cq=1536, d_rope=64)


@dataclass(frozen=True)
class Workload:
    name: str
    dims: Dims
    batch: int
    cached: int | tuple[int, int]   # tokens already cached per sequence, or (lo, hi) drawn uniformly
    layers: int
    sigma_w: float
    paging: str                     # "contiguous" or "shuffled"
    seed: int = 0
    chunk: int = 1                  # new tokens per sequence per step (1 = decode; more = chunked prefill)
    cache: str = "elem"             # "elem": element-type rows; "fp8": e4m3 pages with two scales per token

    @property
    def ragged(self) -> bool:
        return isinstance(self.cached, tuple)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("running_b1_n256_fp16", RUNNING.with_(dtype="fp16"), 1, 256, 1, 0.02, "contiguous"),
        Workload("running_b16_n4096_l12_bf16", RUNNING, 16, 4096, 12, 0.02, "contiguous"),
        Workload("production_b64_n4096_bf16", PRODUCTION, 64, 4096, 1, 0.006, "contiguous"),
        Workload("production_b128_ragged_paged_bf16", PRODUCTION, 128, (512, 32768), 1, 0.006, "shuffled"),
        Workload("production_b4_n131072_bf16", PRODUCTION, 4, 131072, 1, 0.006, "contiguous"),
        Workload("production_b8_n4096_chunk128_bf16", PRODUCTION, 8, 4096, 1, 0.006, "contiguous", chunk=128),
        # chunked prefill over a prefix larger than L2 (64 x 4096 cached rows = 302 MB)
        Workload("production_b64_n4096_chunk32_bf16", PRODUCTION, 64, 4096, 1, 0.006, "contiguous", chunk=32),
        # the decode shape above over an FP8 latent cache (584 bytes per token instead of 1152)
        Workload("production_b64_n4096_fp8", PRODUCTION, 64, 4096, 1, 0.006, "contiguous", cache="fp8"),
    ]
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def storage_dtype(dims: Dims) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp16": torch.float16}[dims.dtype]


def to_storage(x: np.ndarray | torch.Tensor, dims: Dims) -> torch.Tensor:
    """Round float values to the storage dtype (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(x)) if isinstance(x, np.ndarray) else x
    return t.to(storage_dtype(dims))


# Fixed order in which the per-layer matrices are drawn; the stacked forms are the
# layouts the C ABI takes (rows of W^DKV then W^KR; rows of W^UQ then W^QR).
WEIGHT_ORDER = ("w_dkv_kr", "w_dq", "w_uq_qr", "w_uk", "w_uv", "w_o")


def _weight_shapes(d: Dims) -> dict[str, tuple[int, int]]:
    return {
        "w_dkv_kr": (d.d_c + d.d_rope, d.d_model),
        "w_dq": (d.d_cq, d.d_model),
        "w_uq_qr": (d.n_heads * (d.d_head + d.d_rope), d.d_cq),
        "w_uk": (d.n_heads * d.d_head, d.d_c),
        "w_uv": (d.n_heads * d.d_head, d.d_c),
        "w_o": (d.d_model, d.n_heads * d.d_head),
    }


def weights(w: Workload, layer: int = 0, overrides: dict | None = None) -> dict[str, torch.Tensor]:
    """All weight matrices of one layer in the storage dtype (host tensors)."""
    out = {}
    for tag, name in enumerate(WEIGHT_ORDER):
        shape = _weight_shapes(w.dims)[name]
        rng = np.random.default_rng([w.seed, layer, 100 + tag])
        x = rng.standard_normal(shape, dtype=np.float32)
        x *= np.float32(w.sigma_w)
        out[name] = to_storage(x, w.dims)
    if overrides:
        out.update({k: to_storage(v, w.dims) if isinstance(v, np.ndarray) else v for k, v in overrides.items()})
    return out


def hidden(w: Workload, step: int = 0, layer: int = 0, batch: int | None = None) -> torch.Tensor:
    """New-token hidden states h_t, N(0, 1), [B, d] in the storage dtype (host)."""
    b = w.batch if batch is None else batch
    rng = np.random.default_rng([w.seed, layer, 200 + step])
    return to_storage(rng.standard_normal((b, w.dims.d_model), dtype=np.float32), w.dims)


def cached_lengths(w: Workload) -> np.ndarray:
    """N_b, the tokens already in the cache of each sequence before the step."""
    if w.ragged:
        lo, hi = w.cached
        rng = np.random.default_rng([w.seed, 1])
        return rng.integers(lo, hi, size=w.batch, endpoint=True).astype(np.int64)
    return np.full(w.batch, int(w.cached), dtype=np.int64)


def page_table(cached: np.ndarray, page_size: int, paging: str, seed: int = 0,
               spare_tokens: int = 1) -> tuple[np.ndarray, int]:
    """Block table int32[B, max_pages] holding room for N_b + spare_tokens tokens.

    Physical page ids are consecutive ("contiguous") or a seeded permutation ("shuffled").
    Entries past a sequence's last page are -1.
    """
    need = (cached + spare_tokens + page_size - 1) // page_size
    total = int(need.sum())
    max_pages = int(need.max()) if len(need) else 1
    if paging == "shuffled":
        ids = np.random.default_rng([seed, 2]).permutation(total).astype(np.int32)
    elif paging == "contiguous":
        ids = np.arange(total, dtype=np.int32)
    else:
        raise ValueError(paging)
    bt = np.full((len(cached), max_pages), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(need):
        bt[b, :n] = ids[off:off + n]
        off += n
    return bt, total


def prefix_rows(w: Workload, cached: np.ndarray, layer: int = 0, device: str = "cpu",
                std: float | None = None) -> torch.Tensor:
    """Logical cached rows of all sequences, concatenated: [sum N_b, D] storage dtype."""
    d = w.dims
    n = int(cached.sum())
    s = float(std) if std is not None else w.sigma_w * math.sqrt(d.d_model)
    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.default_rng([w.seed, layer, 3]).integers(0, 2**62)))
    out = torch.empty((n, d.D), dtype=storage_dtype(d), device=device)
    chunk = 1 << 24
    flat = out.view(-1)
    for a in range(0, flat.numel(), chunk):
        m = min(chunk, flat.numel() - a)
        flat[a:a + m] = (torch.randn(m, generator=g, device=device, dtype=torch.float32) * s).to(out.dtype)
    return out


def paged_pool(rows: torch.Tensor, cached: np.ndarray, block_table: np.ndarray, num_pages: int,
               page_size: int, fill: float = 0.0) -> torch.Tensor:
    """Place logical rows into a pool [num_pages, page_size, D]; other slots hold ``fill``."""
    D = rows.shape[1]
    pool = torch.full((num_pages, page_size, D), fill, dtype=rows.dtype, device=rows.device)
    slots = []
    for b, n in enumerate(cached):
        j = np.arange(int(n), dtype=np.int64)
        slots.append(block_table[b, j // page_size].astype(np.int64) * page_size + j % page_size)
    idx = torch.from_numpy(np.concatenate(slots) if slots else np.zeros(0, np.int64)).to(rows.device)
    pool.view(-1, D).index_copy_(0, idx, rows)
    return pool


def fp8_pages(w: Workload, num_pages: int, layer: int = 0, device: str = "cpu") -> torch.Tensor:
    """An FP8 cache of ``num_pages`` pages (uint8 [num_pages, page_size * (D + 8)]) filled with
    random bytes in the cache format: every row byte a uniformly drawn non-NaN e4m3 code, every
    scale pair uniform in [0.5, 1.5] / 448 (decoded magnitudes up to about 1.5, as the 16-bit
    prefix rows have). Drawn, not computed from rows: a timing input for the FP8 decode."""
    d = w.dims
    g = torch.Generator().manual_seed(w.seed * 1000003 + layer * 7919 + 17)
    P, D = d.page_size, d.D
    codes = torch.randint(0, 0x7F, (num_pages, P * D), generator=g, dtype=torch.int32)  # 0x00 .. 0x7E
    codes |= torch.randint(0, 2, (num_pages, P * D), generator=g, dtype=torch.int32) << 7
    scales = (0.5 + torch.rand((num_pages, P * 2), generator=g)) / 448.0
    pages = torch.cat([codes.to(torch.uint8), scales.contiguous().view(torch.uint8).view(num_pages, -1)], dim=1)
    return pages.to(device)


def synthetic_query(w: Workload, batch: int, scale: float = 1.0, seed_tag: int = 0) -> torch.Tensor:
    """A stand-in absorbed query [B, n_h, D] = [q~ ‖ q^R] with the magnitudes the weight law gives.

    sigma(c^Q) = sigma_w sqrt(d); sigma(q^C) = sigma_w sqrt(d_c') sigma(c^Q);
    sigma(q~) = sigma_w sqrt(d_h) sigma(q^C); sigma(q^R) = sigma(q^C). ``scale`` multiplies
    both parts (large values make the softmax peaked).
    """
    d = w.dims
    s_cq = w.sigma_w * math.sqrt(d.d_model)
    s_qc = w.sigma_w * math.sqrt(d.d_cq) * s_cq
    s_qt = w.sigma_w * math.sqrt(d.d_head) * s_qc
    rng = np.random.default_rng([w.seed, 4, seed_tag])
    q = rng.standard_normal((batch, d.n_heads, d.D), dtype=np.float32)
    q[..., :d.d_c] *= np.float32(s_qt * scale)
    q[..., d.d_c:] *= np.float32(s_qc * scale)
    return to_storage(q, d)


def yarn_inv_freq(d_rope: int, base: float, factor: float = 40.0, original_ctx: int = 4096, beta_fast: float = 32.0,
                  beta_slow: float = 1.0) -> tuple:
    """An example caller-supplied RoPE frequency table (an input to the library, not part of its
    arithmetic): YaRN's "NTK-by-parts" interpolation of theta_k = base^(-2k/d_rope) for a context
    `factor` times `original_ctx`. Pair k makes r_k = original_ctx * theta_k / (2 pi) turns over the
    original context; pairs with r_k >= beta_fast keep theta_k, pairs with r_k <= beta_slow take
    theta_k / factor, and the ramp between is linear in r_k. The constants are illustrative."""
    out = []
    for k in range(d_rope // 2):
        theta = base ** (-2.0 * k / d_rope)
        r = original_ctx * theta / (2.0 * math.pi)
        gamma = min(1.0, max(0.0, (r - beta_slow) / (beta_fast - beta_slow)))
        out.append((1.0 - gamma) * theta / factor + gamma * theta)
    return tuple(out)
