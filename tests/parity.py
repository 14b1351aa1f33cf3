"""Helpers shared by the parity tests: the tolerance rule and device state builders."""
from __future__ import annotations

import numpy as np
import torch

from mla_latent_kv_42_b200 import synth

# Tolerance fixed for the floating-point outputs (cache rows, q_out, o_lat, u): the error is
# normalised by the largest magnitude of the reference.
MAX_TOL = 2e-2
MEAN_TOL = 2e-3


def normalised_errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    scale = float(np.abs(ref).max())
    err = np.abs(got - ref)
    if scale == 0.0:
        return float(err.max()), float(err.mean())
    return float(err.max() / scale), float(err.mean() / scale)


def assert_parity(got, ref, what="", max_tol=MAX_TOL, mean_tol=MEAN_TOL):
    mx, mean = normalised_errors(got, ref)
    assert np.isfinite(np.asarray(got, dtype=np.float64)).all(), f"{what}: non-finite values"
    assert mx <= max_tol and mean <= mean_tol, f"{what}: max {mx:.3e} (<= {max_tol}), mean {mean:.3e} (<= {mean_tol})"
    return mx, mean


def to64(t) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def device_weights(W: dict, device="cuda") -> dict:
    return {k: v.to(device) for k, v in W.items()}


class CacheCase:
    """A paged cache with N_b prefix rows per sequence (rows drawn by synth) on ``device``."""

    def __init__(self, w: synth.Workload, cached=None, device="cuda", layer=0, paging=None, fill=0.0,
                 row_std=None, spare_tokens=1):
        self.w = w
        d = w.dims
        self.cached = np.asarray(synth.cached_lengths(w) if cached is None else cached, dtype=np.int64)
        self.bt_np, self.num_pages = synth.page_table(self.cached, d.page_size, paging or w.paging, w.seed,
                                                      spare_tokens=spare_tokens)
        self.rows = synth.prefix_rows(w, self.cached, layer=layer, device=device, std=row_std)
        self.offsets = np.concatenate([[0], np.cumsum(self.cached)])
        self.pool = synth.paged_pool(self.rows, self.cached, self.bt_np, self.num_pages, d.page_size, fill=fill)
        self.block_table = torch.from_numpy(self.bt_np).to(device)

    def prefix(self, b: int) -> torch.Tensor:
        return self.rows[int(self.offsets[b]):int(self.offsets[b + 1])]
