"""The stream-K GEMM plan the projection calls use (no GPU): every (tile, k block) iteration is owned by
exactly one CTA, partial slots (tile + CTA) are unique and fit the partial buffer, shared memory fits, and
two CTAs share an SM only when both fit. The plan comes from the library itself (mla_debug_gemm_plan)."""
import ctypes
import math

import numpy as np
import pytest

import mla_latent_kv_42_b200 as M
from mla_latent_kv_42_b200 import build, synth

SMS = 148
SMEM_MAX = 232448
SMEM_HALF = 113 * 1024


@pytest.fixture(scope="module")
def lib():
    build.build()
    lib = M.load_library()
    lib.mla_debug_gemm_plan.restype = ctypes.c_int
    lib.mla_debug_gemm_plan.argtypes = [ctypes.c_int32] * 6 + [ctypes.POINTER(ctypes.c_int64)]
    return lib


def plan(lib, Mr, N, K, batch, fused, d_rope):
    out = (ctypes.c_int64 * 11)()
    assert lib.mla_debug_gemm_plan(Mr, N, K, batch, int(fused), d_rope, out) == 0
    keys = ("bn", "m_tiles", "n_tiles", "kb", "tiles", "G", "stages", "aligned", "split", "smem", "part_bytes")
    return dict(zip(keys, list(out)))


def check_plan(p, Mr, N, K, batch, fused, d_rope):
    bn, kb, tiles, G = p["bn"], p["kb"], p["tiles"], p["G"]
    assert bn in (32, 64, 128, 256) and (bn >= N or p["n_tiles"] > 1)
    assert p["m_tiles"] == math.ceil(Mr / 128) and p["n_tiles"] == math.ceil(N / bn) and kb == math.ceil(K / 64)
    assert tiles == p["m_tiles"] * p["n_tiles"] * batch
    iters = tiles * kb
    assert 1 <= G <= min(iters, 2 * SMS)
    start = [(tiles * c // G) * kb if p["aligned"] else iters * c // G for c in range(G + 1)]
    assert start[0] == 0 and start[-1] == iters
    assert all(start[c + 1] > start[c] for c in range(G)), "a CTA with no work"
    # ownership, segments and partial slots, as the kernel walks its range
    owner = np.full(iters, -1)
    slots = set()
    split = False
    for c in range(G):
        owner[start[c]:start[c + 1]] = c
        i = start[c]
        while i < start[c + 1]:
            t = i // kb
            end = min(start[c + 1], (t + 1) * kb)
            if not (i % kb == 0 and end == (t + 1) * kb):
                split = True
                assert (t + c) not in slots
                slots.add(t + c)
            i = end
    assert (owner >= 0).all()
    assert bool(p["split"]) == split
    if p["aligned"]:
        assert not split
    if split:
        assert max(slots) < tiles + G
        assert p["part_bytes"] >= (tiles + G) * 128 * bn * 4
    # shared memory: ring + RoPE table + control, one or two CTAs per SM
    stage = (128 + bn) * 64 * 2
    table = bn * (d_rope // 2) * 8 + bn * 8 if fused else 0
    assert p["stages"] >= 2 and p["smem"] == 1024 + table + 256 + p["stages"] * stage
    assert p["smem"] <= SMEM_MAX
    if G > SMS:
        assert p["aligned"] and p["smem"] <= SMEM_HALF
        # short tiles: the whole range resident; long tiles (>= 16 k blocks, at least one per SM):
        # whole tiles per CTA through a half-size ring
        assert p["stages"] >= start[1] - start[0] or kb >= 16, "two CTAs per SM only with the whole range resident"


def products(d):
    D, nq, nhd = d.d_c + d.d_rope, d.n_heads * (d.d_head + d.d_rope), d.n_heads * d.d_head
    return [(D, d.d_model, 1, True), (d.d_cq, d.d_model, 1, False), (nq, d.d_cq, 1, True),
            (d.d_c, d.d_head, d.n_heads, False), (d.d_head, d.d_c, d.n_heads, False), (d.d_model, nhd, 1, False)]


@pytest.mark.parametrize("dims", [synth.RUNNING, synth.PRODUCTION], ids=["running", "production"])
@pytest.mark.parametrize("N", [1, 4, 16, 64, 128, 257, 300, 1024, 4096])
def test_projection_plans(lib, dims, N):
    for Mr, K, batch, fused in products(dims):
        check_plan(plan(lib, Mr, N, K, batch, fused, dims.d_rope), Mr, N, K, batch, fused, dims.d_rope)


def test_random_plans(lib):
    rng = np.random.default_rng(3)
    for _ in range(300):
        Mr = int(rng.integers(1, 30000))
        N = int(rng.integers(1, 600))
        K = int(rng.integers(1, 20000))
        batch = int(rng.choice([1, 1, 1, 2, 8, 128]))
        fused = bool(rng.integers(0, 2))
        check_plan(plan(lib, Mr, N, K, batch, fused, 64), Mr, N, K, batch, fused, 64)


def test_plan_rejects_bad_sizes(lib):
    out = (ctypes.c_int64 * 11)()
    assert lib.mla_debug_gemm_plan(0, 64, 64, 1, 0, 64, out) == -1
    assert lib.mla_debug_gemm_plan(64, 64, 64, 1, 0, 64, None) == -1
