"""Host-side checks of the C ABI (no GPU): the library loads, exports every declared symbol,
returns the pages' cache sizes, and rejects bad arguments before queueing anything."""
import ctypes
import os
import re

import pytest

import mla_latent_kv_42_b200 as M
from mla_latent_kv_42_b200 import build, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return M.load_library()


def declared_functions():
    inc = os.path.join(ROOT, "include")
    text = "".join(open(os.path.join(inc, f)).read() for f in sorted(os.listdir(inc)) if f.endswith(".h"))
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_calls():
    names = declared_functions()
    for n in ("mla_append_kv", "mla_absorb_query", "mla_decode_attention", "mla_out_proj", "mla_prefill_attention"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    # and the symbols are plain C (unmangled) in the dynamic table
    out = os.popen(f"nm -D --defined-only {M.library_path()}").read()
    for n in names:
        assert re.search(rf"\bT {n}$", out, flags=re.M), n


def dims(d):
    return M.c_dims(d)


def test_cache_elems_per_token_matches_pages(lib):
    """160 (running model, from-scratch page §4.5) and 576 (production, visual explainer)."""
    assert M.cache_elems_per_token(synth.RUNNING) == 160
    assert M.cache_elems_per_token(synth.PRODUCTION) == 576


@pytest.mark.parametrize("field,value,code", [
    ("n_heads", 129, -2), ("d_c", 520, -2), ("d_rope", 6, -2), ("d_model", 0, -1), ("dtype", 7, -1),
    ("page_size", 0, -1), ("rope_base", 0.0, -1), ("d_head", 12, -2),
])
def test_check_dims_rejects(lib, field, value, code):
    cd = dims(synth.PRODUCTION)
    setattr(cd, field, value)
    assert lib.mla_check_dims(ctypes.byref(cd)) == code
    assert lib.mla_cache_elems_per_token(ctypes.byref(cd)) == code


def test_check_dims_accepts_both_families(lib):
    for d in (synth.RUNNING, synth.PRODUCTION, synth.RUNNING.with_(dtype="fp16")):
        cd = dims(d)
        assert lib.mla_check_dims(ctypes.byref(cd)) == 0


def test_null_dims_is_invalid(lib):
    assert lib.mla_check_dims(None) == -1
    assert lib.mla_workspace_size(None, 0, 1, 1) == 0


FAKE = ctypes.c_void_p(1 << 20)        # aligned, never dereferenced on the host
MISALIGNED = ctypes.c_void_p((1 << 20) + 8)


def test_decode_argument_errors_queue_nothing(lib):
    cd = dims(synth.PRODUCTION)
    f = lib.mla_decode_attention
    args = [ctypes.byref(cd), FAKE, FAKE, 10, FAKE, 4, FAKE, 2, 256, FAKE, None, FAKE, 1 << 30, None]
    bad = list(args)
    bad[1] = None
    assert f(*bad) == -1                                  # null q
    bad = list(args)
    bad[9] = MISALIGNED
    assert f(*bad) == -4                                  # misaligned o_lat
    bad = list(args)
    bad[8] = 0
    assert f(*bad) == -1                                  # max_seq_len < 1
    bad = list(args)
    bad[8] = 257
    assert f(*bad) == -1                                  # max_pages * page_size < max_seq_len
    bad = list(args)
    bad[12] = 0
    need = lib.mla_workspace_size(ctypes.byref(cd), M.CALL_DECODE_ATTENTION, 2, 256)
    assert f(*bad) == (-3 if need > 0 else f(*bad))        # too-small workspace
    bad = list(args)
    bad[8] = (1 << 30) + 1
    bad[5] = 1 << 25
    assert f(*bad) == -1                                  # max_seq_len beyond 2^30
    bad = list(args)
    bad[7] = 0
    assert f(*bad) == 0                                   # B == 0 is a no-op


def test_append_absorb_out_argument_errors(lib):
    cd = dims(synth.RUNNING)
    assert lib.mla_append_kv(ctypes.byref(cd), FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, FAKE, 8, -1, FAKE, 1 << 20,
                             None) == -1
    assert lib.mla_append_kv(ctypes.byref(cd), FAKE, MISALIGNED, FAKE, FAKE, FAKE, 1, 4, FAKE, 8, 3, FAKE, 1 << 20,
                             None) == -4
    cp = dims(synth.PRODUCTION)  # its append splits the reduction over CTAs and needs scratch
    assert M.workspace_size(synth.PRODUCTION, M.CALL_APPEND_KV, 3, 1) > 4
    assert lib.mla_append_kv(ctypes.byref(cp), FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, FAKE, 8, 3, FAKE, 4,
                             None) == -3
    assert lib.mla_append_kv(ctypes.byref(cd), FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, FAKE, 8, 0, None, 0,
                             None) == 0
    assert lib.mla_absorb_query(ctypes.byref(cd), FAKE, FAKE, None, FAKE, FAKE, FAKE, 2, FAKE, 1 << 20, None) == -1
    assert lib.mla_absorb_query(ctypes.byref(cd), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, FAKE, 8, None) == -3
    assert lib.mla_out_proj(ctypes.byref(cd), FAKE, FAKE, FAKE, MISALIGNED, 2, FAKE, 1 << 20, None) == -4
    assert lib.mla_out_proj(ctypes.byref(cd), FAKE, FAKE, FAKE, FAKE, -1, FAKE, 1 << 20, None) == -1


def test_decode_timing_hook_arguments(lib):
    fake = ctypes.c_void_p(0x100000)
    assert lib.mla_set_decode_timing_events(fake, None) == -1
    assert lib.mla_set_decode_timing_events(None, fake) == -1
    assert lib.mla_set_decode_timing_events(None, None) == 0


def test_workspace_sizes_are_consistent(lib):
    for d in (synth.RUNNING, synth.PRODUCTION):
        for call in range(5):
            a = M.workspace_size(d, call, 64, 4097)
            b = M.workspace_size(d, call, 128, 32769)
            assert a >= 0 and b >= a
            assert a % 256 == 0
    assert M.workspace_size(synth.PRODUCTION, 9, 1, 1) == 0


def test_error_strings(lib):
    for code in range(0, -9, -1):
        s = lib.mla_error_string(code).decode()
        assert s and s != "unknown status"
    assert lib.mla_error_string(-99).decode() == "unknown status"


def test_product_path_fails_loudly_without_the_library(tmp_path):
    with pytest.raises(RuntimeError, match="not built"):
        M.load_library(str(tmp_path / "missing.so"))


def test_prefill_argument_errors_queue_nothing(lib):
    cd = dims(synth.PRODUCTION)
    f = lib.mla_prefill_attention
    # dims, q, pool, num_pages, block_table, num_seqs, max_pages, seq_idx, pos, T, max_seq_len, o_lat, lse,
    # ws, ws_bytes, stream
    args = [ctypes.byref(cd), FAKE, FAKE, 10, FAKE, 2, 4, FAKE, FAKE, 5, 256, FAKE, None, FAKE, 1 << 30, None]

    def call(**kw):
        a = list(args)
        for k, v in kw.items():
            a[int(k[1:])] = v
        return f(*a)

    assert call(a7=None) == -1                            # null seq_idx
    assert call(a8=None) == -1                            # null pos
    assert call(a13=None) == -1                           # the per-token tables need a workspace
    assert call(a12=MISALIGNED) == -4                     # misaligned lse_out
    assert call(a5=0) == -1                               # no sequences
    assert call(a9=-1) == -1                              # negative token count
    assert call(a10=257) == -1                            # max_pages * page_size < max_seq_len
    assert call(a10=(1 << 30) + 1, a6=1 << 25) == -1      # max_seq_len beyond 2^30
    assert call(a14=16) == -3                             # too-small workspace
    assert call(a9=0, a1=None, a13=None) == 0             # T == 0 is a no-op
    assert lib.mla_last_launch_count(M.CALL_PREFILL_ATTENTION) == 0
    assert lib.mla_last_launch_count(8) == -1


def test_layer_step_small_argument_errors_queue_nothing(lib):
    """The fused single-launch layer step: argument checks return before anything is queued."""
    assert lib.mla_layer_step_small_supported(ctypes.byref(dims(synth.RUNNING))) == 0
    assert lib.mla_layer_step_small_supported(ctypes.byref(dims(synth.PRODUCTION))) == -2
    cd = dims(synth.RUNNING)
    ws_need = lib.mla_workspace_size(ctypes.byref(cd), M.CALL_LAYER_STEP_SMALL, 4, 300)
    assert ws_need > 0
    assert lib.mla_workspace_size(ctypes.byref(cd), M.CALL_LAYER_STEP_SMALL, 4, (1 << 30) + 1) == 0
    assert lib.mla_workspace_size(ctypes.byref(dims(synth.PRODUCTION)), M.CALL_LAYER_STEP_SMALL, 4, 300) == 0
    f = lib.mla_layer_step_small
    # dims, h, w_dkv_kr, w_dq, w_uq_qr, w_uk, w_uv, w_o, pool, num_pages, block_table, max_pages,
    # seq_lens, B, max_seq_len, q_out, o_lat, lse_out, u, ws, ws_bytes, stream
    args = [ctypes.byref(cd), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 100, FAKE, 8, FAKE, 4, 300, FAKE,
            FAKE, None, FAKE, FAKE, ws_need, None]

    def call(**kw):
        a = list(args)
        for k, v in kw.items():
            a[int(k[1:])] = v
        return f(*a)

    assert call(a0=ctypes.byref(dims(synth.PRODUCTION))) == -2  # dims outside the fused kernel
    assert call(a1=None) == -1                            # null h
    assert call(a8=None) == -1                            # null pool
    assert call(a19=None) == -1                           # null workspace
    assert call(a16=MISALIGNED) == -4                     # misaligned o_lat
    assert call(a13=-1) == -1                             # negative batch
    assert call(a14=0) == -1                              # max_seq_len < 1
    assert call(a14=(1 << 30) + 1) == -1                  # max_seq_len beyond 2^30
    assert call(a20=ws_need - 1) == -3                    # too-small workspace
    assert call(a13=0, a1=None) == 0                      # B == 0 is a no-op
    assert lib.mla_last_launch_count(M.CALL_LAYER_STEP_SMALL) == 0


def test_prefill_workspace_covers_decode_and_stops_growing():
    """Tokens run in launch groups of at most 1024, so past one group the workspace stays put,
    and it always holds a decode call's workspace for one group plus the per-token tables."""
    for d in (synth.RUNNING, synth.PRODUCTION):
        for T in (1, 7, 1000, 1024, 1025, 5000):
            g = min(T, 1024)
            need = M.workspace_size(d, M.CALL_PREFILL_ATTENTION, T, 4097)
            assert need % 256 == 0
            assert need >= M.workspace_size(d, M.CALL_DECODE_ATTENTION, g, 4097) + 4 * g * (-(-4097 // d.page_size))
            assert need >= M.workspace_size(d, M.CALL_DECODE_ATTENTION, T % 1024 or g, 4097)
    P = synth.PRODUCTION
    assert (M.workspace_size(P, M.CALL_PREFILL_ATTENTION, 1024, 4097)
            == M.workspace_size(P, M.CALL_PREFILL_ATTENTION, 4096, 4097)
            == M.workspace_size(P, M.CALL_PREFILL_ATTENTION, 100000, 4097))


def test_binding_refuses_host_tensors_before_calling_the_library(lib):
    """The binding checks placement, layout and dtype itself: host, strided or mistyped tensors
    raise ValueError and reach no C call (so nothing is queued)."""
    import torch
    d = synth.RUNNING
    q = torch.zeros((3, d.n_heads, d.D), dtype=torch.bfloat16)
    i32 = torch.zeros(3, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        M.prefill_attention(d, q, q, i32.view(1, 3), i32, i32, 4)
    with pytest.raises(ValueError, match="CUDA"):
        M.decode_attention(d, q, q, i32.view(1, 3), i32, 4)


def test_page_totals_beyond_int32_are_rejected(lib):
    """The attention planner sums page counts over a launch in int32: a batch whose worst case
    (B x pages of max_seq_len) passes INT32_MAX is rejected before anything is queued, by both the
    workspace and the allocation-free entry point."""
    cd = dims(synth.PRODUCTION)
    big = 1 << 30                     # 2^24 pages of 64 tokens
    args = [ctypes.byref(cd), FAKE, FAKE, 10, FAKE, 1 << 24, FAKE, 128, big, FAKE, None, FAKE, 1 << 40, None]
    assert lib.mla_decode_attention(*args) == -1           # 128 x 2^24 = 2^31 pages
    na = [ctypes.byref(cd), FAKE, FAKE, 10, FAKE, 1 << 24, FAKE, 128, big, FAKE, None, None]
    assert lib.mla_decode_attention_noalloc(*na) == -1
    na[8] = big + 1                                         # beyond the 2^30 length limit
    na[7] = 1
    assert lib.mla_decode_attention_noalloc(*na) == -1
    na[8] = 0
    assert lib.mla_decode_attention_noalloc(*na) == -1


def test_workspace_size_is_zero_for_out_of_range_lengths(lib):
    for call in (M.CALL_DECODE_ATTENTION, M.CALL_PREFILL_ATTENTION):
        for d in (synth.RUNNING, synth.PRODUCTION):
            assert M.workspace_size(d, call, 4, 2**31 - 1) == 0
            assert M.workspace_size(d, call, 4, 0) == 0


def test_prefill_groups_shrink_to_keep_page_totals_in_int32():
    """At max_seq_len = 2^30 (2^24 pages) a launch group holds at most INT32_MAX // 2^24 = 127
    tokens, so the workspace stops growing there instead of at 1024 tokens."""
    P = synth.PRODUCTION
    big = 1 << 30
    a = M.workspace_size(P, M.CALL_PREFILL_ATTENTION, 127, big)
    assert a > 0
    assert a == M.workspace_size(P, M.CALL_PREFILL_ATTENTION, 128, big) == M.workspace_size(
        P, M.CALL_PREFILL_ATTENTION, 4096, big)
    assert a >= 127 * (1 << 24) * 4


def test_fp8_calls_argument_errors_queue_nothing(lib):
    """The FP8 cache calls: page size, shape support and argument checks, before anything is
    queued (no GPU)."""
    P, R = dims(synth.PRODUCTION), dims(synth.RUNNING)
    assert lib.mla_fp8_page_bytes(ctypes.byref(P)) == 64 * 584
    assert lib.mla_fp8_supported(ctypes.byref(P)) == 0
    assert lib.mla_fp8_supported(ctypes.byref(R)) == -2
    assert lib.mla_workspace_size(ctypes.byref(R), M.CALL_DECODE_ATTENTION_FP8, 4, 256) == 0
    need = lib.mla_workspace_size(ctypes.byref(P), M.CALL_APPEND_KV_FP8, 64, 0)
    assert need >= 64 * 576 * 2 and need % 256 == 0
    args = [ctypes.byref(P), FAKE, FAKE, FAKE, FAKE, FAKE, 2, 4, FAKE, 8, 64, FAKE, need, None]

    def append(**kw):
        a = list(args)
        for k, v in kw.items():
            a[int(k[1:])] = v
        return lib.mla_append_kv_fp8(*a)
    assert append(a0=ctypes.byref(R)) == -2
    assert append(a12=need - 16) == -3
    assert append(a8=MISALIGNED) == -4
    assert append(a10=0, a1=None) == 0
    assert lib.mla_last_launch_count(M.CALL_APPEND_KV_FP8) == 0
    dneed = lib.mla_workspace_size(ctypes.byref(P), M.CALL_DECODE_ATTENTION_FP8, 2, 256)
    assert dneed > 0
    dargs = [ctypes.byref(P), FAKE, FAKE, 10, FAKE, 4, FAKE, 2, 256, FAKE, None, FAKE, dneed, None]

    def decode(**kw):
        a = list(dargs)
        for k, v in kw.items():
            a[int(k[1:])] = v
        return lib.mla_decode_attention_fp8(*a)
    assert decode(a0=ctypes.byref(R)) == -2
    assert decode(a12=dneed - 16) == -3
    assert decode(a8=257 * 64) == -1                      # max_pages * page_size < max_seq_len
    assert decode(a7=0) == 0
    assert lib.mla_last_launch_count(M.CALL_DECODE_ATTENTION_FP8) == 0
