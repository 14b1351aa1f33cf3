"""Python binding of libmla, the MLA absorbed-decode library for B200 (sm_100a).

Argument marshalling only: every step of the path runs in libmla's CUDA kernels, reached
through the C ABI of ``include/mla.h``. Torch supplies device memory and streams. If the
shared library is missing, every call raises; there is no fallback of any kind.

Method: "DeepSeek-V2 from Scratch", §6 (the complete MLA algorithm) in the absorbed form of
§5.3: append the new token's latent row, absorb W^UK into the query, attend in latent space,
fold W^UV into the output projection.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

__all__ = [
    "MLAError", "load_library", "library_path", "c_dims", "workspace_size", "cache_elems_per_token",
    "append_kv", "absorb_query", "decode_attention", "decode_attention_noalloc", "prefill_attention", "out_proj",
    "read_device_status", "last_launch_count", "LayerState", "layer_step", "layer_step_small",
    "layer_step_small_supported", "fp8_page_bytes", "fp8_supported", "append_kv_fp8", "decode_attention_fp8",
    "CALL_APPEND_KV", "CALL_ABSORB_QUERY", "CALL_DECODE_ATTENTION", "CALL_OUT_PROJ", "CALL_PREFILL_ATTENTION",
    "CALL_LAYER_STEP_SMALL", "CALL_APPEND_KV_FP8", "CALL_DECODE_ATTENTION_FP8",
]

CALL_APPEND_KV, CALL_ABSORB_QUERY, CALL_DECODE_ATTENTION, CALL_OUT_PROJ, CALL_PREFILL_ATTENTION = 0, 1, 2, 3, 4
CALL_LAYER_STEP_SMALL = 5
CALL_APPEND_KV_FP8, CALL_DECODE_ATTENTION_FP8 = 6, 7
_PKG = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(_PKG, "libmla.so")


class MLAError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {_lib().mla_error_string(code).decode()} ({code})")


class _Dims(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("d_head", ctypes.c_int32),
                ("d_c", ctypes.c_int32), ("d_cq", ctypes.c_int32), ("d_rope", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("dtype", ctypes.c_int32), ("rope_base", ctypes.c_double),
                ("rope_inv_freq", ctypes.c_void_p)]


_LIB = None
_P, _I32, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
_SIGS = {
    "mla_check_dims": (ctypes.c_int, [_P]),
    "mla_cache_elems_per_token": (_I32, [_P]),
    "mla_workspace_size": (_SZ, [_P, _I32, _I32, _I32]),
    "mla_append_kv": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I32, _I32, _P, _I32, _I32, _P, _SZ, _P]),
    "mla_absorb_query": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _I32, _P, _SZ, _P]),
    "mla_decode_attention": (ctypes.c_int, [_P, _P, _P, _I32, _P, _I32, _P, _I32, _I32, _P, _P, _P, _SZ, _P]),
    "mla_prefill_attention": (ctypes.c_int, [_P, _P, _P, _I32, _P, _I32, _I32, _P, _P, _I32, _I32, _P, _P, _P, _SZ,
                                             _P]),
    "mla_out_proj": (ctypes.c_int, [_P, _P, _P, _P, _P, _I32, _P, _SZ, _P]),
    "mla_read_device_status": (ctypes.c_int, [_P, ctypes.POINTER(_I32)]),
    "mla_error_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mla_last_launch_count": (_I32, [_I32]),
    "mla_decode_attention_noalloc": (ctypes.c_int, [_P, _P, _P, _I32, _P, _I32, _P, _I32, _I32, _P, _P, _P]),
    "mla_set_decode_timing_events": (ctypes.c_int, [_P, _P]),
    "mla_debug_inject_missing_load": (ctypes.c_int, [_I32]),
    "mla_layer_step_small_supported": (ctypes.c_int, [_P]),
    "mla_fp8_page_bytes": (ctypes.c_int64, [_P]),
    "mla_fp8_supported": (ctypes.c_int, [_P]),
    "mla_append_kv_fp8": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I32, _I32, _P, _I32, _I32, _P, _SZ, _P]),
    "mla_decode_attention_fp8": (ctypes.c_int, [_P, _P, _P, _I32, _P, _I32, _P, _I32, _I32, _P, _P, _P, _SZ, _P]),
    "mla_layer_step_small": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _I32, _P, _I32, _I32, _P, _P,
                                            _P, _P, _P, _SZ, _P]),
}


def load_library(path: str | None = None):
    """Load libmla.so (built by ``python -m mla_latent_kv_42_b200.build``); raise if absent."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    p = path or library_path()
    if not os.path.exists(p):
        raise RuntimeError(f"libmla.so is not built ({p}); run `python -m mla_latent_kv_42_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    if path is None:
        _LIB = lib
    return lib


_lib = load_library


_ROPE_TABLES = {}


def _rope_table_ptr(d):
    """Device copy (float64, current device) of a dims' RoPE frequency table, or None. The copies are
    kept for the life of the process so that queued kernels can still read them."""
    table = getattr(d, "rope_inv_freq", None)
    if table is None:
        return None
    import torch
    key = (tuple(float(x) for x in table), torch.cuda.current_device())
    t = _ROPE_TABLES.get(key)
    if t is None:
        if len(key[0]) != d.d_rope // 2:
            raise ValueError(f"rope_inv_freq has {len(key[0])} entries, d_rope/2 = {d.d_rope // 2}")
        t = torch.tensor(key[0], dtype=torch.float64, device="cuda")
        _ROPE_TABLES[key] = t
    return t.data_ptr()


def c_dims(d) -> _Dims:
    """mla_dims from a ``synth.Dims`` (or anything with the same attributes). A dims with a RoPE
    frequency table (``rope_inv_freq``, d_rope/2 floats) gets a device copy of it."""
    return _Dims(d.d_model, d.n_heads, d.d_head, d.d_c, d.d_cq, d.d_rope, d.page_size,
                 {"bf16": 0, "fp16": 1}[d.dtype], float(d.rope_base), _rope_table_ptr(d))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(code: int, what: str):
    if code != 0:
        raise MLAError(code, what)


def _need(t, dtype, name, dims=None):
    import torch
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _elem(d):
    import torch
    return {"bf16": torch.bfloat16, "fp16": torch.float16}[d.dtype]


def workspace_size(dims, call: int, B: int, max_seq_len: int = 0) -> int:
    cd = c_dims(dims)
    return int(_lib().mla_workspace_size(ctypes.byref(cd), call, B, max_seq_len))


def cache_elems_per_token(dims) -> int:
    cd = c_dims(dims)
    return int(_lib().mla_cache_elems_per_token(ctypes.byref(cd)))


def _ws(dims, call, B, max_seq_len, ws, device):
    import torch
    n = workspace_size(dims, call, B, max_seq_len)
    if ws is None:
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device=device)
    return ws, ws.numel() * ws.element_size()


def append_kv(dims, h, w_dkv_kr, seq_idx, pos, block_table, pool, ws=None, stream=None):
    """mla_append_kv: write [c ‖ RoPE(k^)] of each new token into its paged slot of ``pool``."""
    import torch
    e = _elem(dims)
    for t, n, dt in ((h, "h", e), (w_dkv_kr, "w_dkv_kr", e), (seq_idx, "seq_idx", torch.int32),
                     (pos, "pos", torch.int32), (block_table, "block_table", torch.int32), (pool, "pool", e)):
        _need(t, dt, n)
    T = h.shape[0]
    ws, nbytes = _ws(dims, CALL_APPEND_KV, T, 0, ws, h.device)
    cd = c_dims(dims)
    _check(_lib().mla_append_kv(ctypes.byref(cd), _ptr(h), _ptr(w_dkv_kr), _ptr(seq_idx), _ptr(pos),
                                _ptr(block_table), block_table.shape[0], block_table.shape[1], _ptr(pool),
                                pool.shape[0], T, _ptr(ws), nbytes, _stream(stream)), "mla_append_kv")
    return pool


def absorb_query(dims, h, w_dq, w_uq_qr, w_uk, pos, q_out=None, ws=None, stream=None):
    """mla_absorb_query: q_out[b][i] = [(W^UK_i)^T q^C_i ‖ RoPE(q^_i, pos[b])]."""
    import torch
    e = _elem(dims)
    for t, n, dt in ((h, "h", e), (w_dq, "w_dq", e), (w_uq_qr, "w_uq_qr", e), (w_uk, "w_uk", e),
                     (pos, "pos", torch.int32)):
        _need(t, dt, n)
    B = h.shape[0]
    if q_out is None:
        q_out = torch.empty((B, dims.n_heads, dims.d_c + dims.d_rope), dtype=e, device=h.device)
    _need(q_out, e, "q_out")
    ws, nbytes = _ws(dims, CALL_ABSORB_QUERY, B, 0, ws, h.device)
    cd = c_dims(dims)
    _check(_lib().mla_absorb_query(ctypes.byref(cd), _ptr(h), _ptr(w_dq), _ptr(w_uq_qr), _ptr(w_uk), _ptr(pos),
                                   _ptr(q_out), B, _ptr(ws), nbytes, _stream(stream)), "mla_absorb_query")
    return q_out


def decode_attention(dims, q, pool, block_table, seq_lens, max_seq_len, o_lat=None, lse=None, want_lse=True,
                     ws=None, stream=None):
    """mla_decode_attention: latent-space softmax attention of every head over its sequence's cache."""
    import torch
    e = _elem(dims)
    for t, n, dt in ((q, "q", e), (pool, "pool", e), (block_table, "block_table", torch.int32),
                     (seq_lens, "seq_lens", torch.int32)):
        _need(t, dt, n)
    B = q.shape[0]
    if o_lat is None:
        o_lat = torch.empty((B, dims.n_heads, dims.d_c), dtype=e, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, dims.n_heads), dtype=torch.float32, device=q.device)
    _need(o_lat, e, "o_lat")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    ws, nbytes = _ws(dims, CALL_DECODE_ATTENTION, B, max_seq_len, ws, q.device)
    cd = c_dims(dims)
    _check(_lib().mla_decode_attention(ctypes.byref(cd), _ptr(q), _ptr(pool), pool.shape[0], _ptr(block_table),
                                       block_table.shape[1], _ptr(seq_lens), B, int(max_seq_len), _ptr(o_lat),
                                       _ptr(lse), _ptr(ws), nbytes, _stream(stream)), "mla_decode_attention")
    return o_lat, lse


def fp8_page_bytes(dims) -> int:
    """Bytes of one FP8 cache page: page_size rows of d_c + d_rope e4m3 bytes, then page_size
    float32 pairs (s_c, s_r)."""
    cd = c_dims(dims)
    return int(_lib().mla_fp8_page_bytes(ctypes.byref(cd)))


def fp8_supported(dims) -> bool:
    cd = c_dims(dims)
    return _lib().mla_fp8_supported(ctypes.byref(cd)) == 0


def append_kv_fp8(dims, h, w_dkv_kr, seq_idx, pos, block_table, pool, ws=None, stream=None):
    """mla_append_kv_fp8: the rows of mla_append_kv, quantised to e4m3 with two scales per token,
    into ``pool`` (uint8 [num_pages, fp8_page_bytes(dims)])."""
    import torch
    e = _elem(dims)
    for t, n, dt in ((h, "h", e), (w_dkv_kr, "w_dkv_kr", e), (seq_idx, "seq_idx", torch.int32),
                     (pos, "pos", torch.int32), (block_table, "block_table", torch.int32), (pool, "pool", torch.uint8)):
        _need(t, dt, n)
    if pool.dim() != 2 or pool.shape[1] != fp8_page_bytes(dims):
        raise ValueError("pool must be uint8 [num_pages, fp8_page_bytes(dims)]")
    T = h.shape[0]
    ws, nbytes = _ws(dims, CALL_APPEND_KV_FP8, T, 0, ws, h.device)
    cd = c_dims(dims)
    _check(_lib().mla_append_kv_fp8(ctypes.byref(cd), _ptr(h), _ptr(w_dkv_kr), _ptr(seq_idx), _ptr(pos),
                                    _ptr(block_table), block_table.shape[0], block_table.shape[1], _ptr(pool),
                                    pool.shape[0], T, _ptr(ws), nbytes, _stream(stream)), "mla_append_kv_fp8")
    return pool


def decode_attention_fp8(dims, q, pool, block_table, seq_lens, max_seq_len, o_lat=None, lse=None, want_lse=True,
                         ws=None, stream=None):
    """mla_decode_attention_fp8: mla_decode_attention over an FP8 cache (uint8 [num_pages,
    fp8_page_bytes(dims)])."""
    import torch
    e = _elem(dims)
    for t, n, dt in ((q, "q", e), (pool, "pool", torch.uint8), (block_table, "block_table", torch.int32),
                     (seq_lens, "seq_lens", torch.int32)):
        _need(t, dt, n)
    if pool.dim() != 2 or pool.shape[1] != fp8_page_bytes(dims):
        raise ValueError("pool must be uint8 [num_pages, fp8_page_bytes(dims)]")
    B = q.shape[0]
    if o_lat is None:
        o_lat = torch.empty((B, dims.n_heads, dims.d_c), dtype=e, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, dims.n_heads), dtype=torch.float32, device=q.device)
    _need(o_lat, e, "o_lat")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    ws, nbytes = _ws(dims, CALL_DECODE_ATTENTION_FP8, B, max_seq_len, ws, q.device)
    cd = c_dims(dims)
    _check(_lib().mla_decode_attention_fp8(ctypes.byref(cd), _ptr(q), _ptr(pool), pool.shape[0], _ptr(block_table),
                                           block_table.shape[1], _ptr(seq_lens), B, int(max_seq_len), _ptr(o_lat),
                                           _ptr(lse), _ptr(ws), nbytes, _stream(stream)), "mla_decode_attention_fp8")
    return o_lat, lse


def prefill_attention(dims, q, pool, block_table, seq_idx, pos, max_seq_len, o_lat=None, lse=None, want_lse=True,
                      ws=None, stream=None):
    """mla_prefill_attention: causal latent attention of several new tokens per sequence.

    Token t (sequence ``seq_idx[t]``, position ``pos[t]``) attends to its sequence's cached
    positions 0..pos[t]; the new tokens' rows must already be appended.
    """
    import torch
    e = _elem(dims)
    for t, n, dt in ((q, "q", e), (pool, "pool", e), (block_table, "block_table", torch.int32),
                     (seq_idx, "seq_idx", torch.int32), (pos, "pos", torch.int32)):
        _need(t, dt, n)
    T = q.shape[0]
    if o_lat is None:
        o_lat = torch.empty((T, dims.n_heads, dims.d_c), dtype=e, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, dims.n_heads), dtype=torch.float32, device=q.device)
    _need(o_lat, e, "o_lat")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    ws, nbytes = _ws(dims, CALL_PREFILL_ATTENTION, T, max_seq_len, ws, q.device)
    cd = c_dims(dims)
    _check(_lib().mla_prefill_attention(ctypes.byref(cd), _ptr(q), _ptr(pool), pool.shape[0], _ptr(block_table),
                                        block_table.shape[0], block_table.shape[1], _ptr(seq_idx), _ptr(pos), T,
                                        int(max_seq_len), _ptr(o_lat), _ptr(lse), _ptr(ws), nbytes,
                                        _stream(stream)), "mla_prefill_attention")
    return o_lat, lse


def decode_attention_noalloc(dims, q, pool, block_table, seq_lens, max_seq_len, o_lat=None, lse=None,
                             want_lse=True, stream=None):
    """mla_decode_attention_noalloc: the same attention with the library's static scratch.

    For callers that cannot allocate device memory when they decode (memory reserved up front
    by their own allocator, no tolerance for cudaMalloc's synchronisation, no workspace
    allocator). Problems needing more than 64 MiB of split-KV scratch raise MLAError (-3).
    The scratch is shared by every call on the device: calls overlapping on the GPU race.
    """
    import torch
    e = _elem(dims)
    for t, n, dt in ((q, "q", e), (pool, "pool", e), (block_table, "block_table", torch.int32),
                     (seq_lens, "seq_lens", torch.int32)):
        _need(t, dt, n)
    B = q.shape[0]
    if o_lat is None:
        o_lat = torch.empty((B, dims.n_heads, dims.d_c), dtype=e, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, dims.n_heads), dtype=torch.float32, device=q.device)
    _need(o_lat, e, "o_lat")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    cd = c_dims(dims)
    _check(_lib().mla_decode_attention_noalloc(ctypes.byref(cd), _ptr(q), _ptr(pool), pool.shape[0],
                                               _ptr(block_table), block_table.shape[1], _ptr(seq_lens), B,
                                               int(max_seq_len), _ptr(o_lat), _ptr(lse), _stream(stream)),
           "mla_decode_attention_noalloc")
    return o_lat, lse


def out_proj(dims, o_lat, w_uv, w_o, u=None, ws=None, stream=None):
    """mla_out_proj: u = W^O [W^UV_1 o_lat_1; ...; W^UV_n_h o_lat_n_h]."""
    import torch
    e = _elem(dims)
    for t, n in ((o_lat, "o_lat"), (w_uv, "w_uv"), (w_o, "w_o")):
        _need(t, e, n)
    B = o_lat.shape[0]
    if u is None:
        u = torch.empty((B, dims.d_model), dtype=e, device=o_lat.device)
    _need(u, e, "u")
    ws, nbytes = _ws(dims, CALL_OUT_PROJ, B, 0, ws, o_lat.device)
    cd = c_dims(dims)
    _check(_lib().mla_out_proj(ctypes.byref(cd), _ptr(o_lat), _ptr(w_uv), _ptr(w_o), _ptr(u), B, _ptr(ws), nbytes,
                               _stream(stream)), "mla_out_proj")
    return u


def read_device_status(stream=None) -> int:
    """Synchronise the stream; return and clear the device status word (0 = no device-side error)."""
    v = ctypes.c_int32(0)
    _check(_lib().mla_read_device_status(_stream(stream), ctypes.byref(v)), "mla_read_device_status")
    return int(v.value)


def last_launch_count(call: int) -> int:
    return int(_lib().mla_last_launch_count(call))


def set_decode_timing_events(before=None, after=None):
    """mla_set_decode_timing_events: record two torch.cuda.Event objects around the attention
    kernel of this thread's later decode calls (None, None: stop). The events must have been
    recorded once (so that they exist) before they are handed over."""
    h = lambda e: None if e is None else ctypes.c_void_p(e.cuda_event)
    r = _lib().mla_set_decode_timing_events(h(before), h(after))
    if r != 0:
        raise MLAError(r, "mla_set_decode_timing_events")



@dataclass
class LayerState:
    """Device-resident state of one layer: weights and its paged latent cache."""
    dims: object
    w: dict            # w_dkv_kr, w_dq, w_uq_qr, w_uk, w_uv, w_o (CUDA tensors)
    pool: object       # [num_pages, page_size, d_c + d_rope]
    block_table: object  # int32 [B, max_pages]


def layer_step(st: LayerState, h, pos, seq_idx, seq_lens, max_seq_len, ws=None, out=None, stream=None):
    """One decode step of one layer through the four C-ABI calls; returns (u, q, o_lat, lse).

    ``pos`` = cached length of each sequence (the new token's position), ``seq_lens`` = pos + 1.
    ``ws`` is one byte buffer at least as large as the largest of the four workspaces (the calls
    run in order on one stream, so they can share it).
    """
    d, w = st.dims, st.w
    out = out or {}
    append_kv(d, h, w["w_dkv_kr"], seq_idx, pos, st.block_table, st.pool, ws=ws, stream=stream)
    q = absorb_query(d, h, w["w_dq"], w["w_uq_qr"], w["w_uk"], pos, q_out=out.get("q"), ws=ws, stream=stream)
    o_lat, lse = decode_attention(d, q, st.pool, st.block_table, seq_lens, max_seq_len, o_lat=out.get("o_lat"),
                                  lse=out.get("lse"), want_lse=out.get("want_lse", True), ws=ws, stream=stream)
    u = out_proj(d, o_lat, w["w_uv"], w["w_o"], u=out.get("u"), ws=ws, stream=stream)
    return u, q, o_lat, lse


def layer_step_small_supported(dims) -> bool:
    cd = c_dims(dims)
    return _lib().mla_layer_step_small_supported(ctypes.byref(cd)) == 0


def layer_step_small(st: LayerState, h, seq_lens, max_seq_len, ws=None, out=None, stream=None):
    """mla_layer_step_small: the same decode step as ``layer_step`` (one new token per sequence,
    sequence b = batch row b, new token at position seq_lens[b] - 1) in one launch, for small head
    counts; returns (u, q, o_lat, lse)."""
    import torch
    d, w = st.dims, st.w
    out = out or {}
    e = _elem(d)
    B = h.shape[0]
    dev = h.device
    q = out.get("q")
    if q is None:
        q = torch.empty((B, d.n_heads, d.d_c + d.d_rope), dtype=e, device=dev)
    o_lat = out.get("o_lat")
    if o_lat is None:
        o_lat = torch.empty((B, d.n_heads, d.d_c), dtype=e, device=dev)
    lse = out.get("lse")
    if lse is None and out.get("want_lse", True):
        lse = torch.empty((B, d.n_heads), dtype=torch.float32, device=dev)
    u = out.get("u")
    if u is None:
        u = torch.empty((B, d.d_model), dtype=e, device=dev)
    ws, nbytes = _ws(d, CALL_LAYER_STEP_SMALL, B, max_seq_len, ws, dev)
    cd = c_dims(d)
    pool, bt = st.pool, st.block_table
    _check(_lib().mla_layer_step_small(ctypes.byref(cd), _ptr(h), _ptr(w["w_dkv_kr"]), _ptr(w["w_dq"]),
                                       _ptr(w["w_uq_qr"]), _ptr(w["w_uk"]), _ptr(w["w_uv"]), _ptr(w["w_o"]),
                                       _ptr(pool), pool.shape[0], _ptr(bt), bt.shape[1], _ptr(seq_lens), B,
                                       max_seq_len, _ptr(q), _ptr(o_lat), _ptr(lse), _ptr(u), _ptr(ws), nbytes,
                                       _stream(stream)), "mla_layer_step_small")
    return u, q, o_lat, lse


def step_workspace_bytes(dims, B: int, max_seq_len: int) -> int:
    return max(workspace_size(dims, c, B, max_seq_len) for c in range(4))
