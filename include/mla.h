/*
 * mla.h — C ABI of libmla: Multi-head Latent Attention (DeepSeek-V2) at decode time, in its
 * weight-absorbed form, on NVIDIA B200 (sm_100a).
 *
 * Method source: "DeepSeek-V2 from Scratch: Multi-head Latent Attention and DeepSeekMoE",
 * §2 (joint KV compression), §4 (decoupled RoPE), §5 (matrix absorption), §6 (the complete
 * algorithm). Notation: d = d_model, n_h heads of d_h, KV latent d_c, query latent d_c'
 * (d_cq), decoupled RoPE width d_h^R (d_rope). One cache row is [c^KV (d_c) ‖ k^R (d_rope)].
 *
 * Conventions for every call
 *   - Matrices follow the pages' y = W x convention: W is [out, in], row-major. Head i of
 *     W^UQ / W^UK / W^UV is the contiguous row block [i*d_h, (i+1)*d_h); head i of W^QR the
 *     row block [i*d_rope, (i+1)*d_rope); head i of W^O its column block [i*d_h, (i+1)*d_h).
 *   - Element type of every activation, weight and cache buffer is dims->dtype (bf16 or
 *     fp16); accumulation is fp32. Results are rounded to the element type to nearest even.
 *   - RoPE rotates adjacent pairs (x[2k], x[2k+1]) by the angle pos * theta_k with
 *     theta_k = rope_base^(-2k/d_rope) (or the caller's table, mla_dims.rope_inv_freq), formed in
 *     double precision; positions are 0-based.
 *   - Ownership: the caller owns every buffer. All pointer arguments are DEVICE pointers,
 *     16-byte aligned, on the current device. The library allocates no device memory and
 *     keeps no per-call state besides one device status word per device.
 *   - Asynchrony: work is queued on `stream` (NULL = the legacy default stream) and the call
 *     returns without synchronising. Calls on different streams may run concurrently if their
 *     buffers (including workspaces) do not overlap.
 *   - Threads: any host thread may call at any time. The library's own host state is per-device
 *     caches of device properties (atomic) and, per thread, the launch counts and the timing
 *     hook below; mla_decode_attention_noalloc's static scratch is the one shared buffer.
 *   - Overlap of consecutive kernels: every kernel is launched with programmatic dependent
 *     launch, so it may start while the kernel queued just before it on `stream` still runs.
 *     Each kernel waits for that predecessor to complete, with its memory visible, before it
 *     touches activations, caches, workspaces or outputs. The one read issued earlier is the
 *     first few k blocks of a projection's WEIGHT matrix (W^DKV, W^KR, W^DQ, W^UQ, W^QR, W^UK,
 *     W^UV, W^O). So a kernel that writes a weight buffer must be separated from the calls that
 *     read it by an event record on `stream` or a host synchronisation (weights loaded once and
 *     synchronised meet this); no library call writes a weight.
 *   - Errors: calls return MLA_OK (0) or a negative mla_status. Argument checks run before
 *     anything is queued, so an error return from a check means no work was queued. A launch
 *     failure returns MLA_ERR_CUDA. Kernels never trap or assert: a bad page id or sequence
 *     length found on the device is recorded in the device status word (see
 *     mla_read_device_status) and the offending row is skipped (written as zeros).
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t / CUstream). */
typedef struct CUstream_st* mla_stream_t;

enum mla_dtype { MLA_BF16 = 0, MLA_FP16 = 1 };

typedef struct mla_dims {
  int32_t d_model;   /* d */
  int32_t n_heads;   /* n_h, 1..128 */
  int32_t d_head;    /* d_h */
  int32_t d_c;       /* KV latent width */
  int32_t d_cq;      /* query latent width d_c' */
  int32_t d_rope;    /* d_h^R, even */
  int32_t page_size; /* tokens per cache page */
  int32_t dtype;     /* enum mla_dtype */
  double rope_base;  /* RoPE frequency base, e.g. 10000 */
  /* Optional RoPE frequency table: DEVICE pointer to d_rope/2 doubles theta_k (8-byte aligned),
   * used in place of rope_base^(-2k/d_rope) by mla_append_kv (k^R) and mla_absorb_query (q^R),
   * e.g. YaRN-interpolated frequencies for context extension (the velog DeepSeek-V2 review §4.1
   * applies YaRN to the decoupled key; its constants are not on the pages, so the caller supplies
   * the table; an amplitude factor of YaRN folds into W^QR and W^KR). NULL: the base formula. The
   * table must stay valid until the calls that read it have completed. */
  const double* rope_inv_freq;
} mla_dims;
/* The softmax scale is derived, 1/sqrt(d_head + d_rope) (from-scratch page, §4.4). */

enum mla_status {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = -1,         /* null pointer, negative size, bad enum */
  MLA_ERR_UNSUPPORTED_DIMS = -2,    /* dims outside what the kernels support (see mla_check_dims) */
  MLA_ERR_WORKSPACE_TOO_SMALL = -3, /* ws_bytes < mla_workspace_size(...) */
  MLA_ERR_ALIGNMENT = -4,           /* a pointer is not 16-byte aligned */
  MLA_ERR_CUDA = -5,                /* a CUDA runtime call or launch failed */
  MLA_ERR_TIMEOUT = -6,             /* device status: a bounded wait in a kernel gave up */
  MLA_ERR_BAD_PAGE = -7,            /* device status: block-table entry outside [0, num_pages) */
  MLA_ERR_BAD_SEQ_LEN = -8          /* device status: seq_len < 1, > max_seq_len or > max_pages*page_size */
};

enum mla_call {
  MLA_CALL_APPEND_KV = 0,
  MLA_CALL_ABSORB_QUERY = 1,
  MLA_CALL_DECODE_ATTENTION = 2,
  MLA_CALL_OUT_PROJ = 3,
  MLA_CALL_PREFILL_ATTENTION = 4,
  MLA_CALL_LAYER_STEP_SMALL = 5,
  MLA_CALL_APPEND_KV_FP8 = 6,
  MLA_CALL_DECODE_ATTENTION_FP8 = 7
};

/* Returns MLA_OK if every call supports `dims`, else MLA_ERR_UNSUPPORTED_DIMS or
 * MLA_ERR_INVALID_ARG (MLA_ERR_ALIGNMENT for a rope_inv_freq table not 8-byte aligned).
 * Supported: all widths positive multiples of 8 (d_rope a multiple of 8), n_heads <= 128,
 * d_c <= 512, d_c + d_rope <= 576, page_size >= 1, dtype bf16/fp16, rope_base > 0. */
int mla_check_dims(const mla_dims* dims);

/* Elements cached per token per layer, d_c + d_rope ("What Gets Cached", from-scratch page
 * §4.5; 160 for the running model, 576 at DeepSeek-V2 dims). Negative on invalid dims. */
int32_t mla_cache_elems_per_token(const mla_dims* dims);

/* Bytes of workspace the call `call` needs for batch B (new tokens T for append and prefill
 * attention) and longest attended length max_seq_len, on the current device. 0 on invalid
 * arguments. */
size_t mla_workspace_size(const mla_dims* dims, int32_t call, int32_t B, int32_t max_seq_len);

/*
 * mla_append_kv — KV pathway and cache write (from-scratch page §2.1 and §4.2, boxed in §6).
 * For each of the T new tokens t:
 *   [c ; k^] = W_dkv_kr h_t            (W^DKV rows then W^KR rows, fp32 accumulate)
 *   k^R = RoPE(k^, pos[t])
 *   pool row  bt[seq_idx[t]][pos[t] / page_size] * page_size + pos[t] % page_size
 *        <- [c ‖ k^R] rounded to the element type.
 * h         [T, d_model]
 * w_dkv_kr  [d_c + d_rope, d_model]
 * seq_idx   int32 [T], each in [0, num_seqs)        pos int32 [T], >= 0
 * block_table int32 [num_seqs, max_pages]; pool [num_pages, page_size, d_c + d_rope]
 * ws        at least mla_workspace_size(dims, MLA_CALL_APPEND_KV, T, 0) bytes (may be NULL if 0)
 * A token whose page entry is outside [0, num_pages) or whose pos/page_size >= max_pages is
 * not written; the device status records MLA_ERR_BAD_PAGE. T == 0 is a no-op.
 */
int mla_append_kv(const mla_dims* dims, const void* h, const void* w_dkv_kr,
                  const int32_t* seq_idx, const int32_t* pos,
                  const int32_t* block_table, int32_t num_seqs, int32_t max_pages,
                  void* pool, int32_t num_pages, int32_t T,
                  void* ws, size_t ws_bytes, mla_stream_t stream);

/*
 * mla_absorb_query — query pathway with W^UK absorbed (from-scratch page §4.1 and §5.1,
 * step 1 of §5.3):
 *   c^Q = W^DQ h;  [q^C ; q^] = [W^UQ ; W^QR] c^Q;  q^R_i = RoPE(q^_i, pos)
 *   q~_i = (W^UK_i)^T q^C_i
 *   q_out[b][i] = [q~_i (d_c) ‖ q^R_i (d_rope)]   — the same layout as a cache row.
 * h [B, d_model]; w_dq [d_cq, d_model]; w_uq_qr [n_heads*(d_head + d_rope), d_cq] (W^UQ rows
 * then W^QR rows); w_uk [n_heads*d_head, d_c]; pos int32 [B]; q_out [B, n_heads, d_c + d_rope].
 * c^Q and q^C are rounded to the element type before their next product. 0 <= B <= 65535
 * (MLA_ERR_INVALID_ARG otherwise); B == 0 is a no-op.
 */
int mla_absorb_query(const mla_dims* dims, const void* h, const void* w_dq, const void* w_uq_qr,
                     const void* w_uk, const int32_t* pos, void* q_out, int32_t B,
                     void* ws, size_t ws_bytes, mla_stream_t stream);

/*
 * mla_decode_attention — latent attention (from-scratch page §4.4 with §5.3 steps 2-3):
 * for every sequence b and head i, over the attended tokens j = 0 .. seq_lens[b]-1
 *   s_j = (q~_i . c_j + q^R_i . k^R_j) / sqrt(d_head + d_rope)
 *   p = softmax_j(s);   o_lat[b][i] = sum_j p_j c_j                      (d_c values)
 *   lse_out[b][i] = log sum_j exp(s_j)   (natural log; skipped if lse_out is NULL)
 * q [B, n_heads, d_c + d_rope]; pool, block_table as in mla_append_kv (num_seqs = B);
 * seq_lens int32 [B], 1 <= seq_lens[b] <= max_seq_len, the new token already appended;
 * o_lat [B, n_heads, d_c] element type; lse_out float [B, n_heads] or NULL.
 * Long sequences are split across SMs and the partials merged by log-sum-exp; the result is
 * bitwise reproducible run to run. A bad seq_len or page id zeroes that sequence's output and
 * records the error in the device status. 0 <= B <= 65535, 1 <= max_seq_len <= 2^30 and
 * max_pages * page_size >= max_seq_len (MLA_ERR_INVALID_ARG otherwise); B == 0 is a no-op.
 */
int mla_decode_attention(const mla_dims* dims, const void* q, const void* pool, int32_t num_pages,
                         const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens,
                         int32_t B, int32_t max_seq_len, void* o_lat, float* lse_out,
                         void* ws, size_t ws_bytes, mla_stream_t stream);

/*
 * mla_prefill_attention — latent attention for a step that brings several new tokens per
 * sequence (chunked prefill), causal (from-scratch page §6: the attention sum of the token at
 * position t runs over the cached positions j <= t; §5.3 steps 2-3 for each new token).
 * For every new token t and head i, over j = 0 .. pos[t] of sequence seq_idx[t]:
 *   s_j = (q~_i . c_j + q^R_i . k^R_j) / sqrt(d_head + d_rope);  p = softmax_j(s)
 *   o_lat[t][i] = sum_j p_j c_j;   lse_out[t][i] = log sum_j exp(s_j)   (skipped if NULL)
 * So a token sees its sequence's prefix, the new tokens before it and itself, and no later
 * token. Every new token's cache row must already be written (mla_append_kv with the same
 * seq_idx and pos), and q is mla_absorb_query's output for the same tokens and positions.
 * q [T, n_heads, d_c + d_rope]; seq_idx int32 [T] in [0, num_seqs); pos int32 [T] in
 * [0, max_seq_len); block_table int32 [num_seqs, max_pages] and pool as in mla_append_kv,
 * max_pages * page_size >= max_seq_len, 1 <= max_seq_len <= 2^30; o_lat [T, n_heads, d_c] element type; lse_out float
 * [T, n_heads] or NULL; ws at least mla_workspace_size(dims, MLA_CALL_PREFILL_ATTENTION, T,
 * max_seq_len) bytes. Tokens may come in any order; each is computed on its own, with the
 * arithmetic of mla_decode_attention for a sequence of length pos[t] + 1 (where split-KV
 * boundaries fall may differ, so agreement is to rounding). The result is bitwise
 * reproducible run to run. A token with an out-of-range seq_idx or pos gets a zero
 * output (lse -inf) and records MLA_ERR_BAD_SEQ_LEN in the device status; a bad page id
 * records MLA_ERR_BAD_PAGE. T == 0 is a no-op.
 */
int mla_prefill_attention(const mla_dims* dims, const void* q, const void* pool, int32_t num_pages,
                          const int32_t* block_table, int32_t num_seqs, int32_t max_pages,
                          const int32_t* seq_idx, const int32_t* pos, int32_t T, int32_t max_seq_len,
                          void* o_lat, float* lse_out, void* ws, size_t ws_bytes, mla_stream_t stream);

/*
 * mla_out_proj — output projection with W^UV absorbed (from-scratch page §5.2, step 4 of
 * §5.3, and u = W^O [o_1; ...; o_n_h] of §6):
 *   o_i = W^UV_i o_lat_i   (d_head values, rounded to the element type)
 *   u   = W^O [o_1 ; ... ; o_n_h]
 * o_lat [B, n_heads, d_c]; w_uv [n_heads*d_head, d_c]; w_o [d_model, n_heads*d_head];
 * u [B, d_model]. 0 <= B <= 65535 (MLA_ERR_INVALID_ARG otherwise); B == 0 is a no-op.
 */
int mla_out_proj(const mla_dims* dims, const void* o_lat, const void* w_uv, const void* w_o,
                 void* u, int32_t B, void* ws, size_t ws_bytes, mla_stream_t stream);

/* Synchronises `stream`, returns the current device's status word in *status_out (MLA_OK or
 * the first device-side error recorded since the last read) and clears it. */
/*
 * mla_layer_step_small — one decode step of one layer (the four calls above for one new token per
 * sequence: mla_append_kv, mla_absorb_query, mla_decode_attention, mla_out_proj) in a single
 * cooperative launch, for small head counts such as the running model of the from-scratch page
 * (§6: 8 heads, d_c = 128, d_h^R = 32). Where the four-call path is bound by its launches, the
 * phases here meet at grid-wide barriers instead.
 * Sequence b's new token sits at position seq_lens[b] - 1 (its row is computed, written to the
 * cache, and attended by the token itself); h [B, d_model]; the weights as in the four calls
 * (w_dkv_kr [d_c + d_rope, d_model], w_dq [d_cq, d_model], w_uq_qr [n_h*(d_h + d_rope), d_cq],
 * w_uk and w_uv [n_h*d_h, d_c], w_o [d_model, n_h*d_h]); pool, block_table [B, max_pages] and
 * seq_lens as in mla_decode_attention (sequence b of the block table is batch row b).
 * Outputs: q_out [B, n_h, d_c + d_rope] (the absorbed query), o_lat [B, n_h, d_c], lse_out
 * [B, n_h] (or NULL) and u [B, d_model], each as the corresponding call writes it; every
 * product accumulates in fp32 and rounds where that call stores, so the two paths agree to
 * rounding. ws at least mla_workspace_size(dims, MLA_CALL_LAYER_STEP_SMALL, B, max_seq_len)
 * bytes. Supported dims: mla_layer_step_small_supported. 0 <= B <= 65535, B == 0 is a no-op.
 * A bad sequence length or page id is recorded in the device status as in the four calls (the
 * row is not written; the output is zero).
 */
int mla_layer_step_small_supported(const mla_dims* dims); /* MLA_OK or MLA_ERR_UNSUPPORTED_DIMS:
  n_heads <= 16, d_c + d_rope <= 192 and a multiple of 16, d_c <= 128 and a multiple of 16,
  page_size a multiple of 16, d_model, d_cq and n_heads*d_head multiples of 8. */
int mla_layer_step_small(const mla_dims* dims, const void* h, const void* w_dkv_kr, const void* w_dq,
                         const void* w_uq_qr, const void* w_uk, const void* w_uv, const void* w_o, void* pool,
                         int32_t num_pages, const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens,
                         int32_t B, int32_t max_seq_len, void* q_out, void* o_lat, float* lse_out, void* u, void* ws,
                         size_t ws_bytes, mla_stream_t stream);

/*
 * FP8 latent cache (DeepSeek-V2 paper review (velog) §4.2 and the DeepSeek-V2 summary page:
 * the deployed model quantises its KV cache to about 6 bits per element; the pages give no
 * format, so this cache takes e4m3 with two float32 scales per token). A page of page_size
 * tokens is page_size rows of d_c + d_rope e4m3 bytes (token order), then page_size pairs of
 * float32 scales (s_c, s_r): mla_fp8_page_bytes(dims) = page_size * (d_c + d_rope + 8) bytes.
 * Row j of a token stands for
 *   c_j = s_c * e4m3(row[0 .. d_c)),   k^R_j = s_r * e4m3(row[d_c .. d_c + d_rope)),
 * with s = max|part| / 448 in float32 (1 for an all-zero part) and each byte the nearest e4m3
 * value (ties to even) of the element-type value divided by s in float32, saturated to +-448.
 * The FP8 cache serves decode steps (mla_append_kv_fp8, mla_decode_attention_fp8);
 * mla_prefill_attention and mla_layer_step_small read the element-type cache only.
 */
int64_t mla_fp8_page_bytes(const mla_dims* dims); /* negative on invalid dims */

/* MLA_OK if the FP8 calls support `dims`: the DeepSeek-V2 cache shape of the tensor-core decode
 * (d_c = 512, d_rope = 64, page_size = 64, 65 <= n_heads <= 128), else MLA_ERR_UNSUPPORTED_DIMS. */
int mla_fp8_supported(const mla_dims* dims);

/*
 * mla_append_kv_fp8 — mla_append_kv into an FP8 cache: the rows [c ‖ k^R] are computed and
 * rounded to the element type exactly as mla_append_kv computes them, then quantised as above
 * and written, with their scales, to the token's slot of `pool` (FP8 pages, num_pages of
 * mla_fp8_page_bytes each, 16-byte aligned). Arguments, checks and error behaviour as
 * mla_append_kv; ws at least mla_workspace_size(dims, MLA_CALL_APPEND_KV_FP8, T, 0) bytes.
 */
int mla_append_kv_fp8(const mla_dims* dims, const void* h, const void* w_dkv_kr,
                      const int32_t* seq_idx, const int32_t* pos,
                      const int32_t* block_table, int32_t num_seqs, int32_t max_pages,
                      void* pool, int32_t num_pages, int32_t T,
                      void* ws, size_t ws_bytes, mla_stream_t stream);

/*
 * mla_decode_attention_fp8 — mla_decode_attention over an FP8 cache: the attention of every
 * sequence and head over the rows the cache stands for. Its tensor-core products run in fp16
 * with fp32 accumulation: each cached value is converted in shared memory as its e4m3 value
 * (exact in fp16) times its token's scale rounded to fp16, the product rounded once to fp16; the
 * queries are rounded to fp16 and the softmax weights are fp16. So the queries and the values the
 * cache stands for must lie within fp16's range (|x| < 65504), and scales below 2^-14 (parts
 * whose largest magnitude is below about 0.027) lose relative precision. Arguments, outputs,
 * checks and error behaviour as mla_decode_attention, with pool the FP8 pages; ws at least
 * mla_workspace_size(dims, MLA_CALL_DECODE_ATTENTION_FP8, B, max_seq_len) bytes.
 */
int mla_decode_attention_fp8(const mla_dims* dims, const void* q, const void* pool, int32_t num_pages,
                             const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens,
                             int32_t B, int32_t max_seq_len, void* o_lat, float* lse_out,
                             void* ws, size_t ws_bytes, mla_stream_t stream);

int mla_read_device_status(mla_stream_t stream, int32_t* status_out);

/* Static string for a status code. */
const char* mla_error_string(int code);

/* Number of kernel launches the last successful call of `call` on this thread queued
 * (for launch accounting in benchmarks). */
int32_t mla_last_launch_count(int32_t call);

typedef struct CUevent_st* mla_event_t;

/* Profiling hook (not part of the method): from this call on, every mla_decode_attention (and
 * _noalloc) call made by this host thread records `before` on its stream immediately before the
 * attention kernel and `after` immediately after it (mla_prefill_attention records them around the
 * attention kernel of each of its launch groups, so afterwards they bracket the last group's), so that the kernel's own duration can be
 * read with cudaEventElapsedTime apart from the planner and the split-KV merge launched in the
 * same call. Pass NULL for both to stop. The events belong to the caller, who creates them
 * (with timing) and destroys them. An event recorded between two launches keeps the second
 * from starting early into the first one's tail, so leave the hook off where throughput
 * matters. Returns MLA_OK, or MLA_ERR_INVALID_ARG if exactly one of the two is NULL. */
int mla_set_decode_timing_events(mla_event_t before, mla_event_t after);

/*
 * mla_decode_attention_noalloc — mla_decode_attention without a caller-supplied workspace.
 * The paper has no counterpart: it is a convenience for callers that cannot allocate device
 * memory at the moment they run a decode step, such as a serving process whose device memory
 * is reserved up front by its own allocator, code that must not stall on the device-wide
 * synchronisation that cudaMalloc/cudaFree can cause, or a plain C caller with no workspace
 * allocator of its own. The caller still passes q, the cache, the block table, the lengths
 * and the outputs, with the same meaning, layout and checks as mla_decode_attention.
 *
 * The split-KV partials go to one static device array of the library instead:
 * 64 MiB (67108864 bytes), created with the library's module on every GPU that loads it and
 * held until the process exits. A call whose workspace need, mla_workspace_size(dims,
 * MLA_CALL_DECODE_ATTENTION, B, max_seq_len), exceeds 64 MiB is rejected with
 * MLA_ERR_WORKSPACE_TOO_SMALL before anything is queued. The call allocates nothing.
 *
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current; make that first call before any stream capture on the device.
 * Every call on a device shares the one array and it keeps the last call's contents (no part
 * of it needs to start at zero: every partial a call reads was written by that call), so calls
 * whose work overlaps on the GPU race: keep them on one stream or order them yourself.
 */
int mla_decode_attention_noalloc(const mla_dims* dims, const void* q, const void* pool, int32_t num_pages,
                                 const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens,
                                 int32_t B, int32_t max_seq_len, void* o_lat, float* lse_out,
                                 mla_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
