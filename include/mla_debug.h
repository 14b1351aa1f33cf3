/*
 * mla_debug.h — introspection of libmla's host-side planning, for tests (not part of the method).
 *
 * The projection calls (mla_append_kv, mla_absorb_query, mla_out_proj) run every product
 * D[z][m][n] = sum_k A[z][m][k] * B[z][n][k] (z < batch, m < M, n < N, k < K) on one persistent
 * tcgen05 GEMM whose iteration space (tile, 64-wide k block) is cut into G contiguous CTA ranges.
 * This call returns the plan those calls would use on the current device (148 SMs assumed when no
 * device is available), so that its invariants can be checked without a GPU.
 */
#ifndef MLA_DEBUG_H_
#define MLA_DEBUG_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Plan of the GEMM for an M x N x K product batched `batch` times; `fused_rope` != 0 for the
 * output steps that apply RoPE (they keep a cos/sin table in shared memory), d_rope its width.
 * On success writes 11 values to out[0..10] (caller-owned host array):
 *   out[0] BN (tile width over N), out[1] m tiles, out[2] n tiles, out[3] k blocks per tile,
 *   out[4] tiles (= m tiles * n tiles * batch), out[5] G (CTAs), out[6] ring stages,
 *   out[7] 1 if CTA ranges start at tile boundaries (else iterations are split evenly),
 *   out[8] 1 if some tile is shared by several CTAs (fp32 partials + a reduction launch),
 *   out[9] dynamic shared memory per CTA in bytes, out[10] partial-buffer bytes.
 * CTA c owns iterations [start(c), start(c+1)): start(c) = (tiles*c/G)*k_blocks when aligned,
 * else tiles*k_blocks*c/G (integer division). Returns 0, or -1 (MLA_ERR_INVALID_ARG) if a size
 * is not positive or `out` is NULL. Queues nothing. */
int mla_debug_gemm_plan(int32_t M, int32_t N, int32_t K, int32_t batch, int32_t fused_rope, int32_t d_rope,
                        int64_t* out);

/* Fault injection for testing the bounded waits (not part of the method). In the library built
 * with MLA_FAULT_INJECT (libmla_faultinj.so, used only by tests), every wait inside a kernel gives
 * up after 20 ms instead of 2 s, and this call makes the next mla_decode_attention calls on the
 * current device leave one cache load unissued: the first latent load of 128-token tile `tile` of
 * the call's concatenated tile list (the tiles of sequence 0, then of sequence 1, ...; -1: none).
 * The waits of the SM pair that owns it then run out; its kernel records MLA_ERR_TIMEOUT
 * in the device status, waits for the loads it did issue, releases its tensor memory and
 * returns, and later calls on the stream run normally once the injection is cleared (-1). The
 * output of the call with a missing load is undefined. Returns 0 (set), MLA_ERR_INVALID_ARG in
 * the regular library (which has no injection) or for tile < -1, MLA_ERR_CUDA if the copy to the
 * device fails. */
int mla_debug_inject_missing_load(int32_t tile);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DEBUG_H_ */
