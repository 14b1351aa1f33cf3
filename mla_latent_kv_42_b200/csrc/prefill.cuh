// Attention for a step that brings several new tokens per sequence (chunked prefill), over the
// paged latent cache. The attention sum of the complete algorithm ("DeepSeek-V2 from Scratch",
// §6) runs over the cached positions j <= t of the token at position t, so each new token is an
// independent attention item: its attended length is pos + 1 and its pages are its sequence's.
// The tokens therefore run through the decode attention kernels as items of their own. At
// n_h = 128 one token's fp32 output (128 heads x 512 latents) fills a whole SM's tensor memory,
// so tokens cannot share a cache tile inside one SM; tokens of a sequence sit next to each other
// in item order instead, so the clusters working on them read the same pages at about the same
// time and the repeat reads come from L2.
#pragma once

#include "common.cuh"

namespace mla {

// Per-token attention items: length pos[t] + 1 and a copy of the block-table row of
// seq_idx[t], cut to the pages that length covers (the attention kernels read no further).
// A token whose sequence index is outside [0, num_seqs) or whose position is outside
// [0, max_seq_len) gets length 0, which the attention planner rejects (zero output and
// MLA_ERR_BAD_SEQ_LEN in the device status). One warp per token: grid ceil(T / 8), 256 threads.
// item_pages = ceil(max_seq_len / page_size) <= max_pages, so every copy stays in both rows.
__global__ void __launch_bounds__(256) k_prefill_items(const int* __restrict__ seq_idx, const int* __restrict__ pos,
                                                       const int* __restrict__ bt, int num_seqs, int max_pages,
                                                       int page_size, int max_seq_len, int T, int item_pages,
                                                       int* __restrict__ item_bt, int* __restrict__ item_len) {
  griddep_wait();  // positions, the block table and the item buffers belong to earlier kernels
  if (threadIdx.x == 0) griddep_launch();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= T) return;
  const int s = seq_idx[t], p = pos[t];
  const bool ok = s >= 0 && s < num_seqs && p >= 0 && p < max_seq_len;
  const int L = ok ? p + 1 : 0;
  const int n = (L + page_size - 1) / page_size;
  const int* src = bt + (long)(ok ? s : 0) * max_pages;
  int* dst = item_bt + (long)t * item_pages;
  for (int j = lane; j < n; j += 32) dst[j] = src[j];
  if (lane == 0) item_len[t] = L;
}

}  // namespace mla
