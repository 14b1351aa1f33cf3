// CUDA-core latent attention (any supported dims; the path for small head counts):
// one warp per head, tokens streamed with an online softmax, split-KV partials merged by
// log-sum-exp in a fixed order (bitwise reproducible).
#pragma once

#include "common.cuh"

namespace mla {


// grid (n_splits, B, ceil(n_h / 8)), block 256 (warp w -> head blockIdx.z*8 + w).
// NPAIR = ceil(D / 64): element pairs of one row held per lane.
template <typename T, int NPAIR>
__global__ void __launch_bounds__(256) k_decode_simt(
    const T* __restrict__ q, const T* __restrict__ pool, const int* __restrict__ bt, int max_pages,
    const int* __restrict__ seq_lens, int max_seq_len, int num_pages, int n_h, int d_c, int D, int page_size,
    float scale_log2, int split_len, int n_splits, T* __restrict__ o_lat, float* __restrict__ lse_out,
    float* __restrict__ o_part, float* __restrict__ lse_part) {
  using P = Pack<T>;
  using T2 = typename P::T2;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.z * 8 + (threadIdx.x >> 5);
  const int split = blockIdx.x, b = blockIdx.y;
  if (h >= n_h) return;
  int L = seq_lens[b];
  if (L < 1 || L > max_seq_len || (L + page_size - 1) / page_size > max_pages) {
    if (split == 0 && h == 0 && lane == 0) record_error(MLA_ERR_BAD_SEQ_LEN);
    L = 0;  // the sequence's output becomes zeros
  }
  const int npairs = D / 2, lpairs = d_c / 2;
  const T2* qp = reinterpret_cast<const T2*>(q + ((long)b * n_h + h) * D);
  float2 qf[NPAIR], o[NPAIR];
#pragma unroll
  for (int r = 0; r < NPAIR; ++r) {
    const int p = lane + 32 * r;
    float2 v = make_float2(0.f, 0.f);
    if (p < npairs) v = P::f2(qp[p]);
    qf[r] = make_float2(v.x * scale_log2, v.y * scale_log2);
    o[r] = make_float2(0.f, 0.f);
  }
  float m = -INFINITY, l = 0.f;  // running max (log2 units) and denominator
  const int t0 = split * split_len;
  const int t1 = min(L, t0 + split_len);
  const int* btb = bt + (long)b * max_pages;
  for (int t = t0; t < t1; ++t) {
    const int page = btb[t / page_size];
    if (page < 0 || page >= num_pages) {
      if (lane == 0) record_error(MLA_ERR_BAD_PAGE);
      continue;
    }
    const T2* row = reinterpret_cast<const T2*>(pool + ((long)page * page_size + t % page_size) * D);
    float2 c[NPAIR];
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < NPAIR; ++r) {
      const int p = lane + 32 * r;
      c[r] = make_float2(0.f, 0.f);
      if (p < npairs) c[r] = P::f2(row[p]);
      s = fmaf(qf[r].x, c[r].x, fmaf(qf[r].y, c[r].y, s));
    }
    s = warp_sum(s);
    const float m_new = fmaxf(m, s);
    const float alpha = exp2f(m - m_new);
    const float pj = exp2f(s - m_new);
    l = fmaf(l, alpha, pj);
#pragma unroll
    for (int r = 0; r < NPAIR; ++r) {
      if (lane + 32 * r < lpairs) {
        o[r].x = fmaf(o[r].x, alpha, pj * c[r].x);
        o[r].y = fmaf(o[r].y, alpha, pj * c[r].y);
      }
    }
    m = m_new;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const float lse = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
  const long bh = (long)b * n_h + h;
  if (n_splits == 1) {
    T2* out = reinterpret_cast<T2*>(o_lat + bh * d_c);
#pragma unroll
    for (int r = 0; r < NPAIR; ++r) {
      const int p = lane + 32 * r;
      if (p < lpairs) out[p] = P::make(o[r].x * inv, o[r].y * inv);
    }
    if (lse_out != nullptr && lane == 0) lse_out[bh] = lse;
  } else {
    float2* out = reinterpret_cast<float2*>(o_part + (bh * n_splits + split) * d_c);
#pragma unroll
    for (int r = 0; r < NPAIR; ++r) {
      const int p = lane + 32 * r;
      if (p < lpairs) out[p] = make_float2(o[r].x * inv, o[r].y * inv);
    }
    if (lane == 0) lse_part[bh * n_splits + split] = lse;
  }
}

// Merge of split-KV partials: o = sum_s w_s o_s / sum_s w_s with w_s = e^{lse_s - max lse},
// summed in split order. One warp per (b, head), grid ceil(B n_h / 8), 256 threads; lane l takes
// columns 4l + 128q (d_c a multiple of 4, <= 512). Lane s holds w_s (splits past 32 recompute it);
// each lane keeps eight partial rows' loads in flight. o_part [BH][S][d_c], lse_part [BH][S].
template <typename T>
__global__ void __launch_bounds__(256) k_lse_merge_warp(const float* __restrict__ o_part,
                                                         const float* __restrict__ lse_part, int n_splits, int d_c,
                                                         long BH, T* __restrict__ o_lat, float* __restrict__ lse_out) {
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch();
  const long bh = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (bh >= BH) return;
  const float* lp = lse_part + bh * n_splits;
  const float l_lane = lane < n_splits ? lp[lane] : -INFINITY;
  float mx = l_lane;
  for (int s = lane + 32; s < n_splits; s += 32) mx = fmaxf(mx, lp[s]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  auto weight = [&](float l) { return l > -INFINITY ? exp2f((l - mx) * kLog2e) : 0.f; };  // -inf: no tokens
  const float w_lane = weight(l_lane);
  float z = w_lane;
  for (int s = lane + 32; s < n_splits; s += 32) z += weight(lp[s]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  const float inv = z > 0.f ? 1.f / z : 0.f;
  const float* src0 = o_part + bh * n_splits * d_c;
  for (int c = 4 * lane; c < d_c; c += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < n_splits; s0 += 8) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = s0 + u < n_splits ? *reinterpret_cast<const float4*>(src0 + (long)(s0 + u) * d_c + c)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int s = s0 + u;
        const float w = s < 32 ? __shfl_sync(0xffffffffu, w_lane, s & 31) : (s < n_splits ? weight(lp[s]) : 0.f);
        acc.x = fmaf(w, v[u].x, acc.x);
        acc.y = fmaf(w, v[u].y, acc.y);
        acc.z = fmaf(w, v[u].z, acc.z);
        acc.w = fmaf(w, v[u].w, acc.w);
      }
    }
    T* out = o_lat + bh * d_c + c;
    Out<T>::put(out, acc.x * inv);
    Out<T>::put(out + 1, acc.y * inv);
    Out<T>::put(out + 2, acc.z * inv);
    Out<T>::put(out + 3, acc.w * inv);
  }
  if (lse_out != nullptr && lane == 0) lse_out[bh] = z > 0.f ? mx + logf(z) : -INFINITY;
}

}  // namespace mla
