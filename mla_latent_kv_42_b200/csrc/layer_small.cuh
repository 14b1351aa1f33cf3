// One decode step of one layer in a single launch, for small head counts (the pages' running
// model: 8 heads, d_c = 128, a 160-wide cache row): the four calls mla_append_kv,
// mla_absorb_query, mla_decode_attention and mla_out_proj as the phases of one cooperative kernel
// ("DeepSeek-V2 from Scratch" §6, the decode step, in the absorbed form of §5.3). At these sizes
// every product is a few hundred thousand multiply-adds and the attention a few MB of cache, so
// the four-call path is bound by its launches; here the phases are separated by grid-wide
// barriers instead.
//
//   1  [c ; k^] = W^DKV;KR h, k^R = RoPE(k^, pos) -> the new cache row;  c' = W^DQ h
//   2  q^C_i = W^UQ_i c',  q^R_i = RoPE(W^QR_i c', pos)
//   3  q~_i = (W^UK_i)^T q^C_i                      (q = [q~ ; q^R], the attention query)
//   4  latent attention of every head over the sequence's cache (the warp-MMA item of
//      decode_mma.cuh, split over the grid)
//   5  log-sum-exp merge of the splits -> o_lat, lse
//   6  o_i = W^UV_i o_lat_i
//   7  u = W^O [o_1 ; ... ; o_n_h]
// The new token of sequence b sits at position seq_lens[b] - 1. Every product accumulates in fp32
// and rounds to the element type where the four-call path stores (c', q^C, q, o_lat, o, u, and the
// cache row), so the two paths agree to rounding.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "decode_mma.cuh"

namespace mla {

struct SmallStepArgs {
  int B;
  const void* h;         // [B, d_model]
  const void* w_dkv_kr;  // [d_c + d_rope, d_model]
  const void* w_dq;      // [d_cq, d_model]
  const void* w_uq_qr;   // [n_h d_h + n_h d_rope, d_cq]
  const void* w_uk;      // [n_h d_h, d_c]
  const void* w_uv;      // [n_h d_h, d_c]
  const void* w_o;       // [d_model, n_h d_h]
  int d_model, n_h, d_h, d_c, d_cq, d_rope;
  double rope_base;
  const double* rope_table;  // [d_rope / 2] or null
  void* pool;            // [num_pages, page_size, d_c + d_rope]
  void* cq;              // workspace [B, d_cq]
  void* qc;              // workspace [B, n_h, d_h]
  void* q;               // [B, n_h, d_c + d_rope]
  void* o;               // workspace [B, n_h d_h]
  void* u;               // [B, d_model]
  MmaAttnArgs attn;      // phases 4-5 (q, pool, block table, lengths, o_lat, lse, partials)
};

// Dot products of weight rows w0, w1 with vectors x0, x1 (K elements, K % 8 == 0, 16-byte
// aligned) by one warp, fp32, each reduced over the lanes in a fixed order: two rows at a time,
// all their loads in flight together. The vectors are written earlier in the same launch (by other
// CTAs), so they are read at L2 (coherent); the weights through the read-only path.
template <typename T>
__device__ __forceinline__ float2 warp_dot2(const T* __restrict__ w0, const T* x0, const T* __restrict__ w1,
                                            const T* x1, int K, int lane) {
  float acc0 = 0.f, acc1 = 0.f;
  for (int k = 8 * lane; k < K; k += 256) {
    const uint4 a0 = ldg16(w0 + k), a1 = ldg16(w1 + k);
    const uint4 b0 = __ldcg(reinterpret_cast<const uint4*>(x0 + k)), b1 = __ldcg(reinterpret_cast<const uint4*>(x1 + k));
    float fa0[8], fa1[8], fb0[8], fb1[8];
    unpack8<T>(a0, fa0);
    unpack8<T>(a1, fa1);
    unpack8<T>(b0, fb0);
    unpack8<T>(b1, fb1);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      acc0 = fmaf(fa0[e], fb0[e], acc0);
      acc1 = fmaf(fa1[e], fb1[e], acc1);
    }
  }
  return make_float2(warp_sum(acc0), warp_sum(acc1));
}

// Items [0, n) of a phase, two per warp at a time: f(item0, item1, both) computes item0 and, when
// `both`, item1 (else item1 = item0 and its result is dropped).
template <typename F>
__device__ __forceinline__ void pairs_over_warps(int n, int gwarp, int nwarps, F&& f) {
  for (int it = 2 * gwarp; it < n; it += 2 * nwarps) f(it, it + 1 < n ? it + 1 : it, it + 1 < n);
}

// Rotation of the pair (x0, x1) = rows (2k, 2k + 1) by the RoPE angle of pair k at position pos.
__device__ __forceinline__ void rope_pair(float& x0, float& x1, int pos, int k, int d_rope, double base,
                                          const double* table) {
  float c, s;
  rope_cos_sin(pos, k, d_rope, base, table, c, s);
  const float r0 = fmaf(x0, c, -x1 * s), r1 = fmaf(x1, c, x0 * s);
  x0 = r0;
  x1 = r1;
}

// grid: cooperative, 128 threads (the warp-MMA attention item's CTA); dynamic shared memory
// dmma::smem_bytes(d_c + d_rope).
template <typename T>
__global__ void __launch_bounds__(128) k_layer_small(const SmallStepArgs a) {
  namespace cg = cooperative_groups;
  cg::grid_group grid = cg::this_grid();
  extern __shared__ __align__(16) uint8_t sm[];
  const int lane = threadIdx.x & 31;
  const int gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int gthread = blockIdx.x * blockDim.x + threadIdx.x, nthreads = gridDim.x * blockDim.x;
  const MmaAttnArgs& at = a.attn;
  const int B = a.B, D = a.d_c + a.d_rope, half = a.d_rope / 2;
  const T* h = static_cast<const T*>(a.h);
  auto pos_of = [&](int b) { return at.seq_lens[b] - 1; };
  auto len_ok = [&](int b) {
    const int L = at.seq_lens[b];
    return L >= 1 && L <= at.max_seq_len && (L - 1) / at.page_size < at.max_pages;
  };

  // ---- 1: the new cache row and c'. Per token: d_c latent rows, d_rope / 2 rope pairs (a warp
  // each), d_cq rows of c'.
  {
    const T* wk = static_cast<const T*>(a.w_dkv_kr);
    const T* wq = static_cast<const T*>(a.w_dq);
    // cache row of token b, or -1 (error recorded once per token)
    auto row_of = [&](int b, bool record) -> long {
      if (!len_ok(b)) {
        if (record) record_error(MLA_ERR_BAD_SEQ_LEN);
        return -1;
      }
      const int pos = pos_of(b);
      const int page = at.bt[(long)b * at.max_pages + pos / at.page_size];
      if (page < 0 || page >= at.num_pages) {
        if (record) record_error(MLA_ERR_BAD_PAGE);
        return -1;
      }
      return ((long)page * at.page_size + pos % at.page_size) * D;
    };
    const int n_lat = B * a.d_c, n_cq = B * a.d_cq;
    pairs_over_warps(n_lat + n_cq, gwarp, nwarps, [&](int i0, int i1, bool both) {
      auto src = [&](int it, const T*& w, const T*& x) {
        if (it < n_lat) {
          const int b = it / a.d_c;
          w = wk + (long)(it - b * a.d_c) * a.d_model;
          x = h + (long)b * a.d_model;
        } else {
          const int b = (it - n_lat) / a.d_cq;
          w = wq + (long)(it - n_lat - b * a.d_cq) * a.d_model;
          x = h + (long)b * a.d_model;
        }
      };
      const T *w0, *x0, *w1, *x1;
      src(i0, w0, x0);
      src(i1, w1, x1);
      const float2 v = warp_dot2<T>(w0, x0, w1, x1, a.d_model, lane);
      if (lane == 0)
        for (int u = 0; u < (both ? 2 : 1); ++u) {
          const int it = u ? i1 : i0;
          const float val = u ? v.y : v.x;
          if (it < n_lat) {
            const int b = it / a.d_c, r = it - b * a.d_c;
            const long row = row_of(b, r == 0);
            if (row >= 0) Out<T>::put(static_cast<T*>(a.pool) + row + r, val);
          } else {
            const int b = (it - n_lat) / a.d_cq;
            Out<T>::put(static_cast<T*>(a.cq) + (long)b * a.d_cq + (it - n_lat - b * a.d_cq), val);
          }
        }
    });
    for (int it = gwarp; it < B * half; it += nwarps) {  // rope pairs
      const int b = it / half, k = it - b * half, m = a.d_c + 2 * k;
      const T* x = h + (long)b * a.d_model;
      const float2 v = warp_dot2<T>(wk + (long)m * a.d_model, x, wk + (long)(m + 1) * a.d_model, x, a.d_model, lane);
      const long row = row_of(b, false);
      if (lane == 0 && row >= 0) {
        float x0 = v.x, x1 = v.y;
        rope_pair(x0, x1, pos_of(b), k, a.d_rope, a.rope_base, a.rope_table);
        T* dst = static_cast<T*>(a.pool) + row;
        Out<T>::put(dst + m, x0);
        Out<T>::put(dst + m + 1, x1);
      }
    }
  }
  grid.sync();
  // ---- 2: q^C_i = W^UQ_i c' (rows two per warp) and q^R_i = RoPE(W^QR_i c') (a pair per warp)
  {
    const int nq = a.n_h * a.d_h;
    const T* w = static_cast<const T*>(a.w_uq_qr);
    const T* cq = static_cast<const T*>(a.cq);
    pairs_over_warps(B * nq, gwarp, nwarps, [&](int i0, int i1, bool both) {
      const int b0 = i0 / nq, b1 = i1 / nq;
      const float2 v = warp_dot2<T>(w + (long)(i0 - b0 * nq) * a.d_cq, cq + (long)b0 * a.d_cq,
                                    w + (long)(i1 - b1 * nq) * a.d_cq, cq + (long)b1 * a.d_cq, a.d_cq, lane);
      if (lane == 0) {
        Out<T>::put(static_cast<T*>(a.qc) + i0, v.x);
        if (both) Out<T>::put(static_cast<T*>(a.qc) + i1, v.y);
      }
    });
    for (int it = gwarp; it < B * a.n_h * half; it += nwarps) {
      const int b = it / (a.n_h * half), pr = it - b * a.n_h * half, i = pr / half, k = pr - i * half;
      const int m = nq + i * a.d_rope + 2 * k;
      const T* x = cq + (long)b * a.d_cq;
      const float2 v = warp_dot2<T>(w + (long)m * a.d_cq, x, w + (long)(m + 1) * a.d_cq, x, a.d_cq, lane);
      if (lane == 0) {
        float x0 = v.x, x1 = v.y;
        rope_pair(x0, x1, len_ok(b) ? pos_of(b) : 0, k, a.d_rope, a.rope_base, a.rope_table);
        T* dst = static_cast<T*>(a.q) + ((long)b * a.n_h + i) * D + a.d_c + 2 * k;
        Out<T>::put(dst, x0);
        Out<T>::put(dst + 1, x1);
      }
    }
  }
  grid.sync();
  // ---- 3: q~_i[m] = sum_k W^UK[i d_h + k][m] q^C_i[k], a thread per output (coalesced over m)
  {
    const T* wk = static_cast<const T*>(a.w_uk);
    const T* qc = static_cast<const T*>(a.qc);
    const int per = a.n_h * a.d_c;
    for (int it = gthread; it < B * per; it += nthreads) {
      const int b = it / per, r = it - b * per, i = r / a.d_c, m = r - i * a.d_c;
      const T* qi = qc + ((long)b * a.n_h + i) * a.d_h;
      const T* col = wk + (long)i * a.d_h * a.d_c + m;
      float acc = 0.f;
      for (int k = 0; k < a.d_h; ++k) acc = fmaf(Pack<T>::f(col[(long)k * a.d_c]), Pack<T>::f(__ldcg(qi + k)), acc);
      Out<T>::put(static_cast<T*>(a.q) + ((long)b * a.n_h + i) * D + m, acc);
    }
  }
  grid.sync();
  // ---- 4: attention items (sequence, split), one per CTA at a time
  for (int it = blockIdx.x; it < B * at.n_splits; it += gridDim.x) attn_mma_item<T>(at, it / at.n_splits, it % at.n_splits, sm);
  grid.sync();
  // ---- 5: merge of the splits in split order (a warp per sequence and head)
  if (at.n_splits > 1) {
    for (int bh = gwarp; bh < B * a.n_h; bh += nwarps) {
      const float* lp = at.lse_part + (long)bh * at.n_splits;
      float mx = -INFINITY;
      for (int s = lane; s < at.n_splits; s += 32) mx = fmaxf(mx, __ldcg(lp + s));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      float z = 0.f;
      if (mx != -INFINITY)
        for (int s = 0; s < at.n_splits; ++s) {
          const float w = exp2f((__ldcg(lp + s) - mx) * kLog2e);  // -inf partials (no tokens) weigh 0
          z += w;
          const float* src = at.o_part + ((long)bh * at.n_splits + s) * a.d_c;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (lane + 32 * j < a.d_c) acc[j] = fmaf(w, __ldcg(src + lane + 32 * j), acc[j]);
        }
      const float inv = z > 0.f ? 1.f / z : 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (lane + 32 * j < a.d_c) Out<T>::put(static_cast<T*>(at.o_lat) + (long)bh * a.d_c + lane + 32 * j, acc[j] * inv);
      if (at.lse_out != nullptr && lane == 0) at.lse_out[bh] = z > 0.f ? mx + logf(z) : -INFINITY;
    }
  }
  grid.sync();
  // ---- 6: o_i = W^UV_i o_lat_i (rows two per warp)
  {
    const int nq = a.n_h * a.d_h;
    const T* w = static_cast<const T*>(a.w_uv);
    const T* ol = static_cast<const T*>(at.o_lat);
    pairs_over_warps(B * nq, gwarp, nwarps, [&](int i0, int i1, bool both) {
      const int b0 = i0 / nq, b1 = i1 / nq;
      const int h0 = (i0 - b0 * nq) / a.d_h, h1 = (i1 - b1 * nq) / a.d_h;
      const float2 v = warp_dot2<T>(w + (long)(i0 - b0 * nq) * a.d_c, ol + ((long)b0 * a.n_h + h0) * a.d_c,
                                    w + (long)(i1 - b1 * nq) * a.d_c, ol + ((long)b1 * a.n_h + h1) * a.d_c, a.d_c,
                                    lane);
      if (lane == 0) {
        Out<T>::put(static_cast<T*>(a.o) + i0, v.x);
        if (both) Out<T>::put(static_cast<T*>(a.o) + i1, v.y);
      }
    });
  }
  grid.sync();
  // ---- 7: u = W^O o (rows two per warp)
  {
    const int nq = a.n_h * a.d_h;
    const T* w = static_cast<const T*>(a.w_o);
    const T* o = static_cast<const T*>(a.o);
    pairs_over_warps(B * a.d_model, gwarp, nwarps, [&](int i0, int i1, bool both) {
      const int b0 = i0 / a.d_model, b1 = i1 / a.d_model;
      const float2 v = warp_dot2<T>(w + (long)(i0 - b0 * a.d_model) * nq, o + (long)b0 * nq,
                                    w + (long)(i1 - b1 * a.d_model) * nq, o + (long)b1 * nq, nq, lane);
      if (lane == 0) {
        Out<T>::put(static_cast<T*>(a.u) + i0, v.x);
        if (both) Out<T>::put(static_cast<T*>(a.u) + i1, v.y);
      }
    });
  }
}

}  // namespace mla
