// CUDA-core projection kernels (any supported dims): skinny products Y = X W^T for a handful of
// tokens, the per-head (W^UK_i)^T q^C_i absorption, and the RoPE / cache-write epilogues.
// Weight rows are read with 16-byte loads; one warp owns one output feature.
#pragma once

#include "common.cuh"

namespace mla {

// Y[z][t][m] = sum_k W[z][m][k] * X[z][t][k] for t < T, m < M (fp32 accumulate).
// W row-major [M, K] (K % 8 == 0); X rows stride ldx; Y rows stride ldy. blockIdx.z = batch z.
template <typename T, typename OutT, int TT>
__global__ void __launch_bounds__(256) k_rowdot(const T* __restrict__ W, const T* __restrict__ X,
                                                OutT* __restrict__ Y, int M, int K, int T_, long ldx, long ldy,
                                                long sW, long sX, long sY) {
  const int lane = threadIdx.x & 31;
  const int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (m >= M) return;
  const long z = blockIdx.z;
  const T* w = W + z * sW + (long)m * K;
  const T* x = X + z * sX;
  OutT* y = Y + z * sY;
  for (int t0 = 0; t0 < T_; t0 += TT) {
    float acc[TT];
#pragma unroll
    for (int i = 0; i < TT; ++i) acc[i] = 0.f;
    for (int k = lane * 8; k < K; k += 256) {
      float wf[8];
      unpack8<T>(ldg16(w + k), wf);
#pragma unroll
      for (int i = 0; i < TT; ++i) {
        if (t0 + i < T_) {
          float xf[8];
          unpack8<T>(ldg16(x + (long)(t0 + i) * ldx + k), xf);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[i] = fmaf(wf[e], xf[e], acc[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < TT; ++i) {
      const float v = warp_sum(acc[i]);
      if (lane == i && t0 + i < T_) Out<OutT>::put(y + (long)(t0 + i) * ldy + m, v);
    }
  }
}

// q_out[b][i][m] = sum_k W^UK[i*d_h + k][m] * q^C[b][i*d_h + k]  for m < d_c (the absorbed
// content query, from-scratch page §5.1). W^UK_i^T is read row by row (m contiguous).
// grid (ceil(d_c/2 / blockDim.x), n_h); dynamic smem BT * d_h floats.
template <typename T, int BT>
__global__ void __launch_bounds__(256) k_absorb_uk(const T* __restrict__ w_uk, const T* __restrict__ qc,
                                                   T* __restrict__ q_out, int B, int n_h, int d_h, int d_c, int D) {
  using P = Pack<T>;
  using T2 = typename P::T2;
  extern __shared__ float xs[];
  const int i = blockIdx.y;
  const int m2 = blockIdx.x * blockDim.x + threadIdx.x;  // pair of latent features
  const T2* w = reinterpret_cast<const T2*>(w_uk + (long)i * d_h * d_c);
  for (int b0 = 0; b0 < B; b0 += BT) {
    __syncthreads();
    for (int e = threadIdx.x; e < BT * d_h; e += blockDim.x) {
      const int bb = e / d_h, k = e % d_h;
      xs[e] = (b0 + bb < B) ? P::f(qc[(long)(b0 + bb) * n_h * d_h + (long)i * d_h + k]) : 0.f;
    }
    __syncthreads();
    if (m2 < d_c / 2) {
      float a0[BT], a1[BT];
#pragma unroll
      for (int bb = 0; bb < BT; ++bb) a0[bb] = a1[bb] = 0.f;
      for (int k = 0; k < d_h; ++k) {
        const float2 wv = P::f2(w[(long)k * (d_c / 2) + m2]);
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) {
          const float xv = xs[bb * d_h + k];
          a0[bb] = fmaf(wv.x, xv, a0[bb]);
          a1[bb] = fmaf(wv.y, xv, a1[bb]);
        }
      }
#pragma unroll
      for (int bb = 0; bb < BT; ++bb)
        if (b0 + bb < B)
          reinterpret_cast<T2*>(q_out + ((long)(b0 + bb) * n_h + i) * D)[m2] = P::make(a0[bb], a1[bb]);
    }
  }
}

// Cache-write epilogue of mla_append_kv: row = [c ‖ RoPE(k^, pos)] rounded, stored at the
// token's paged slot. Y holds `splits` fp32 partial products [T, D], `split_off` apart, summed
// in split order. One block per token.
template <typename T>
__global__ void k_append_epilogue(const float* __restrict__ Y, int splits, long split_off,
                                  const int* __restrict__ seq_idx, const int* __restrict__ pos,
                                  const int* __restrict__ bt, int num_seqs, int max_pages, T* __restrict__ pool,
                                  int num_pages, int page_size, int d_c, int d_rope, double base) {
  using P = Pack<T>;
  const int t = blockIdx.x;
  const int D = d_c + d_rope;
  const int s = seq_idx[t], p = pos[t];
  const int lp = p / page_size;
  int page = -1;
  if (s >= 0 && s < num_seqs && p >= 0 && lp < max_pages) page = bt[(long)s * max_pages + lp];
  if (page < 0 || page >= num_pages) {
    if (threadIdx.x == 0) record_error(MLA_ERR_BAD_PAGE);
    return;
  }
  T* row = pool + ((long)page * page_size + p % page_size) * D;
  const float* y = Y + (long)t * D;
  extern __shared__ float2 cs[];  // cos/sin of each RoPE pair at this position
  for (int k = threadIdx.x; k < d_rope / 2; k += blockDim.x) rope_cos_sin(p, k, d_rope, base, cs[k].x, cs[k].y);
  __syncthreads();
  for (int e = threadIdx.x; e < D / 2; e += blockDim.x) {
    float a = 0.f, b = 0.f;
    for (int k = 0; k < splits; ++k) {
      a += y[k * split_off + 2 * e];
      b += y[k * split_off + 2 * e + 1];
    }
    if (2 * e >= d_c) {
      const float2 r = cs[e - d_c / 2];
      const float ra = a * r.x - b * r.y, rb = a * r.y + b * r.x;
      a = ra;
      b = rb;
    }
    reinterpret_cast<typename P::T2*>(row)[e] = P::make(a, b);
  }
}

// Query epilogue of mla_absorb_query: Y = [q^C ; q^] fp32 [B, n_h*(d_h + d_r)] as `splits`
// partials `split_off` apart (summed in order). q^C -> qc (element type, [B, n_h*d_h]);
// q^R_i = RoPE(q^_i, pos[b]) -> q_out[b][i][d_c:].
template <typename T>
__global__ void k_query_epilogue(const float* __restrict__ Y, int splits, long split_off, const int* __restrict__ pos,
                                 T* __restrict__ qc, T* __restrict__ q_out, int n_h, int d_h, int d_r, int d_c,
                                 double base) {
  using P = Pack<T>;
  using T2 = typename P::T2;
  const int b = blockIdx.x;
  const int nc = n_h * d_h, D = d_c + d_r;
  const float* y = Y + (long)b * n_h * (d_h + d_r);
  const int p = pos[b];
  extern __shared__ float2 cs[];  // cos/sin of each RoPE pair at this position (shared by all heads)
  for (int k = threadIdx.x; k < d_r / 2; k += blockDim.x) rope_cos_sin(p, k, d_r, base, cs[k].x, cs[k].y);
  __syncthreads();
  for (int e = threadIdx.x; e < n_h * (d_h + d_r) / 2; e += blockDim.x) {
    float a = 0.f, c2 = 0.f;
    for (int k = 0; k < splits; ++k) {
      a += y[k * split_off + 2 * e];
      c2 += y[k * split_off + 2 * e + 1];
    }
    if (2 * e < nc) {
      reinterpret_cast<T2*>(qc + (long)b * nc)[e] = P::make(a, c2);
    } else {
      const int r = 2 * e - nc;  // index inside the W^QR block
      const int i = r / d_r, k = (r % d_r) / 2;
      const float2 q = cs[k];
      reinterpret_cast<T2*>(q_out + ((long)b * n_h + i) * D + d_c)[k] =
          P::make(a * q.x - c2 * q.y, a * q.y + c2 * q.x);
    }
  }
}

}  // namespace mla
