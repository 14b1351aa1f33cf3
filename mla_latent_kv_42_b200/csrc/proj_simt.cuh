// CUDA-core kernels for the two per-head projection products when a head's slice is not a whole
// number of 64-wide blocks (the tensor-core GEMM batches heads by whole blocks): the batched
// skinny product W^UV_i o_lat_i and the absorption (W^UK_i)^T q^C_i.
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

}  // namespace mla
