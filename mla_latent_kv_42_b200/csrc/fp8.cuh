// FP8 latent cache: DeepSeek-V2 paper review (velog) §4.2 and the DeepSeek-V2 summary page
// ("The Model") quantise the deployed model's KV cache to about 6 bits per element without
// giving the format; this cache stores e4m3 bytes with two float32 scales per token.
//
// Page layout (page_size tokens): page_size rows of D = d_c + d_rope bytes in token order, then
// page_size float2 scales (s_c, s_r). A byte is the nearest e4m3 value (ties to even, saturated
// to +-448) of the element-type value divided by its part's scale max|part| / 448 in float32
// (1 for an all-zero part), so the largest magnitude of each part lands on 448.
//
// Writer: k_quant_fp8 below, after the append GEMM has staged the element-type rows. Reader: the
// decode kernel of decode_tc.cuh instantiated with F8 = true, where four more warps convert each
// landed e4m3 box in place to fp16 (dequant16_f16) and the products run as fp16 MMAs.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace mla {
namespace fp8 {
constexpr float kE4m3Max = 448.f;
constexpr int kMaxGroups = 3;  // 8-element groups per lane: D <= 768
__host__ __device__ constexpr long page_bytes(int page_size, int D) { return (long)page_size * (D + 8); }
}  // namespace fp8

// One warp per new token: the token's row (element type, staged by the append GEMM) is
// quantised into its cache slot, with the two scales after the page's rows. A token whose slot
// is outside the block table or the pool records MLA_ERR_BAD_PAGE and is not written.
template <typename T>
__global__ void __launch_bounds__(256) k_quant_fp8(const T* __restrict__ rows, const int* __restrict__ seq_idx,
                                                   const int* __restrict__ pos, const int* __restrict__ bt,
                                                   int num_seqs, int max_pages, int num_pages, int page_size, int d_c,
                                                   int D, int T_, uint8_t* __restrict__ pool) {
  griddep_wait();  // the rows come from the GEMM before
  const int t = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
  if (t >= T_) return;
  const int s = seq_idx[t], p = pos[t];
  const int lp = p >= 0 ? p / page_size : -1;
  int page = -1;
  if (s >= 0 && s < num_seqs && p >= 0 && lp < max_pages) page = bt[(long)s * max_pages + lp];
  if (page < 0 || page >= num_pages) {
    if (lane == 0) record_error(MLA_ERR_BAD_PAGE);
    return;
  }
  const int row = p % page_size;
  const T* src = rows + (long)t * D;
  const int G = D / 8;  // d_c % 8 == 0: a group lies in one part
  float v[fp8::kMaxGroups][8];
  float mc = 0.f, mr = 0.f;
#pragma unroll
  for (int i = 0; i < fp8::kMaxGroups; ++i) {
    const int g = lane + 32 * i;
    if (g < G) {
      const uint4 raw = *reinterpret_cast<const uint4*>(src + 8 * g);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = Pack<T>::f2(*reinterpret_cast<const typename Pack<T>::T2*>(&w[e]));
        v[i][2 * e] = f.x;
        v[i][2 * e + 1] = f.y;
        a = fmaxf(a, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
      if (8 * g < d_c) mc = fmaxf(mc, a);
      else mr = fmaxf(mr, a);
    }
  }
  // non-negative floats order as their bit patterns
  mc = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mc)));
  mr = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mr)));
  const float sc = mc > 0.f ? mc / fp8::kE4m3Max : 1.f;
  const float sr = mr > 0.f ? mr / fp8::kE4m3Max : 1.f;
  uint8_t* const pg = pool + (long)page * fp8::page_bytes(page_size, D);
  uint8_t* const dst = pg + (long)row * D;
#pragma unroll
  for (int i = 0; i < fp8::kMaxGroups; ++i) {
    const int g = lane + 32 * i;
    if (g < G) {
      const float sg = 8 * g < d_c ? sc : sr;
      uint32_t q[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const __nv_fp8x2_storage_t lo =
            __nv_cvt_float2_to_fp8x2(make_float2(v[i][4 * h] / sg, v[i][4 * h + 1] / sg), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
            make_float2(v[i][4 * h + 2] / sg, v[i][4 * h + 3] / sg), __NV_SATFINITE, __NV_E4M3);
        q[h] = (uint32_t)lo | ((uint32_t)hi << 16);
      }
      *reinterpret_cast<uint2*>(dst + 8 * g) = make_uint2(q[0], q[1]);
    }
  }
  if (lane == 0) *reinterpret_cast<float2*>(pg + (long)page_size * D + 8 * row) = make_float2(sc, sr);
}

// 16 e4m3 values (16 bytes, element order) as fp16 times the fp16 scale `s` (the e4m3 value is
// exact in fp16; the product is rounded once): two 16-byte groups of eight elements.
__device__ __forceinline__ void dequant16_f16(const uint4& in, __half2 s, uint4& out0, uint4& out1) {
  const uint32_t w[4] = {in.x, in.y, in.z, in.w};
  uint32_t o[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const __nv_fp8x2_storage_t two = (__nv_fp8x2_storage_t)(w[e >> 1] >> (16 * (e & 1)));
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(two, __NV_E4M3);
    const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&hr), s);
    o[e] = *reinterpret_cast<const uint32_t*>(&v);
  }
  out0 = make_uint4(o[0], o[1], o[2], o[3]);
  out1 = make_uint4(o[4], o[5], o[6], o[7]);
}

}  // namespace mla
