// Latent attention for small head counts (n_h <= 16; the pages' running model has 8 heads of a
// 160-wide cache row): "DeepSeek-V2 from Scratch" §4.4 with the absorbed steps 2-3 of §5.3.
//
// With 8 heads the score and value products are matrices of 8 rows, far below the 64-128 rows of
// a tcgen05 MMA, and at 4608 flops per 320-byte token the bound is HBM with the tensor pipe
// mostly idle either way. The kernel therefore uses warp-level mma.sync m16n8k16 (heads on
// M = 16, padded): S = Q C^T takes B from the cache tile with ldmatrix, and the bf16/fp16 P
// fragment of O = P C_lat is the S accumulator itself (the accumulator layout of two n8 tiles is
// the A layout of one k16 step), so P never leaves registers.
//
// A CTA (4 warps) owns tokens [t0, t1) of one sequence and streams them in 64-token stages
// (cp.async, 16-byte copies, three buffers, rows padded by 16 bytes so that ldmatrix is
// conflict-free); warp w takes tokens [16w, 16w + 16) of each stage and keeps its own online
// softmax (fp32, lazy rescaling) and O accumulators. The four warps are merged in a fixed order at
// the end into the sequence's output or a split-KV partial that k_lse_merge_warp combines.
#pragma once

#include "common.cuh"

namespace mla {

namespace dmma {
constexpr int kWarps = 4;
constexpr int kStageTokens = 64;
constexpr int kStages = 3;
constexpr int kMaxKD = 12;  // D <= 192 (D / 16 k steps of the score product)
constexpr int kMaxND = 16;  // d_c <= 128 (d_c / 8 n tiles of the value product)
constexpr float kLazy = 8.f;
__host__ __device__ constexpr int row_stride(int D) { return 2 * D + 16; }  // bytes
__host__ __device__ constexpr size_t smem_bytes(int D) { return (size_t)kStages * kStageTokens * row_stride(D); }
}  // namespace dmma

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D (16x8 fp32) += A (16x16) B (16x8), 16-bit inputs of type T.
template <typename T>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct MmaAttnArgs {
  const void* q;            // [B, n_h, D]
  const void* pool;         // [num_pages, page_size, D]
  const int* bt;            // [B, max_pages]
  int max_pages;
  const int* seq_lens;      // [B]
  int max_seq_len, num_pages, n_h, d_c, D, page_size;
  float scale_log2;
  int split_len, n_splits;
  void* o_lat;              // [B, n_h, d_c] (n_splits == 1)
  float* lse_out;           // [B, n_h] or null (n_splits == 1)
  float* o_part;            // [B * n_h][n_splits][d_c] (n_splits > 1)
  float* lse_part;          // [B * n_h][n_splits]
};

// One work item: tokens [split * split_len, min(L, (split + 1) * split_len)) of sequence b, by the
// first 128 threads of the calling CTA (four warps); `sm` holds smem_bytes(D) bytes, 16-aligned.
// Requirements (checked by the host): n_h <= 16, D % 16 == 0, D <= 192, d_c % 16 == 0, d_c <= 128,
// page_size % 16 == 0, split_len a multiple of 64.
template <typename T>
__device__ void attn_mma_item(const MmaAttnArgs& a, int b, int split, uint8_t* sm) {
  using namespace dmma;
  using P2 = typename Pack<T>::T2;
  const T* __restrict__ q = static_cast<const T*>(a.q);
  const T* __restrict__ pool = static_cast<const T*>(a.pool);
  const int* __restrict__ bt = a.bt;
  const int max_pages = a.max_pages, max_seq_len = a.max_seq_len, num_pages = a.num_pages, n_h = a.n_h;
  const int d_c = a.d_c, D = a.D, page_size = a.page_size, split_len = a.split_len, n_splits = a.n_splits;
  const float scale_log2 = a.scale_log2;
  T* __restrict__ o_lat = static_cast<T*>(a.o_lat);
  float* __restrict__ lse_out = a.lse_out;
  float* __restrict__ o_part = a.o_part;
  float* __restrict__ lse_part = a.lse_part;
  __shared__ int stage_page[kStages][kStageTokens / 16];  // page of each 16-token group of a stage
  __shared__ float w_ml[kWarps][16][2];                   // per warp and head row: reference max, denominator
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;  // mma fragment coordinates
  const int KD = D / 16, ND = d_c / 8;
  const int stride = row_stride(D);
  const uint32_t sm_u32 = static_cast<uint32_t>(__cvta_generic_to_shared(sm));

  int L = a.seq_lens[b];
  bool bad_len = L < 1 || L > max_seq_len || (L + page_size - 1) / page_size > max_pages;
  if (bad_len) {
    if (split == 0 && tid == 0) record_error(MLA_ERR_BAD_SEQ_LEN);
    L = 0;
  }
  const int t0 = split * split_len, t1 = min(L, t0 + split_len);
  const int n_stages = t1 > t0 ? (t1 - t0 + kStageTokens - 1) / kStageTokens : 0;
  const int* btb = bt + (long)b * max_pages;
  bool bad_page = false;

  // Q as A fragments: rows = heads (>= n_h: zero), k = D columns in steps of 16
  uint32_t qa[kMaxKD][4];
  {
    const T* qb = q + (long)b * n_h * D;
#pragma unroll
    for (int ks = 0; ks < kMaxKD; ++ks) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = g + ((e & 1) ? 8 : 0), col = 16 * ks + 2 * tq + ((e & 2) ? 8 : 0);
        uint32_t v = 0;
        // read at L2: the fused layer step writes q earlier in the same launch
        if (ks < KD && row < n_h) v = __ldcg(reinterpret_cast<const unsigned*>(qb + (long)row * D + col));
        qa[ks][e] = v;
      }
    }
  }

  // stage s of the loop -> buffer s % kStages: 64 rows of the cache (zero rows past t1)
  const int chunks_per_row = D / 8;  // 16-byte chunks
  auto issue_stage = [&](int st) {
    const int buf = st % kStages;
    const int s0 = t0 + st * kStageTokens;
    if (tid < kStageTokens / 16) {
      const int tok = s0 + 16 * tid;
      int pg = -1;
      if (tok < t1) {
        pg = btb[tok / page_size];
        if (pg < 0 || pg >= num_pages) {
          bad_page = true;
          pg = -1;
        }
      }
      stage_page[buf][tid] = pg;
    }
    __syncthreads();
    const uint32_t base = sm_u32 + buf * kStageTokens * stride;
    for (int c = tid; c < kStageTokens * chunks_per_row; c += 128) {
      const int row = c / chunks_per_row, col = c - row * chunks_per_row;
      const int tok = s0 + row;
      const int pg = stage_page[buf][row >> 4];
      const bool valid = tok < t1 && pg >= 0;
      const T* src = valid ? pool + ((long)pg * page_size + tok % page_size) * D + col * 8 : pool;
      cp_async16(base + row * stride + col * 16, src, valid ? 16u : 0u);
    }
  };

  float oacc[kMaxND][4];
#pragma unroll
  for (int j = 0; j < kMaxND; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[j][e] = 0.f;
  float m_ref[2] = {-INFINITY, -INFINITY};  // rows g and g + 8, log2 units
  float lsum[2] = {0.f, 0.f};               // this thread's tokens only (summed over the quad at the end)

  for (int st = 0; st < kStages - 1; ++st) {
    if (st < n_stages) issue_stage(st);
    cp_async_commit();
  }
  for (int st = 0; st < n_stages; ++st) {
    if (st + kStages - 1 < n_stages) issue_stage(st + kStages - 1);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncthreads();
    const int buf = st % kStages;
    const int tok0 = t0 + st * kStageTokens + 16 * warp;  // this warp's 16 tokens
    const uint32_t tile = sm_u32 + buf * kStageTokens * stride + (16 * warp) * stride;
    if (tok0 < t1) {
      // S = Q C^T for 16 tokens: two n8 tiles
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      const int mi = lane >> 3, ri = lane & 7;  // ldmatrix: matrix index, row within it
#pragma unroll
      for (int ks = 0; ks < kMaxKD; ++ks) {
        if (ks < KD) {
          uint32_t bfr[4];
          // matrices: (tokens 0-7, k 0-7), (tokens 0-7, k 8-15), (tokens 8-15, k 0-7), (tokens 8-15, k 8-15)
          ldsm_x4(tile + (ri + 8 * (mi >> 1)) * stride + (16 * ks + 8 * (mi & 1)) * 2, bfr);
          mma16816<T>(s[0], qa[ks], bfr[0], bfr[1]);
          mma16816<T>(s[1], qa[ks], bfr[2], bfr[3]);
        }
      }
      // online softmax per head row (g, g + 8): scores of tokens 2tq, 2tq+1 (tile 0) and 8+2tq, 9+2tq
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        float v[4] = {s[0][2 * h2], s[0][2 * h2 + 1], s[1][2 * h2], s[1][2 * h2 + 1]};
        const int toks[4] = {tok0 + 2 * tq, tok0 + 2 * tq + 1, tok0 + 8 + 2 * tq, tok0 + 9 + 2 * tq};
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = toks[e] < t1 ? v[e] * scale_log2 : -INFINITY;
        float mx = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        if (mx > m_ref[h2] + kLazy) {  // the quad agrees: the same mx and m_ref in its four lanes
          const float alpha = exp2f(m_ref[h2] - mx);
          lsum[h2] *= alpha;
#pragma unroll
          for (int j = 0; j < kMaxND; ++j) {
            oacc[j][2 * h2] *= alpha;
            oacc[j][2 * h2 + 1] *= alpha;
          }
          m_ref[h2] = mx;
        }
        // p = 2^(s - m_ref), rounded; the denominator sums the rounded weights
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pe = exp2f(v[e] - m_ref[h2]);
          v[e] = pe;
        }
        const P2 p01 = Pack<T>::make(v[0], v[1]), p23 = Pack<T>::make(v[2], v[3]);
        const float2 f01 = Pack<T>::f2(p01), f23 = Pack<T>::f2(p23);
        lsum[h2] += (f01.x + f01.y) + (f23.x + f23.y);
        s[0][2 * h2] = __uint_as_float(*reinterpret_cast<const uint32_t*>(&p01));  // reuse as packed storage
        s[1][2 * h2] = __uint_as_float(*reinterpret_cast<const uint32_t*>(&p23));
      }
      // P as the A fragment of O += P C_lat (rows g / g+8, k = tokens 2tq.., 8+2tq..)
      const uint32_t pa[4] = {__float_as_uint(s[0][0]), __float_as_uint(s[0][2]), __float_as_uint(s[1][0]),
                              __float_as_uint(s[1][2])};
#pragma unroll
      for (int jp = 0; jp < kMaxND / 2; ++jp) {
        if (2 * jp < ND) {
          uint32_t bfr[4];
          // matrices: (tokens 0-7, n 0-7), (tokens 8-15, n 0-7), (tokens 0-7, n 8-15), (tokens 8-15, n 8-15)
          ldsm_x4_t(tile + (ri + 8 * (mi & 1)) * stride + (16 * jp + 8 * (mi >> 1)) * 2, bfr);
          mma16816<T>(oacc[2 * jp], pa, bfr[0], bfr[1]);
          mma16816<T>(oacc[2 * jp + 1], pa, bfr[2], bfr[3]);
        }
      }
    }
    __syncthreads();  // every warp is done with this buffer before it is refilled
  }
  cp_async_wait<0>();
  if (bad_page) record_error(MLA_ERR_BAD_PAGE);

  // ---- merge the four warps in a fixed order
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    lsum[h2] += __shfl_xor_sync(0xffffffffu, lsum[h2], 1);
    lsum[h2] += __shfl_xor_sync(0xffffffffu, lsum[h2], 2);
  }
  __syncthreads();
  float* wo = reinterpret_cast<float*>(sm);  // [warp][16 rows][d_c]
  if (tq == 0) {
    w_ml[warp][g][0] = m_ref[0];
    w_ml[warp][g][1] = lsum[0];
    w_ml[warp][g + 8][0] = m_ref[1];
    w_ml[warp][g + 8][1] = lsum[1];
  }
#pragma unroll
  for (int j = 0; j < kMaxND; ++j) {
    if (j < ND) {
      const int col = 8 * j + 2 * tq;
      wo[(warp * 16 + g) * d_c + col] = oacc[j][0];
      wo[(warp * 16 + g) * d_c + col + 1] = oacc[j][1];
      wo[(warp * 16 + g + 8) * d_c + col] = oacc[j][2];
      wo[(warp * 16 + g + 8) * d_c + col + 1] = oacc[j][3];
    }
  }
  __syncthreads();
  for (int e = tid; e < n_h * d_c; e += 128) {
    const int row = e / d_c, col = e - row * d_c;
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, w_ml[w][row][0]);
    float l = 0.f, acc = 0.f;
    if (m != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = w_ml[w][row][0] == -INFINITY ? 0.f : exp2f(w_ml[w][row][0] - m);
        l = fmaf(f, w_ml[w][row][1], l);
        acc = fmaf(f, wo[(w * 16 + row) * d_c + col], acc);
      }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const long bh = (long)b * n_h + row;
    if (n_splits == 1) {
      Out<T>::put(o_lat + bh * d_c + col, acc * inv);
      if (col == 0 && lse_out != nullptr) lse_out[bh] = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
    } else {
      o_part[(bh * n_splits + split) * d_c + col] = acc * inv;
      if (col == 0) lse_part[bh * n_splits + split] = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
  }
}

// grid (n_splits, B), 128 threads: one work item per CTA.
template <typename T>
__global__ void __launch_bounds__(128) k_decode_mma(const MmaAttnArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch();
  attn_mma_item<T>(a, blockIdx.y, blockIdx.x, sm);
}

}  // namespace mla
