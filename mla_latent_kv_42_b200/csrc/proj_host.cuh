// Host side of the three projection calls (mla_append_kv, mla_absorb_query, mla_out_proj):
// GEMM planning, TMA tensor maps, workspace layout and launches. Every product runs on the
// tcgen05 GEMM; the CUDA-core kernels remain as a second implementation, selected by setting
// MLA_PROJ_IMPL=simt in the environment (used to cross-check the two in tests).
// Included once, from libmla.cu.
#pragma once

#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "gemm_tc.cuh"
#include "proj_simt.cuh"

namespace mla {
namespace host {

constexpr int kMaxDev = 64;

inline int sm_count() {
  static int cache[kMaxDev] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

inline size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

struct Carver {
  char* base;
  size_t off = 0;
  template <typename X>
  X* take(size_t count) {
    X* p = base ? reinterpret_cast<X*>(base + off) : nullptr;
    off += a256(count * sizeof(X));
    return p;
  }
};

inline bool proj_uses_simt() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("MLA_PROJ_IMPL");
    v = (e != nullptr && std::strcmp(e, "simt") == 0) ? 1 : 0;
  }
  return v == 1;
}

// ------------------------------------------------------------------ TMA tensor maps
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major tensor [outer][inner] of 16-bit elements, rows `row_bytes` apart; boxes of
// box_inner x box_outer elements, 128-byte swizzle, zero fill outside the tensor.
inline bool encode_2d(CUtensorMap* map, const void* base, bool bf16, uint64_t inner, uint64_t outer,
                      uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base),
            dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ GEMM planning
struct GemmPlan {
  int bn, n_tiles, m_tiles, splits, kbps;
};

inline GemmPlan plan_gemm(int M, int N, int K, int batch, bool allow_split) {
  GemmPlan g;
  g.bn = N <= 16 ? 16 : N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
  g.n_tiles = (N + g.bn - 1) / g.bn;
  g.m_tiles = (M + 127) / 128;
  const int kb = (K + 63) / 64;
  const long base = (long)g.m_tiles * g.n_tiles * batch;
  long s = 1;
  if (allow_split && base < sm_count()) s = std::max(1L, std::min((long)sm_count() / base, (long)kb / 4));
  g.kbps = (int)((kb + s - 1) / s);
  g.splits = (kb + g.kbps - 1) / g.kbps;
  return g;
}

// A operand: K-major -> rows = all M rows (heads stacked), cols = K; MN-major -> rows = all K
// rows, cols = M. `batch_off` advances the row coordinate (K-major) or K-row coordinate
// (MN-major) per batch z. B operand: rows = N tokens, cols = full row length; `batch_off`
// advances the K (column) coordinate per batch z.
struct Operand {
  const void* base;
  long rows, cols;
  int batch_off;
};

template <typename T, int BN, bool MN>
cudaError_t run_gemm(const CUtensorMap& ma, const CUtensorMap& mb, const tc::GemmParams& p, dim3 grid,
                     cudaStream_t st) {
  using C = tc::GemmCfg<BN>;
  static bool attr_done[kMaxDev] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < kMaxDev && !attr_done[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(tc::k_gemm_tc<T, BN, MN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  tc::k_gemm_tc<T, BN, MN><<<grid, 192, C::SMEM, st>>>(ma, mb, p);
  return cudaGetLastError();
}

// out[z][n][m] (or fp32 partial [split][z][n][m]) = sum_k A[z][m][k] B[z][n][k].
template <typename T>
int gemm_tc(const Operand& A, bool a_mn, const Operand& B, int M, int N, int K, int batch, const GemmPlan& g,
            void* out, bool out_f32, long out_ld, long out_batch_off, long out_split_off, cudaStream_t st) {
  constexpr bool bf16 = tc::IsBf16<T>::value;
  CUtensorMap ma, mb;
  const bool ok_a = a_mn ? encode_2d(&ma, A.base, bf16, A.cols, A.rows, A.cols * 2, 64, 64)
                         : encode_2d(&ma, A.base, bf16, A.cols, A.rows, A.cols * 2, 64, 128);
  const bool ok_b = encode_2d(&mb, B.base, bf16, B.cols, B.rows, B.cols * 2, 64, g.bn);
  if (!ok_a || !ok_b) return MLA_ERR_CUDA;
  tc::GemmParams p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.kb_per_split = g.kbps;
  p.n_tiles = g.n_tiles;
  p.a_batch_off = A.batch_off;
  p.b_batch_off = B.batch_off;
  p.out = out;
  p.out_ld = out_ld;
  p.out_batch_off = out_batch_off;
  p.out_split_off = out_split_off;
  p.out_f32 = out_f32 ? 1 : 0;
  const dim3 grid(g.m_tiles, g.splits * g.n_tiles, batch);
  cudaError_t e;
#define MLA_GEMM_CASE(BNV)                                                              \
  case BNV:                                                                             \
    e = a_mn ? run_gemm<T, BNV, true>(ma, mb, p, grid, st) : run_gemm<T, BNV, false>(ma, mb, p, grid, st); \
    break;
  switch (g.bn) {
    MLA_GEMM_CASE(16)
    MLA_GEMM_CASE(32)
    MLA_GEMM_CASE(64)
    MLA_GEMM_CASE(128)
    MLA_GEMM_CASE(256)
    default: return MLA_ERR_CUDA;
  }
#undef MLA_GEMM_CASE
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

template <typename T>
void launch_reduce(const float* part, int splits, long split_off, long rows, long row_len, long out_ld, T* out,
                   cudaStream_t st) {
  const long n = rows * row_len;
  const int threads = 256;
  const long blocks = std::min((n + threads - 1) / threads, 4L * sm_count());
  tc::k_splitk_reduce<T><<<(unsigned)blocks, threads, 0, st>>>(part, splits, split_off, n, rows, row_len, out_ld, out);
}

template <typename T, typename OutT>
void launch_rowdot(const T* W, const T* X, OutT* Y, int M, int K, int Tn, long ldx, long ldy, int batch, long sW,
                   long sX, long sY, cudaStream_t st, int32_t& launches) {
  if (Tn <= 0 || M <= 0 || batch <= 0) return;
  dim3 grid((M + 7) / 8, 1, batch);
  if (Tn <= 8)
    k_rowdot<T, OutT, 8><<<grid, 256, 0, st>>>(W, X, Y, M, K, Tn, ldx, ldy, sW, sX, sY);
  else
    k_rowdot<T, OutT, 16><<<grid, 256, 0, st>>>(W, X, Y, M, K, Tn, ldx, ldy, sW, sX, sY);
  ++launches;
}

// ------------------------------------------------------------------ mla_append_kv
struct AppendLayout {
  GemmPlan g;
  float* Y;
  size_t bytes;
};
inline AppendLayout append_layout(const mla_dims* d, int T_, void* ws) {
  AppendLayout L;
  const int D = d->d_c + d->d_rope;
  L.g = plan_gemm(D, T_, d->d_model, 1, true);
  const int splits = proj_uses_simt() ? 1 : L.g.splits;
  Carver c{static_cast<char*>(ws)};
  L.Y = c.take<float>((size_t)splits * T_ * D);
  L.bytes = c.off;
  return L;
}

template <typename T>
int append_run(const mla_dims* d, const void* h, const void* w, const int32_t* seq_idx, const int32_t* pos,
               const int32_t* bt, int32_t num_seqs, int32_t max_pages, void* pool, int32_t num_pages, int32_t T_,
               void* ws, cudaStream_t st, int32_t& n) {
  const int D = d->d_c + d->d_rope;
  const AppendLayout L = append_layout(d, T_, ws);
  int splits = 1;
  if (proj_uses_simt()) {
    launch_rowdot<T, float>(static_cast<const T*>(w), static_cast<const T*>(h), L.Y, D, d->d_model, T_, d->d_model,
                            D, 1, 0, 0, 0, st, n);
  } else {
    const int r = gemm_tc<T>({w, D, d->d_model, 0}, false, {h, T_, d->d_model, 0}, D, T_, d->d_model, 1, L.g, L.Y,
                             true, D, 0, (long)T_ * D, st);
    if (r != MLA_OK) return r;
    ++n;
    splits = L.g.splits;
  }
  k_append_epilogue<T><<<T_, 128, (d->d_rope / 2) * sizeof(float2), st>>>(L.Y, splits, (long)T_ * D, seq_idx, pos, bt, num_seqs, max_pages,
                                          static_cast<T*>(pool), num_pages, d->page_size, d->d_c, d->d_rope,
                                          d->rope_base);
  ++n;
  return MLA_OK;
}

// ------------------------------------------------------------------ mla_absorb_query
struct AbsorbLayout {
  GemmPlan g1, g2, g3;
  float* P1;   // split partials of c^Q (fp32), when g1.splits > 1
  void* cq;    // c^Q, element type [B, d_cq]
  float* Y2;   // [q^C ; q^] partials, fp32 [g2.splits][B][nq]
  void* qc;    // q^C, element type [B, n_h*d_h]
  size_t bytes;
  bool tc_uk;  // the per-head (W^UK_i)^T product runs on the tensor-core GEMM
};
inline AbsorbLayout absorb_layout(const mla_dims* d, int B, void* ws) {
  AbsorbLayout L;
  const int nq = d->n_heads * (d->d_head + d->d_rope);
  const bool simt = proj_uses_simt();
  L.g1 = plan_gemm(d->d_cq, B, d->d_model, 1, true);
  L.g2 = plan_gemm(nq, B, d->d_cq, 1, true);
  L.g3 = plan_gemm(d->d_c, B, d->d_head, d->n_heads, false);
  L.tc_uk = !simt && d->d_head % 64 == 0;
  Carver c{static_cast<char*>(ws)};
  L.P1 = (!simt && L.g1.splits > 1) ? c.take<float>((size_t)L.g1.splits * B * d->d_cq) : nullptr;
  L.cq = c.take<uint16_t>((size_t)B * d->d_cq);
  L.Y2 = c.take<float>((size_t)(simt ? 1 : L.g2.splits) * B * nq);
  L.qc = c.take<uint16_t>((size_t)B * d->n_heads * d->d_head);
  L.bytes = c.off;
  return L;
}

template <typename T>
int absorb_run(const mla_dims* d, const void* h, const void* w_dq, const void* w_uq_qr, const void* w_uk,
               const int32_t* pos, void* q_out, int32_t B, void* ws, cudaStream_t st, int32_t& n) {
  const int nq = d->n_heads * (d->d_head + d->d_rope);
  const int nhd = d->n_heads * d->d_head;
  const int D = d->d_c + d->d_rope;
  const AbsorbLayout L = absorb_layout(d, B, ws);
  T* cq = static_cast<T*>(L.cq);
  T* qc = static_cast<T*>(L.qc);
  int splits2 = 1;
  if (proj_uses_simt()) {
    launch_rowdot<T, T>(static_cast<const T*>(w_dq), static_cast<const T*>(h), cq, d->d_cq, d->d_model, B,
                        d->d_model, d->d_cq, 1, 0, 0, 0, st, n);
    launch_rowdot<T, float>(static_cast<const T*>(w_uq_qr), cq, L.Y2, nq, d->d_cq, B, d->d_cq, nq, 1, 0, 0, 0, st, n);
  } else {
    // c^Q = W^DQ h
    int r;
    if (L.g1.splits > 1) {
      r = gemm_tc<T>({w_dq, d->d_cq, d->d_model, 0}, false, {h, B, d->d_model, 0}, d->d_cq, B, d->d_model, 1, L.g1,
                     L.P1, true, d->d_cq, 0, (long)B * d->d_cq, st);
      if (r != MLA_OK) return r;
      launch_reduce<T>(L.P1, L.g1.splits, (long)B * d->d_cq, B, d->d_cq, d->d_cq, cq, st);
      n += 2;
    } else {
      r = gemm_tc<T>({w_dq, d->d_cq, d->d_model, 0}, false, {h, B, d->d_model, 0}, d->d_cq, B, d->d_model, 1, L.g1,
                     cq, false, d->d_cq, 0, 0, st);
      if (r != MLA_OK) return r;
      ++n;
    }
    // [q^C ; q^] = [W^UQ ; W^QR] c^Q
    r = gemm_tc<T>({w_uq_qr, nq, d->d_cq, 0}, false, {cq, B, d->d_cq, 0}, nq, B, d->d_cq, 1, L.g2, L.Y2, true, nq, 0,
                   (long)B * nq, st);
    if (r != MLA_OK) return r;
    ++n;
    splits2 = L.g2.splits;
  }
  k_query_epilogue<T><<<B, 256, (d->d_rope / 2) * sizeof(float2), st>>>(L.Y2, splits2, (long)B * nq, pos, qc, static_cast<T*>(q_out), d->n_heads,
                                         d->d_head, d->d_rope, d->d_c, d->rope_base);
  ++n;
  // q~_i = (W^UK_i)^T q^C_i
  if (L.tc_uk) {
    const int r = gemm_tc<T>({w_uk, nhd, d->d_c, d->d_head}, true, {qc, B, nhd, d->d_head}, d->d_c, B, d->d_head,
                             d->n_heads, L.g3, q_out, false, (long)d->n_heads * D, D, 0, st);
    if (r != MLA_OK) return r;
  } else {
    const int threads = 128;
    dim3 grid((d->d_c / 2 + threads - 1) / threads, d->n_heads);
    k_absorb_uk<T, 16><<<grid, threads, 16 * d->d_head * sizeof(float), st>>>(
        static_cast<const T*>(w_uk), qc, static_cast<T*>(q_out), B, d->n_heads, d->d_head, d->d_c, D);
  }
  ++n;
  return MLA_OK;
}

// ------------------------------------------------------------------ mla_out_proj
struct OutLayout {
  GemmPlan g_o, g_u;
  void* o;    // element type [B, n_h*d_h]
  float* P;   // split partials of u (fp32), when g_u.splits > 1
  size_t bytes;
  bool tc_o;
};
inline OutLayout out_layout(const mla_dims* d, int B, void* ws) {
  OutLayout L;
  const int nhd = d->n_heads * d->d_head;
  const bool simt = proj_uses_simt();
  L.g_o = plan_gemm(d->d_head, B, d->d_c, d->n_heads, false);
  L.g_u = plan_gemm(d->d_model, B, nhd, 1, true);
  L.tc_o = !simt && d->d_c % 64 == 0;
  Carver c{static_cast<char*>(ws)};
  L.o = c.take<uint16_t>((size_t)B * nhd);
  L.P = (!simt && L.g_u.splits > 1) ? c.take<float>((size_t)L.g_u.splits * B * d->d_model) : nullptr;
  L.bytes = c.off;
  return L;
}

template <typename T>
int out_run(const mla_dims* d, const void* o_lat, const void* w_uv, const void* w_o, void* u, int32_t B, void* ws,
            cudaStream_t st, int32_t& n) {
  const int nhd = d->n_heads * d->d_head;
  const OutLayout L = out_layout(d, B, ws);
  T* o = static_cast<T*>(L.o);
  // o_i = W^UV_i o_lat_i (row block i of W^UV, head i of o_lat)
  if (L.tc_o) {
    const int r = gemm_tc<T>({w_uv, nhd, d->d_c, d->d_head}, false, {o_lat, B, (long)d->n_heads * d->d_c, d->d_c},
                             d->d_head, B, d->d_c, d->n_heads, L.g_o, o, false, nhd, d->d_head, 0, st);
    if (r != MLA_OK) return r;
    ++n;
  } else {
    launch_rowdot<T, T>(static_cast<const T*>(w_uv), static_cast<const T*>(o_lat), o, d->d_head, d->d_c, B,
                        (long)d->n_heads * d->d_c, nhd, d->n_heads, (long)d->d_head * d->d_c, d->d_c, d->d_head, st, n);
  }
  // u = W^O [o_1; ...; o_n_h]
  if (proj_uses_simt()) {
    launch_rowdot<T, T>(static_cast<const T*>(w_o), o, static_cast<T*>(u), d->d_model, nhd, B, nhd, d->d_model, 1, 0,
                        0, 0, st, n);
  } else if (L.g_u.splits > 1) {
    const int r = gemm_tc<T>({w_o, d->d_model, nhd, 0}, false, {o, B, nhd, 0}, d->d_model, B, nhd, 1, L.g_u, L.P,
                             true, d->d_model, 0, (long)B * d->d_model, st);
    if (r != MLA_OK) return r;
    launch_reduce<T>(L.P, L.g_u.splits, (long)B * d->d_model, B, d->d_model, d->d_model, static_cast<T*>(u), st);
    n += 2;
  } else {
    const int r = gemm_tc<T>({w_o, d->d_model, nhd, 0}, false, {o, B, nhd, 0}, d->d_model, B, nhd, 1, L.g_u, u, false,
                             d->d_model, 0, 0, st);
    if (r != MLA_OK) return r;
    ++n;
  }
  return MLA_OK;
}

}  // namespace host
}  // namespace mla
