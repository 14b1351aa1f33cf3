// Host side of the three projection calls (mla_append_kv, mla_absorb_query, mla_out_proj):
// GEMM planning, TMA tensor maps, workspace layout and launches. Every product runs on the
// tcgen05 GEMM, except the two per-head products when the head's slice is not a whole number of
// 64-wide blocks (d_h % 64 for (W^UK_i)^T q^C_i, d_c % 64 for W^UV_i o_lat_i): the GEMM batches
// heads by whole blocks, so those shapes take the CUDA-core kernels of proj_simt.cuh.
// Included once, from libmla.cu.
#pragma once

#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "fp8.cuh"
#include "gemm_sk.cuh"
#include "proj_simt.cuh"

namespace mla {
namespace host {

constexpr int kMaxDev = 64;

// Per-device values cached on first use; atomics, since host threads may call concurrently (a race
// only computes the same value twice).
inline int sm_count() {
  static std::atomic<int> cache[kMaxDev];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
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

// 3-D view of a row-major [rows][9 * 64] tensor of 16-bit elements, rows `row_bytes` apart, as
// (64 columns, rows, 9 column chunks): one box of (64, 64, depth) lands in shared memory as
// `depth` consecutive 64 x 64 chunks, each in the 128-byte-swizzled layout of a 2-D 64 x 64 box.
inline bool encode_chunks(CUtensorMap* map, const void* base, bool bf16, uint64_t rows, uint64_t row_bytes,
                          uint32_t depth) {
  auto fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {64, rows, 9};
  cuuint64_t strides[2] = {row_bytes, 128};
  cuuint32_t box[3] = {64, 64, depth};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base),
            dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D view of a paged cache [pages][64 rows][9 * 64] of 16-bit elements, rows `row_bytes` apart, as
// (64 columns, 64 rows of a page, pages, 9 column chunks) with boxes of (64, 64, 1, depth). A box
// started at row nv - 64 (nv = rows of the page that hold tokens) lands with the page's rows
// [0, nv) in the box's last nv rows and zeros (the fill outside the tensor) in the rows before.
inline bool encode_pages(CUtensorMap* map, const void* base, bool bf16, uint64_t pages, uint64_t row_bytes,
                         uint32_t depth) {
  auto fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  cuuint64_t dims[4] = {64, 64, pages, 9};
  cuuint64_t strides[3] = {row_bytes, 64 * row_bytes, 128};
  cuuint32_t box[4] = {64, 64, 1, depth};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(base),
            dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// FP8 pages (see fp8.cuh) viewed as (576 byte columns, 64 rows, pages): rows of 576 bytes, pages
// of 64 rows plus their 512 bytes of scales; boxes of `width` bytes x 64 rows x 1 page, no
// swizzle. Rows outside the page read as zeros.
inline bool encode_pages_fp8(CUtensorMap* map, const void* base, uint64_t pages, uint32_t width) {
  auto fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {576, 64, pages};
  cuuint64_t strides[2] = {576, 64 * (576 + 8)};
  cuuint32_t box[3] = {width, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same view with 32-byte x 32-head boxes, unswizzled: the attention epilogue's half rounds.
inline bool encode_heads_out32(CUtensorMap* map, void* base, CUtensorMapDataType dtype, uint32_t elem_bytes,
                               uint64_t n_h, uint64_t rows) {
  auto fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {512, n_h, rows};
  cuuint64_t strides[2] = {512 * elem_bytes, 512 * elem_bytes * n_h};
  cuuint32_t box[3] = {32 / elem_bytes, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, dtype, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view of an output [rows][n_h][512] (fp32, bf16 or fp16) as (512 columns, n_h heads, rows)
// with boxes of 64 bytes x 32 heads x 1 row in the 64-byte swizzle: the attention epilogue's
// staging layout. Heads past n_h fall outside the tensor and are not written by a store.
inline bool encode_heads_out(CUtensorMap* map, void* base, CUtensorMapDataType dtype, uint32_t elem_bytes,
                             uint64_t n_h, uint64_t rows) {
  auto fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {512, n_h, rows};
  cuuint64_t strides[2] = {512 * elem_bytes, 512 * elem_bytes * n_h};
  cuuint32_t box[3] = {64 / elem_bytes, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, dtype, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ GEMM planning
// One stream-K GEMM launch (see gemm_sk.cuh): tile sizes, CTA count, ring depth, and whether
// any tile is shared by several CTAs (then fp32 partials and a reduction launch are needed).
struct SkPlan {
  int bn, m_tiles, n_tiles, batch, kb, tiles, G, stages;
  long iters;
  bool aligned, split;
  size_t smem, part_bytes;
};

constexpr int kSkMinIters = 8;       // k blocks per CTA at least, when tiles are split
constexpr int kSkLongTile = 16;      // tiles of at least this many k blocks are split (stream-K)
constexpr size_t kSkSmemMax = 232448;
constexpr size_t kSkSmemHalf = 113 * 1024;  // two CTAs per SM (228 KB per SM, 1 KB reserved per CTA)

inline SkPlan plan_sk(int M, int N, int K, int batch, bool fused_epi, int d_rope) {
  SkPlan g;
  g.bn = N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
  g.n_tiles = (N + g.bn - 1) / g.bn;
  g.m_tiles = (M + 127) / 128;
  g.batch = batch;
  g.kb = (K + 63) / 64;
  g.tiles = g.m_tiles * g.n_tiles * batch;
  g.iters = (long)g.tiles * g.kb;
  const int sms = sm_count();
  const size_t stage = (size_t)(128 + g.bn) * 64 * 2;
  const size_t table = fused_epi ? (size_t)g.bn * (d_rope / 2) * 8 + (size_t)g.bn * 8 : 0;
  const size_t fixed = 1024 + table + 256;
  // Long tiles, at least one per SM: whole tiles per CTA, two CTAs per SM (half-size rings), so
  // no tile is split and no reduction launch follows ([W^UQ; W^QR] at decode sizes: 192 tiles of
  // 24 k blocks).
  const bool long_many = g.kb >= kSkLongTile && g.tiles >= sms && fixed + 2 * stage <= kSkSmemHalf;
  if (g.kb >= kSkLongTile && !long_many) {
    g.aligned = false;
    g.G = (int)std::max(1L, std::min((long)sms, g.iters / kSkMinIters));
  } else {
    g.aligned = true;
    const int per = (g.tiles + (long_many ? 2 : 1) * sms - 1) / ((long_many ? 2 : 1) * sms);
    g.G = (g.tiles + per - 1) / per;
  }
  g.split = false;
  if (!g.aligned)
    for (int c = 1; c < g.G && !g.split; ++c) g.split = (g.iters * c / g.G) % g.kb != 0;
  g.stages = (int)std::min<size_t>(12, ((long_many ? kSkSmemHalf : kSkSmemMax) - fixed) / stage);
  // Many short tiles (the per-head products): when a CTA's whole range fits a half-size ring,
  // run two CTAs per SM, so that two sets of epilogue warps drain tiles side by side.
  if (g.aligned && g.tiles > sms) {
    const int per2 = (g.tiles + 2 * sms - 1) / (2 * sms);
    const int need = per2 * g.kb;  // every stage of the range resident at once
    if (need >= 2 && fixed + (size_t)need * stage <= kSkSmemHalf) {
      g.G = (g.tiles + per2 - 1) / per2;
      g.stages = need;
    }
  }
  g.smem = fixed + (size_t)g.stages * stage;
  g.part_bytes = g.split ? (size_t)(g.tiles + g.G) * 128 * g.bn * sizeof(float) : 0;
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

template <typename T, int BN, bool MN, int MODE>
cudaError_t run_sk(const CUtensorMap& ma, const CUtensorMap& mb, const tc::SkParams& p, const SkPlan& g,
                   cudaStream_t st, int32_t& n) {
  static std::atomic<bool> attr_done[kMaxDev];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < kMaxDev && !attr_done[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(tc::k_gemm_sk<T, BN, MN, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSkSmemMax);
    if (e != cudaSuccess) return e;
    attr_done[dev].store(true, std::memory_order_release);
  }
  cudaError_t e = launch_pdl(tc::k_gemm_sk<T, BN, MN, MODE>, dim3(g.G), dim3(192), g.smem, st, ma, mb, p);
  if (e != cudaSuccess) return e;
  ++n;
  if (g.split) {
    e = launch_pdl(tc::k_sk_reduce<T, BN, MODE>, dim3(g.tiles, BN / 4), dim3(256), 0, st, p, g.G);
    if (e != cudaSuccess) return e;
    ++n;
  }
  return cudaGetLastError();
}

template <typename T, int BN>
cudaError_t run_sk_mode(const CUtensorMap& ma, const CUtensorMap& mb, bool a_mn, const tc::SkParams& p,
                        const SkPlan& g, cudaStream_t st, int32_t& n) {
  switch (p.epi.mode) {
    case tc::kEpiPlain:
      return a_mn ? run_sk<T, BN, true, tc::kEpiPlain>(ma, mb, p, g, st, n)
                  : run_sk<T, BN, false, tc::kEpiPlain>(ma, mb, p, g, st, n);
    case tc::kEpiAppend:  // the fused steps read K-major weights
      return a_mn ? cudaErrorInvalidValue : run_sk<T, BN, false, tc::kEpiAppend>(ma, mb, p, g, st, n);
    case tc::kEpiQuery:
      return a_mn ? cudaErrorInvalidValue : run_sk<T, BN, false, tc::kEpiQuery>(ma, mb, p, g, st, n);
    default:
      return cudaErrorInvalidValue;
  }
}

// D[z][m][n] = sum_k A[z][m][k] B[z][n][k], finished by the output step `epi`; `part` holds
// g.part_bytes of scratch when g.split.
template <typename T>
int gemm_sk(const Operand& A, bool a_mn, const Operand& B, int M, int N, int K, const SkPlan& g,
            const tc::EpiParams& epi, float* part, cudaStream_t st, int32_t& n) {
  if (N <= 0 || M <= 0) return MLA_OK;
  if (g.stages < 2 || g.smem > kSkSmemMax) return MLA_ERR_CUDA;  // no shape of the library reaches this
  constexpr bool bf16 = tc::IsBf16<T>::value;
  CUtensorMap ma, mb;
  const bool ok_a = a_mn ? encode_2d(&ma, A.base, bf16, A.cols, A.rows, A.cols * 2, 64, 64)
                         : encode_2d(&ma, A.base, bf16, A.cols, A.rows, A.cols * 2, 64, 128);
  const bool ok_b = encode_2d(&mb, B.base, bf16, B.cols, B.rows, B.cols * 2, 64, g.bn);
  if (!ok_a || !ok_b) return MLA_ERR_CUDA;
  tc::SkParams p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.m_tiles = g.m_tiles;
  p.n_tiles = g.n_tiles;
  p.kb = g.kb;
  p.iters = g.iters;
  p.aligned = g.aligned ? 1 : 0;
  p.tiles = g.tiles;
  p.stages = g.stages;
  p.a_batch_off = A.batch_off;
  p.b_batch_off = B.batch_off;
  p.part = part;
  p.epi = epi;
  cudaError_t e;
  switch (g.bn) {
    case 32: e = run_sk_mode<T, 32>(ma, mb, a_mn, p, g, st, n); break;
    case 64: e = run_sk_mode<T, 64>(ma, mb, a_mn, p, g, st, n); break;
    case 128: e = run_sk_mode<T, 128>(ma, mb, a_mn, p, g, st, n); break;
    case 256: e = run_sk_mode<T, 256>(ma, mb, a_mn, p, g, st, n); break;
    default: return MLA_ERR_CUDA;
  }
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

inline tc::EpiParams epi_plain(void* out, long ld, long batch_off) {
  tc::EpiParams e{};
  e.mode = tc::kEpiPlain;
  e.out = out;
  e.out_ld = ld;
  e.out_batch_off = batch_off;
  e.d_rope = 2;
  return e;
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
  SkPlan g;
  float* part;  // stream-K partials
  float2* cs;   // RoPE cos/sin per token for the reduction of split tiles
  size_t bytes;
};
inline AppendLayout append_layout(const mla_dims* d, int T_, void* ws) {
  AppendLayout L;
  const int D = d->d_c + d->d_rope;
  L.g = plan_sk(D, T_, d->d_model, 1, true, d->d_rope);
  Carver c{static_cast<char*>(ws)};
  L.part = L.g.split ? c.take<float>(L.g.part_bytes / sizeof(float)) : nullptr;
  L.cs = (L.g.split && L.g.n_tiles == 1) ? c.take<float2>((size_t)T_ * (d->d_rope / 2)) : nullptr;
  L.bytes = c.off;
  return L;
}

template <typename T>
int append_run(const mla_dims* d, const void* h, const void* w, const int32_t* seq_idx, const int32_t* pos,
               const int32_t* bt, int32_t num_seqs, int32_t max_pages, void* pool, int32_t num_pages, int32_t T_,
               void* ws, cudaStream_t st, int32_t& n) {
  const int D = d->d_c + d->d_rope;
  const AppendLayout L = append_layout(d, T_, ws);
  // [c^KV ; k^R] = W^{DKV,KR} h, RoPE on k^R, written to each token's cache slot
  tc::EpiParams e{};
  e.mode = tc::kEpiAppend;
  e.out = pool;
  e.rope_lo = d->d_c;
  e.d_rope = d->d_rope;
  e.rope_base = d->rope_base;
  e.rope_table = d->rope_inv_freq;
  e.pos = pos;
  e.seq_idx = seq_idx;
  e.bt = bt;
  e.num_seqs = num_seqs;
  e.max_pages = max_pages;
  e.num_pages = num_pages;
  e.page_size = d->page_size;
  e.d_c = d->d_c;
  e.cs_glob = L.cs;
  return gemm_sk<T>({w, D, d->d_model, 0}, false, {h, T_, d->d_model, 0}, D, T_, d->d_model, L.g, e, L.part, st, n);
}

// ------------------------------------------------------------------ mla_append_kv_fp8
// The append GEMM writes the rows (element type, RoPE applied) to a staging area after its own
// workspace; k_quant_fp8 then quantises each into its FP8 cache slot.
inline size_t append_fp8_bytes(const mla_dims* d, int T_) {
  return ((append_layout(d, T_, nullptr).bytes + 255) & ~size_t(255)) + (size_t)T_ * (d->d_c + d->d_rope) * 2;
}

template <typename T>
int append_fp8_run(const mla_dims* d, const void* h, const void* w, const int32_t* seq_idx, const int32_t* pos,
                   const int32_t* bt, int32_t num_seqs, int32_t max_pages, void* pool, int32_t num_pages, int32_t T_,
                   void* ws, cudaStream_t st, int32_t& n) {
  const int D = d->d_c + d->d_rope;
  const AppendLayout L = append_layout(d, T_, ws);
  T* rows = reinterpret_cast<T*>(static_cast<char*>(ws) + ((L.bytes + 255) & ~size_t(255)));
  tc::EpiParams e{};
  e.mode = tc::kEpiAppend;
  e.out = rows;
  e.stage_rows = 1;
  e.rope_lo = d->d_c;
  e.d_rope = d->d_rope;
  e.rope_base = d->rope_base;
  e.rope_table = d->rope_inv_freq;
  e.pos = pos;
  e.seq_idx = seq_idx;
  e.bt = bt;
  e.num_seqs = num_seqs;
  e.max_pages = max_pages;
  e.num_pages = num_pages;
  e.page_size = d->page_size;
  e.d_c = d->d_c;
  e.cs_glob = L.cs;
  const int r = gemm_sk<T>({w, D, d->d_model, 0}, false, {h, T_, d->d_model, 0}, D, T_, d->d_model, L.g, e, L.part, st, n);
  if (r != MLA_OK) return r;
  if (launch_pdl(k_quant_fp8<T>, dim3((unsigned)((T_ + 7) / 8)), dim3(256), 0, st, static_cast<const T*>(rows),
                 seq_idx, pos, bt, (int)num_seqs, (int)max_pages, (int)num_pages, (int)d->page_size, (int)d->d_c, D,
                 (int)T_, static_cast<uint8_t*>(pool)) != cudaSuccess)
    return MLA_ERR_CUDA;
  ++n;
  return MLA_OK;
}

// ------------------------------------------------------------------ mla_absorb_query
struct AbsorbLayout {
  SkPlan g1, g2, g3;
  void* cq;     // c^Q, element type [B, d_cq]
  void* qc;     // q^C, element type [B, n_h*d_h]
  float* part;  // stream-K partials, shared by the three products (they run one after another)
  float2* cs;   // RoPE cos/sin per token, filled by the W^DQ product for the query product
  size_t bytes;
  bool tc_uk;   // the per-head (W^UK_i)^T product runs on the tensor-core GEMM
};
inline AbsorbLayout absorb_layout(const mla_dims* d, int B, void* ws) {
  AbsorbLayout L;
  const int nq = d->n_heads * (d->d_head + d->d_rope);
  L.g1 = plan_sk(d->d_cq, B, d->d_model, 1, false, d->d_rope);
  L.g2 = plan_sk(nq, B, d->d_cq, 1, true, d->d_rope);
  L.g3 = plan_sk(d->d_c, B, d->d_head, d->n_heads, false, d->d_rope);
  L.tc_uk = d->d_head % 64 == 0;
  Carver c{static_cast<char*>(ws)};
  L.cq = c.take<uint16_t>((size_t)B * d->d_cq);
  L.qc = c.take<uint16_t>((size_t)B * d->n_heads * d->d_head);
  const size_t part = std::max(L.g1.part_bytes, std::max(L.g2.part_bytes, L.tc_uk ? L.g3.part_bytes : 0));
  L.part = part ? c.take<float>(part / sizeof(float)) : nullptr;
  L.cs = c.take<float2>((size_t)B * (d->d_rope / 2));
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
  {
    // c^Q = W^DQ h; its CTAs also tabulate the query's RoPE cos/sin for the next product
    tc::EpiParams e1 = epi_plain(cq, d->d_cq, 0);
    e1.cs_prefill = L.cs;
    e1.pos = pos;
    e1.d_rope = d->d_rope;
    e1.rope_base = d->rope_base;
    e1.rope_table = d->rope_inv_freq;
    int r = gemm_sk<T>({w_dq, d->d_cq, d->d_model, 0}, false, {h, B, d->d_model, 0}, d->d_cq, B, d->d_model, L.g1, e1,
                       L.part, st, n);
    if (r != MLA_OK) return r;
    // [q^C ; q^] = [W^UQ ; W^QR] c^Q; q^C -> qc, q^R_i = RoPE(q^_i) -> q_out[b][i][d_c:]
    tc::EpiParams e{};
    e.mode = tc::kEpiQuery;
    e.out = q_out;
    e.rope_lo = nhd;
    e.d_rope = d->d_rope;
    e.rope_base = d->rope_base;
    e.rope_table = d->rope_inv_freq;
    e.pos = pos;
    e.qc = qc;
    e.n_h = d->n_heads;
    e.d_c = d->d_c;
    e.cs_glob = L.cs;
    e.cs_ready = L.cs != nullptr;
    // one n tile: rope tiles go through the reduction, which runs anyway, instead of rotating from
    // a shared-memory table while the next tile streams in; several n tiles: whole tiles read the
    // cos/sin per element from the global table
    e.rope_in_reduce = L.g2.split && L.g2.n_tiles == 1 && L.cs != nullptr;
    r = gemm_sk<T>({w_uq_qr, nq, d->d_cq, 0}, false, {cq, B, d->d_cq, 0}, nq, B, d->d_cq, L.g2, e, L.part, st, n);
    if (r != MLA_OK) return r;
  }
  // q~_i = (W^UK_i)^T q^C_i -> q_out[b][i][:d_c]
  if (L.tc_uk) {
    const int r = gemm_sk<T>({w_uk, nhd, d->d_c, d->d_head}, true, {qc, B, nhd, d->d_head}, d->d_c, B, d->d_head,
                             L.g3, epi_plain(q_out, (long)d->n_heads * D, D), L.part, st, n);
    if (r != MLA_OK) return r;
  } else {
    const int threads = 128;
    dim3 grid((d->d_c / 2 + threads - 1) / threads, d->n_heads);
    k_absorb_uk<T, 16><<<grid, threads, 16 * d->d_head * sizeof(float), st>>>(
        static_cast<const T*>(w_uk), qc, static_cast<T*>(q_out), B, d->n_heads, d->d_head, d->d_c, D);
    ++n;
  }
  return MLA_OK;
}

// ------------------------------------------------------------------ mla_out_proj
struct OutLayout {
  SkPlan g_o, g_u;
  void* o;      // element type [B, n_h*d_h]
  float* part;  // stream-K partials, shared by the two products
  size_t bytes;
  bool tc_o;
};
inline OutLayout out_layout(const mla_dims* d, int B, void* ws) {
  OutLayout L;
  const int nhd = d->n_heads * d->d_head;
  L.g_o = plan_sk(d->d_head, B, d->d_c, d->n_heads, false, d->d_rope);
  L.g_u = plan_sk(d->d_model, B, nhd, 1, false, d->d_rope);
  L.tc_o = d->d_c % 64 == 0;
  Carver c{static_cast<char*>(ws)};
  L.o = c.take<uint16_t>((size_t)B * nhd);
  const size_t part = std::max(L.tc_o ? L.g_o.part_bytes : 0, L.g_u.part_bytes);
  L.part = part ? c.take<float>(part / sizeof(float)) : nullptr;
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
    const int r = gemm_sk<T>({w_uv, nhd, d->d_c, d->d_head}, false, {o_lat, B, (long)d->n_heads * d->d_c, d->d_c},
                             d->d_head, B, d->d_c, L.g_o, epi_plain(o, nhd, d->d_head), L.part, st, n);
    if (r != MLA_OK) return r;
  } else {
    launch_rowdot<T, T>(static_cast<const T*>(w_uv), static_cast<const T*>(o_lat), o, d->d_head, d->d_c, B,
                        (long)d->n_heads * d->d_c, nhd, d->n_heads, (long)d->d_head * d->d_c, d->d_c, d->d_head, st, n);
  }
  // u = W^O [o_1; ...; o_n_h]
  return gemm_sk<T>({w_o, d->d_model, nhd, 0}, false, {o, B, nhd, 0}, d->d_model, B, nhd, L.g_u,
                    epi_plain(u, d->d_model, 0), L.part, st, n);
}

}  // namespace host
}  // namespace mla
