// libmla — C ABI of the MLA absorbed-decode path (declared in include/mla.h and include/mla_debug.h).
// One translation unit: the kernels are included from the .cuh files beside this one.
// Host code here validates arguments (before anything is queued), carves the caller's
// workspace, picks kernels and launches them on the caller's stream. It allocates nothing.
#include "mla_debug.h"
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "decode_mma.cuh"
#include "decode_simt.cuh"
#include "decode_tc.cuh"
#include "layer_small.cuh"
#include "prefill.cuh"
#include "proj_host.cuh"

using namespace mla;

namespace {

// NVTX range around each entry point (host side: the argument checks and the launches), named
// after the call, for timelines taken with a profiler; without one attached it costs a few ns.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

thread_local int32_t t_launches[8] = {0, 0, 0, 0, 0, 0, 0, 0};
// Profiling hook: events recorded around the attention kernel of this thread's decode calls.
thread_local cudaEvent_t t_ev_before = nullptr, t_ev_after = nullptr;
inline void mark_before(cudaStream_t st) {
  if (t_ev_before != nullptr) cudaEventRecord(t_ev_before, st);
}
inline void mark_after(cudaStream_t st) {
  if (t_ev_after != nullptr) cudaEventRecord(t_ev_after, st);
}

constexpr int kMaxDevices = 64;
// Longest attended length the attention calls accept: page counts and token indices stay far
// from int32 overflow in every kernel.
constexpr int32_t kMaxSeqLen = 1 << 30;

// Per-device values cached on first use. Host threads may call concurrently: the caches are
// atomics, and a race only computes the same value twice.
int device_sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Sequential sub-allocation of the caller's workspace (256-byte aligned pieces).
struct Carve {
  char* base;
  size_t off = 0;
  template <typename X>
  X* take(size_t count) {
    X* p = reinterpret_cast<X*>(base + off);
    off += align256(count * sizeof(X));
    return p;
  }
};

int check_dims_impl(const mla_dims* d) {
  if (d == nullptr) return MLA_ERR_INVALID_ARG;
  if (d->dtype != MLA_BF16 && d->dtype != MLA_FP16) return MLA_ERR_INVALID_ARG;
  if (!(d->rope_base > 0.0) || !std::isfinite(d->rope_base)) return MLA_ERR_INVALID_ARG;
  const int32_t w[] = {d->d_model, d->n_heads, d->d_head, d->d_c, d->d_cq, d->d_rope, d->page_size};
  for (int32_t v : w)
    if (v <= 0) return MLA_ERR_INVALID_ARG;
  if (d->d_model % 8 || d->d_head % 8 || d->d_c % 8 || d->d_cq % 8 || d->d_rope % 8) return MLA_ERR_UNSUPPORTED_DIMS;
  if (d->n_heads > 128 || d->d_c > 512 || d->d_c + d->d_rope > 576) return MLA_ERR_UNSUPPORTED_DIMS;
  if ((reinterpret_cast<uintptr_t>(d->rope_inv_freq) & 7u) != 0) return MLA_ERR_ALIGNMENT;
  return MLA_OK;
}

// ---------------------------------------------------------------- decode planning
struct DecodePlan {
  int n_splits;
  int split_len;
  int head_groups;
};

// The warp-MMA kernel for small head counts (decode_mma.cuh): up to 16 heads of a row of at most
// 192 columns, latent at most 128, everything in 16-column steps.
bool decode_mma_eligible(const mla_dims* d) {
  const int D = d->d_c + d->d_rope;
  return d->n_heads <= 16 && D % 16 == 0 && D <= 16 * dmma::kMaxKD && d->d_c % 16 == 0 &&
         d->d_c <= 8 * dmma::kMaxND && d->page_size % 16 == 0;
}

// Split-KV plan of the warp-MMA kernel: about three CTAs per SM in one wave, each a whole number
// of 64-token stages.
DecodePlan plan_decode_mma(int B, int max_seq_len) {
  DecodePlan p;
  p.head_groups = 1;
  const long ctas_wanted = 3L * device_sm_count();
  long s = (ctas_wanted + B - 1) / B;
  const long stages = ((long)max_seq_len + dmma::kStageTokens - 1) / dmma::kStageTokens;
  if (s > stages) s = stages;
  if (s < 1) s = 1;
  const long per = (stages + s - 1) / s;  // stages per split
  p.split_len = (int)(per * dmma::kStageTokens);
  p.n_splits = (int)(((long)max_seq_len + p.split_len - 1) / p.split_len);
  return p;
}

DecodePlan plan_decode(const mla_dims* d, int B, int max_seq_len) {
  if (decode_mma_eligible(d)) return plan_decode_mma(B, max_seq_len);
  DecodePlan p;
  p.head_groups = (d->n_heads + 7) / 8;
  const long blocks_wanted = 4L * device_sm_count();
  const long base = (long)B * p.head_groups;
  long s = (blocks_wanted + base - 1) / base;
  const long by_len = ((long)max_seq_len + 255) / 256;  // at least 256 tokens per split
  if (s > by_len) s = by_len;
  if (s < 1) s = 1;
  p.n_splits = (int)s;
  p.split_len = (int)((max_seq_len + s - 1) / s);
  return p;
}

size_t ws_append(const mla_dims* d, int T) { return T > 0 ? host::append_layout(d, T, nullptr).bytes : 0; }
size_t ws_append_fp8(const mla_dims* d, int T) { return T > 0 ? host::append_fp8_bytes(d, T) : 0; }
size_t ws_absorb(const mla_dims* d, int B) { return B > 0 ? host::absorb_layout(d, B, nullptr).bytes : 0; }
size_t ws_out(const mla_dims* d, int B) { return B > 0 ? host::out_layout(d, B, nullptr).bytes : 0; }

int finish_launches(int call, int32_t launches) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  t_launches[call] = launches;
  return MLA_OK;
}

template <typename T>
int append_impl(const mla_dims* d, const void* h, const void* w, const int32_t* seq_idx, const int32_t* pos,
                const int32_t* bt, int32_t num_seqs, int32_t max_pages, void* pool, int32_t num_pages, int32_t T_,
                void* ws, cudaStream_t st) {
  int32_t n = 0;
  const int r = host::append_run<T>(d, h, w, seq_idx, pos, bt, num_seqs, max_pages, pool, num_pages, T_, ws, st, n);
  if (r != MLA_OK) return r;
  return finish_launches(MLA_CALL_APPEND_KV, n);
}

template <typename T>
int absorb_impl(const mla_dims* d, const void* h, const void* w_dq, const void* w_uq_qr, const void* w_uk,
                const int32_t* pos, void* q_out, int32_t B, void* ws, cudaStream_t st) {
  int32_t n = 0;
  const int r = host::absorb_run<T>(d, h, w_dq, w_uq_qr, w_uk, pos, q_out, B, ws, st, n);
  if (r != MLA_OK) return r;
  return finish_launches(MLA_CALL_ABSORB_QUERY, n);
}

// ---------------------------------------------------------------- tensor-core decode
// The tcgen05 path serves DeepSeek-V2-shaped caches (d_c = 512, d_h^R = 64, 64-token pages,
// 65..128 heads: one pair of SMs holds the heads' 512-column accumulators); other shapes, the
// running model's eight heads among them, take the CUDA-core kernel.
bool decode_tc_eligible(const mla_dims* d) {
  return d->n_heads > 64 && d->n_heads <= 128 && d->d_c == tc::dec::kDc &&
         d->d_c + d->d_rope == tc::dec::kD && d->page_size == tc::dec::kPage;
}

// The FP8 cache serves the tensor-core decode's shape only.
int fp8_dims(const mla_dims* d) {
  const int r = check_dims_impl(d);
  if (r != MLA_OK) return r;
  return decode_tc_eligible(d) ? MLA_OK : MLA_ERR_UNSUPPORTED_DIMS;
}

template <typename T, bool F8 = false>
bool decode_tc_set_smem() {
  static std::atomic<bool> done[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (!done[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(tc::k_decode_tc<T, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::dec::kSmem) !=
        cudaSuccess)
      return false;
    done[dev].store(true, std::memory_order_release);
  }
  return true;
}

// Clusters of two CTAs that can be resident at once: the work is split statically over them.
int decode_clusters() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return device_sm_count() / 2;
  int c = cache[dev].load(std::memory_order_relaxed);
  if (c == 0) {
    int n = 0;
    if (decode_tc_set_smem<__nv_bfloat16>()) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (device_sm_count() / 2), 1, 1);
      cfg.blockDim = dim3(tc::dec::kThreads, 1, 1);
      cfg.dynamicSmemBytes = tc::dec::kSmem;
      if (cudaOccupancyMaxActiveClusters(&n, tc::k_decode_tc<__nv_bfloat16>, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    c = std::min(n > 0 ? n : device_sm_count() / 2, tc::kMaxDecodeClusters);
    cache[dev].store(c, std::memory_order_relaxed);
  }
  return c;
}

size_t ws_decode_tc(const mla_dims* d, int B) {
  const size_t slots = (size_t)B + decode_clusters();
  return align256((size_t)(B + 1) * 4) + align256((size_t)B * 4) + align256((tc::kMaxDecodeClusters + 1) * 4) +
         align256(slots * d->n_heads * tc::dec::kDc * 4) + align256(slots * d->n_heads * 4);
}

// Pages of the longest sequence; the planner's page counts, summed over a launch, must stay in
// int32.
inline long pages_of(const mla_dims* d, int32_t max_seq_len) {
  return ((long)max_seq_len + d->page_size - 1) / d->page_size;
}
inline bool page_total_fits(const mla_dims* d, long items, int32_t max_seq_len) {
  return items * pages_of(d, max_seq_len) <= (long)INT32_MAX;
}

size_t ws_decode(const mla_dims* d, int B, int max_seq_len) {
  if (B <= 0 || max_seq_len < 1 || max_seq_len > kMaxSeqLen) return 0;
  if (decode_tc_eligible(d)) return ws_decode_tc(d, B);
  const DecodePlan p = plan_decode(d, B, max_seq_len);
  if (p.n_splits == 1) return 0;
  const size_t bh = (size_t)B * d->n_heads;
  return align256(bh * p.n_splits * d->d_c * 4) + align256(bh * p.n_splits * 4);
}

// caller_inputs: seq_lens and bt come from the caller (no kernel of this call wrote them), so the
// planner may read them before waiting for the kernel before it.
template <typename T, bool F8 = false>
int decode_tc_impl(const mla_dims* d, const void* q, const void* pool, int32_t num_pages, const int32_t* bt,
                   int32_t max_pages, const int32_t* seq_lens, int32_t B, int32_t max_seq_len, void* o_lat,
                   float* lse_out, void* ws, cudaStream_t st, int32_t& launches, bool caller_inputs) {
  const int C = decode_clusters();
  if (!decode_tc_set_smem<T, F8>()) return MLA_ERR_CUDA;
  Carve c{static_cast<char*>(ws)};
  int* prefix = c.take<int>((size_t)B + 1);
  int* seq_pairs = c.take<int>((size_t)B);
  int* pair_start = c.take<int>(tc::kMaxDecodeClusters + 1);
  float* o_part = c.take<float>(((size_t)B + C) * d->n_heads * tc::dec::kDc);
  float* lse_part = c.take<float>(((size_t)B + C) * d->n_heads);
  constexpr bool bf16 = tc::IsBf16<T>::value;
  tc::DecodeTcMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const bool pages_ok =
      F8 ? host::encode_pages_fp8(&maps.f8_256, pool, (uint64_t)num_pages, 256) &&
               host::encode_pages_fp8(&maps.f8_128, pool, (uint64_t)num_pages, 128) &&
               host::encode_pages_fp8(&maps.f8_64, pool, (uint64_t)num_pages, 64)
         : host::encode_pages(&maps.page1, pool, bf16, (uint64_t)num_pages, tc::dec::kD * 2, 1) &&
               host::encode_pages(&maps.page2, pool, bf16, (uint64_t)num_pages, tc::dec::kD * 2, 2) &&
               host::encode_pages(&maps.page4, pool, bf16, (uint64_t)num_pages, tc::dec::kD * 2, 4);
  if (!pages_ok ||
      !host::encode_chunks(&maps.q9, q, bf16, (uint64_t)B * d->n_heads, tc::dec::kD * 2, 9) ||
      !host::encode_heads_out(&maps.o_lat, o_lat, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                              2, (uint64_t)d->n_heads, (uint64_t)B) ||
      !host::encode_heads_out(&maps.o_part, o_part, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)d->n_heads,
                              (uint64_t)B + C) ||
      !host::encode_heads_out32(&maps.o_lat_h, o_lat,
                                bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                                (uint64_t)d->n_heads, (uint64_t)B) ||
      !host::encode_heads_out32(&maps.o_part_h, o_part, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)d->n_heads,
                                (uint64_t)B + C))
    return MLA_ERR_CUDA;
  if (launch_pdl(tc::k_decode_plan, dim3(1), dim3(1024), 0, st, seq_lens, bt, (int)B, (int)max_pages, (int)num_pages,
                 (int)max_seq_len, C, (int)caller_inputs, prefix, seq_pairs, pair_start) != cudaSuccess)
    return MLA_ERR_CUDA;
  tc::DecodeTcParams p;
  p.bt = bt;
  p.max_pages = max_pages;
  p.seq_lens = seq_lens;
  p.tile_prefix = prefix;
  p.B = B;
  p.n_h = d->n_heads;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)(d->d_head + d->d_rope)));
  p.o_lat = o_lat;
  p.lse_out = lse_out;
  p.o_part = o_part;
  p.lse_part = lse_part;
  p.f8_pool = F8 ? static_cast<const uint8_t*>(pool) : nullptr;
  mark_before(st);
  if (launch_pdl(tc::k_decode_tc<T, F8>, dim3(2 * C), dim3(F8 ? tc::dec::kThreadsF8 : tc::dec::kThreads),
                 tc::dec::kSmem, st, maps, p) != cudaSuccess)
    return MLA_ERR_CUDA;
  mark_after(st);
  if (launch_pdl(tc::k_decode_tc_merge<T>, dim3(B, (d->n_heads + 31) / 32), dim3(512), 0, st,
                 static_cast<const float*>(o_part), static_cast<const float*>(lse_part),
                 static_cast<const int*>(seq_pairs), static_cast<const int*>(pair_start), (int)d->n_heads,
                 static_cast<T*>(o_lat), lse_out) != cudaSuccess)
    return MLA_ERR_CUDA;
  launches += 3;
  return MLA_OK;
}

template <typename T>
bool decode_mma_set_smem(size_t smem) {
  static std::atomic<bool> done[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (!done[dev].load(std::memory_order_acquire)) {
    // the largest row the kernel takes, so that one setting serves every eligible shape
    if (cudaFuncSetAttribute(k_decode_mma<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)dmma::smem_bytes(16 * dmma::kMaxKD)) != cudaSuccess)
      return false;
    done[dev].store(true, std::memory_order_release);
  }
  return smem <= dmma::smem_bytes(16 * dmma::kMaxKD);
}

template <typename T, int NPAIR>
void launch_decode_simt(const mla_dims* d, const DecodePlan& p, const void* q, const void* pool, int32_t num_pages,
                        const int32_t* bt, int32_t max_pages, const int32_t* seq_lens, int32_t B, int32_t max_seq_len,
                        void* o_lat, float* lse_out, float* o_part, float* lse_part, cudaStream_t st) {
  const float scale_log2 = (float)(1.0 / std::sqrt((double)(d->d_head + d->d_rope)) * 1.4426950408889634);
  dim3 grid(p.n_splits, B, p.head_groups);
  mark_before(st);
  k_decode_simt<T, NPAIR><<<grid, 256, 0, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(pool), bt, max_pages, seq_lens, max_seq_len, num_pages,
      d->n_heads, d->d_c, d->d_c + d->d_rope, d->page_size, scale_log2, p.split_len, p.n_splits,
      static_cast<T*>(o_lat), lse_out, o_part, lse_part);
  mark_after(st);
}

template <typename T>
int decode_impl(const mla_dims* d, const void* q, const void* pool, int32_t num_pages, const int32_t* bt,
                int32_t max_pages, const int32_t* seq_lens, int32_t B, int32_t max_seq_len, void* o_lat,
                float* lse_out, void* ws, cudaStream_t st, int32_t& launches, bool caller_inputs) {
  if (decode_tc_eligible(d))
    return decode_tc_impl<T>(d, q, pool, num_pages, bt, max_pages, seq_lens, B, max_seq_len, o_lat, lse_out, ws, st,
                             launches, caller_inputs);
  const DecodePlan p = plan_decode(d, B, max_seq_len);
  const size_t bh = (size_t)B * d->n_heads;
  float* o_part = nullptr;
  float* lse_part = nullptr;
  if (p.n_splits > 1) {
    Carve c{static_cast<char*>(ws)};
    o_part = c.take<float>(bh * p.n_splits * d->d_c);
    lse_part = c.take<float>(bh * p.n_splits);
  }
  const int D = d->d_c + d->d_rope;
  int32_t& n = launches;
  if (decode_mma_eligible(d)) {
    const float scale_log2 = (float)(1.0 / std::sqrt((double)(d->d_head + d->d_rope)) * 1.4426950408889634);
    const size_t smem = dmma::smem_bytes(D);
    if (!decode_mma_set_smem<T>(smem)) return MLA_ERR_CUDA;
    mark_before(st);
    const MmaAttnArgs a{q, pool, bt, (int)max_pages, seq_lens, (int)max_seq_len, (int)num_pages, (int)d->n_heads,
                        (int)d->d_c, D, (int)d->page_size, scale_log2, p.split_len, p.n_splits, o_lat, lse_out,
                        o_part, lse_part};
    if (launch_pdl(k_decode_mma<T>, dim3(p.n_splits, B), dim3(128), smem, st, a) != cudaSuccess) return MLA_ERR_CUDA;
    mark_after(st);
    ++n;
  } else {
    if (D <= 192)
      launch_decode_simt<T, 3>(d, p, q, pool, num_pages, bt, max_pages, seq_lens, B, max_seq_len, o_lat, lse_out,
                               o_part, lse_part, st);
    else if (D <= 384)
      launch_decode_simt<T, 6>(d, p, q, pool, num_pages, bt, max_pages, seq_lens, B, max_seq_len, o_lat, lse_out,
                               o_part, lse_part, st);
    else
      launch_decode_simt<T, 9>(d, p, q, pool, num_pages, bt, max_pages, seq_lens, B, max_seq_len, o_lat, lse_out,
                               o_part, lse_part, st);
    ++n;
  }
  if (p.n_splits > 1) {
    if (launch_pdl(k_lse_merge_warp<T>, dim3((unsigned)((bh + 7) / 8)), dim3(256), 0, st,
                   static_cast<const float*>(o_part), static_cast<const float*>(lse_part), p.n_splits, (int)d->d_c,
                   (long)bh, static_cast<T*>(o_lat), lse_out) != cudaSuccess)
      return MLA_ERR_CUDA;
    ++n;
  }
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// New tokens per group of attention launches in mla_prefill_attention: bounds its workspace
// (per-token items and split-KV partials) while leaving thousands of attention tiles per launch.
constexpr int kPrefillGroup = 1024;

// Tokens per launch group: at most kPrefillGroup, and few enough that the group's page count
// (tokens x pages of the longest sequence) stays in int32.
inline int prefill_group(const mla_dims* d, int T, int max_seq_len) {
  long G = T < kPrefillGroup ? T : kPrefillGroup;
  const long cap = (long)INT32_MAX / pages_of(d, max_seq_len);
  if (G > cap) G = cap;
  return G < 1 ? 1 : (int)G;
}

size_t ws_prefill(const mla_dims* d, int T, int max_seq_len) {
  if (T <= 0 || max_seq_len < 1 || max_seq_len > kMaxSeqLen) return 0;
  const int G = prefill_group(d, T, max_seq_len);
  const size_t item_pages = ((size_t)max_seq_len + d->page_size - 1) / d->page_size;
  size_t dec = ws_decode(d, G, max_seq_len);
  if (T % G != 0) {  // the last, smaller group may split sequences further
    const size_t last = ws_decode(d, T % G, max_seq_len);
    if (last > dec) dec = last;
  }
  return align256((size_t)G * item_pages * 4) + align256((size_t)G * 4) + dec;
}

template <typename T>
int prefill_impl(const mla_dims* d, const void* q, const void* pool, int32_t num_pages, const int32_t* bt,
                 int32_t num_seqs, int32_t max_pages, const int32_t* seq_idx, const int32_t* pos, int32_t T_,
                 int32_t max_seq_len, void* o_lat, float* lse_out, void* ws, cudaStream_t st) {
  const int G = prefill_group(d, T_, max_seq_len);
  const int item_pages = (int)(((long)max_seq_len + d->page_size - 1) / d->page_size);
  Carve c{static_cast<char*>(ws)};
  int* item_bt = c.take<int>((size_t)G * item_pages);
  int* item_len = c.take<int>((size_t)G);
  void* dec_ws = static_cast<char*>(ws) + c.off;
  const size_t q_row = (size_t)d->n_heads * (d->d_c + d->d_rope) * sizeof(T);
  const size_t o_row = (size_t)d->n_heads * d->d_c * sizeof(T);
  int32_t n = 0;
  // The groups reuse the item tables and the attention workspace. Each group's k_prefill_items
  // waits (griddep_wait) for the kernel before it, the previous group's last launch, which itself
  // waited for that group's attention kernel, the last reader of those buffers.
  for (int g0 = 0; g0 < T_; g0 += G) {
    const int g = T_ - g0 < G ? T_ - g0 : G;
    if (launch_pdl(k_prefill_items, dim3((g + 7) / 8), dim3(256), 0, st, seq_idx + g0, pos + g0, bt, (int)num_seqs,
                   (int)max_pages, (int)d->page_size, (int)max_seq_len, g, item_pages, item_bt,
                   item_len) != cudaSuccess)
      return MLA_ERR_CUDA;
    ++n;
    const int r = decode_impl<T>(d, static_cast<const char*>(q) + g0 * q_row, pool, num_pages, item_bt, item_pages,
                                 item_len, g, max_seq_len, static_cast<char*>(o_lat) + g0 * o_row,
                                 lse_out != nullptr ? lse_out + (size_t)g0 * d->n_heads : nullptr, dec_ws, st, n,
                                 false);
    if (r != MLA_OK) return r;
  }
  return finish_launches(MLA_CALL_PREFILL_ATTENTION, n);
}

template <typename T>
int out_impl(const mla_dims* d, const void* o_lat, const void* w_uv, const void* w_o, void* u, int32_t B, void* ws,
             cudaStream_t st) {
  int32_t n = 0;
  const int r = host::out_run<T>(d, o_lat, w_uv, w_o, u, B, ws, st, n);
  if (r != MLA_OK) return r;
  return finish_launches(MLA_CALL_OUT_PROJ, n);
}

}  // namespace

// ------------------------------------------------------------------ fused small-head layer step
bool layer_small_eligible(const mla_dims* d) {
  return decode_mma_eligible(d) && d->d_model % 8 == 0 && d->d_cq % 8 == 0 && (d->n_heads * d->d_head) % 8 == 0;
}

struct SmallLayout {
  DecodePlan p;
  size_t cq, qc, o, o_part, lse_part, bytes;
};
// Attention split over `ctas` CTAs of the fused kernel: about one (sequence, split) item per CTA,
// each a whole number of 64-token stages.
DecodePlan plan_small(int B, int max_seq_len, long ctas) {
  DecodePlan p;
  p.head_groups = 1;
  const long stages = ((long)max_seq_len + dmma::kStageTokens - 1) / dmma::kStageTokens;
  long s = std::max(1L, ctas / B);
  if (s > stages) s = stages;
  const long per = (stages + s - 1) / s;
  p.split_len = (int)(per * dmma::kStageTokens);
  p.n_splits = (int)(((long)max_seq_len + p.split_len - 1) / p.split_len);
  return p;
}
// ctas: the grid the call launches (the workspace query assumes the largest, 3 per SM)
SmallLayout small_layout(const mla_dims* d, int B, int max_seq_len, long ctas) {
  SmallLayout L;
  L.p = plan_small(B, max_seq_len, ctas);
  const size_t e = 2, nq = (size_t)d->n_heads * d->d_head, bh = (size_t)B * d->n_heads;
  L.cq = 0;
  L.qc = L.cq + align256((size_t)B * d->d_cq * e);
  L.o = L.qc + align256((size_t)B * nq * e);
  L.o_part = L.o + align256((size_t)B * nq * e);
  L.lse_part = L.o_part + (L.p.n_splits > 1 ? align256(bh * L.p.n_splits * d->d_c * 4) : 0);
  L.bytes = L.lse_part + (L.p.n_splits > 1 ? align256(bh * L.p.n_splits * 4) : 0);
  return L;
}
size_t ws_layer_small(const mla_dims* d, int B, int max_seq_len) {
  if (B <= 0 || max_seq_len < 1 || max_seq_len > kMaxSeqLen || !layer_small_eligible(d)) return 0;
  // the most splits any grid of the call gives: the smallest grid (one CTA per SM)
  size_t most = 0;
  for (int per_sm = 1; per_sm <= 3; ++per_sm)
    most = std::max(most, small_layout(d, B, max_seq_len, (long)per_sm * device_sm_count()).bytes);
  return most;
}

template <typename T>
int layer_small_impl(const mla_dims* d, const void* h, const void* w_dkv_kr, const void* w_dq, const void* w_uq_qr,
                     const void* w_uk, const void* w_uv, const void* w_o, void* pool, int32_t num_pages,
                     const int32_t* bt, int32_t max_pages, const int32_t* seq_lens, int32_t B, int32_t max_seq_len,
                     void* q_out, void* o_lat, float* lse_out, void* u, void* ws, cudaStream_t st) {
  const int D = d->d_c + d->d_rope;
  const size_t smem = dmma::smem_bytes(D);
  // resident CTAs per SM for this row width (the cooperative grid must fit at once), cached per
  // device and width (D / 16 <= kMaxKD)
  static std::atomic<int> blocks_per_sm[kMaxDevices][dmma::kMaxKD + 1];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
  int bps = blocks_per_sm[dev][D / 16].load(std::memory_order_acquire);
  if (bps == 0) {
    // the largest row the kernel takes, so that one setting serves every eligible shape
    if (cudaFuncSetAttribute(k_layer_small<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)dmma::smem_bytes(16 * dmma::kMaxKD)) != cudaSuccess)
      return MLA_ERR_CUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, k_layer_small<T>, 128, smem) != cudaSuccess || bps < 1)
      return MLA_ERR_CUDA;
    blocks_per_sm[dev][D / 16].store(bps, std::memory_order_release);
  }
  // As many CTAs as the largest phase has warp items for (two rows per warp, four warps per CTA),
  // at least one per SM and at most what fits at once: with little work (one sequence) fewer CTAs
  // make each grid-wide barrier cheaper.
  const long nq = (long)d->n_heads * d->d_head, half = d->d_rope / 2;
  const long warps = std::max({(long)B * (d->d_c + d->d_cq) / 2 + (long)B * half, (long)B * nq / 2 + (long)B * d->n_heads * half,
                               (long)B * d->d_model / 2});
  const int grid = (int)std::max<long>(device_sm_count(),
                                       std::min<long>((long)std::min(bps, 3) * device_sm_count(), (warps + 3) / 4));
  // attention items (sequence, split) for one round over the grid
  SmallLayout L = small_layout(d, B, max_seq_len, grid);
  char* w = static_cast<char*>(ws);
  SmallStepArgs a;
  a.B = B;
  a.h = h;
  a.w_dkv_kr = w_dkv_kr;
  a.w_dq = w_dq;
  a.w_uq_qr = w_uq_qr;
  a.w_uk = w_uk;
  a.w_uv = w_uv;
  a.w_o = w_o;
  a.d_model = d->d_model;
  a.n_h = d->n_heads;
  a.d_h = d->d_head;
  a.d_c = d->d_c;
  a.d_cq = d->d_cq;
  a.d_rope = d->d_rope;
  a.rope_base = d->rope_base;
  a.rope_table = d->rope_inv_freq;
  a.pool = pool;
  a.cq = w + L.cq;
  a.qc = w + L.qc;
  a.q = q_out;
  a.o = w + L.o;
  a.u = u;
  const float scale_log2 = (float)(1.0 / std::sqrt((double)(d->d_head + d->d_rope)) * 1.4426950408889634);
  a.attn = MmaAttnArgs{q_out, pool, bt, (int)max_pages, seq_lens, (int)max_seq_len, (int)num_pages, (int)d->n_heads,
                       (int)d->d_c, D, (int)d->page_size, scale_log2, L.p.split_len, L.p.n_splits, o_lat, lse_out,
                       L.p.n_splits > 1 ? reinterpret_cast<float*>(w + L.o_part) : nullptr,
                       L.p.n_splits > 1 ? reinterpret_cast<float*>(w + L.lse_part) : nullptr};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k_layer_small<T>, a) != cudaSuccess) return MLA_ERR_CUDA;
  return finish_launches(MLA_CALL_LAYER_STEP_SMALL, 1);
}

extern "C" {

int mla_check_dims(const mla_dims* dims) { return check_dims_impl(dims); }

int32_t mla_cache_elems_per_token(const mla_dims* dims) {
  const int r = check_dims_impl(dims);
  if (r != MLA_OK) return r;
  return dims->d_c + dims->d_rope;
}

size_t mla_workspace_size(const mla_dims* dims, int32_t call, int32_t B, int32_t max_seq_len) {
  if (check_dims_impl(dims) != MLA_OK || B < 0) return 0;
  switch (call) {
    case MLA_CALL_APPEND_KV: return ws_append(dims, B);
    case MLA_CALL_ABSORB_QUERY: return ws_absorb(dims, B);
    case MLA_CALL_DECODE_ATTENTION: return ws_decode(dims, B, max_seq_len);
    case MLA_CALL_OUT_PROJ: return ws_out(dims, B);
    case MLA_CALL_PREFILL_ATTENTION: return ws_prefill(dims, B, max_seq_len);
    case MLA_CALL_LAYER_STEP_SMALL: return ws_layer_small(dims, B, max_seq_len);
    case MLA_CALL_APPEND_KV_FP8: return fp8_dims(dims) == MLA_OK ? ws_append_fp8(dims, B) : 0;
    case MLA_CALL_DECODE_ATTENTION_FP8:
      return fp8_dims(dims) == MLA_OK && B > 0 && max_seq_len >= 1 && max_seq_len <= kMaxSeqLen
                 ? ws_decode_tc(dims, B)
                 : 0;
    default: return 0;
  }
}

int mla_append_kv(const mla_dims* dims, const void* h, const void* w_dkv_kr, const int32_t* seq_idx,
                  const int32_t* pos, const int32_t* block_table, int32_t num_seqs, int32_t max_pages, void* pool,
                  int32_t num_pages, int32_t T, void* ws, size_t ws_bytes, mla_stream_t stream) {
  NvtxRange nvtx_range("mla_append_kv");
  int r = check_dims_impl(dims);
  if (r != MLA_OK) return r;
  if (T < 0 || num_seqs <= 0 || max_pages <= 0 || num_pages <= 0) return MLA_ERR_INVALID_ARG;
  if (T == 0) {
    t_launches[MLA_CALL_APPEND_KV] = 0;
    return MLA_OK;
  }
  if (!h || !w_dkv_kr || !seq_idx || !pos || !block_table || !pool) return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(w_dkv_kr) || !aligned16(pool) || !aligned16(ws)) return MLA_ERR_ALIGNMENT;
  if (ws_bytes < ws_append(dims, T)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (!ws) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims->dtype == MLA_BF16)
    return append_impl<__nv_bfloat16>(dims, h, w_dkv_kr, seq_idx, pos, block_table, num_seqs, max_pages, pool,
                                      num_pages, T, ws, st);
  return append_impl<__half>(dims, h, w_dkv_kr, seq_idx, pos, block_table, num_seqs, max_pages, pool, num_pages, T,
                             ws, st);
}

int mla_absorb_query(const mla_dims* dims, const void* h, const void* w_dq, const void* w_uq_qr, const void* w_uk,
                     const int32_t* pos, void* q_out, int32_t B, void* ws, size_t ws_bytes, mla_stream_t stream) {
  NvtxRange nvtx_range("mla_absorb_query");
  int r = check_dims_impl(dims);
  if (r != MLA_OK) return r;
  if (B < 0 || B > 65535) return MLA_ERR_INVALID_ARG;
  if (B == 0) {
    t_launches[MLA_CALL_ABSORB_QUERY] = 0;
    return MLA_OK;
  }
  if (!h || !w_dq || !w_uq_qr || !w_uk || !pos || !q_out || !ws) return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(w_dq) || !aligned16(w_uq_qr) || !aligned16(w_uk) || !aligned16(q_out) ||
      !aligned16(ws))
    return MLA_ERR_ALIGNMENT;
  if (ws_bytes < ws_absorb(dims, B)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims->dtype == MLA_BF16)
    return absorb_impl<__nv_bfloat16>(dims, h, w_dq, w_uq_qr, w_uk, pos, q_out, B, ws, st);
  return absorb_impl<__half>(dims, h, w_dq, w_uq_qr, w_uk, pos, q_out, B, ws, st);
}

int mla_decode_attention(const mla_dims* dims, const void* q, const void* pool, int32_t num_pages,
                         const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens, int32_t B,
                         int32_t max_seq_len, void* o_lat, float* lse_out, void* ws, size_t ws_bytes,
                         mla_stream_t stream) {
  NvtxRange nvtx_range("mla_decode_attention");
  int r = check_dims_impl(dims);
  if (r != MLA_OK) return r;
  if (B < 0 || B > 65535 || max_seq_len < 1 || max_seq_len > kMaxSeqLen || max_pages <= 0 || num_pages <= 0)
    return MLA_ERR_INVALID_ARG;
  if ((long)max_pages * dims->page_size < (long)max_seq_len) return MLA_ERR_INVALID_ARG;
  if (!page_total_fits(dims, B, max_seq_len)) return MLA_ERR_INVALID_ARG;
  if (B == 0) {
    t_launches[MLA_CALL_DECODE_ATTENTION] = 0;
    return MLA_OK;
  }
  if (!q || !pool || !block_table || !seq_lens || !o_lat) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(pool) || !aligned16(o_lat) || !aligned16(ws) || !aligned16(lse_out))
    return MLA_ERR_ALIGNMENT;
  const size_t need = ws_decode(dims, B, max_seq_len);
  if (ws_bytes < need) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (need > 0 && !ws) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t n = 0;
  r = dims->dtype == MLA_BF16
          ? decode_impl<__nv_bfloat16>(dims, q, pool, num_pages, block_table, max_pages, seq_lens, B, max_seq_len,
                                       o_lat, lse_out, ws, st, n, true)
          : decode_impl<__half>(dims, q, pool, num_pages, block_table, max_pages, seq_lens, B, max_seq_len, o_lat,
                                lse_out, ws, st, n, true);
  if (r != MLA_OK) return r;
  return finish_launches(MLA_CALL_DECODE_ATTENTION, n);
}

int64_t mla_fp8_page_bytes(const mla_dims* dims) {
  const int r = check_dims_impl(dims);
  if (r != MLA_OK) return r;
  return fp8::page_bytes(dims->page_size, dims->d_c + dims->d_rope);
}

int mla_fp8_supported(const mla_dims* dims) {
  if (dims == nullptr) return MLA_ERR_INVALID_ARG;
  const int r = fp8_dims(dims);
  return r == MLA_ERR_INVALID_ARG ? r : (r == MLA_OK ? MLA_OK : MLA_ERR_UNSUPPORTED_DIMS);
}

int mla_append_kv_fp8(const mla_dims* dims, const void* h, const void* w_dkv_kr, const int32_t* seq_idx,
                      const int32_t* pos, const int32_t* block_table, int32_t num_seqs, int32_t max_pages, void* pool,
                      int32_t num_pages, int32_t T, void* ws, size_t ws_bytes, mla_stream_t stream) {
  NvtxRange nvtx_range("mla_append_kv_fp8");
  int r = fp8_dims(dims);
  if (r != MLA_OK) return r;
  if (T < 0 || num_seqs <= 0 || max_pages <= 0 || num_pages <= 0) return MLA_ERR_INVALID_ARG;
  if (T == 0) {
    t_launches[MLA_CALL_APPEND_KV_FP8] = 0;
    return MLA_OK;
  }
  if (!h || !w_dkv_kr || !seq_idx || !pos || !block_table || !pool || !ws) return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(w_dkv_kr) || !aligned16(pool) || !aligned16(ws)) return MLA_ERR_ALIGNMENT;
  if (ws_bytes < ws_append_fp8(dims, T)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t n = 0;
  r = dims->dtype == MLA_BF16 ? host::append_fp8_run<__nv_bfloat16>(dims, h, w_dkv_kr, seq_idx, pos, block_table,
                                                                      num_seqs, max_pages, pool, num_pages, T, ws, st, n)
                              : host::append_fp8_run<__half>(dims, h, w_dkv_kr, seq_idx, pos, block_table, num_seqs,
                                                             max_pages, pool, num_pages, T, ws, st, n);
  if (r != MLA_OK) return r;
  return finish_launches(MLA_CALL_APPEND_KV_FP8, n);
}

int mla_decode_attention_fp8(const mla_dims* dims, const void* q, const void* pool, int32_t num_pages,
                             const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens, int32_t B,
                             int32_t max_seq_len, void* o_lat, float* lse_out, void* ws, size_t ws_bytes,
                             mla_stream_t stream) {
  NvtxRange nvtx_range("mla_decode_attention_fp8");
  int r = fp8_dims(dims);
  if (r != MLA_OK) return r;
  if (B < 0 || B > 65535 || max_seq_len < 1 || max_seq_len > kMaxSeqLen || max_pages <= 0 || num_pages <= 0)
    return MLA_ERR_INVALID_ARG;
  if ((long)max_pages * dims->page_size < (long)max_seq_len) return MLA_ERR_INVALID_ARG;
  if (!page_total_fits(dims, B, max_seq_len)) return MLA_ERR_INVALID_ARG;
  if (B == 0) {
    t_launches[MLA_CALL_DECODE_ATTENTION_FP8] = 0;
    return MLA_OK;
  }
  if (!q || !pool || !block_table || !seq_lens || !o_lat || !ws) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(pool) || !aligned16(o_lat) || !aligned16(ws) || !aligned16(lse_out))
    return MLA_ERR_ALIGNMENT;
  if (ws_bytes < ws_decode_tc(dims, B)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t n = 0;
  r = dims->dtype == MLA_BF16
          ? decode_tc_impl<__nv_bfloat16, true>(dims, q, pool, num_pages, block_table, max_pages, seq_lens, B,
                                                max_seq_len, o_lat, lse_out, ws, st, n, true)
          : decode_tc_impl<__half, true>(dims, q, pool, num_pages, block_table, max_pages, seq_lens, B, max_seq_len,
                                         o_lat, lse_out, ws, st, n, true);
  if (r != MLA_OK) return r;
  return finish_launches(MLA_CALL_DECODE_ATTENTION_FP8, n);
}

int mla_prefill_attention(const mla_dims* dims, const void* q, const void* pool, int32_t num_pages,
                          const int32_t* block_table, int32_t num_seqs, int32_t max_pages, const int32_t* seq_idx,
                          const int32_t* pos, int32_t T, int32_t max_seq_len, void* o_lat, float* lse_out, void* ws,
                          size_t ws_bytes, mla_stream_t stream) {
  NvtxRange nvtx_range("mla_prefill_attention");
  const int r = check_dims_impl(dims);
  if (r != MLA_OK) return r;
  if (T < 0 || max_seq_len < 1 || max_seq_len > kMaxSeqLen || num_seqs <= 0 || max_pages <= 0 || num_pages <= 0)
    return MLA_ERR_INVALID_ARG;
  if ((long)max_pages * dims->page_size < (long)max_seq_len) return MLA_ERR_INVALID_ARG;
  if (T == 0) {
    t_launches[MLA_CALL_PREFILL_ATTENTION] = 0;
    return MLA_OK;
  }
  if (!q || !pool || !block_table || !seq_idx || !pos || !o_lat || !ws) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(pool) || !aligned16(o_lat) || !aligned16(ws) || !aligned16(lse_out))
    return MLA_ERR_ALIGNMENT;
  if (ws_bytes < ws_prefill(dims, T, max_seq_len)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims->dtype == MLA_BF16)
    return prefill_impl<__nv_bfloat16>(dims, q, pool, num_pages, block_table, num_seqs, max_pages, seq_idx, pos, T,
                                       max_seq_len, o_lat, lse_out, ws, st);
  return prefill_impl<__half>(dims, q, pool, num_pages, block_table, num_seqs, max_pages, seq_idx, pos, T,
                              max_seq_len, o_lat, lse_out, ws, st);
}

int mla_out_proj(const mla_dims* dims, const void* o_lat, const void* w_uv, const void* w_o, void* u, int32_t B,
                 void* ws, size_t ws_bytes, mla_stream_t stream) {
  NvtxRange nvtx_range("mla_out_proj");
  int r = check_dims_impl(dims);
  if (r != MLA_OK) return r;
  if (B < 0 || B > 65535) return MLA_ERR_INVALID_ARG;
  if (B == 0) {
    t_launches[MLA_CALL_OUT_PROJ] = 0;
    return MLA_OK;
  }
  if (!o_lat || !w_uv || !w_o || !u || !ws) return MLA_ERR_INVALID_ARG;
  if (!aligned16(o_lat) || !aligned16(w_uv) || !aligned16(w_o) || !aligned16(u) || !aligned16(ws))
    return MLA_ERR_ALIGNMENT;
  if (ws_bytes < ws_out(dims, B)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims->dtype == MLA_BF16) return out_impl<__nv_bfloat16>(dims, o_lat, w_uv, w_o, u, B, ws, st);
  return out_impl<__half>(dims, o_lat, w_uv, w_o, u, B, ws, st);
}

int mla_layer_step_small_supported(const mla_dims* dims) {
  const int r = check_dims_impl(dims);
  if (r != MLA_OK) return r;
  return layer_small_eligible(dims) ? MLA_OK : MLA_ERR_UNSUPPORTED_DIMS;
}

int mla_layer_step_small(const mla_dims* dims, const void* h, const void* w_dkv_kr, const void* w_dq,
                         const void* w_uq_qr, const void* w_uk, const void* w_uv, const void* w_o, void* pool,
                         int32_t num_pages, const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens,
                         int32_t B, int32_t max_seq_len, void* q_out, void* o_lat, float* lse_out, void* u, void* ws,
                         size_t ws_bytes, mla_stream_t stream) {
  NvtxRange nvtx_range("mla_layer_step_small");
  int r = mla_layer_step_small_supported(dims);
  if (r != MLA_OK) return r;
  if (B < 0 || B > 65535 || num_pages < 0 || max_pages < 1 || max_seq_len < 1 || max_seq_len > kMaxSeqLen)
    return MLA_ERR_INVALID_ARG;
  if (B == 0) {
    t_launches[MLA_CALL_LAYER_STEP_SMALL] = 0;
    return MLA_OK;
  }
  if (!page_total_fits(dims, B, max_seq_len)) return MLA_ERR_INVALID_ARG;
  if (!h || !w_dkv_kr || !w_dq || !w_uq_qr || !w_uk || !w_uv || !w_o || !pool || !block_table || !seq_lens ||
      !q_out || !o_lat || !u || !ws)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(w_dkv_kr) || !aligned16(w_dq) || !aligned16(w_uq_qr) || !aligned16(w_uk) ||
      !aligned16(w_uv) || !aligned16(w_o) || !aligned16(pool) || !aligned16(q_out) || !aligned16(o_lat) ||
      !aligned16(u) || !aligned16(ws))
    return MLA_ERR_ALIGNMENT;
  if (ws_bytes < ws_layer_small(dims, B, max_seq_len)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims->dtype == MLA_BF16)
    return layer_small_impl<__nv_bfloat16>(dims, h, w_dkv_kr, w_dq, w_uq_qr, w_uk, w_uv, w_o, pool, num_pages,
                                           block_table, max_pages, seq_lens, B, max_seq_len, q_out, o_lat, lse_out, u,
                                           ws, st);
  return layer_small_impl<__half>(dims, h, w_dkv_kr, w_dq, w_uq_qr, w_uk, w_uv, w_o, pool, num_pages, block_table,
                                  max_pages, seq_lens, B, max_seq_len, q_out, o_lat, lse_out, u, ws, st);
}

int mla_read_device_status(mla_stream_t stream, int32_t* status_out) {
  if (!status_out) return MLA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MLA_ERR_CUDA;
  int v = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&v, mla::g_status, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaMemcpyToSymbol(mla::g_status, &zero, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  *status_out = v;
  return MLA_OK;
}

const char* mla_error_string(int code) {
  switch (code) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED_DIMS: return "unsupported dims";
    case MLA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MLA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_TIMEOUT: return "device wait timed out";
    case MLA_ERR_BAD_PAGE: return "block-table entry out of range";
    case MLA_ERR_BAD_SEQ_LEN: return "sequence length out of range";
    default: return "unknown status";
  }
}

int32_t mla_last_launch_count(int32_t call) { return (call >= 0 && call < 8) ? t_launches[call] : -1; }

int mla_debug_gemm_plan(int32_t M, int32_t N, int32_t K, int32_t batch, int32_t fused_rope, int32_t d_rope,
                        int64_t* out) {
  if (M <= 0 || N <= 0 || K <= 0 || batch <= 0 || d_rope <= 0 || out == nullptr) return MLA_ERR_INVALID_ARG;
  const host::SkPlan g = host::plan_sk(M, N, K, batch, fused_rope != 0, d_rope);
  const int64_t v[11] = {g.bn, g.m_tiles, g.n_tiles, g.kb, g.tiles, g.G, g.stages, g.aligned ? 1 : 0,
                         g.split ? 1 : 0, (int64_t)g.smem, (int64_t)g.part_bytes};
  for (int i = 0; i < 11; ++i) out[i] = v[i];
  return MLA_OK;
}

int mla_debug_inject_missing_load(int32_t tile) {
#ifdef MLA_FAULT_INJECT
  if (tile < -1) return MLA_ERR_INVALID_ARG;
  return cudaMemcpyToSymbol(tc::g_inject_missing_tile, &tile, sizeof(int)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
#else
  (void)tile;
  return MLA_ERR_INVALID_ARG;
#endif
}

int mla_set_decode_timing_events(mla_event_t before, mla_event_t after) {
  if ((before == nullptr) != (after == nullptr)) return MLA_ERR_INVALID_ARG;
  t_ev_before = reinterpret_cast<cudaEvent_t>(before);
  t_ev_after = reinterpret_cast<cudaEvent_t>(after);
  return MLA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- allocation-free decode
// Scratch of mla_decode_attention_noalloc: one file-scope device array per GPU that loads this
// module. Host code must not pass the symbol itself to a kernel (on the host it names a
// host-side stand-in); its device address is looked up once per device and cached.
namespace {
constexpr size_t kStaticScratchBytes = size_t(64) << 20;
__device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

int static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return MLA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MLA_OK;
}
}  // namespace

extern "C" {

int mla_decode_attention_noalloc(const mla_dims* dims, const void* q, const void* pool, int32_t num_pages,
                                 const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens, int32_t B,
                                 int32_t max_seq_len, void* o_lat, float* lse_out, mla_stream_t stream) {
  NvtxRange nvtx_range("mla_decode_attention_noalloc");
  const int r = check_dims_impl(dims);
  if (r != MLA_OK) return r;
  // the argument checks of mla_decode_attention come first, so that the size below is defined
  if (B < 0 || B > 65535 || max_seq_len < 1 || max_seq_len > kMaxSeqLen || max_pages <= 0 || num_pages <= 0)
    return MLA_ERR_INVALID_ARG;
  if ((long)max_pages * dims->page_size < (long)max_seq_len || !page_total_fits(dims, B, max_seq_len))
    return MLA_ERR_INVALID_ARG;
  if (ws_decode(dims, B, max_seq_len) > kStaticScratchBytes) return MLA_ERR_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  const int s = static_scratch_address(&ws);
  if (s != MLA_OK) return s;
  return mla_decode_attention(dims, q, pool, num_pages, block_table, max_pages, seq_lens, B, max_seq_len, o_lat,
                              lse_out, ws, kStaticScratchBytes, stream);
}

}  // extern "C"
