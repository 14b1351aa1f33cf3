// Latent attention on tcgen05 for DeepSeek-V2 dims (65..128 heads, d_c = 512, d_h^R = 64,
// 64-token pages): "DeepSeek-V2 from Scratch" §4.4 with the absorbed steps 2-3 of §5.3.
//
// A work unit is a pair of CTAs (a 2-CTA cluster, one TPC) that shares every MMA (tcgen05
// cta_group::2, M = 128). CTA r owns heads [64r, 64r + 64): their absorbed queries Q_r
// [64 x 576] sit in its shared memory and their fp32 accumulator O_r [64 x 512] in its tensor
// memory (256 columns). Cached tokens go in 128-token tiles of two pages:
//   S = Q C^T      N = 128 tokens. CTA r supplies page r of the tile, all 576 columns; each CTA
//                  receives its 64 heads x 128 tokens (TMEM lanes 0-63: page 0, 64-127: page 1).
//   softmax        eight warps per CTA, four threads per head (two pages x two halves of 32
//                  tokens), online in fp32 with lazy rescaling (the reference max moves only
//                  when a score exceeds it by 2^8); P (bf16) is written to shared memory.
//   O += P C_lat   N = 256 latent columns per MMA, two of them: CTA r supplies columns
//                  [256j + 128r, 256j + 128r + 128) of all 128 tokens.
// So CTA r reads its own page whole and only the latent half it supplies of the other page:
// 1.44x the unique bytes per SM, against 2x for two SMs that each stream whole pages. The own
// page's latent half stays in shared memory from S to O, and the other page's half is loaded
// into the slots that the own page's remaining latent half held during S.
//
// Shared memory (per CTA): Q (9 chunks of 64 rows x 64 columns, 128-byte swizzle), P (two
// chunks: 64 heads x the tokens of page g), one rope slot (the own page's k^R columns, shared by
// consecutive tiles) and two sets of 8 latent chunks (tile i uses set i & 1). Latent chunks
// 2p and 2p+1 of a set form pair p = 2j + g: during S they hold the own page's columns
// [128p, 128p + 128); during O they hold the columns CTA r supplies for n-half j of page g.
//
// The pages of all sequences are split evenly over the pairs by 128-token tile; a sequence that
// spans pairs is merged afterwards by log-sum-exp in a fixed order.
#pragma once

#include <type_traits>

#include "fp8.cuh"
#include "tc_common.cuh"

namespace mla {
namespace tc {

#ifdef MLA_FAULT_INJECT
// Fault-injection test builds only: the global tile (index in the concatenated tile list of the
// call) whose first latent load the rank-0 loader of its pair leaves unissued, after arming its
// barrier; -1 = none. The S MMAs then wait for bytes that never come, and every role of the pair
// gives up after the build's short wait limit. Set with mla_debug_inject_missing_load.
__device__ int g_inject_missing_tile = -1;
#endif

namespace dec {
constexpr int kPage = 64;          // tokens per cache page
constexpr int kTile = 128;         // tokens per tile: page r of it is supplied by CTA r
constexpr int kDc = 512;           // latent width (O columns)
constexpr int kD = 576;            // cache row width
constexpr int kChunk = 8192;       // 64 rows x 64 columns of 16-bit elements
constexpr int kQOff = 0;           // Q: 9 chunks
constexpr int kPOff = 9 * kChunk;  // P: 2 chunks (tokens of page 0, of page 1)
constexpr int kRopeOff = kPOff + 2 * kChunk;  // own page's k^R columns
constexpr int kSetOff = kRopeOff + kChunk;    // two sets of 8 latent chunks
constexpr int kSetBytes = 8 * kChunk;
constexpr int kDataBytes = kSetOff + 2 * kSetBytes;  // 229376
constexpr float kLazy = 8.f;       // rescale threshold in log2 units
constexpr int kSoftWarps = 8;      // warps 0-7: softmax, rescale, epilogue
constexpr int kLoadWarp = 8;       // Q, rope and own-page latent loads
constexpr int kMmaWarp = 9;        // TMEM allocation; rank 0: S MMA issue
constexpr int kPairWarp = 10;      // the other page's latent half
constexpr int kOWarp = 11;        // rank 0: O MMA issue
constexpr int kThreads = 12 * 32;
// FP8 cache (see fp8.cuh): warps 12-15 turn the e4m3 boxes the two loaders bring into the chunks
// above, so that the MMAs are those of the 16-bit cache.
constexpr int kConvWarp0 = 12;
constexpr int kThreadsF8 = 16 * 32;
constexpr int kF8Page = kPage * (kD + 8);  // 64 rows of 576 bytes, then 64 (s_c, s_r) pairs
// TMEM columns
constexpr uint32_t kOCol = 0;      // O: n-half j in columns [128j, 128j + 128)
constexpr uint32_t kSCol = 256;    // S buffer b in columns [256 + 64b, 320 + 64b)
constexpr uint32_t kTmemCols = 512;

struct Ctrl {
  // Barriers arrived by both CTAs (two arrivals, plus the TMA bytes) live in rank 0, the issuer.
  uint64_t qk_full[2][2];  // set s, chunks [4h, 4h + 4) of the own page loaded in both CTAs
  uint64_t pv_full[2][4];  // set s, pair p ready for O in both CTAs
  uint64_t rope_full, q_full;
  uint64_t s_free[2];      // S buffer b read by all 16 softmax warps
  uint64_t p_full;         // P written (and O rescaled) by all 16 softmax warps
  uint64_t o_free;         // O read out by all 16 softmax warps (end of a sequence's item)
  // Barriers arrived by rank 0's MMA commits, multicast to both CTAs.
  uint64_t qk_done[2][4];  // set s, the S MMAs of pair p are complete (its slots may be reused)
  uint64_t set_free[2][2];  // the O MMAs of the tile using set s are done with its chunks [4h, 4h + 4)
  uint64_t rope_done, q_free;
  uint64_t s_full[2], p_free;
  // Local barriers.
  uint64_t mx_full[2][2];  // exchanges among the softmax warps: [head group][buffer xm, xh]
  uint64_t f8_qk[2][2], f8_pv[2][2], f8_rope;  // FP8: an e4m3 box has landed in this CTA
  uint64_t f8_q;                               // FP8: this CTA's queries have landed
  uint64_t drain;
  float xm[2][128];          // [column half][TMEM lane]: partial maxima or sums
  __nv_bfloat16 xh[2][128];  // the same, for maxima only (the second buffer)
  uint32_t tmem_slot;
  int abort_flag;
};
constexpr size_t kSmem = 1024 + kDataBytes + sizeof(Ctrl);
static_assert(kSmem <= 232448, "decode kernel shared memory");
}  // namespace dec

struct DecodeTcParams {
  const int* bt;          // [B, max_pages]
  int max_pages;
  const int* seq_lens;    // [B]
  const int* tile_prefix;  // [B + 1] 128-token tiles before each sequence (0 tiles for a rejected one)
  int B, n_h;
  float scale_log2;       // log2(e) / sqrt(d_h + d_h^R)
  void* o_lat;            // [B, n_h, 512] element type
  float* lse_out;         // [B, n_h] or null
  float* o_part;          // [B + C][n_h][512]
  float* lse_part;        // [B + C][n_h]
  const uint8_t* f8_pool;  // FP8 pages (their scales are read directly), or null
};

// Tensor maps of the attention kernel: the paged pool viewed as (64 columns, 64 rows of a page,
// pages, 9 column chunks) with boxes of 1, 2 and 4 chunks of one page; the queries viewed as
// (64 columns, B * n_h rows, 9 chunks) with a box of 9 chunks. (Prefetching pages into L2 ahead
// of their loads was measured slower: the prefetches take the same per-SM copy engine.)
//
// A page that holds nv < 64 tokens of its sequence (the last one) is loaded from row nv - 64:
// its tokens land in slot rows [64 - nv, 64) and the rows before are the tensor map's zero fill,
// so whatever the pool holds past the end of a sequence never reaches shared memory, and a page
// wholly past the end (nv = 0) loads as zeros. Softmax masks slot rows r < 64 - nv.
//
// FP8 pages are viewed as (576 byte columns, 64 rows, pages) with boxes of 256, 128 and 64 bytes
// x 64 rows, unswizzled, loaded the same way into the upper half of the chunks they become.
struct DecodeTcMaps {
  CUtensorMap page1, page2, page4, q9;
  CUtensorMap f8_256, f8_128, f8_64;
  CUtensorMap o_lat, o_part;  // outputs as (512 columns, n_h heads, rows), 64-byte x 32-head boxes
  CUtensorMap o_lat_h, o_part_h;  // the same with 32-byte x 32-head boxes, unswizzled
};

// Tiles [t0, t1) of sequence b handled by this pair (n_b = tiles of the sequence).
struct Item {
  int b, t0, t1, n_b;
};
struct ItemIter {
  long g, g_end;
  int b;
};

__device__ __forceinline__ ItemIter item_iter(const int* prefix, int B, int cluster, int nclusters) {
  ItemIter it;
  const long T = prefix[B];
  it.g = T * cluster / nclusters;
  it.g_end = T * (cluster + 1) / nclusters;
  int lo = 0, hi = B - 1;  // largest b with prefix[b] <= g
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= it.g) lo = mid; else hi = mid - 1;
  }
  it.b = lo;
  return it;
}
__device__ __forceinline__ bool next_item(ItemIter& it, const int* prefix, Item& out) {
  if (it.g >= it.g_end) return false;
  while (prefix[it.b + 1] <= it.g) ++it.b;
  const int base = prefix[it.b];
  out.b = it.b;
  out.n_b = prefix[it.b + 1] - base;
  out.t0 = (int)(it.g - base);
  out.t1 = (int)(min(it.g_end, (long)prefix[it.b + 1]) - base);
  it.g = base + out.t1;
  return true;
}

// The pair's tiles in order. Every role walks the same sequence with a cursor of its own:
// ti counts the pair's tiles, ii its items, t is the tile within sequence item.b (tokens
// [128t, 128t + 128)).
struct Cursor {
  ItemIter it;
  Item item;
  int t, ti, ii;
  bool valid;
  __device__ __forceinline__ void start(const int* prefix, int B, int cluster, int nclusters) {
    it = item_iter(prefix, B, cluster, nclusters);
    valid = next_item(it, prefix, item);
    t = valid ? item.t0 : 0;
    ti = 0;
    ii = 0;
  }
  __device__ __forceinline__ bool first() const { return t == item.t0; }
  __device__ __forceinline__ bool last() const { return t + 1 == item.t1; }
  __device__ __forceinline__ void advance(const int* prefix) {
    ++ti;
    if (++t == item.t1) {
      ++ii;
      valid = next_item(it, prefix, item);
      if (valid) t = item.t0;
    }
  }
};

// Most SM pairs one call spreads its tiles over (the merge kernel lists a sequence's pairs).
constexpr int kMaxDecodeClusters = 128;
// A sequence whose tiles fall to pairs c0 < c1 is merged by the merge kernel from the pairs'
// partials (fp32 o / l and lse in slot b + c). The planner gives each sequence
// c0 | c1 << 16 | all << 28 (all: every pair has tiles, so the slots are b + c0 .. b + c1),
// or -1 without tiles.

// Pair that owns global tile g when T tiles are split over C pairs as [T c / C, T (c+1) / C).
__device__ __forceinline__ int cluster_of(long g, long T, int C) { return (int)(((g + 1) * C - 1) / T); }

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t cluster_bar, int x,
                                                 int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(cluster_bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Box of page `page` of a paged map, rows from `row0` (negative: zero fill before the page's
// first row), chunks from `chunk`.
__device__ __forceinline__ void tma_load_page_pair(uint32_t dst, const CUtensorMap* map, uint32_t cluster_bar, int row0,
                                                   int page, int chunk) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(cluster_bar), "r"(0), "r"(row0), "r"(page), "r"(chunk)
      : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t a, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
// Named barrier with a vote: true on every thread iff `v` was true on all `count` threads.
__device__ __forceinline__ bool named_bar_and(uint32_t id, uint32_t count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

template <typename T, bool F8 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(F8 ? dec::kThreadsF8 : dec::kThreads, 1)
    k_decode_tc(const __grid_constant__ DecodeTcMaps maps, const DecodeTcParams p) {
  using namespace dec;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* data = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl* ctl = reinterpret_cast<Ctrl*>(data + kDataBytes);
  volatile int* abort_flag = &ctl->abort_flag;
  const uint32_t data_u32 = smem_u32(data);
  const uint32_t rank = cluster_ctarank();
  const int cluster = (int)cluster_id_x(), nclusters = (int)num_clusters_x();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };
  auto lead = [&](uint64_t& b) { return mapa(smem_u32(&b), 0u); };  // the barrier in rank 0
  constexpr bool kBf16 = IsBf16<T>::value;
  // With the FP8 cache the products run in fp16: a cached value is then one hardware conversion
  // and one fp16 multiply by its scale; the queries are converted once per sequence and P is fp16.
  constexpr bool kMmaBf16 = kBf16 && !F8;
  using PT = std::conditional_t<F8, __half, T>;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      for (int h = 0; h < 2; ++h) mbar_init(bar(ctl->qk_full[s][h]), 2);
      for (int q = 0; q < 4; ++q) {
        mbar_init(bar(ctl->pv_full[s][q]), 2);
        mbar_init(bar(ctl->qk_done[s][q]), 1);
      }
      mbar_init(bar(ctl->s_free[s]), 2 * kSoftWarps);
      mbar_init(bar(ctl->set_free[s][0]), 1);
      mbar_init(bar(ctl->set_free[s][1]), 1);
      mbar_init(bar(ctl->s_full[s]), 1);
    }
    mbar_init(bar(ctl->rope_full), 2);
    mbar_init(bar(ctl->q_full), 2);
    mbar_init(bar(ctl->p_full), 2 * kSoftWarps);
    mbar_init(bar(ctl->o_free), 2 * kSoftWarps);
    mbar_init(bar(ctl->rope_done), 1);
    mbar_init(bar(ctl->q_free), 1);
    mbar_init(bar(ctl->p_free), 1);
    for (int g2 = 0; g2 < 2; ++g2)
      for (int b2 = 0; b2 < 2; ++b2) mbar_init(bar(ctl->mx_full[g2][b2]), kSoftWarps / 2);
    mbar_init(bar(ctl->drain), 2);
    for (int s = 0; s < 2; ++s)
      for (int h = 0; h < 2; ++h) {
        mbar_init(bar(ctl->f8_qk[s][h]), 1);
        mbar_init(bar(ctl->f8_pv[s][h]), 1);
      }
    mbar_init(bar(ctl->f8_rope), 1);
    mbar_init(bar(ctl->f8_q), 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc2(smem_u32(&ctl->tmem_slot), kTmemCols);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_arrive();  // barriers of both CTAs are initialised before any remote arrive
  cluster_wait();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_slot;
  if (threadIdx.x == 0) griddep_launch();
  griddep_wait();  // the plan, the query and the cache come from earlier kernels
  const int* prefix = p.tile_prefix;
  const bool has_work = [&] {
    const long T_ = prefix[p.B];
    return T_ * (cluster + 1) / nclusters > T_ * cluster / nclusters;
  }();
  const uint32_t peer_abort = mapa(smem_u32(&ctl->abort_flag), rank ^ 1u);
  // A wait that gives up also releases the peer CTA's waiters. The warp-uniform variant is for
  // warps whose lanes then run warp-collective instructions: a give-up seen by any lane is taken
  // by the whole warp.
  auto wait = [&](uint64_t& b, uint32_t parity) {
    if (mbar_wait(bar(b), parity, abort_flag)) return true;
    st_cluster_u32(peer_abort, 1u);
    return false;
  };
  auto wwait = [&](uint64_t& b, uint32_t parity) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar(b), parity, abort_flag));
    if (!ok && lane == 0) st_cluster_u32(peer_abort, 1u);
    return ok;
  };
  const uint32_t set_u32 = data_u32 + kSetOff;

  if (has_work) {
    if (warp == kLoadWarp) {
      // ---------------------------------------------------------------- Q, rope and own-page loads
      if (lane == 0) {
        if constexpr (F8) {  // the maps of the other cache type are left zero
          tma_prefetch_map(&maps.f8_256);
          tma_prefetch_map(&maps.f8_128);
          tma_prefetch_map(&maps.f8_64);
        } else {
          tma_prefetch_map(&maps.page1);
          tma_prefetch_map(&maps.page2);
          tma_prefetch_map(&maps.page4);
        }
        tma_prefetch_map(&maps.q9);
        Cursor c;
        c.start(prefix, p.B, cluster, nclusters);
        int L = 0;
        while (c.valid) {
          const int s = c.ti & 1, b = c.item.b, t = c.t;
          // global reads first: their latency overlaps the waits below
          if (c.first()) L = p.seq_lens[b];
          const int* btb = p.bt + (long)b * p.max_pages;
          const int page_idx = 2 * t + (int)rank;
          const int nv = min(kPage, max(0, L - kPage * page_idx));  // tokens in page r of the tile
          const int page = nv > 0 ? btb[page_idx] : 0;
          if (c.first()) {  // this CTA's 64 heads of the sequence's queries, after the last S MMA of the item before
            if (!wait(ctl->q_free, (c.ii & 1) ^ 1)) break;
            if constexpr (F8) {  // the converting warps turn them into fp16 and publish them
              mbar_arrive_expect_tx(bar(ctl->f8_q), 9 * kChunk);
              tma_load_3d(data_u32 + kQOff, &maps.q9, bar(ctl->f8_q), 0, b * p.n_h + 64 * (int)rank, 0);
            } else {
              mbar_arrive_expect_tx_cl(lead(ctl->q_full), 9 * kChunk);
              tma_load_3d_pair(data_u32 + kQOff, &maps.q9, lead(ctl->q_full), 0, b * p.n_h + 64 * (int)rank, 0);
            }
          }
          if (!wait(ctl->rope_done, (c.ti & 1) ^ 1)) break;
          if constexpr (F8) {
            mbar_arrive_expect_tx(bar(ctl->f8_rope), kPage * 64);
            tma_load_3d(data_u32 + kRopeOff + kChunk / 2, &maps.f8_64, bar(ctl->f8_rope), kDc, nv - kPage, page);
          } else {
            mbar_arrive_expect_tx_cl(lead(ctl->rope_full), kChunk);
            tma_load_page_pair(data_u32 + kRopeOff, &maps.page1, lead(ctl->rope_full), nv - kPage, page, 8);
          }
          bool ok = true;
          for (int h = 0; h < 2; ++h) {
            // the O MMAs of tile ti - 2 are done with chunks [4h, 4h + 4) of set s
            if (!wait(ctl->set_free[s][h], ((c.ti >> 1) & 1) ^ 1)) {
              ok = false;
              break;
            }
            if constexpr (F8) {
              mbar_arrive_expect_tx(bar(ctl->f8_qk[s][h]), kPage * 256);
              tma_load_3d(set_u32 + s * kSetBytes + 4 * h * kChunk + 2 * kChunk, &maps.f8_256, bar(ctl->f8_qk[s][h]),
                          256 * h, nv - kPage, page);
              continue;
            }
#ifdef MLA_FAULT_INJECT
            if (h == 0 && rank == 0 && prefix[b] + t == g_inject_missing_tile) {
              mbar_arrive_expect_tx_cl(lead(ctl->qk_full[s][h]), 4 * kChunk);
              continue;
            }
#endif
            mbar_arrive_expect_tx_cl(lead(ctl->qk_full[s][h]), 4 * kChunk);
            tma_load_page_pair(set_u32 + s * kSetBytes + 4 * h * kChunk, &maps.page4, lead(ctl->qk_full[s][h]),
                               nv - kPage, page, 4 * h);
          }
          if (!ok) break;
          c.advance(prefix);
        }
      }
      __syncwarp();
    } else if (warp == kPairWarp) {
      // ---------------------------------------------------------------- the other page's latent half
      // Pair p = 2j + g of set s holds, for O, the columns this CTA supplies for n-half j of page
      // g. Page g = r is already there (loaded for S); page 1 - r is loaded once the S MMAs are
      // done with the own page's columns in those slots (a tail page with its zero-filled rows).
      if (lane == 0) {
        Cursor c;
        c.start(prefix, p.B, cluster, nclusters);
        int L = 0;
        const int g = 1 - (int)rank;
        while (c.valid) {
          const int s = c.ti & 1, b = c.item.b, t = c.t;
          if (c.first()) L = p.seq_lens[b];
          const uint32_t ph = (c.ti >> 1) & 1;
          const int nv = min(kPage, max(0, L - kTile * t - kPage * g));  // tokens in page g of the tile
          const int page = nv > 0 ? p.bt[(long)b * p.max_pages + 2 * t + g] : 0;  // read ahead of the waits
          // the O MMAs of tile ti - 2 are complete, so every barrier of set s is in this tile's phase
          if (!wait(ctl->set_free[s][1], ph ^ 1)) break;
          mbar_arrive_cl(lead(ctl->pv_full[s][(int)rank]));      // j = 0, g = r
          mbar_arrive_cl(lead(ctl->pv_full[s][2 + (int)rank]));  // j = 1, g = r
          bool ok = true;
          for (int j = 0; j < 2; ++j) {
            const int pr = 2 * j + g;
            if (!wait(ctl->qk_done[s][pr], ph)) {
              ok = false;
              break;
            }
            if constexpr (F8) {
              mbar_arrive_expect_tx(bar(ctl->f8_pv[s][j]), kPage * 128);
              tma_load_3d(set_u32 + s * kSetBytes + 2 * pr * kChunk + kChunk, &maps.f8_128, bar(ctl->f8_pv[s][j]),
                          256 * j + 128 * (int)rank, nv - kPage, page);
            } else {
              mbar_arrive_expect_tx_cl(lead(ctl->pv_full[s][pr]), 2 * kChunk);
              tma_load_page_pair(set_u32 + s * kSetBytes + 2 * pr * kChunk, &maps.page2, lead(ctl->pv_full[s][pr]),
                                 nv - kPage, page, 4 * j + 2 * (int)rank);
            }
          }
          if (!ok) break;
          c.advance(prefix);
        }
      }
      __syncwarp();
    } else if (warp == kMmaWarp || warp == kOWarp) {
      // ---------------------------------------------------------------- MMA issue (rank 0)
      // Two issuing threads, one per stream of MMAs: warp kMmaWarp issues S(i) for the tiles in
      // order (the rope chunk and latent chunks 0-3 once the first box lands, chunks 4-7 once the
      // second does), warp kOWarp issues O(i) once P(i) is written and each pair's chunks are in
      // place. The two streams touch disjoint tensor memory (S buffers, O) and are ordered through
      // the softmax barriers, so neither waits behind the other's inputs. Each thread's commits
      // track its own MMAs. A single thread runs dependent instructions and branches at a few
      // cycles each, so each step is straight-line code: a wait, MMAs with compile-time operand
      // offsets, commits. A descriptor is a fixed high word and a low word stepped by 32-bit adds
      // (16-byte units: a K-step of 16 elements is +2 along a K-major row and +128, i.e. 16 rows,
      // down an MN-major operand).
      if (rank == 0 && lane == 0) {
        constexpr uint32_t idesc_qk = idesc_f16(128, kTile, kMmaBf16, false, false);
        constexpr uint32_t idesc_pv = idesc_f16(128, 256, kMmaBf16, false, true);
        constexpr uint32_t hi = desc_sw128_hi(1024);
        constexpr uint32_t kChunkD = kChunk >> 4, kSetD = kSetBytes >> 4;
        const uint32_t b_qk_full = bar(ctl->qk_full[0][0]), b_pv_full = bar(ctl->pv_full[0][0]);
        const uint32_t b_qk_done = bar(ctl->qk_done[0][0]), b_set_free = bar(ctl->set_free[0][0]);
        const uint32_t b_s_free = bar(ctl->s_free[0]), b_s_full = bar(ctl->s_full[0]);
        auto wt = [&](uint32_t b, uint32_t parity) {
          if (mbar_wait(b, parity, abort_flag)) return true;
          st_cluster_u32(peer_abort, 1u);
          return false;
        };
        Cursor c;
        c.start(prefix, p.B, cluster, nclusters);
        if (warp == kMmaWarp) {
          // S(i) = Q C^T into S buffer i & 1
          const uint32_t q_lo = desc_sw128_lo(data_u32 + kQOff, 16);
          const uint32_t rope_lo = desc_sw128_lo(data_u32 + kRopeOff, 16);
          const uint32_t k_lo = desc_sw128_lo(set_u32, 16);  // latent chunks as K-major B
          for (; c.valid; c.advance(prefix)) {
            const int ti = c.ti, s = ti & 1;
            const uint32_t ph = (ti >> 1) & 1;
            const uint32_t d = tmem + kSCol + 64 * s;
            const uint32_t kb = k_lo + s * kSetD;
            if (!wt(b_s_free + 8 * s, ph ^ 1)) break;  // softmax has read S(i - 2)
            if (c.first() && !wt(bar(ctl->q_full), c.ii & 1)) break;
            if (!wt(bar(ctl->rope_full), ti & 1)) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma2_ss_lohi(d, q_lo + 8 * kChunkD + 2 * ks, rope_lo + 2 * ks, hi, idesc_qk, ks != 0);
            mma_commit2(bar(ctl->rope_done), 3);
            bool ok = true;
#pragma unroll
            for (int grp = 0; grp < 2; ++grp) {
              if (!wt(b_qk_full + 8 * (2 * s + grp), ph)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int k4 = 0; k4 < 4; ++k4) {
                const int kc = 4 * grp + k4;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                  mma2_ss_lohi(d, q_lo + kc * kChunkD + 2 * ks, kb + kc * kChunkD + 2 * ks, hi, idesc_qk, 1);
                if (k4 & 1) mma_commit2(b_qk_done + 8 * (4 * s + (kc >> 1)), 3);
              }
            }
            if (!ok) break;
            mma_commit2(b_s_full + 8 * s, 3);
            if (c.last()) mma_commit2(bar(ctl->q_free), 3);
          }
        } else {
          // O += P C_lat, pairs (g, j) = (0,0), (1,0), (0,1), (1,1); chunks 0-3 of the set are
          // released after the first two
          const uint32_t p_lo = desc_sw128_lo(data_u32 + kPOff, 16);
          const uint32_t v_lo = desc_sw128_lo(set_u32, kChunk);  // chunk pairs as MN-major B
          for (; c.valid; c.advance(prefix)) {
            const int ti = c.ti, s = ti & 1;
            const uint32_t ph = (ti >> 1) & 1;
            const bool first = c.first();
            const uint32_t vb = v_lo + s * kSetD;
            if (!wt(bar(ctl->p_full), ti & 1)) break;  // P written, O rescaled
            if (first && !wt(bar(ctl->o_free), (c.ii & 1) ^ 1)) break;  // O of the item before read out
            bool ok = true;
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
              const int g = gq & 1, jh = gq >> 1, pr = 2 * jh + g;
              if (!wt(b_pv_full + 8 * (4 * s + pr), ph)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t d = tmem + kOCol + 128 * jh;
              mma2_ss_lohi(d, p_lo + g * kChunkD, vb + 2 * pr * kChunkD, hi, idesc_pv, g != 0 || !first);
#pragma unroll
              for (int ks = 1; ks < 4; ++ks)
                mma2_ss_lohi(d, p_lo + g * kChunkD + 2 * ks, vb + 2 * pr * kChunkD + 128 * ks, hi, idesc_pv, 1);
              if (gq == 1) mma_commit2(b_set_free + 8 * (2 * s), 3);
            }
            if (!ok) break;
            mma_commit2(bar(ctl->p_free), 3);
            mma_commit2(b_set_free + 8 * (2 * s + 1), 3);
          }
        }
        mma_commit2(bar(ctl->drain), 1);  // once all of this thread's MMAs are complete
      }
      __syncwarp();
    } else if (F8 && warp >= kConvWarp0) {
      // ---------------------------------------------------------------- FP8: e4m3 boxes -> fp16 chunks
      // Each box (64 slot rows, unswizzled, rows of 256, 128 or 64 bytes) lies in the upper half
      // of the chunks it becomes: a latent group (4 chunks), a pair (2 chunks), the rope chunk.
      // The four warps convert it in place, each value times its token's scale in float32: first
      // the units whose output lies below the box, then, once every thread holds its share of the
      // rest in registers (a named barrier), the units whose output overwrites it. Thread ct takes
      // slot row ct / 2 and half ct % 2 of its units, in an order rotated by the row so that a
      // warp's 16-byte reads spread over the banks. Tiles go in order, each tile's own page (rope,
      // latent groups) and then its pairs: the next tile's own page was loaded while this tile's S
      // ran, so it is ready by the time the pairs are done.
      const int ct = (int)threadIdx.x - 32 * kConvWarp0;
      const int row = ct >> 1, half = ct & 1;
      const uint32_t sw = (uint32_t)(row & 7);
      const float2* const scale_base =
          reinterpret_cast<const float2*>(p.f8_pool + (size_t)kPage * kD);  // page 0's scales
      // (s_c, s_r) of slot row `row` of a page with nv tokens (rows before 64 - nv are zero fill)
      auto scales = [&](int page, int nv) {
        const int pr = row - (kPage - nv);
        if (pr < 0) return make_float2(0.f, 0.f);
        return __ldg(reinterpret_cast<const float2*>(reinterpret_cast<const uint8_t*>(scale_base) +
                                                     (size_t)page * kF8Page) + pr);
      };
      auto put16 = [&](uint32_t dst, int v, const uint4& in, __half2 sc) {
        uint4 o0, o1;
        dequant16_f16(in, sc, o0, o1);
        const uint32_t rb = dst + (v >> 2) * kChunk + row * 128;
        const uint32_t u = 2u * (v & 3);
        sts128(rb + ((u ^ sw) << 4), o0);
        sts128(rb + (((u + 1) ^ sw) << 4), o1);
      };
      auto cwait = [&](uint64_t& b, uint32_t parity) {
        const bool all = named_bar_and(1, 128, mbar_wait(bar(b), parity, abort_flag));
        if (!all && ct == 0) st_cluster_u32(peer_abort, 1u);
        return all;
      };
      auto publish = [&](uint64_t& full) {  // the chunks are written: both CTAs' MMAs may read them
        fence_proxy_async_cta();
        named_bar_sync(1, 128);
        if (ct == 0) mbar_arrive_cl(lead(full));
      };
      // latent group: 4 chunks from dst, box of 256-byte rows at dst + 2 chunks
      auto conv_group = [&](uint32_t dst, __half2 sc) {
        const uint32_t box = dst + 2 * kChunk + row * 256;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int v = 4 * half + ((j + row) & 3);
          put16(dst, v, lds128(box + 16 * v), sc);
        }
        uint4 keep[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) keep[j] = lds128(box + 16 * (8 + 4 * half + ((j + row) & 3)));
        named_bar_sync(1, 128);
#pragma unroll
        for (int j = 0; j < 4; ++j) put16(dst, 8 + 4 * half + ((j + row) & 3), keep[j], sc);
      };
      // pair: 2 chunks from dst, box of 128-byte rows at dst + 1 chunk
      auto conv_pair = [&](uint32_t dst, __half2 sc) {
        const uint32_t box = dst + kChunk + row * 128;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int v = 2 * half + ((j + row) & 1);
          put16(dst, v, lds128(box + 16 * v), sc);
        }
        uint4 keep[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) keep[j] = lds128(box + 16 * (4 + 2 * half + ((j + row) & 1)));
        named_bar_sync(1, 128);
#pragma unroll
        for (int j = 0; j < 2; ++j) put16(dst, 4 + 2 * half + ((j + row) & 1), keep[j], sc);
      };
      // rope chunk, box of 64-byte rows in its upper half: output rows 32-63 overwrite the box
      auto conv_rope = [&](uint32_t dst, __half2 sr) {
        const uint32_t box = dst + kChunk / 2 + row * 64;
        uint4 keep[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) keep[j] = lds128(box + 16 * (2 * half + j));
        named_bar_sync(1, 128);
#pragma unroll
        for (int j = 0; j < 2; ++j) put16(dst, 2 * half + j, keep[j], sr);
      };
      // an item's queries: bf16 -> fp16 in place, each thread its own 16-byte units
      auto conv_q = [&](const Cursor& c) {
        if (!cwait(ctl->f8_q, c.ii & 1)) return false;
        if constexpr (kBf16) {
          for (int u = ct; u < 9 * kChunk / 16; u += 128) {
            const uint32_t a = data_u32 + kQOff + 16 * u;
            const uint4 v = lds128(a);
            uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
              const __half2 hv = __floats2half2_rn(f.x, f.y);
              w[e] = *reinterpret_cast<const uint32_t*>(&hv);
            }
            sts128(a, make_uint4(w[0], w[1], w[2], w[3]));
          }
        }
        publish(ctl->q_full);
        return true;
      };
      // the own page of a tile: rope, then latent groups 0 and 1
      auto conv_own = [&](const Cursor& c, float2 sc) {
        const int s = c.ti & 1;
        const __half2 hc = __float2half2_rn(sc.x), hr = __float2half2_rn(sc.y);
        if (!cwait(ctl->f8_rope, c.ti & 1)) return false;
        conv_rope(data_u32 + kRopeOff, hr);
        publish(ctl->rope_full);
        for (int h = 0; h < 2; ++h) {
          if (!cwait(ctl->f8_qk[s][h], (c.ti >> 1) & 1)) return false;
          conv_group(set_u32 + s * kSetBytes + 4 * h * kChunk, hc);
          publish(ctl->qk_full[s][h]);
        }
        return true;
      };
      // the other page's latent half of a tile: pairs 2j + g, j = 0, 1
      auto conv_pairs = [&](const Cursor& c, float sc) {
        const int s = c.ti & 1, g = 1 - (int)rank;
        for (int j = 0; j < 2; ++j) {
          const int pr = 2 * j + g;
          if (!cwait(ctl->f8_pv[s][j], (c.ti >> 1) & 1)) return false;
          conv_pair(set_u32 + s * kSetBytes + 2 * pr * kChunk, __float2half2_rn(sc));
          publish(ctl->pv_full[s][pr]);
        }
        return true;
      };
      // this thread's scales for a tile: the own page's (s_c, s_r) and the other page's s_c (their
      // page ids and values are read a tile ahead, so that their latency hides behind a tile)
      struct TileScales {
        float2 own;
        float pair;
      };
      auto tile_scales = [&](const Cursor& c, int L) {
        const int pi = 2 * c.t + (int)rank, g = 1 - (int)rank;
        const int nv_o = min(kPage, max(0, L - kPage * pi));
        const int nv_p = min(kPage, max(0, L - kTile * c.t - kPage * g));
        const long bt0 = (long)c.item.b * p.max_pages;
        const int pg_o = nv_o > 0 ? p.bt[bt0 + pi] : 0;
        const int pg_p = nv_p > 0 ? p.bt[bt0 + 2 * c.t + g] : 0;
        return TileScales{scales(pg_o, nv_o), scales(pg_p, nv_p).x};
      };
      if constexpr (F8) {
        Cursor c;
        c.start(prefix, p.B, cluster, nclusters);
        int L = c.valid ? p.seq_lens[c.item.b] : 0;
        TileScales cur = c.valid ? tile_scales(c, L) : TileScales{};
        while (c.valid) {
          Cursor nx = c;
          nx.advance(prefix);
          int Ln = L;
          TileScales nxt{};
          if (nx.valid) {
            if (nx.first()) Ln = p.seq_lens[nx.item.b];
            nxt = tile_scales(nx, Ln);
          }
          if ((c.first() && !conv_q(c)) || !conv_own(c, cur.own) || !conv_pairs(c, cur.pair)) break;
          c = nx;
          L = Ln;
          cur = nxt;
        }
      }
    } else if (warp < kSoftWarps) {
      // ---------------------------------------------------------------- softmax, rescale, epilogue
      // Thread: TMEM lane lt = 32 (warp % 4) + lane, head h = lt % 64 of this CTA, page g = lt / 64,
      // column half ch = warp / 4: tokens [64g + 32ch, 64g + 32ch + 32) of the tile, and O
      // columns [128ch, 128ch + 128) (latent columns 256ch + 128g + [0, 128)).
      const int qd = warp & 3, ch = warp >> 2;
      const int lt = 32 * qd + lane, h = lt & 63, g = lt >> 6;
      const int head = 64 * (int)rank + h;
      const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
      const uint32_t p_row = data_u32 + kPOff + g * kChunk + (h >> 3) * 1024 + (h & 7) * 128;
      uint8_t* const p_row_ptr = data + (p_row - data_u32);
      // Exchange one value among the four threads of a head; returns the four in a fixed order
      // (page 0 half 0, page 0 half 1, page 1 half 0, page 1 half 1). A head's four threads sit
      // in the four warps of one parity, so each group of four warps exchanges on barriers of its
      // own: one barrier round per exchange. Successive maxima alternate between two buffers, the
      // fp32 xm and the bf16 xh (a reference maximum need not be exact, only the same for the
      // four threads), so that a writer never waits for the readers of the exchange before: they
      // have arrived at the one in between. The denominator exchange at an item's end is fp32
      // (xm); the tile before it is complete (its O MMAs have read every thread's P, which each
      // thread writes after reading that tile's maxima), and the next maximum goes to xh.
      const int xg = warp & 1;
      uint32_t xuse0 = 0, xuse1 = 0;  // completed exchanges on xm / xh (their barriers' phases)
      int xnext = 0;                  // buffer of the next maximum: 0 = xm, 1 = xh
      auto exchange = [&](float v, int buf, float (&out)[4]) {
        const int l0 = lt & 63;
        if (buf == 0) ctl->xm[ch][lt] = v;
        else ctl->xh[ch][lt] = __float2bfloat16_rn(v);
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ctl->mx_full[xg][buf]));
        if (!wwait(ctl->mx_full[xg][buf], (buf == 0 ? xuse0 : xuse1) & 1)) return false;
        if (buf == 0) {
          ++xuse0;
          out[0] = ctl->xm[0][l0];
          out[1] = ctl->xm[1][l0];
          out[2] = ctl->xm[0][l0 + 64];
          out[3] = ctl->xm[1][l0 + 64];
        } else {
          ++xuse1;
          out[0] = __bfloat162float(ctl->xh[0][l0]);
          out[1] = __bfloat162float(ctl->xh[1][l0]);
          out[2] = __bfloat162float(ctl->xh[0][l0 + 64]);
          out[3] = __bfloat162float(ctl->xh[1][l0 + 64]);
        }
        return true;
      };
      Cursor c;
      c.start(prefix, p.B, cluster, nclusters);
      float m_ref = -INFINITY, lsum = 0.f;
      int L = 0;
      bool ok = true;
      while (ok && c.valid) {
        const int ti = c.ti, sb = ti & 1, t = c.t;
        if (c.first()) {
          m_ref = -INFINITY;
          lsum = 0.f;
          L = p.seq_lens[c.item.b];
        }
        if (!wwait(ctl->s_full[sb], (ti >> 1) & 1)) break;
        tc_fence_after();
        uint32_t sr[32];
        tmem_ld32(tmem + lane_base + kSCol + 64 * sb + 32 * ch, sr);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cl(lead(ctl->s_free[sb]));
        // Slot rows before 64 - nv of a tail page (nv tokens) are zero fill: -inf, weight exactly 0.
        const int lo = kPage - min(kPage, max(0, L - kTile * t - kPage * g)) - 32 * ch;  // first valid k
        if (lo > 0) {
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (k < lo) sr[k] = __float_as_uint(-INFINITY);
        }
        float mxs[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mxs[k] = u2f(sr[k]);
#pragma unroll
        for (int k = 8; k < 32; ++k) mxs[k & 7] = fmaxf(mxs[k & 7], u2f(sr[k]));
        float four[4];
        if (!exchange(fmaxf(fmaxf(fmaxf(mxs[0], mxs[1]), fmaxf(mxs[2], mxs[3])),
                            fmaxf(fmaxf(mxs[4], mxs[5]), fmaxf(mxs[6], mxs[7]))),
                      xnext, four))
          break;
        xnext ^= 1;
        const float mx = fmaxf(fmaxf(four[0], four[1]), fmaxf(four[2], four[3])) * p.scale_log2;
        float alpha = 1.f;
        if (mx > m_ref + kLazy) {
          alpha = ex2_approx(m_ref - mx);
          lsum *= alpha;
          m_ref = mx;
        }
        // the O MMAs of the previous tile are done: P may be overwritten and O rescaled
        if (!wwait(ctl->p_free, (ti & 1) ^ 1)) break;
        if (!c.first() && __any_sync(0xffffffffu, alpha != 1.f)) {
          tc_fence_after();
          // two TMEM loads in flight per wait (one with the FP8 cache's smaller register budget)
          constexpr int kRl = F8 ? 1 : 2;
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 32 * kRl) {
            uint32_t r[kRl][32];
#pragma unroll
            for (int q2 = 0; q2 < kRl; ++q2) tmem_ld32(tmem + lane_base + kOCol + 128 * ch + c0 + 32 * q2, r[q2]);
            tmem_wait_ld();
#pragma unroll
            for (int q2 = 0; q2 < kRl; ++q2) {
#pragma unroll
              for (int k = 0; k < 32; ++k) r[q2][k] = __float_as_uint(u2f(r[q2][k]) * alpha);
              tmem_st32(tmem + lane_base + kOCol + 128 * ch + c0 + 32 * q2, r[q2]);
            }
          }
          tmem_wait_st();
        }
        // P row h, tokens [32ch, 32ch + 32) of page g: p = 2^(s * scale - m_ref), one FFMA and one
        // ex2 per token. The sum of the rounded weights is the denominator (it matches what the
        // MMA accumulates).
        float sums[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int u4 = 0; u4 < 4; ++u4) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k = 8 * u4 + 2 * e;
            const typename Pack<PT>::T2 pr2 = Pack<PT>::make(ex2_approx(fmaf(u2f(sr[k]), p.scale_log2, -m_ref)),
                                                           ex2_approx(fmaf(u2f(sr[k + 1]), p.scale_log2, -m_ref)));
            const float2 back = Pack<PT>::f2(pr2);
            sums[e] += back.x + back.y;
            w[e] = *reinterpret_cast<const uint32_t*>(&pr2);
          }
          *reinterpret_cast<uint4*>(p_row_ptr + ((((4 * ch + u4) ^ (h & 7))) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        lsum += (sums[0] + sums[1]) + (sums[2] + sums[3]);
        fence_proxy_async_cta();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cl(lead(ctl->p_full));

        if (c.last()) {  // ---- epilogue of the item: O / l for this thread's head and columns
          if (!wwait(ctl->p_free, ti & 1)) break;  // the last O MMAs are done
          tc_fence_after();
          if (!exchange(lsum, 0, four)) break;
          xnext = 1;
          const float l = (four[0] + four[1]) + (four[2] + four[3]);
          const float inv = l > 0.f ? 1.f / l : 0.f;
          const float lse = l > 0.f ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
          const Item& it = c.item;
          const bool whole = it.t0 == 0 && it.t1 == it.n_b;
          const long slot = (long)it.b + cluster;
          const int col0 = 256 * ch + 128 * g;  // latent columns [col0, col0 + 128)
          // The warp writes its 32 heads x 128 columns in rounds of 64 bytes per head through
          // shared memory: each lane puts its head's segment in row `lane` of a 2 KB box in the
          // 64-byte swizzle (16-byte chunk c of row r at c ^ (r/2 % 4), conflict-free), and lane 0
          // stores the 32 x 64-byte box with one TMA store, which heads past n_h fall outside of.
          // Mid-range the warp's 2 KB of the P buffer (free: the last O MMAs are done) holds two
          // 1 KB boxes of 32 bytes per head, used in turn by half rounds, so a box waits only for
          // the store two half rounds back; at the pair's last item every round gets a 2 KB box
          // of its own in the latent sets, which no tile needs any more, so nothing waits.
          const bool last_item = c.it.g >= c.it.g_end;
          const uint32_t wsw = (lane >> 1) & 3;
          const int head0 = 64 * (int)rank + 32 * (qd & 1);
          int round = 0;
          auto stage_store = [&](const uint32_t (&w)[16], int col) {
            if (!last_item) {
              // mid-range: two half rounds of 32 bytes per head through the warp's two 1 KB boxes
              // of P (unswizzled), each box reused once the store two half rounds back has read it
#pragma unroll
              for (int hf = 0; hf < 2; ++hf) {
                const uint32_t box_u32 = data_u32 + kPOff + warp * 2048 + (round & 1) * 1024;
                uint8_t* const box = data + (box_u32 - data_u32);
                ++round;
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
                *reinterpret_cast<uint4*>(box + lane * 32) = make_uint4(w[8 * hf], w[8 * hf + 1], w[8 * hf + 2], w[8 * hf + 3]);
                *reinterpret_cast<uint4*>(box + lane * 32 + 16) =
                    make_uint4(w[8 * hf + 4], w[8 * hf + 5], w[8 * hf + 6], w[8 * hf + 7]);
                fence_proxy_async_cta();
                __syncwarp();
                if (lane == 0) {
                  const int c = col + hf * (whole ? 16 : 8);  // 32 bytes of columns
                  if (whole) tma_store_3d(&maps.o_lat_h, box_u32, c, head0, it.b);
                  else tma_store_3d(&maps.o_part_h, box_u32, c, head0, (int)slot);
                  bulk_commit_group();
                }
              }
              return;
            }
            const uint32_t stage_u32 = set_u32 + warp * 16384 + round * 2048;
            uint8_t* const stage = data + (stage_u32 - data_u32);
            ++round;
#pragma unroll
            for (int i2 = 0; i2 < 4; ++i2)
              *reinterpret_cast<uint4*>(stage + lane * 64 + ((i2 ^ wsw) << 4)) =
                  make_uint4(w[4 * i2], w[4 * i2 + 1], w[4 * i2 + 2], w[4 * i2 + 3]);
            fence_proxy_async_cta();
            __syncwarp();
            if (lane == 0) {
              if (whole) tma_store_3d(&maps.o_lat, stage_u32, col, head0, it.b);
              else tma_store_3d(&maps.o_part, stage_u32, col, head0, (int)slot);
              bulk_commit_group();
            }
          };
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_base + kOCol + 128 * ch + c0, r);
            tmem_wait_ld();
            if (whole) {  // 32 columns of bf16 / fp16 per round
              uint32_t w[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const typename Pack<T>::T2 v = Pack<T>::make(u2f(r[2 * e]) * inv, u2f(r[2 * e + 1]) * inv);
                w[e] = *reinterpret_cast<const uint32_t*>(&v);
              }
              stage_store(w, col0 + c0);
            } else {  // 16 columns of fp32 per round
#pragma unroll
              for (int half = 0; half < 2; ++half) {
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(u2f(r[16 * half + e]) * inv);
                stage_store(w, col0 + c0 + 16 * half);
              }
            }
          }
          if (head < p.n_h && g == 0 && ch == 0) {
            if (whole) {
              if (p.lse_out != nullptr) p.lse_out[(long)it.b * p.n_h + head] = lse;
            } else {
              p.lse_part[slot * p.n_h + head] = lse;
            }
          }
          // the boxes have left shared memory before the next tile's softmax writes P, or before
          // the CTA exits
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cl(lead(ctl->o_free));
        }
        c.advance(prefix);
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  if (has_work && warp == kMmaWarp && rank == 0) {
    // every pair MMA (of both issuing threads) has completed before either CTA releases its
    // tensor memory
    if (lane == 0) mbar_wait_slow<false>(bar(ctl->drain), 0, nullptr);
    __syncwarp();
  }
  if (*abort_flag && threadIdx.x == 0) {
    // A wait gave up: loads already issued (to this CTA's slots, signalling rank 0's barriers)
    // land within microseconds; give them 200 us before either CTA of the pair exits.
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 200000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_arrive();  // neither CTA leaves while its peer may still touch its shared memory
  cluster_wait();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc2(tmem, kTmemCols);
  }
}

// Tiles per sequence (0 for a sequence whose length or pages are invalid) and their exclusive
// prefix sum, in one block of 1024 threads: a warp checks a sequence's pages (lanes stride over
// its block-table row), then a block-wide scan turns the counts into offsets in place. The host
// keeps the total (B x tiles of max_seq_len) within int32.
__global__ void __launch_bounds__(1024) k_decode_plan(const int* __restrict__ seq_lens, const int* __restrict__ bt,
                                                      int B, int max_pages, int num_pages, int max_seq_len, int C,
                                                      int caller_inputs, int* __restrict__ tile_prefix,
                                                      int* __restrict__ seq_pairs,
                                                      int* __restrict__ pair_start) {
  // When the lengths and block tables come from the caller (caller_inputs: no kernel of this
  // call wrote them), up to kPlanEarlySeqs sequences are checked, their tile counts kept in shared
  // memory, before the wait for the kernel before, which may still be using the workspace this
  // kernel writes. (Prefill's per-token tables are written by the kernel before: it waits first.)
  constexpr int kPlanEarlySeqs = 4096;
  __shared__ int s_count[kPlanEarlySeqs];
  const bool early = caller_inputs != 0 && B <= kPlanEarlySeqs;
  if (!early) griddep_wait();
  if (threadIdx.x == 0) griddep_launch();
  int* const count = early ? s_count : tile_prefix;
  __shared__ int warp_total[32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Tiles of each sequence (0 for a rejected one), a half-warp per sequence, 64 sequences per
  // pass; every lane runs every pass so the ballot below is warp-uniform.
  const int grp = 2 * warp + (lane >> 4), sub = lane & 15;
  const unsigned half = (lane >> 4) ? 0xffff0000u : 0x0000ffffu;
  for (int b0 = 0; b0 < B; b0 += 64) {
    const int b = b0 + grp;
    int L = 0, n = 0;
    bool ok = false;
    if (b < B) {
      L = seq_lens[b];
      n = (int)(((long)L + dec::kPage - 1) / dec::kPage);
      ok = L >= 1 && L <= max_seq_len && n <= max_pages;
      if (!ok && sub == 0) record_error(MLA_ERR_BAD_SEQ_LEN);
    }
    bool bad = false;
    if (ok)
      for (int t = sub; t < n; t += 16) {
        const int pg = bt[(long)b * max_pages + t];
        bad |= pg < 0 || pg >= num_pages;
      }
    const bool any_bad = (__ballot_sync(0xffffffffu, bad) & half) != 0;
    if (ok && any_bad) {
      ok = false;
      if (sub == 0) record_error(MLA_ERR_BAD_PAGE);
    }
    if (b < B && sub == 0) count[b] = ok ? (int)(((long)L + dec::kTile - 1) / dec::kTile) : 0;
  }
  __syncthreads();
  if (early) griddep_wait();
  // exclusive scan: thread tid sums the counts of sequences [tid * per, tid * per + per), then a
  // two-level warp-shuffle scan over the 1024 thread sums
  const int per = (B + 1023) / 1024;
  const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
  int sum = 0;
  for (int b = b0; b < b1; ++b) sum += count[b];
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_total[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_total[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += v;
    }
    warp_total[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  // Pair c takes tiles [T c / C, T (c+1) / C) (T = all tiles); each sequence gets the first and
  // last pair its tiles fall to (c0 | c1 << 16, or -1 without tiles), for the merge.
  const long T_ = warp_total[31];
  int run = incl - sum + (warp > 0 ? warp_total[warp - 1] : 0);
  for (int b = b0; b < b1; ++b) {
    const int n = count[b];
    tile_prefix[b] = run;
    if (n > 0) {
      const int c0 = cluster_of(run, T_, C), c1 = cluster_of(run + n - 1, T_, C);
      seq_pairs[b] = c0 | (c1 << 16) | ((T_ >= C ? 1 : 0) << 28);
    } else {
      seq_pairs[b] = -1;
    }
    run += n;
  }
  if (tid <= C) pair_start[tid] = (int)(T_ * tid / C);
  if (tid == 1023) tile_prefix[B] = (int)T_;
}

// Merge of the partials of sequences that span pairs, in pair order; zero output for rejected
// sequences. grid (B, ceil(n_h / 8)), 256 threads: one warp per head, each lane 16 of the 512
// latent values (four 16-byte loads per contributing pair, all in flight together).
template <typename T>
__global__ void __launch_bounds__(512) k_decode_tc_merge(const float* __restrict__ o_part,
                                                          const float* __restrict__ lse_part,
                                                          const int* __restrict__ seq_pairs,
                                                          const int* __restrict__ pair_start, int n_h,
                                                          T* __restrict__ o_lat, float* __restrict__ lse_out) {
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch();
  // grid (B, ceil(n_h / 32)), 16 warps of two heads each. Warp 0 lists the partial slots of
  // sequence b (the pairs its tiles fall to, in pair order, skipping pairs without tiles): n = -1
  // when one pair wrote it whole, 0 when it has no tiles (rejected: zero output).
  __shared__ int s_slot[kMaxDecodeClusters];
  __shared__ int s_n;
  const int b = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    const int sp = seq_pairs[b];
    int n = 0;
    if (sp >= 0) {
      const int c0 = sp & 0xffff, c1 = (sp >> 16) & 0xfff;
      if (c0 == c1) {
        n = -1;
      } else if ((sp >> 28) & 1) {  // every pair has tiles
        n = c1 - c0 + 1;
        for (int k = lane; k < n; k += 32) s_slot[k] = b + c0 + k;
      } else {
        for (int cb = c0; cb <= c1; cb += 32) {
          const int c = cb + lane;
          const bool own = c <= c1 && pair_start[c + 1] > pair_start[c];
          const unsigned m = __ballot_sync(0xffffffffu, own);
          if (own) s_slot[n + __popc(m & ((1u << lane) - 1u))] = b + c;
          n += __popc(m);
        }
      }
    }
    if (lane == 0) s_n = n;
  }
  __syncthreads();
  const int n = s_n, h0 = blockIdx.y * 32 + 2 * warp;
  if (n < 0 || h0 >= n_h) return;
  const int nh = min(2, n_h - h0);
  if (n == 0) {
    for (int hh = 0; hh < nh; ++hh) {
      T* out = o_lat + ((long)b * n_h + h0 + hh) * dec::kDc;
      for (int e = lane; e < dec::kDc; e += 32) Out<T>::put(out + e, 0.f);
      if (lse_out != nullptr && lane == 0) lse_out[(long)b * n_h + h0 + hh] = -INFINITY;
    }
    return;
  }
  auto row = [&](int i, int hh) {
    return reinterpret_cast<const float4*>(o_part + ((long)s_slot[i] * n_h + h0 + hh) * dec::kDc);
  };
  auto lse_of = [&](int i, int hh) { return lse_part[(long)s_slot[i] * n_h + h0 + hh]; };
  // The first two partial rows of both heads are requested before the weights are formed, so
  // that a sequence split over two pairs takes one round trip.
  float4 pre[2][2][4];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh)
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        pre[hh][i][j] = hh < nh && i < n ? row(i, hh)[lane + 32 * j] : make_float4(0.f, 0.f, 0.f, 0.f);
  // weights e^{lse_i - max}: lane i holds lse_i (i < 32); the sums run over lanes in a fixed order
  float lp[2], mx[2], z[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    lp[hh] = hh < nh && lane < n ? lse_of(lane, hh) : -INFINITY;
    float m = lp[hh];
    for (int i = lane + 32; i < n; i += 32) m = fmaxf(m, hh < nh ? lse_of(i, hh) : -INFINITY);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    mx[hh] = m;
    float zz = lp[hh] > -INFINITY ? exp2f((lp[hh] - m) * kLog2e) : 0.f;
    for (int i = lane + 32; i < n; i += 32) zz += hh < nh ? exp2f((lse_of(i, hh) - m) * kLog2e) : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) zz += __shfl_xor_sync(0xffffffffu, zz, o);
    z[hh] = zz;
  }
  float4 acc[2][4];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[hh][j] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  auto add = [&](int hh, float w, const float4 (&v)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc[hh][j].x = fmaf(w, v[j].x, acc[hh][j].x);
      acc[hh][j].y = fmaf(w, v[j].y, acc[hh][j].y);
      acc[hh][j].z = fmaf(w, v[j].z, acc[hh][j].z);
      acc[hh][j].w = fmaf(w, v[j].w, acc[hh][j].w);
    }
  };
  auto weight = [&](int i, int hh) {
    const float li = i < 32 ? __shfl_sync(0xffffffffu, lp[hh], i) : lse_of(i, hh);
    return li > -INFINITY ? exp2f((li - mx[hh]) * kLog2e) : 0.f;
  };
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {  // the prefetched rows (weight 0 past n or nh: zero rows)
    const float w0 = weight(0, hh), w1 = weight(1, hh);
    add(hh, hh < nh ? w0 : 0.f, pre[hh][0]);
    add(hh, hh < nh && n > 1 ? w1 : 0.f, pre[hh][1]);
  }
  for (int i = 2; i < n; ++i) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const float w = weight(i, hh);
      if (hh >= nh) continue;
      float4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = row(i, hh)[lane + 32 * j];
      add(hh, w, v);
    }
  }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    if (hh >= nh) continue;
    const float inv = z[hh] > 0.f ? 1.f / z[hh] : 0.f;
    typename Pack<T>::T2* dst = reinterpret_cast<typename Pack<T>::T2*>(o_lat + ((long)b * n_h + h0 + hh) * dec::kDc);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = 4 * (lane + 32 * j);
      dst[e / 2] = Pack<T>::make(acc[hh][j].x * inv, acc[hh][j].y * inv);
      dst[e / 2 + 1] = Pack<T>::make(acc[hh][j].z * inv, acc[hh][j].w * inv);
    }
    if (lse_out != nullptr && lane == 0)
      lse_out[(long)b * n_h + h0 + hh] = z[hh] > 0.f ? mx[hh] + logf(z[hh]) : -INFINITY;
  }
}

}  // namespace tc
}  // namespace mla
