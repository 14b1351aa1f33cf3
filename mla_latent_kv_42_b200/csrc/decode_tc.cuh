// Latent attention on tcgen05 for DeepSeek-V2 dims (n_h <= 128 heads, d_c = 512, d_h^R = 64,
// 64-token pages): "DeepSeek-V2 from Scratch" §4.4 with the absorbed steps 2-3 of §5.3.
//
// For 128 heads the fp32 accumulator O = sum_j p_j c_j is 128 x 512 x 4 B = 256 KB, all of
// one SM's tensor memory, so one work unit runs on a cluster of two CTAs:
//   score CTA (rank 0): Q [128 x 576] lives in TMEM as the A operand; S = Q C^T for each
//     64-token page (36 MMAs of K = 16, N = 64) from TMA-loaded 64 x 64 chunks; four warps
//     run the online softmax in fp32 (one head per thread, lazy rescaling: the reference
//     max moves only when a score exceeds it by 2^8) and write P (bf16) and the per-head
//     rescale factor straight into the value CTA's shared memory.
//   value CTA (rank 1): O in TMEM (512 columns); O += P C_lat per page (two N = 256
//     halves, C_lat read MN-major from TMA-loaded chunks); four warps apply rescales and
//     write the result (or a split-KV partial) out.
// The pages of all sequences are split evenly over the clusters; a sequence that spans
// clusters is merged afterwards by log-sum-exp in a fixed order.
#pragma once

#include "tc_common.cuh"

namespace mla {
namespace tc {

namespace dec {
constexpr int kPage = 64;         // tokens per cache page
constexpr int kTile = 128;        // tokens per tile: two pages (S = Q C^T with N = 128)
constexpr int kDc = 512;          // latent width (O columns)
constexpr int kD = 576;           // cache row width
constexpr int kChunk = 8192;      // one 64 x 64 box of 16-bit elements
constexpr int kPair = 2 * kChunk;  // column chunk kc of both pages of a tile, rows 0-63 then 64-127
constexpr int kScoreSlots = 8;    // score ring: 8 x 16 KB
constexpr int kValSlots = 4;      // value ring: 4 x 32 KB (one page's half latent: 4 chunks)
constexpr int kPBufs = 2;         // P buffers in the value CTA
constexpr int kPTile = 2 * 16384;  // P tile: 128 heads x 128 tokens bf16, two 64-token swizzled halves
constexpr int kPBytes = kPTile + 512;  // + 128 rescale factors
constexpr int kPStride = 33792;   // 1024-aligned stride of P buffers / staging buffers
constexpr int kStg = 2;           // score CTA: P staging buffers
constexpr int kStageOff = kScoreSlots * kPair;   // score CTA: kStg staging buffers
constexpr int kPOff = kValSlots * 4 * kChunk;    // value CTA: kPBufs P buffers
constexpr float kLazy = 8.f;      // rescale threshold in log2 units
constexpr int kDataBytes = 204800;
static_assert(kStageOff + kStg * kPStride <= kDataBytes, "score layout");
static_assert(kPOff + kPBufs * kPStride <= kDataBytes, "value layout");
constexpr int kThreads = 224;     // 7 warps
// TMEM columns
constexpr uint32_t kSCol = 0;     // score: S, 128 columns
constexpr uint32_t kQCol = 128;   // score: Q, 288 columns
constexpr uint32_t kOCol = 0;     // value: O, 512 columns
constexpr uint32_t kTmemCols = 512;

struct Ctrl {
  uint64_t full[kScoreSlots];
  uint64_t empty[kScoreSlots];
  uint64_t s_full, s_empty, q_ready;
  uint64_t stg_ready[kStg], stg_free[kStg];  // score CTA: staging buffers (softmax warps <-> sender warp)
  uint64_t p_empty[kPBufs];  // score CTA; arrived by the value CTA's multicast commit
  uint64_t stats_empty;      // score CTA; arrived remotely by the value CTA
  uint64_t p_full[kPBufs];   // value CTA; armed and completed by the score CTA's bulk copy
  uint64_t p_ready[kPBufs];  // value CTA
  // value CTA: O complete through the last tile that used P buffer pb. One barrier per P buffer
  // keeps every parity wait on it at most one phase behind: the P ring only guarantees that the
  // MMAs of tile t-2 are done when tile t's P arrives, so one shared barrier could lag by two.
  uint64_t o_done[kPBufs];
  uint64_t stats_full, o_free, drain;
  float stats[128][2];       // value CTA: reference max (log2 units) and denominator
  uint32_t tmem_slot;
  int abort_flag;
};
constexpr size_t kSmem = 1024 + kDataBytes + sizeof(Ctrl);
}  // namespace dec

struct DecodeTcParams {
  const void* q;          // [B, n_h, 576]
  const int* bt;          // [B, max_pages]
  int max_pages;
  const int* seq_lens;    // [B]
  const int* tile_prefix;  // [B + 1] pages before each sequence (0 pages for a rejected one)
  int B, n_h;
  float scale_log2;       // log2(e) / sqrt(d_h + d_h^R)
  void* o_lat;            // [B, n_h, 512] element type
  float* lse_out;         // [B, n_h] or null
  float* o_part;          // [B + C][n_h][512]
  float* lse_part;        // [B + C][n_h]
};

// Pages [t0, t1) of sequence b handled by this cluster (n_b = pages of the sequence).
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

// Cluster owning global page g when T pages are split over C clusters as [T c / C, T (c+1) / C).
__device__ __forceinline__ int cluster_of(long g, long T, int C) { return (int)(((g + 1) * C - 1) / T); }

template <typename T>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(dec::kThreads, 1)
    k_decode_tc(const __grid_constant__ CUtensorMap pool_map, const DecodeTcParams p) {
  using namespace dec;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* data = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl* ctl = reinterpret_cast<Ctrl*>(data + kDataBytes);
  volatile int* abort_flag = &ctl->abort_flag;
  const uint32_t data_u32 = smem_u32(data);
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int cluster = (int)cluster_id_x(), nclusters = (int)num_clusters_x();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kScoreSlots; ++i) {
      mbar_init(bar(ctl->full[i]), 1);
      mbar_init(bar(ctl->empty[i]), 1);
    }
    mbar_init(bar(ctl->s_full), 1);
    mbar_init(bar(ctl->s_empty), 128);
    for (int i = 0; i < kStg; ++i) {
      mbar_init(bar(ctl->stg_ready[i]), 128);
      mbar_init(bar(ctl->stg_free[i]), 1);
    }
    mbar_init(bar(ctl->q_ready), 128);
    for (int i = 0; i < kPBufs; ++i) {
      mbar_init(bar(ctl->p_empty[i]), 1);
      mbar_init(bar(ctl->p_full[i]), 1);
      mbar_init(bar(ctl->p_ready[i]), 128);
      mbar_init(bar(ctl->o_done[i]), 1);
    }
    mbar_init(bar(ctl->stats_empty), 128);
    mbar_init(bar(ctl->stats_full), 128);
    mbar_init(bar(ctl->o_free), 128);
    mbar_init(bar(ctl->drain), 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(&ctl->tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_arrive();  // barriers of both CTAs are initialised before any remote arrive
  cluster_wait();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_slot;
  if (threadIdx.x == 0) griddep_launch();
  griddep_wait();  // the plan, the query and the cache come from earlier kernels
  const bool has_work = [&] {
    const long T_ = p.tile_prefix[p.B];
    return T_ * (cluster + 1) / nclusters > T_ * cluster / nclusters;
  }();
  const uint32_t peer_abort = mapa(smem_u32(&ctl->abort_flag), peer);
  // A wait that gives up also releases the peer CTA's waiters.
  auto wait = [&](uint64_t& b, uint32_t parity) {
    if (mbar_wait(bar(b), parity, abort_flag)) return true;
    st_cluster_u32(peer_abort, 1u);
    return false;
  };
  auto wait_cl = [&](uint64_t& b, uint32_t parity) {
    if (mbar_wait_cluster(bar(b), parity, abort_flag)) return true;
    st_cluster_u32(peer_abort, 1u);
    return false;
  };
  // Warp-uniform variants for warps whose lanes all wait and then run warp-collective
  // instructions: a give-up seen by any lane is taken by the whole warp.
  auto wwait = [&](uint64_t& b, uint32_t parity) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar(b), parity, abort_flag));
    if (!ok && lane == 0) st_cluster_u32(peer_abort, 1u);
    return ok;
  };
  auto wwait_cl = [&](uint64_t& b, uint32_t parity) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(b), parity, abort_flag));
    if (!ok && lane == 0) st_cluster_u32(peer_abort, 1u);
    return ok;
  };
  constexpr bool kBf16 = IsBf16<T>::value;

  if (has_work) {
    if (rank == 0) {
      // =========================================================== score CTA
      if (warp == 4) {  // ---------------- TMA producer: chunk kc (64 columns) of both pages of a tile
        if (lane == 0) {
          tma_prefetch_map(&pool_map);
          int slot_i = 0;
          bool ok = true;
          ItemIter it = item_iter(p.tile_prefix, p.B, cluster, nclusters);
          Item item;
          while (ok && next_item(it, p.tile_prefix, item)) {
            const int* btb = p.bt + (long)item.b * p.max_pages;
            int page_a = btb[item.t0];
            int page_b = item.t0 + 1 < item.t1 ? btb[item.t0 + 1] : -1;
            for (int t = item.t0; ok && t < item.t1; t += 2) {
              const int next_a = t + 2 < item.t1 ? btb[t + 2] : 0;  // read ahead of their use
              const int next_b = t + 3 < item.t1 ? btb[t + 3] : -1;
              for (int kc = 0; kc < 9; ++kc, ++slot_i) {
                const int s = slot_i % kScoreSlots;
                if (!wait(ctl->empty[s], ((slot_i / kScoreSlots) & 1) ^ 1)) {
                  ok = false;
                  break;
                }
                mbar_arrive_expect_tx(bar(ctl->full[s]), page_b >= 0 ? kPair : kChunk);
                tma_load_2d(data_u32 + s * kPair, &pool_map, bar(ctl->full[s]), kc * 64, page_a * kPage);
                if (page_b >= 0)
                  tma_load_2d(data_u32 + s * kPair + kChunk, &pool_map, bar(ctl->full[s]), kc * 64, page_b * kPage);
              }
              page_a = next_a;
              page_b = next_b;
            }
          }
          if (!ok)  // copies in flight must land before the CTA exits
            for (int i = max(0, slot_i - kScoreSlots); i < slot_i; ++i)
              mbar_wait_slow<false>(bar(ctl->full[i % kScoreSlots]), (i / kScoreSlots) & 1, nullptr);
        }
        __syncwarp();
      } else if (warp == 5) {  // ---------------- MMA issue: S = Q C^T, 128 heads x 128 tokens
        if (lane == 0) {
          const uint32_t idesc = idesc_f16(128, kTile, kBf16, false, false);
          int slot_i = 0, tile = 0, item_i = 0;
          bool ok = true;
          ItemIter it = item_iter(p.tile_prefix, p.B, cluster, nclusters);
          Item item;
          while (ok && next_item(it, p.tile_prefix, item)) {
            if (!wait(ctl->q_ready, item_i & 1)) break;
            tc_fence_after();
            for (int t = item.t0; ok && t < item.t1; t += 2, ++tile) {
              if (!wait(ctl->s_empty, (tile & 1) ^ 1)) {
                ok = false;
                break;
              }
              tc_fence_after();
              for (int kc = 0; kc < 9; ++kc, ++slot_i) {
                const int s = slot_i % kScoreSlots;
                if (!wait(ctl->full[s], (slot_i / kScoreSlots) & 1)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
                const uint32_t sa = data_u32 + s * kPair;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                  mma_ts(tmem + kSCol, tmem + kQCol + kc * 32 + ks * 8, desc_sw128(sa + ks * 32, 16, 1024), idesc,
                         (kc | ks) != 0);
                mma_commit(bar(ctl->empty[s]));
              }
              if (ok) mma_commit(bar(ctl->s_full));
            }
            ++item_i;
          }
        }
        __syncwarp();
      } else if (warp == 6) {  // ---------------- sender: staged P tiles -> value CTA, one bulk copy each
        if (lane == 0) {
          int tile = 0;
          bool ok = true;
          ItemIter it = item_iter(p.tile_prefix, p.B, cluster, nclusters);
          Item item;
          while (ok && next_item(it, p.tile_prefix, item)) {
            for (int t = item.t0; t < item.t1; t += 2, ++tile) {
              const int sb = tile % kStg, pb = tile % kPBufs;
              if (!wait(ctl->stg_ready[sb], (tile / kStg) & 1) ||
                  !wait_cl(ctl->p_empty[pb], ((tile / kPBufs) & 1) ^ 1)) {
                ok = false;
                break;
              }
              const uint32_t full_remote = mapa(bar(ctl->p_full[pb]), 1u);
              mbar_arrive_expect_tx_remote(full_remote, kPBytes);
              bulk_copy_to_peer(mapa(data_u32 + kPOff + pb * kPStride, 1u), data_u32 + kStageOff + sb * kPStride,
                                kPBytes, full_remote);
              bulk_commit_group();
              bulk_wait_read<1>();  // the previous tile's staging buffer has been read: hand it back
              if (tile > 0) mbar_arrive(bar(ctl->stg_free[(tile - 1) % kStg]));
            }
          }
          bulk_wait<0>();
          // The value CTA's last commits arrive on p_empty asynchronously: let them land first.
          if (ok)
            for (int j = max(0, tile - kPBufs); j < tile; ++j)
              if (!wait_cl(ctl->p_empty[j % kPBufs], (j / kPBufs) & 1)) break;
        }
        __syncwarp();
      } else {  // ---------------- softmax warps 0-3: thread = head row = TMEM lane
        const int h = warp * 32 + lane;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const uint32_t row_off = (uint32_t)((h >> 3) * 1024 + (h & 7) * 128);
        int tile = 0, item_i = 0;
        bool ok = true;
        ItemIter it = item_iter(p.tile_prefix, p.B, cluster, nclusters);
        Item item;
        while (ok && next_item(it, p.tile_prefix, item)) {
          // Q row h of sequence b into TMEM columns [kQCol, kQCol + 288): two elements per column,
          // loaded in three batches of 24 x 16 bytes so that the loads overlap
          const uint4* qrow = reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) +
                                                             ((long)item.b * p.n_h + (h < p.n_h ? h : 0)) * kD);
#pragma unroll 1
          for (int c0 = 0; c0 < kD / 2; c0 += 96) {
            uint4 x[24];
#pragma unroll
            for (int v = 0; v < 24; ++v) x[v] = h < p.n_h ? __ldg(qrow + c0 / 4 + v) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int part = 0; part < 3; ++part) {
              uint32_t r[32];
#pragma unroll
              for (int v = 0; v < 8; ++v) {
                r[4 * v] = x[part * 8 + v].x;
                r[4 * v + 1] = x[part * 8 + v].y;
                r[4 * v + 2] = x[part * 8 + v].z;
                r[4 * v + 3] = x[part * 8 + v].w;
              }
              tmem_st32(tmem + lane_base + kQCol + c0 + part * 32, r);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(ctl->q_ready));

          const int L = p.seq_lens[item.b];
          float m_ref = -INFINITY, l = 0.f;
          for (int t = item.t0; t < item.t1; t += 2, ++tile) {
            if (!wwait(ctl->s_full, tile & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // S row h: four TMEM loads in flight, one wait
            uint32_t sr[4][32];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tmem + lane_base + kSCol + c4 * 32, sr[c4]);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bar(ctl->s_empty));

            // tokens of this tile: page t (0..63) and, if it belongs to this item, page t+1 (64..127);
            // masked tokens become -inf and get weight exactly 0
            const int nv = min(t + 1 < item.t1 ? kTile : kPage, L - t * kPage);
            if (nv < kTile) {
#pragma unroll
              for (int k = 0; k < kTile; ++k)
                if (k >= nv) sr[k >> 5][k & 31] = __float_as_uint(-INFINITY);
            }
            // running maximum on the raw scores (the scale is positive, so the order is the same),
            // eight independent chains
            float mxs[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) mxs[j] = u2f(sr[0][j]);
#pragma unroll
            for (int k = 8; k < kTile; ++k) mxs[k & 7] = fmaxf(mxs[k & 7], u2f(sr[k >> 5][k & 31]));
            const float mx = fmaxf(fmaxf(fmaxf(mxs[0], mxs[1]), fmaxf(mxs[2], mxs[3])),
                                   fmaxf(fmaxf(mxs[4], mxs[5]), fmaxf(mxs[6], mxs[7]))) * p.scale_log2;
            float alpha = 1.f;
            if (mx > m_ref + kLazy) {
              alpha = ex2_approx(m_ref - mx);
              l *= alpha;
              m_ref = mx;
            }
            const int sb = tile % kStg;
            if (!wwait(ctl->stg_free[sb], ((tile / kStg) & 1) ^ 1)) {
              ok = false;
              break;
            }
            // P row h in the 128-byte-swizzled K-major layout (two 64-token halves):
            // p = 2^(s * scale - m_ref), one FFMA and one ex2 per token. The sum of the rounded
            // weights is the denominator (it matches what the MMA accumulates); four chains.
            uint8_t* stage = data + kStageOff + sb * kPStride;
            float sums[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              uint32_t w[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int k = 8 * c + 2 * j;
                const typename Pack<T>::T2 pr =
                    Pack<T>::make(ex2_approx(fmaf(u2f(sr[k >> 5][k & 31]), p.scale_log2, -m_ref)),
                                  ex2_approx(fmaf(u2f(sr[(k + 1) >> 5][(k + 1) & 31]), p.scale_log2, -m_ref)));
                const float2 back = Pack<T>::f2(pr);
                sums[j] += back.x + back.y;
                w[j] = *reinterpret_cast<const uint32_t*>(&pr);
              }
              *reinterpret_cast<uint4*>(stage + (c >> 3) * 16384 + row_off + (((c & 7) ^ (h & 7)) << 4)) =
                  make_uint4(w[0], w[1], w[2], w[3]);
            }
            const float sum = (sums[0] + sums[1]) + (sums[2] + sums[3]);
            l += sum;
            reinterpret_cast<float*>(stage + kPTile)[h] = alpha;
            fence_proxy_async_cta();
            mbar_arrive(bar(ctl->stg_ready[sb]));
          }
          if (!ok) break;
          if (!wwait_cl(ctl->stats_empty, (item_i & 1) ^ 1)) break;
          st_cluster_f32(mapa(smem_u32(&ctl->stats[h][0]), 1u), m_ref);
          st_cluster_f32(mapa(smem_u32(&ctl->stats[h][1]), 1u), l);
          mbar_arrive_remote(mapa(bar(ctl->stats_full), 1u));
          ++item_i;
        }
      }
    } else {
      // =========================================================== value CTA
      if (warp == 4) {  // ---------------- TMA producer: half the latent of one page per slot
        if (lane == 0) {
          tma_prefetch_map(&pool_map);
          int vslot = 0;
          bool ok = true;
          ItemIter it = item_iter(p.tile_prefix, p.B, cluster, nclusters);
          Item item;
          while (ok && next_item(it, p.tile_prefix, item)) {
            const int* btb = p.bt + (long)item.b * p.max_pages;
            for (int t = item.t0; ok && t < item.t1; t += 2) {
              const int np = t + 1 < item.t1 ? 2 : 1;
              const int pages[2] = {btb[t], np == 2 ? btb[t + 1] : 0};
              for (int hf = 0; ok && hf < 2; ++hf)
                for (int g = 0; g < np; ++g, ++vslot) {
                  const int s = vslot % kValSlots;
                  if (!wait(ctl->empty[s], ((vslot / kValSlots) & 1) ^ 1)) {
                    ok = false;
                    break;
                  }
                  mbar_arrive_expect_tx(bar(ctl->full[s]), 4 * kChunk);
#pragma unroll
                  for (int q4 = 0; q4 < 4; ++q4)
                    tma_load_2d(data_u32 + (s * 4 + q4) * kChunk, &pool_map, bar(ctl->full[s]), (hf * 4 + q4) * 64,
                                pages[g] * kPage);
                }
            }
          }
          if (!ok)
            for (int i = max(0, vslot - kValSlots); i < vslot; ++i)
              mbar_wait_slow<false>(bar(ctl->full[i % kValSlots]), (i / kValSlots) & 1, nullptr);
        }
        __syncwarp();
      } else if (warp == 5) {  // ---------------- MMA issue: O += P C_lat (whole warp waits; lane 0 issues)
        const uint32_t idesc = idesc_f16(128, 256, kBf16, false, true);
        int vslot = 0, tile = 0, item_i = 0;
        bool ok = true;
        ItemIter it = item_iter(p.tile_prefix, p.B, cluster, nclusters);
        Item item;
        while (ok && next_item(it, p.tile_prefix, item)) {
          if (!wwait(ctl->o_free, (item_i & 1) ^ 1)) break;
          tc_fence_after();
          const int L = p.seq_lens[item.b];
          for (int t = item.t0; ok && t < item.t1; t += 2, ++tile) {
            const int pb = tile % kPBufs;
            if (!wwait(ctl->p_ready[pb], (tile / kPBufs) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t pa = data_u32 + kPOff + pb * kPStride;
            const int np = t + 1 < item.t1 ? 2 : 1;
            for (int hf = 0; ok && hf < 2; ++hf)
              for (int g = 0; g < np; ++g, ++vslot) {
                const int s = vslot % kValSlots;
                if (!wwait(ctl->full[s], (vslot / kValSlots) & 1)) {
                  ok = false;
                  break;
                }
                const int nv = min(kPage, L - (t + g) * kPage);
                if (nv < kPage) {  // rows past the sequence end may hold anything (even NaN): zero them
                  uint8_t* slot = data + s * 4 * kChunk;
                  const int per_chunk = (kPage - nv) * 8;
                  for (int e = lane; e < 4 * per_chunk; e += 32) {
                    const int q4 = e / per_chunk, rem = e % per_chunk;
                    *reinterpret_cast<uint4*>(slot + q4 * kChunk + (nv + rem / 8) * 128 + (rem % 8) * 16) =
                        make_uint4(0, 0, 0, 0);
                  }
                  fence_proxy_async_cta();
                  __syncwarp();
                }
                tc_fence_after();
                if (lane == 0) {
                  const uint32_t sb = data_u32 + s * 4 * kChunk;
#pragma unroll
                  for (int ks = 0; ks < 4; ++ks)
                    mma_ss(tmem + kOCol + hf * 256, desc_sw128(pa + g * 16384 + ks * 32, 16, 1024),
                           desc_sw128(sb + ks * 2048, 4 * 2048, 1024), idesc, !(t == item.t0 && g == 0 && ks == 0));
                  mma_commit(bar(ctl->empty[s]));
                }
                __syncwarp();
              }
            if (ok && lane == 0) {
              mma_commit_mc(bar(ctl->p_empty[pb]), (uint16_t)1u);  // P buffer free: tell the score CTA
              mma_commit(bar(ctl->o_done[pb]));
            }
            __syncwarp();
          }
          ++item_i;
        }
      } else if (warp < 4) {  // ---------------- correction + epilogue warps 0-3: thread = head row
        const int h = warp * 32 + lane;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const uint32_t stats_empty_remote = mapa(bar(ctl->stats_empty), 0u);
        int tile = 0, item_i = 0;
        bool ok = true;
        ItemIter it = item_iter(p.tile_prefix, p.B, cluster, nclusters);
        Item item;
        while (ok && next_item(it, p.tile_prefix, item)) {
          for (int t = item.t0; t < item.t1; t += 2, ++tile) {
            const int pb = tile % kPBufs;
            if (!wwait_cl(ctl->p_full[pb], (tile / kPBufs) & 1)) {
              ok = false;
              break;
            }
            const float alpha = reinterpret_cast<const float*>(data + kPOff + pb * kPStride + kPTile)[h];
            if (t != item.t0 && __any_sync(0xffffffffu, alpha != 1.f)) {
              if (!wwait(ctl->o_done[(tile - 1) % kPBufs], ((tile - 1) / kPBufs) & 1)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll 1
              for (int c0 = 0; c0 < kDc; c0 += 128) {  // four TMEM loads in flight per wait
                uint32_t r[4][32];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tmem + lane_base + kOCol + c0 + 32 * q4, r[q4]);
                tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
                  for (int j = 0; j < 32; ++j) r[q4][j] = __float_as_uint(u2f(r[q4][j]) * alpha);
                  tmem_st32(tmem + lane_base + kOCol + c0 + 32 * q4, r[q4]);
                }
              }
              tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar(ctl->p_ready[pb]));
          }
          if (!ok) break;
          if (!wwait_cl(ctl->stats_full, item_i & 1)) break;
          const float m_ref = ctl->stats[h][0], l = ctl->stats[h][1];
          mbar_arrive_remote(stats_empty_remote);
          // O holds every tile of the item once the last one is done; the other buffer's last
          // arrival is waited for as well so that none is still in flight when the CTA exits
          if (!wwait(ctl->o_done[(tile - 1) % kPBufs], ((tile - 1) / kPBufs) & 1)) break;
          if (tile >= 2 && !wwait(ctl->o_done[(tile - 2) % kPBufs], ((tile - 2) / kPBufs) & 1)) break;
          tc_fence_after();
          const float inv = l > 0.f ? 1.f / l : 0.f;
          const float lse = l > 0.f ? (m_ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
          const bool whole = item.t0 == 0 && item.t1 == item.n_b;
          const long slot = (long)item.b + cluster;
#pragma unroll 1
          for (int c0 = 0; c0 < kDc; c0 += 128) {  // four TMEM loads in flight per wait
            uint32_t r[4][32];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tmem + lane_base + kOCol + c0 + 32 * q4, r[q4]);
            tmem_wait_ld();
            if (h < p.n_h) {
              if (whole) {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<T*>(p.o_lat) + ((long)item.b * p.n_h + h) * kDc + c0);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                  uint32_t w[4];
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const int k = 8 * j + 2 * e;
                    const typename Pack<T>::T2 v =
                        Pack<T>::make(u2f(r[k >> 5][k & 31]) * inv, u2f(r[(k + 1) >> 5][(k + 1) & 31]) * inv);
                    w[e] = *reinterpret_cast<const uint32_t*>(&v);
                  }
                  dst[j] = make_uint4(w[0], w[1], w[2], w[3]);
                }
              } else {
                float4* dst = reinterpret_cast<float4*>(p.o_part + (slot * p.n_h + h) * kDc + c0);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                  const int k = 4 * j;
                  dst[j] = make_float4(u2f(r[k >> 5][k & 31]) * inv, u2f(r[k >> 5][(k & 31) + 1]) * inv,
                                       u2f(r[k >> 5][(k & 31) + 2]) * inv, u2f(r[k >> 5][(k & 31) + 3]) * inv);
                }
              }
            }
          }
          if (h < p.n_h) {
            if (whole) {
              if (p.lse_out != nullptr) p.lse_out[(long)item.b * p.n_h + h] = lse;
            } else {
              p.lse_part[slot * p.n_h + h] = lse;
            }
          }
          tc_fence_before();
          mbar_arrive(bar(ctl->o_free));
          ++item_i;
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  if (has_work && warp == 5) {
    if (lane == 0) {  // every MMA this thread issued has completed before TMEM is released
      mma_commit(bar(ctl->drain));
      mbar_wait_slow<false>(bar(ctl->drain), 0, nullptr);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  cluster_arrive();  // neither CTA leaves while its peer may still touch its shared memory
  cluster_wait();
}

// Pages per sequence (0 for a sequence whose length or pages are invalid) and their exclusive
// prefix sum, in one block of 1024 threads: a warp checks a sequence's pages (lanes stride over
// its block-table row), then a block-wide scan turns the counts into offsets in place.
__global__ void __launch_bounds__(1024) k_decode_plan(const int* __restrict__ seq_lens, const int* __restrict__ bt,
                                                      int B, int max_pages, int num_pages, int max_seq_len,
                                                      int* __restrict__ tile_prefix) {
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch();
  __shared__ int part[1024];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int b = warp; b < B; b += 32) {
    const int L = seq_lens[b];
    const int n = (L + dec::kPage - 1) / dec::kPage;
    bool ok = L >= 1 && L <= max_seq_len && n <= max_pages;
    if (!ok && lane == 0) record_error(MLA_ERR_BAD_SEQ_LEN);
    if (ok) {
      bool bad = false;
      for (int t = lane; t < n; t += 32) {
        const int pg = bt[(long)b * max_pages + t];
        bad |= pg < 0 || pg >= num_pages;
      }
      if (__any_sync(0xffffffffu, bad)) {
        ok = false;
        if (lane == 0) record_error(MLA_ERR_BAD_PAGE);
      }
    }
    if (lane == 0) tile_prefix[b] = ok ? n : 0;
  }
  __syncthreads();
  const int per = (B + 1023) / 1024;
  const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
  int sum = 0;
  for (int b = b0; b < b1; ++b) sum += tile_prefix[b];
  part[tid] = sum;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const int v = tid >= off ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int run = tid > 0 ? part[tid - 1] : 0;
  for (int b = b0; b < b1; ++b) {
    const int n = tile_prefix[b];
    tile_prefix[b] = run;
    run += n;
  }
  if (tid == 1023) tile_prefix[B] = part[1023];
}

// Merge of the partials of sequences that span clusters, in cluster order; zero output for
// rejected sequences. grid (B, ceil(n_h / 8)), 256 threads: one warp per head, each lane 16 of
// the 512 latent values (four 16-byte loads per contributing cluster, all in flight together).
template <typename T>
__global__ void __launch_bounds__(256) k_decode_tc_merge(const float* __restrict__ o_part,
                                                          const float* __restrict__ lse_part,
                                                          const int* __restrict__ tile_prefix, int B, int C, int n_h,
                                                          T* __restrict__ o_lat, float* __restrict__ lse_out) {
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch();
  const int b = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * 8 + warp;
  if (h >= n_h) return;
  const long T_ = tile_prefix[B];
  const int g0 = tile_prefix[b], g1 = tile_prefix[b + 1];
  T* out = o_lat + ((long)b * n_h + h) * dec::kDc;
  if (g1 == g0) {
    for (int e = lane; e < dec::kDc; e += 32) Out<T>::put(out + e, 0.f);
    if (lse_out != nullptr && lane == 0) lse_out[(long)b * n_h + h] = -INFINITY;
    return;
  }
  const int c0 = cluster_of(g0, T_, C), c1 = cluster_of(g1 - 1, T_, C);
  if (c0 == c1) return;  // written whole by its cluster
  // clusters between c0 and c1 own consecutive pages of this sequence, except those whose range
  // is empty (fewer pages than clusters): they wrote nothing and are skipped
  auto owns = [&](int c) { return T_ * (c + 1) / C > T_ * c / C; };
  const float* lp = lse_part + (long)b * n_h + h;  // slot b + c is at lp[c * n_h]
  float mx = -INFINITY;
  for (int c = c0; c <= c1; ++c)
    if (owns(c)) mx = fmaxf(mx, lp[(long)c * n_h]);
  float z = 0.f;
  for (int c = c0; c <= c1; ++c)
    if (owns(c)) z += exp2f((lp[(long)c * n_h] - mx) * 1.4426950408889634f);
  const float inv = 1.f / z;
  float4 acc[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
  for (int c = c0; c <= c1; ++c) {
    if (!owns(c)) continue;
    const float w = exp2f((lp[(long)c * n_h] - mx) * 1.4426950408889634f);
    const float4* src = reinterpret_cast<const float4*>(o_part + (((long)b + c) * n_h + h) * dec::kDc);
    float4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = src[lane + 32 * j];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc[j].x = fmaf(w, v[j].x, acc[j].x);
      acc[j].y = fmaf(w, v[j].y, acc[j].y);
      acc[j].z = fmaf(w, v[j].z, acc[j].z);
      acc[j].w = fmaf(w, v[j].w, acc[j].w);
    }
  }
  typename Pack<T>::T2* dst = reinterpret_cast<typename Pack<T>::T2*>(out);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = 4 * (lane + 32 * j);
    dst[e / 2] = Pack<T>::make(acc[j].x * inv, acc[j].y * inv);
    dst[e / 2 + 1] = Pack<T>::make(acc[j].z * inv, acc[j].w * inv);
  }
  if (lse_out != nullptr && lane == 0) lse_out[(long)b * n_h + h] = mx + logf(z);
}

}  // namespace tc
}  // namespace mla
