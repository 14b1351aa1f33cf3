// Persistent stream-K GEMM on tcgen05 for the projections, with the projection epilogues fused:
//   D[z][m][n] = sum_k A[z][m][k] * B[z][n][k]
// The weights are the M = 128 side of the MMA and the few tokens of a decode step the N side
// ("swap-AB"), so every launch is a stream of weight bytes: what matters is that all SMs pull
// from HBM without a tail. The iteration space (tile, 64-wide k block), tiles ordered
// (z, m tile, n tile), is cut into G contiguous ranges, one per CTA: either evenly by
// iteration (stream-K, for long tiles) or at tile boundaries (for short ones). A CTA walks its
// range as segments, one per tile it touches; the MMA warp accumulates a segment in one of two
// TMEM buffers while the four epilogue warps drain the other.
//
// A segment that covers a whole tile is finished in the CTA: the epilogue applies the
// projection's output step and stores. A partial segment is written as fp32 to slot
// (tile + cta) of the partial buffer — unique, because both the tile and the CTA index only
// grow along the iteration space — and k_sk_reduce sums a tile's slots in CTA order (a fixed
// order, so results repeat bit for bit) before applying the same output step. With
// rope_in_reduce, tiles holding rope rows go that way even when one CTA finishes them.
//
// Output steps (EpiParams::mode):
//   plain   out[z * batch_off + n * ld + m]
//   append  the DeepSeek-V2 KV row [c^KV ; k^R] of token n: rows at and past rope_lo get RoPE
//           (adjacent pairs, angle at pos[n]) and the row goes to its paged-cache slot
//           (block_table[seq_idx[n]][pos[n] / page_size], row pos[n] % page_size)
//   query   [q^C ; q^R-before-RoPE] of token n: rows below rope_lo are q^C -> qc[n][m];
//           rope rows (head i, element j) get RoPE and go to q_out[n][i][d_c + j]
// ("DeepSeek-V2 from Scratch" §4.2 for the compressed KV and decoupled RoPE key, §5.3 for the
// absorbed query.)
//
// Warp roles (192 threads): 0-3 epilogue (thread = TMEM lane = row m), 4 TMA producer,
// 5 TMEM allocation + MMA issue (one elected lane).
#pragma once

#include "tc_common.cuh"

namespace mla {
namespace tc {

enum EpiMode : int { kEpiPlain = 0, kEpiAppend = 1, kEpiQuery = 2 };

struct EpiParams {
  int mode;
  void* out;            // plain: element type; append: the cache pool; query: q_out
  long out_ld, out_batch_off;
  // RoPE (append, query): rows m >= rope_lo rotate in pairs (m, m ^ 1)
  int rope_lo, d_rope;
  double rope_base;
  const double* rope_table;  // [d_rope/2] theta_k supplied by the caller, or null (base^(-2k/d_rope))
  const int* pos;       // [N]
  float2* cs_glob;      // [N][d_rope/2] cos/sin for split tiles' reduction (or null)
  int cs_ready;         // 1: cs_glob was filled by an earlier kernel (read it, do not compute it)
  int rope_in_reduce;   // 1: tiles with rope rows always go through k_sk_reduce (even whole ones)
  float2* cs_prefill;   // plain mode: fill this [N][d_rope/2] table for the next kernel (or null)
  // append
  const int* seq_idx;   // [N]
  const int* bt;
  int num_seqs, max_pages, num_pages, page_size;
  int stage_rows;       // 1: token n's row goes to row n of `out` ([N][rope_lo + d_rope]), not to the cache
  // query
  void* qc;             // [N][rope_lo] element type
  int n_h, d_c;
};

struct SkParams {
  int M, N, K;
  int m_tiles, n_tiles;
  int kb;               // 64-wide k blocks per tile
  long iters;           // tiles * kb
  int aligned;          // 1: CTA ranges start at tile boundaries
  int tiles;
  int stages;
  int a_batch_off;      // per z: row offset (K-major A) or K-row offset (MN-major A)
  int b_batch_off;      // per z: K (column) offset into B's rows
  float* part;          // [tiles + G][BN][128] fp32 partial slots
  EpiParams epi;
};

// First iteration of CTA c out of G.
__device__ __forceinline__ long sk_start(const SkParams& p, int c, int G) {
  if (p.aligned) return ((long)p.tiles * c / G) * p.kb;
  return p.iters * c / G;
}
// CTA whose range holds iteration i (inverse of sk_start).
__device__ __forceinline__ int sk_owner(const SkParams& p, long i, int G) {
  if (p.aligned) {
    const long t = i / p.kb;
    return (int)(((t + 1) * G - 1) / p.tiles);
  }
  return (int)(((i + 1) * G - 1) / p.iters);
}

template <int BN>
struct SkCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * BN;  // two accumulator buffers
  static constexpr int MAX_STAGES = 12;
};

// Host and device: bytes of the RoPE table kept in shared memory (float2 per token and pair).
__host__ __device__ inline size_t sk_table_bytes(int BN, const EpiParams& e) {
  return e.mode == kEpiPlain ? 0 : (size_t)BN * (e.d_rope / 2) * 8 + (size_t)BN * 8;
}

// Where row m of the output goes, for one tile: element (m, n) is stored at
// base + n * stride (plain, query) or at the token's cache row + m (append, see row_off).
// The per-row part is computed once per tile so that the store loop stays short: the
// epilogue runs once per tile, and its instructions are fetched cold each time.
template <typename T, int MODE>
struct RowDest {
  T* base;
  long stride;
  __device__ __forceinline__ RowDest(const EpiParams& e, int z, int m) {
    if (MODE == kEpiPlain) {
      base = static_cast<T*>(e.out) + (long)z * e.out_batch_off + m;
      stride = e.out_ld;
    } else if (MODE == kEpiAppend) {
      base = static_cast<T*>(e.out) + m;
      stride = 0;
    } else if (m < e.rope_lo) {
      base = static_cast<T*>(e.qc) + m;
      stride = e.rope_lo;
    } else {
      const int r = m - e.rope_lo;
      base = static_cast<T*>(e.out) + (long)(r / e.d_rope) * (e.d_c + e.d_rope) + e.d_c + r % e.d_rope;
      stride = (long)e.n_h * (e.d_c + e.d_rope);
    }
  }
  // row_off: the token's cache row offset (append; negative = no valid slot, nothing stored)
  __device__ __forceinline__ void put(int n, float v, long row_off) const {
    if (MODE == kEpiAppend) {
      if (row_off >= 0) Out<T>::put(base + row_off, v);
    } else {
      Out<T>::put(base + (long)n * stride, v);
    }
  }
};

// cos/sin of the RoPE angle of token n, pair k: read from the per-token table `tab`
// ([N][d_rope/2]) when an earlier kernel filled it, else computed. Kept out of line: the epilogue
// loop that may call it is unrolled and runs with cold instruction fetch, so an inlined
// double-precision pow and sincos in its branch would slow every pass through it.
__device__ __noinline__ float2 rope_cs_out_of_line(const float2* tab, const int* pos, int n, int k, int d_rope,
                                                   double base, const double* table) {
  if (tab != nullptr) return tab[(long)n * (d_rope / 2) + k];
  float2 q;
  rope_cos_sin(pos[n], k, d_rope, base, table, q.x, q.y);
  return q;
}

// Cache row offset (elements) of token n for the append step, or -1 (error recorded).
__device__ __forceinline__ long append_row_base(const EpiParams& e, int n) {
  if (e.stage_rows) return (long)n * (e.rope_lo + e.d_rope);
  const int s = e.seq_idx[n], p = e.pos[n];
  const int lp = p >= 0 ? p / e.page_size : -1;
  int page = -1;
  if (s >= 0 && s < e.num_seqs && p >= 0 && lp < e.max_pages) page = e.bt[(long)s * e.max_pages + lp];
  if (page < 0 || page >= e.num_pages) return -1;
  return ((long)page * e.page_size + p % e.page_size) * (e.rope_lo + e.d_rope);
}

template <typename T, int BN, bool A_MN, int MODE>
__global__ void __launch_bounds__(192, 2)
    k_gemm_sk(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
              const SkParams p) {
  using C = SkCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  const int half_rope = p.epi.d_rope / 2;
  float2* cs_tab = reinterpret_cast<float2*>(smem + (size_t)S * C::STAGE_BYTES);        // [BN][d_rope/2]
  long* row_tab = reinterpret_cast<long*>(cs_tab + (p.epi.mode == kEpiPlain ? 0 : BN * half_rope));  // [BN]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)S * C::STAGE_BYTES + sk_table_bytes(BN, p.epi));
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* acc_full = bars + 2 * S;
  uint64_t* acc_empty = bars + 2 * S + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x, G = gridDim.x;
  const long i0 = sk_start(p, cta, G), i1 = sk_start(p, cta + 1, G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(full + s), 1);
      mbar_init(smem_u32(empty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(acc_full + b), 1);
      mbar_init(smem_u32(acc_empty + b), 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto tile_coords = [&](int tile, int& z, int& mt, int& nt) {
    nt = tile % p.n_tiles;
    mt = (tile / p.n_tiles) % p.m_tiles;
    z = tile / (p.n_tiles * p.m_tiles);
  };

  if (warp == 4) {  // ------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&tma_a);
      tma_prefetch_map(&tma_b);
      // Counters advance incrementally: this single thread paces the whole CTA, so the loop
      // carries no divisions. The weights are written by no kernel, so the first ring stages
      // start streaming them before the wait for the previous kernel; the activations (B)
      // are loaded after it.
      const int n_it = (int)(i1 - i0);
      auto load_a = [&](int s, int z, int mt, int kbi) {
        uint8_t* sa = smem + (size_t)s * C::STAGE_BYTES;
        const uint32_t fb = smem_u32(full + s);
        const int k = kbi * C::BK;
        if (A_MN) {
          tma_load_2d(smem_u32(sa), &tma_a, fb, mt * C::BM, k + z * p.a_batch_off);
          tma_load_2d(smem_u32(sa + 8192), &tma_a, fb, mt * C::BM + 64, k + z * p.a_batch_off);
        } else {
          tma_load_2d(smem_u32(sa), &tma_a, fb, k, mt * C::BM + z * p.a_batch_off);
        }
      };
      auto load_b = [&](int s, int z, int nt, int kbi) {
        tma_load_2d(smem_u32(smem + (size_t)s * C::STAGE_BYTES + C::A_BYTES), &tma_b, smem_u32(full + s),
                    kbi * C::BK + z * p.b_batch_off, nt * BN);
      };
      const int pre = min(S, n_it);
      // (z, m tile, n tile, k block) of iteration i0, stepped with adds: one division per CTA
      int z0, mt0, nt0;
      const int tile0 = (int)(i0 / p.kb), kb0 = (int)(i0 - (long)tile0 * p.kb);
      tile_coords(tile0, z0, mt0, nt0);
      auto step = [&](int& z, int& mt, int& nt, int& kbi) {
        if (++kbi == p.kb) {
          kbi = 0;
          if (++nt == p.n_tiles) {
            nt = 0;
            if (++mt == p.m_tiles) {
              mt = 0;
              ++z;
            }
          }
        }
      };
      {
        int z = z0, mt = mt0, nt = nt0, kbi = kb0;
        for (int j = 0; j < pre; ++j) {  // ring slots start empty: no wait
          mbar_arrive_expect_tx(smem_u32(full + j), C::STAGE_BYTES);
          load_a(j, z, mt, kbi);
          step(z, mt, nt, kbi);
        }
      }
      griddep_wait();
      int z = z0, mt = mt0, nt = nt0, kbi = kb0;
      for (int j = 0; j < pre; ++j) {
        load_b(j, z, nt, kbi);
        step(z, mt, nt, kbi);
      }
      int s = pre % S, it = pre;
      uint32_t ph = pre == S ? 1u : 0u;
      for (; it < n_it; ++it) {
        if (!mbar_wait(smem_u32(empty + s), ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(smem_u32(full + s), C::STAGE_BYTES);
        load_a(s, z, mt, kbi);
        load_b(s, z, nt, kbi);
        if (++s == S) {
          s = 0;
          ph ^= 1;
        }
        step(z, mt, nt, kbi);
      }
      if (*abort_flag) {  // copies still in flight land before the CTA exits
        for (int j = max(0, it - S); j < it; ++j) mbar_wait_slow<false>(smem_u32(full + j % S), (j / S) & 1, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 5) {  // ----------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(C::BM, BN, IsBf16<T>::value, A_MN, false);
      constexpr uint32_t hi = desc_sw128_hi(1024);
      const uint32_t a_lo0 = desc_sw128_lo(smem_u32(smem), A_MN ? 8192 : 16);
      const uint32_t b_lo0 = desc_sw128_lo(smem_u32(smem) + C::A_BYTES, 16);
      const int n_it = (int)(i1 - i0);
      int kbi = (int)(i0 % p.kb), seg = 0, s = 0;
      uint32_t ph = 0, acc_col = 0;
      bool first = true;
      for (int it = 0; it < n_it; ++it) {
        if (it == 0 || kbi == 0) {  // a new segment: wait until its accumulator buffer is drained
          const int b = seg & 1;
          if (!mbar_wait(smem_u32(acc_empty + b), ((seg >> 1) & 1) ^ 1, abort_flag)) break;
          tc_fence_after();
          acc_col = (uint32_t)(b * BN);
          first = true;
        }
        if (!mbar_wait(smem_u32(full + s), ph, abort_flag)) break;
        tc_fence_after();
        // descriptor low words of stage s (16-byte units); a K-step is +2 along a K-major row
        // and +128 (16 rows) down the MN-major A
        const uint32_t a_lo = a_lo0 + (uint32_t)s * (C::STAGE_BYTES >> 4), b_lo = b_lo0 + (uint32_t)s * (C::STAGE_BYTES >> 4);
        mma_ss_lohi(tmem + acc_col, a_lo, b_lo, hi, idesc, !first);
#pragma unroll
        for (int ks = 1; ks < 4; ++ks) mma_ss_lohi(tmem + acc_col, a_lo + (A_MN ? 128 : 2) * ks, b_lo + 2 * ks, hi, idesc, 1);
        mma_commit(smem_u32(empty + s));
        first = false;
        if (it == n_it - 1 || kbi == p.kb - 1) {
          mma_commit(smem_u32(acc_full + (seg & 1)));
          ++seg;
        }
        if (++s == S) {
          s = 0;
          ph ^= 1;
        }
        if (++kbi == p.kb) kbi = 0;
      }
    }
    __syncwarp();
  } else {  // ---------------------------------------------------------- epilogue warps 0-3
    const int ml = warp * 32 + lane;  // row within the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    // Tables of the fused output step for the one n tile (RoPE cos/sin per token and pair,
    // cache row offset per token), built once while the first tiles stream in. With several
    // n tiles the step computes them per element instead.
    // Shared-memory tables are built only by CTAs that finish a whole tile themselves: the cache
    // row offsets for any whole append tile, the RoPE cos/sin for a whole tile with rope rows.
    // The CTA's segments: the first starts at k block kb0 of tile tile0 (one division per CTA),
    // the others at tile starts.
    const int tile0 = (int)(i0 / p.kb), kb0 = (int)(i0 - (long)tile0 * p.kb);
    bool tab_row = false, tab_cs = false;
    if (MODE != kEpiPlain && p.n_tiles == 1) {
      int tile = tile0, kbi0 = kb0;
      for (long i = i0; i < i1; ++tile, kbi0 = 0) {
        const long tile_end = (long)(tile + 1) * p.kb, seg_end = min(i1, tile_end);
        const bool rope_tile = (tile % p.m_tiles) * C::BM + C::BM > p.epi.rope_lo;  // n_tiles == 1
        if (kbi0 == 0 && seg_end == tile_end && !(p.epi.rope_in_reduce && rope_tile)) {
          tab_row |= MODE == kEpiAppend;
          tab_cs |= rope_tile;
        }
        i = seg_end;
      }
    }
    griddep_wait();  // token positions, cache slots and outputs belong to earlier kernels
    // RoPE cos/sin tables in global memory, a slice per CTA: for this kernel's reduction, or
    // (cs_prefill) for the next kernel, whose epilogues then copy it instead of computing it
    float2* const fill = MODE == kEpiPlain ? p.epi.cs_prefill : (p.epi.cs_ready ? nullptr : p.epi.cs_glob);
    if (fill != nullptr)
      for (int e = cta * 128 + ml; e < p.N * half_rope; e += G * 128) {
        float c, sn;
        rope_cos_sin(p.epi.pos[e / half_rope], e % half_rope, p.epi.d_rope, p.epi.rope_base, p.epi.rope_table, c,
                     sn);
        fill[e] = make_float2(c, sn);
      }
    if (tab_cs && p.epi.cs_ready) {
      for (int e = ml; e < BN * half_rope; e += 128)
        cs_tab[e] = e / half_rope < p.N ? p.epi.cs_glob[e] : make_float2(1.f, 0.f);
    } else if (tab_cs) {
      double theta = 0.0;
      int theta_k = -1;
      for (int e = ml; e < BN * half_rope; e += 128) {
        const int n = e / half_rope, k = e % half_rope;
        if (k != theta_k) {  // with half_rope dividing 128 this runs once per thread
          theta = rope_inv_freq(k, p.epi.d_rope, p.epi.rope_base, p.epi.rope_table);
          theta_k = k;
        }
        float c = 1.f, sn = 0.f;
        if (n < p.N) rope_cos_sin_at(p.epi.pos[n], theta, c, sn);
        cs_tab[e] = make_float2(c, sn);
      }
    }
    if (tab_row)
      for (int e = ml; e < BN; e += 128) {
        long rb = -1;
        if (e < p.N) {
          rb = append_row_base(p.epi, e);
          if (rb < 0) record_error(MLA_ERR_BAD_PAGE);
        }
        row_tab[e] = rb;
      }
    if (tab_cs || tab_row) named_bar_sync(1, 128);
    int seg = 0, tile = tile0, kbi0 = kb0;
    long i = i0;
    for (; i < i1; ++tile, kbi0 = 0) {
      const long seg_end = min(i1, (long)(tile + 1) * p.kb);
      int z, mt, nt;
      tile_coords(tile, z, mt, nt);
      // A tile with rope rows may be left to the reduction kernel: rotating it here reads the
      // cos/sin table from shared memory while the next tile streams through it, which is slow.
      const bool whole = kbi0 == 0 && seg_end == (long)(tile + 1) * p.kb &&
                         !(p.epi.rope_in_reduce && mt * C::BM + C::BM > p.epi.rope_lo);
      const int m = mt * C::BM + ml;
      const int n0 = nt * BN;
      const bool rot = MODE != kEpiPlain && m >= p.epi.rope_lo;
      const bool rope_warp = __any_sync(0xffffffffu, rot);
      const int k = rot ? ((m - p.epi.rope_lo) % p.epi.d_rope) >> 1 : 0;
      const RowDest<T, MODE> dst(p.epi, z, m);
      const bool row_ok = m < p.M;
      const int nv = min(BN, p.N - n0);  // valid columns of this tile
      const int b = seg & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(acc_full + b), (seg >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      const uint32_t acc = tmem + lane_base + (uint32_t)(b * BN);
      float* slot = p.part + ((long)tile + cta) * (128L * BN) + ml;
      // 32 columns per TMEM load, the next chunk's load in flight while this one is stored: the
      // load latency is paid about once per tile instead of once per few columns
      uint32_t ra[32], rb[32];
      tmem_ld32(acc, ra);
      tmem_wait_ld();
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        const bool more = c0 + 32 < BN;
        if (more) tmem_ld32(acc + c0 + 32, rb);
        if (!whole) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0 + j < nv) slot[(long)(c0 + j) * 128] = u2f(ra[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float v = u2f(ra[j]);
            const int nl = c0 + j;
            if (MODE != kEpiPlain && rope_warp) {  // warp-uniform: every lane takes part in the exchange
              const float w = __shfl_xor_sync(0xffffffffu, v, 1);  // the pair partner's value
              if (rot && nl < nv) {
                float2 q;
                if (tab_cs) q = cs_tab[nl * half_rope + k];
                else q = rope_cs_out_of_line(p.epi.cs_ready ? p.epi.cs_glob : nullptr, p.epi.pos, n0 + nl, k,
                                             p.epi.d_rope, p.epi.rope_base, p.epi.rope_table);
                v = (m & 1) ? fmaf(w, q.y, v * q.x) : fmaf(v, q.x, -w * q.y);
              }
            }
            if (nl < nv && row_ok)
              dst.put(n0 + nl, v, MODE != kEpiAppend ? 0 : tab_row ? row_tab[nl] : append_row_base(p.epi, n0 + nl));
          }
        }
        if (more) {
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) ra[j] = rb[j];
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(acc_empty + b));
      ++seg;
      i = seg_end;
    }
  }
  tc_fence_before();
  __syncthreads();
  // Dependents may launch only now: a small-block dependent (the split reduction) resident
  // early would share the SMs with the epilogue warps while they still work.
  if (threadIdx.x == 0) griddep_launch();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Tiles split over several CTAs: sum the fp32 partial slots in CTA order and apply the output
// step. Block (tile, 4-column group); thread = row pair (2q, 2q+1) of one column.
template <typename T, int BN, int MODE>
__global__ void __launch_bounds__(256) k_sk_reduce(const SkParams p, int G) {
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch();
  const int tile = blockIdx.x;
  const long t0 = (long)tile * p.kb;
  const int c_lo = sk_owner(p, t0, G), c_hi = sk_owner(p, t0 + p.kb - 1, G);
  const int nt = tile % p.n_tiles, mt = (tile / p.n_tiles) % p.m_tiles, z = tile / (p.n_tiles * p.m_tiles);
  if (c_lo == c_hi && !(p.epi.rope_in_reduce && mt * 128 + 128 > p.epi.rope_lo)) return;  // finished by its CTA
  const int q = threadIdx.x & 63;
  const int m = mt * 128 + 2 * q;
  const int nl = blockIdx.y * 4 + (threadIdx.x >> 6);
  const int n = nt * BN + nl;
  if (nl >= BN || n >= p.N || m >= p.M) return;
  // slot (tile + c) of each contributing CTA c; eight loads in flight, summed in CTA order
  const float* src = p.part + ((long)tile + c_lo) * (128L * BN) + (long)nl * 128 + 2 * q;
  float a = 0.f, b = 0.f;
  for (int c = c_lo; c <= c_hi; c += 8) {
    float2 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      v[u] = c + u <= c_hi ? *reinterpret_cast<const float2*>(src + (long)(c - c_lo + u) * (128L * BN))
                           : make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (c + u <= c_hi) {
        a += v[u].x;
        b += v[u].y;
      }
  }
  long rb = 0;
  if (MODE == kEpiAppend) {
    rb = append_row_base(p.epi, n);
    if (rb < 0) {
      record_error(MLA_ERR_BAD_PAGE);
      return;
    }
  }
  if (MODE != kEpiPlain && m >= p.epi.rope_lo) {
    const int k = ((m - p.epi.rope_lo) % p.epi.d_rope) >> 1;
    float cs, sn;
    if (p.epi.cs_glob != nullptr) {
      const float2 t = p.epi.cs_glob[(long)n * (p.epi.d_rope / 2) + k];
      cs = t.x;
      sn = t.y;
    } else {
      rope_cos_sin(p.epi.pos[n], k, p.epi.d_rope, p.epi.rope_base, p.epi.rope_table, cs, sn);
    }
    const float ra = fmaf(a, cs, -b * sn), rb2 = fmaf(b, cs, a * sn);
    a = ra;
    b = rb2;
  }
  RowDest<T, MODE>(p.epi, z, m).put(n, a, rb);
  if (m + 1 < p.M) RowDest<T, MODE>(p.epi, z, m + 1).put(n, b, rb);
}

}  // namespace tc
}  // namespace mla
