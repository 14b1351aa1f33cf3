// tcgen05 GEMM for the projections: D[m][n] = sum_k A[m][k] * B[n][k] with the weights as the
// M = 128 side and the few tokens of a decode step as N ("swap-AB": a skinny activation
// matrix becomes the N dimension of the MMA). Operands are fed by TMA in 64-element-wide
// (128-byte-swizzled) K blocks through a STAGES-deep mbarrier ring; the fp32 accumulator
// lives in TMEM and is read back by four epilogue warps, one TMEM lane quarter each.
//
// A is K-major ([M, K] row-major, the pages' W in R^{out x in}) or MN-major ([K, M]
// row-major, used for (W^UK_i)^T). B is K-major ([N, K], one token per row). blockIdx.z
// indexes a batch (heads) through coordinate offsets; blockIdx.y = split * n_tiles + n_tile
// splits K, each split writing an fp32 partial that a reduction kernel sums in split order.
//
// Warp roles (192 threads): 0-3 epilogue, 4 TMA producer, 5 TMEM allocation + MMA issue.
#pragma once

#include "tc_common.cuh"

namespace mla {
namespace tc {

struct GemmParams {
  int M, N, K;
  int kb_per_split;   // 64-wide K blocks per split
  int n_tiles;
  int a_batch_off;    // per batch z: row offset (K-major A) or K-row offset (MN-major A)
  int b_batch_off;    // per batch z: K (column) offset into B's rows
  void* out;
  long out_ld;        // elements between consecutive n in the output
  long out_batch_off;  // elements per batch z
  long out_split_off;  // elements per split (fp32 partials)
  int out_f32;        // 1: fp32 output (partials or fp32 result), 0: element type
};

template <int BN>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (192 * 1024) / STAGE_BYTES > 8 ? 8 : (192 * 1024) / STAGE_BYTES;
  static constexpr uint32_t TMEM_COLS = BN < 32 ? 32 : BN;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
};

template <typename T, int BN, bool A_MN>
__global__ void __launch_bounds__(192, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
              const GemmParams p) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tile = blockIdx.x;
  const int split = blockIdx.y / p.n_tiles, n_tile = blockIdx.y % p.n_tiles;
  const int z = blockIdx.z;
  const int kb_total = (p.K + C::BK - 1) / C::BK;
  const int kb0 = split * p.kb_per_split;
  const int nkb = max(0, min(kb_total, kb0 + p.kb_per_split) - kb0);

  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + C::STAGES), acc_bar = smem_u32(bars + 2 * C::STAGES);
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(acc_bar, 1);
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
  const uint32_t tmem_d = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      tma_prefetch_map(&tma_a);
      tma_prefetch_map(&tma_b);
      int issued = 0;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % C::STAGES;
        const uint32_t ph = (i / C::STAGES) & 1;
        if (!mbar_wait(empty0 + 8 * s, ph ^ 1, abort_flag)) break;
        uint8_t* sa = smem + s * C::STAGE_BYTES;
        const uint32_t fb = full0 + 8 * s;
        mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
        const int k = (kb0 + i) * C::BK;
        if (A_MN) {
          tma_load_2d(smem_u32(sa), &tma_a, fb, m_tile * C::BM, k + z * p.a_batch_off);
          tma_load_2d(smem_u32(sa + 8192), &tma_a, fb, m_tile * C::BM + 64, k + z * p.a_batch_off);
        } else {
          tma_load_2d(smem_u32(sa), &tma_a, fb, k, m_tile * C::BM + z * p.a_batch_off);
        }
        tma_load_2d(smem_u32(sa + C::A_BYTES), &tma_b, fb, k + z * p.b_batch_off, n_tile * BN);
        ++issued;
      }
      if (*abort_flag) {  // let copies still in flight land before the CTA exits
        for (int i = max(0, issued - C::STAGES); i < issued; ++i)
          mbar_wait_slow<false>(full0 + 8 * (i % C::STAGES), (i / C::STAGES) & 1, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(C::BM, BN, IsBf16<T>::value, A_MN, false);
      for (int i = 0; i < nkb; ++i) {
        const int s = i % C::STAGES;
        if (!mbar_wait(full0 + 8 * s, (i / C::STAGES) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES), sb = sa + C::A_BYTES;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = A_MN ? desc_sw128(sa + ks * 2048, 8192, 1024) : desc_sw128(sa + ks * 32, 16, 1024);
          const uint64_t bd = desc_sw128(sb + ks * 32, 16, 1024);
          mma_ss(tmem_d, ad, bd, idesc, (i | ks) != 0);
        }
        mma_commit(empty0 + 8 * s);
      }
      mma_commit(acc_bar);
    }
    __syncwarp();
  } else {
    const bool ok = mbar_wait(acc_bar, 0, abort_flag);
    tc_fence_after();
    const int m = m_tile * C::BM + warp * 32 + lane;
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem_d + ((uint32_t)(warp * 32) << 16) + c0, r);
      tmem_wait_ld();
      if (ok && m < p.M) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int n = n_tile * BN + c0 + j;
          if (c0 + j < BN && n < p.N) {
            const float v = nkb > 0 ? u2f(r[j]) : 0.f;
            const long off = (long)z * p.out_batch_off + (long)n * p.out_ld + m;
            if (p.out_f32)
              reinterpret_cast<float*>(p.out)[(long)split * p.out_split_off + off] = v;
            else
              Out<T>::put(reinterpret_cast<T*>(p.out) + off, v);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem_d, C::TMEM_COLS);
  }
}

// out[i] = sum_s part[s][i] (s in order), rounded to the element type; i < n.
template <typename T>
__global__ void k_splitk_reduce(const float* __restrict__ part, int splits, long split_off, long n, long rows,
                                long row_len, long out_ld, T* __restrict__ out) {
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < splits; ++s) acc += part[s * split_off + i];
    const long r = i / row_len, c = i % row_len;
    Out<T>::put(out + r * out_ld + c, acc);
  }
  (void)rows;
}

}  // namespace tc
}  // namespace mla
