// gemm.cuh -- persistent tcgen05 GEMM for sm_100a: C[M,N] = A[M,K] * B, bf16
// operands, fp32 accumulation in tensor memory, bf16 output.
//
// Used for the W_kvb up-projection (A = latent [M, 512], B = W_kvb stored
// [N, K] i.e. K-major) and for the output projection (A = attention output
// [M, H*128], B = W_o stored [K, N] i.e. N-major).
//
// One CTA per SM, 192 threads:
//   warp 0      TMA producer: A and B tiles into a STAGES-deep ring
//   warp 1      tensor-memory allocator and UMMA issuer (one elected lane)
//   warps 2..5  epilogue: tensor memory -> registers -> bf16 -> swizzled
//               shared staging -> TMA store
// Two 128 x BN fp32 accumulators in tensor memory let the epilogue of one
// tile run under the main loop of the next.
#pragma once

#include "ptx.cuh"

namespace mla {

template <int BN_, bool B_MN_MAJOR_>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BN = BN_;
  static constexpr int BK = 64;  // one 128-byte swizzle row of bf16
  static constexpr bool B_MN_MAJOR = B_MN_MAJOR_;
  static constexpr int STAGES = 4;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_WARPS = 4;
  static constexpr int EPI_BUF = 32 * 128;  // 32 rows x 64 bf16 columns
  static constexpr int EPI_BYTES = EPI_WARPS * 2 * EPI_BUF;
  static constexpr int NUM_BARS = 2 * STAGES + 4;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + NUM_BARS * 8 + 16;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN must be a multiple of 64 in [64, 256]");
  static_assert(2 * BN <= 512, "two accumulators must fit in tensor memory");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, int M, int N, int K, int* err) {
  constexpr int BM = Cfg::BM, BN = Cfg::BN, BK = Cfg::BK, S = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi = smem + S * Cfg::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi + Cfg::EPI_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
  int* abort_word = reinterpret_cast<int*>(tmem_slot + 1);

  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + S);
  const uint32_t accf0 = smem_u32(bars + 2 * S);
  const uint32_t acce0 = smem_u32(bars + 2 * S + 2);
  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf0 + 8 * a, 1);
      mbar_init(acce0 + 8 * a, Cfg::EPI_WARPS);
    }
    *abort_word = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Abort ab{abort_word, err};

  const int num_m = (M + BM - 1) / BM;
  const int num_n = N / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = K / BK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int mt = tile % num_m, nt = tile / num_m;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1, ab, kErrWaitConsumer)) {
            ok = false;
            break;
          }
          const uint32_t full = full0 + 8 * s;
          const uint32_t sa = smem_u32(smem + s * Cfg::STAGE_BYTES);
          const uint32_t sb = sa + Cfg::A_BYTES;
          mbar_arrive_expect_tx(full, Cfg::STAGE_BYTES);
          tma_load_2d(sa, &tmA, full, kb * BK, mt * BM);
          if constexpr (!Cfg::B_MN_MAJOR) {
            tma_load_2d(sb, &tmB, full, kb * BK, nt * BN);
          } else {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c) tma_load_2d(sb + c * (BK * 128), &tmB, full, nt * BN + c * 64, kb * BK);
          }
        }
      }
      if (!ok) {
        // Let every load already issued land before the CTA exits.
        for (int i = (it > S ? it - S : 0); i < it; ++i) mbar_wait_drain(full0 + 8 * (i % S), (i / S) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- UMMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, 0, Cfg::B_MN_MAJOR ? 1 : 0);
      int it = 0, t = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++t) {
        const int a = t & 1;
        const uint32_t aph = (t >> 1) & 1;
        if (!mbar_wait(acce0 + 8 * a, aph ^ 1, ab, kErrWaitEpilogue)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + a * BN;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(full0 + 8 * s, ph, ab, kErrWaitTma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * Cfg::STAGE_BYTES);
          const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t adesc = smem_desc_sw128(sa + k * 32, 16, 1024);
            const uint64_t bdesc = Cfg::B_MN_MAJOR ? smem_desc_sw128(sb + k * 16 * 128, BK * 128, 1024)
                                                   : smem_desc_sw128(sb + k * 32, 16, 1024);
            umma_ss(d, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(empty0 + 8 * s);
        }
        if (!ok) break;
        umma_commit(accf0 + 8 * a);
      }
      if (!ok && it > 0) {
        const int i = it - 1;  // the last commit covers every earlier MMA
        mbar_wait_drain(empty0 + 8 * (i % S), (i / S) & 1);
      }
    }
  } else {
    // ---------------- epilogue warps
    const int q = warp & 3;  // tensor-memory lane quarter this warp may access
    uint8_t* bufs = epi + (warp - 2) * 2 * Cfg::EPI_BUF;
    int t = 0, nbuf = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++t) {
      const int mt = tile % num_m, nt = tile / num_m;
      const int a = t & 1;
      const uint32_t aph = (t >> 1) & 1;
      if (!warp_wait(accf0 + 8 * a, aph, ab, kErrWaitMma)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * BN;
      const int row0 = mt * BM + q * 32;
#pragma unroll 1
      for (int c = 0; c < BN / 64; ++c) {
        uint32_t r0[32], r1[32];
        tmem_ld32x2(tb + c * 64, tb + c * 64 + 32, r0, r1);
        uint8_t* buf = bufs + (nbuf & 1) * Cfg::EPI_BUF;
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        uint8_t* rowp = buf + lane * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(r0[8 * j + 0]), __uint_as_float(r0[8 * j + 1]));
          v.y = pack_bf16x2(__uint_as_float(r0[8 * j + 2]), __uint_as_float(r0[8 * j + 3]));
          v.z = pack_bf16x2(__uint_as_float(r0[8 * j + 4]), __uint_as_float(r0[8 * j + 5]));
          v.w = pack_bf16x2(__uint_as_float(r0[8 * j + 6]), __uint_as_float(r0[8 * j + 7]));
          *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) = v;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(r1[8 * j + 0]), __uint_as_float(r1[8 * j + 1]));
          v.y = pack_bf16x2(__uint_as_float(r1[8 * j + 2]), __uint_as_float(r1[8 * j + 3]));
          v.z = pack_bf16x2(__uint_as_float(r1[8 * j + 4]), __uint_as_float(r1[8 * j + 5]));
          v.w = pack_bf16x2(__uint_as_float(r1[8 * j + 6]), __uint_as_float(r1[8 * j + 7]));
          *reinterpret_cast<uint4*>(rowp + (((j + 4) ^ (lane & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < M) {
          tma_store_2d(&tmC, smem_u32(buf), nt * BN + c * 64, row0);
          bulk_commit_group();
        }
        ++nbuf;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce0 + 8 * a);
    }
    if (lane == 0) bulk_wait_group<0>();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
}

}  // namespace mla
