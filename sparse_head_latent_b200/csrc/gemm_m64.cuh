// gemm_m64.cuh -- split-K tcgen05 GEMM for a few rows (the decode step's
// output projection) on sm_100a:
//
//   part[s][m, n] = sum over k in K range s of A[m, k] * B[k, n]   (fp32)
//   out[m, n]     = bf16(sum over s of part[s][m, n])             (sum_splits_kernel)
//
//   A bf16 [M, K] (K contiguous), M small; B bf16 [K, N] (N contiguous).
//
// With one sequence per row, M is the batch (64 at the decode workload): the
// 256-row tiles of the pair GEMM were three quarters zero fill, and with 56
// column tiles only 112 SMs streamed the 235 MB weight, each keeping about
// 48 KB of it in flight (≈ 2.6 TB/s in all). Here each work item is a 64-row
// tile x 128 columns x one K range, the UMMA has M = 64 (cta_group::1), every
// staged byte of B is a weight byte, and eight 24 KB stages keep 128 KB of
// weights in flight per SM; the K ranges give every SM work.
//
// For 64 < M <= 128 the tiles have 128 rows (UMMA M = 128), so that the
// weight is still streamed once.
//
// The same kernel runs the decode step's per-head GEMMs (the absorption of
// q_nope into W_UK and the un-absorption of o_lat through W_UV) as a batch:
// item z of the batch reads A columns, B rows and writes C columns at offsets
// z * step (M64Batch), stores bf16 directly, and may read B K-major.
//
// Roles (192 threads, one CTA per SM, persistent over the work items):
//   warp 0      TMA producer
//   warp 1      tensor-memory allocator (256 columns: two accumulators) and
//               UMMA issuer
//   warps 2..5  epilogue: an M = 64 accumulator occupies lanes 0..15 of each
//               sub-partition, so warp w stores rows [16 (w % 4), +16); an
//               M = 128 one all 32 lanes, rows [32 (w % 4), +32)
#pragma once

#include "ptx.cuh"

namespace mla {

// B_MN_MAJOR_: B stored [K, N] (N contiguous; two 64-column boxes per
// stage) or [N, K] (K contiguous; one 128-row box). OUT_BF16_: items write
// bf16 C columns directly instead of fp32 partial planes.
template <int BM_, bool B_MN_MAJOR_ = true, bool OUT_BF16_ = false>
struct GemmM64Cfg {
  static_assert(BM_ == 64 || BM_ == 128, "row tile");
  static constexpr int BM = BM_, BN = 128, BK = 64;
  static constexpr bool B_MN_MAJOR = B_MN_MAJOR_;
  static constexpr bool OUT_BF16 = OUT_BF16_;
  static constexpr int STAGES = BM_ == 64 ? 8 : 6;
  static constexpr int A_BYTES = BM * BK * 2;   // 8 or 16 KB
  static constexpr int B_BYTES = BK * BN * 2;   // 16 KB: two [64 K rows x 64 columns] boxes
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int NUM_BARS = 2 * STAGES + 4;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + NUM_BARS * 8 + 16;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 256;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Item z of the z dimension (a K range of a split-K GEMM, or a head of a
// batch): A columns from z * a_step, B rows from b_row0 + z * b_step (K rows
// for an N-major B, N rows for a K-major one), output fp32 plane z of `part`
// [count][M][N], or bf16 columns from z * c_step of `out` (row pitch ldc).
struct M64Batch {
  int count;
  int a_step, b_row0, b_step;
  int c_step, ldc;
};

// Work item i = ((z * num_n) + nt) * num_m + mt; each item runs K columns of A.
template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
gemm_m64_splitk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M,
                       int N, int K, const M64Batch bt, float* __restrict__ part, __nv_bfloat16* __restrict__ out,
                       int* err) {
  constexpr int BK = Cfg::BK, S = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * Cfg::STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
  int* abort_word = reinterpret_cast<int*>(tmem_slot + 1);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + S);
  const uint32_t accf0 = smem_u32(bars + 2 * S), acce0 = smem_u32(bars + 2 * S + 2);
  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf0 + 8 * a, 1);
      mbar_init(acce0 + 8 * a, 4);  // the four epilogue warps
    }
    *abort_word = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
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

  const int num_m = (M + Cfg::BM - 1) / Cfg::BM;
  const int num_n = N / Cfg::BN;
  const int items = num_m * num_n * bt.count;
  const int num_kb = K / BK;  // K a multiple of BK (host-checked)

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
        const int mt = item % num_m, nt = (item / num_m) % num_n, sp = item / (num_m * num_n);
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(empty0 + 8 * s, ((it / S) & 1) ^ 1, ab, kErrWaitConsumer)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8 * s;
          mbar_arrive_expect_tx(fb, Cfg::STAGE_BYTES);
          const uint32_t sa = smem_u32(smem + s * Cfg::STAGE_BYTES);
          const uint32_t sb = sa + Cfg::A_BYTES;
          const int k = kb * BK;
          tma_load_2d(sa, &tmA, fb, sp * bt.a_step + k, mt * Cfg::BM);  // rows past M read as zero
          if constexpr (Cfg::B_MN_MAJOR) {
            const int kr = bt.b_row0 + sp * bt.b_step + k;
            tma_load_2d(sb, &tmB, fb, nt * Cfg::BN, kr);
            tma_load_2d(sb + BK * 128, &tmB, fb, nt * Cfg::BN + 64, kr);
          } else {
            tma_load_2d(sb, &tmB, fb, k, bt.b_row0 + sp * bt.b_step + nt * Cfg::BN);  // box 64 K x 128 N rows
          }
        }
      }
      if (!ok) spin_ns(2000000);  // let issued loads land before the CTA can exit
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- UMMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(Cfg::BM, Cfg::BN, 0, Cfg::B_MN_MAJOR ? 1 : 0);
      int it = 0, t = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < items && ok; item += gridDim.x, ++t) {
        const int a = t & 1;
        if (!mbar_wait(acce0 + 8 * a, ((t >> 1) & 1) ^ 1, ab, kErrWaitEpilogue)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + a * Cfg::BN;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(full0 + 8 * s, (it / S) & 1, ab, kErrWaitTma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * Cfg::STAGE_BYTES);
          const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_ss(d, smem_desc_sw128(sa + k * 32, 16, 1024),
                    Cfg::B_MN_MAJOR ? smem_desc_sw128(sb + k * 16 * 128, BK * 128, 1024)
                                    : smem_desc_sw128(sb + k * 32, 16, 1024),
                    idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit(empty0 + 8 * s);
        }
        if (!ok) break;
        umma_commit(accf0 + 8 * a);
      }
      if (!ok && it > 0) {
        const int i = it - 1;
        mbar_wait_drain(empty0 + 8 * (i % S), (i / S) & 1);
      }
    }
  } else {
    // ---------------- epilogue: rows [16q, 16q+16) of the tile in lanes 0..15
    // (M = 64) or [32q, 32q+32) in all lanes (M = 128)
    constexpr int RPW = Cfg::BM / 4;  // rows per warp
    const int q = warp & 3;
    int t = 0;
    for (int item = blockIdx.x; item < items; item += gridDim.x, ++t) {
      const int mt = item % num_m, nt = (item / num_m) % num_n, sp = item / (num_m * num_n);
      const int a = t & 1;
      if (!warp_wait(accf0 + 8 * a, (t >> 1) & 1, ab, kErrWaitMma)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * Cfg::BN;
      const int row = mt * Cfg::BM + RPW * q + static_cast<int>(lane);
#pragma unroll 1
      for (int c = 0; c < Cfg::BN; c += 32) {
        uint32_t v[32];
        tmem_ld32(tb + c, v);
        if (static_cast<int>(lane) < RPW && row < M) {
          if constexpr (Cfg::OUT_BF16) {
            uint4* d4 = reinterpret_cast<uint4*>(out + static_cast<size_t>(row) * bt.ldc + sp * bt.c_step +
                                                 nt * Cfg::BN + c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              d4[i] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * i]), __uint_as_float(v[8 * i + 1])),
                                 pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
                                 pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
                                 pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])));
          } else {
            float4* d4 = reinterpret_cast<float4*>(part + (static_cast<size_t>(sp) * M + row) * N + nt * Cfg::BN + c);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              d4[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                  __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce0 + 8 * a);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
}

// out[m, n] = bf16(sum over s < splits of part[s][m, n]); one thread per 4 columns.
__global__ void __launch_bounds__(256)
sum_splits_kernel(const float* __restrict__ part, int M, int N, int splits, __nv_bfloat16* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const int64_t total = static_cast<int64_t>(M) * N / 4;
  if (i >= total) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const int64_t plane = static_cast<int64_t>(M) * N / 4;
  for (int s = 0; s < splits; ++s) {
    const float4 v = reinterpret_cast<const float4*>(part)[s * plane + i];
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  reinterpret_cast<uint2*>(out)[i] = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
}

}  // namespace mla
