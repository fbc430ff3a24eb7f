// gemm_m64.cuh -- tcgen05 GEMM for a few rows (M <= 256: the decode step,
// one row per sequence) on sm_100a. Two modes:
//
// Stream-K (the output projection, A bf16 [M, K], B bf16 [K, N] N-contiguous):
//   the (row tile, 128-column tile) tiles' 64-deep k-blocks, tile by tile, are
//   cut into gridDim.x contiguous equal shares, one per CTA; a CTA's share
//   covers the end of one tile, whole tiles, and the start of another, and
//   each such segment writes an fp32 partial tile, slot c + t for CTA c and
//   tile t (distinct: along a CTA's shares either c or t grows);
//     out[m, n] = bf16(sum over the segments of tile(m, n), by increasing c)
//   (sum_segments_kernel; deterministic for a given grid).
//
// Batch (the per-head absorption of q_nope into W_UK and un-absorption of
//   o_lat through W_UV): item z reads A columns, B rows and writes bf16 C
//   columns at offsets z * step (M64Batch); B N-major or K-major.
//
// With one sequence per row, M is the batch (64 at the decode workload): the
// 256-row tiles of the pair GEMM were three quarters zero fill, and with 56
// column tiles only 112 SMs streamed the 235 MB weight, each keeping about
// 48 KB of it in flight (≈ 2.6 TB/s in all). Here the UMMA has M = 64
// (cta_group::1; M = 128 tiles for 64 < M <= 256), every staged byte of B is
// a weight byte, and eight 24 KB stages keep 128 KB of weights in flight per
// SM. Equal shares matter: with whole K ranges as work items (448 of them
// over 148 SMs) the last of four rounds ran on four SMs (51.5 us for the
// 64 x 16384 x 7168 projection against 43.7 us with 280 items).
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
// stage) or [N, K] (K contiguous; one 128-row box). BATCH_: batch mode with
// bf16 C, else stream-K with fp32 partial tiles.
template <int BM_, bool B_MN_MAJOR_ = true, bool BATCH_ = false>
struct GemmM64Cfg {
  static_assert(BM_ == 64 || BM_ == 128, "row tile");
  static constexpr int BM = BM_, BN = 128, BK = 64;
  static constexpr bool B_MN_MAJOR = B_MN_MAJOR_;
  static constexpr bool BATCH = BATCH_;
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

// Batch mode: item z reads A columns from z * a_step and B rows from
// b_row0 + z * b_step (K rows for an N-major B, N rows for a K-major one) and
// writes bf16 columns from z * c_step of `out` (row pitch ldc). Stream-K
// mode: count = 1, all offsets 0.
struct M64Batch {
  int count;
  int a_step, b_row0, b_step;
  int c_step, ldc;
};

// First k-block unit of CTA c's share when `units` are cut into g shares.
__host__ __device__ __forceinline__ int64_t stream_k_start(int c, int64_t units, int g) {
  return static_cast<int64_t>(c) * units / g;
}

// One segment of a CTA's work: tile (mt, nt) of batch item z, k-blocks
// [kb0, kb1), output slot (partial tile c + t in stream-K mode).
struct M64Seg {
  int mt, nt, z, kb0, kb1, slot;
};

// The CTA's segments in order. Batch mode: items blockIdx.x + j gridDim.x,
// item i = ((z * num_n) + nt) * num_m + mt, each over all of K. Stream-K:
// units u = t * nkb + kb with tile t = nt * num_m + mt, CTA c taking
// [stream_k_start(c), stream_k_start(c + 1)).
struct M64Work {
  int num_m, num_n, nkb;
  bool batch;
  int item, items;    // batch
  int64_t u, u1;      // stream-K
  __device__ M64Work(int M, int N, int K, int count, int bm, bool batch_) : batch(batch_) {
    num_m = (M + bm - 1) / bm;
    num_n = N / 128;
    nkb = K / 64;
    items = num_m * num_n * count;
    item = blockIdx.x;
    const int64_t units = static_cast<int64_t>(num_m) * num_n * nkb;
    u = stream_k_start(blockIdx.x, units, gridDim.x);
    u1 = stream_k_start(blockIdx.x + 1, units, gridDim.x);
  }
  __device__ bool next(M64Seg& s) {
    if (batch) {
      if (item >= items) return false;
      s.mt = item % num_m;
      s.nt = (item / num_m) % num_n;
      s.z = item / (num_m * num_n);
      s.kb0 = 0;
      s.kb1 = nkb;
      s.slot = s.z;
      item += gridDim.x;
      return true;
    }
    if (u >= u1) return false;
    const int t = static_cast<int>(u / nkb);
    s.mt = t % num_m;
    s.nt = t / num_m;
    s.z = 0;
    s.kb0 = static_cast<int>(u - static_cast<int64_t>(t) * nkb);
    const int64_t end = u1 - static_cast<int64_t>(t) * nkb;
    s.kb1 = end < nkb ? static_cast<int>(end) : nkb;
    s.slot = static_cast<int>(blockIdx.x) + t;
    u = static_cast<int64_t>(t) * nkb + s.kb1;
    return true;
  }
};

// Stream-K mode writes `part` [gridDim.x + tiles][BM][128] fp32 (slots of
// rows past M are left unwritten); batch mode writes `out`.
template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
gemm_m64_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
                int K, const M64Batch bt, float* __restrict__ part, __nv_bfloat16* __restrict__ out, int* err) {
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

  // K, N multiples of BK, BN (host-checked)
  M64Work work(M, N, K, bt.count, Cfg::BM, Cfg::BATCH);
  M64Seg sg;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int it = 0;
      bool ok = true;
      while (ok && work.next(sg)) {
        const int mt = sg.mt, nt = sg.nt, sp = sg.z;
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
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
      for (; ok && work.next(sg); ++t) {
        const int a = t & 1;
        if (!mbar_wait(acce0 + 8 * a, ((t >> 1) & 1) ^ 1, ab, kErrWaitEpilogue)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + a * Cfg::BN;
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
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
                    idesc, (kb != sg.kb0 || k != 0) ? 1u : 0u);
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
    for (; work.next(sg); ++t) {
      const int mt = sg.mt, nt = sg.nt, sp = sg.z;
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
          if constexpr (Cfg::BATCH) {
            uint4* d4 = reinterpret_cast<uint4*>(out + static_cast<size_t>(row) * bt.ldc + sp * bt.c_step +
                                                 nt * Cfg::BN + c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              d4[i] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * i]), __uint_as_float(v[8 * i + 1])),
                                 pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
                                 pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
                                 pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])));
          } else {
            float4* d4 = reinterpret_cast<float4*>(
                part + (static_cast<size_t>(sg.slot) * Cfg::BM + (row - mt * Cfg::BM)) * Cfg::BN + c);
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

// out[m, n] = bf16(sum of the stream-K partial tiles of tile (m / bm, n / 128)
// over the CTAs c whose share meets it, by increasing c); `ctas` is the GEMM's
// grid. One block per tile and 16 rows of it: thread 0 lists the tile's CTAs
// (at most ctas / tiles + 2 of them, since every share holds at least
// tiles * nkb / ctas units), then each thread adds two float4 columns.
constexpr int kSumRows = 16;
constexpr int kSumMaxParts = 64;
__global__ void __launch_bounds__(256)
sum_segments_kernel(const float* __restrict__ part, int M, int N, int K, int bm, int ctas,
                    __nv_bfloat16* __restrict__ out, int* err) {
  __shared__ int parts[kSumMaxParts];
  __shared__ int nparts;
  const int num_m = (M + bm - 1) / bm, nkb = K / 64;
  const int chunks = bm / kSumRows;
  const int t = blockIdx.x / chunks, r0 = (blockIdx.x % chunks) * kSumRows;
  const int mt = t % num_m, nt = t / num_m;
  if (threadIdx.x == 0) {
    const int64_t units = static_cast<int64_t>(num_m) * (N / 128) * nkb;
    const int64_t lo = static_cast<int64_t>(t) * nkb, hi = lo + nkb;
    int c = static_cast<int>(lo * ctas / units);  // the CTA whose share holds unit lo
    while (c + 1 < ctas && stream_k_start(c + 1, units, ctas) <= lo) ++c;
    int n = 0;
    for (; c < ctas; ++c) {
      const int64_t s0 = stream_k_start(c, units, ctas), s1 = stream_k_start(c + 1, units, ctas);
      if (s0 >= hi) break;
      if ((s1 < hi ? s1 : hi) <= (s0 > lo ? s0 : lo)) continue;  // an empty share
      if (n == kSumMaxParts) {
        atomicCAS(err, 0, kErrGeometry);
        break;
      }
      parts[n++] = c;
    }
    nparts = n;
  }
  __syncthreads();
  const int n = nparts;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int q = threadIdx.x + 256 * h;  // float4 index in the 16 x 128 block
    const int r = r0 + q / 32, col = (q % 32) * 4;
    const int m = mt * bm + r;
    if (m >= M) continue;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = 0; i < n; ++i) {
      const float4 v =
          *reinterpret_cast<const float4*>(part + (static_cast<size_t>(parts[i] + t) * bm + r) * 128 + col);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    *reinterpret_cast<uint2*>(out + static_cast<size_t>(m) * N + nt * 128 + col) =
        make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
  }
}

}  // namespace mla
