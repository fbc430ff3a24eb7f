// gemm2.cuh -- persistent tcgen05 GEMM on CTA pairs (cta_group::2) for sm_100a:
// C[M,N] = A[M,K] * B, bf16 operands, fp32 accumulation in tensor memory,
// bf16 output.
//
// A cluster of two CTAs on two SMs computes one 256 x 256 output tile with a
// single M=256, N=256 UMMA per K step, issued by the leader CTA (rank 0):
//   CTA r holds A rows [128r, 128r+128) and B columns [128r, 128r+128) of
//   the tile (each CTA TMA-loads its own halves; nothing is multicast), and
//   its tensor memory receives D rows [128r, 128r+128).
// Per SM this moves (128 + 128) x K operand elements for a 128 x 256 share
// of the output, a third less L2->SM traffic than a 128 x 256 tile with a
// single CTA, which is what bounds the output projection.
//
// Roles per CTA (192 threads), as in the single-CTA kernel:
//   warp 0      TMA producer for this CTA's halves; completion is counted on
//               the leader's full barrier
//   warp 1      tensor-memory allocator (both CTAs, cta_group::2); UMMA
//               issuer in the leader only; commits arrive on both CTAs
//   warps 2..5  epilogue on this CTA's 128 rows; releases the accumulator
//               by arriving on the leader's barrier
#pragma once

#include "ptx.cuh"

namespace mla {

// V_F16: the output columns [128, 256) of every 256-column tile are stored
// as f16 instead of bf16. With N = H*256 that is the v half of each head of
// the up-projection, which the attention kernel consumes as f16.
// BN_: output tile width per pair, 256 or 128.
template <bool B_MN_MAJOR_, bool V_F16_ = false, int BN_ = 256>
struct Gemm2Cfg {
  static_assert(BN_ == 256 || BN_ == 128, "tile width");
  static constexpr int BM = 256;       // per CTA pair
  static constexpr int BN = BN_;       // per CTA pair
  static constexpr int HM = 128;       // A rows per CTA
  static constexpr int HN = BN_ / 2;   // B columns per CTA
  static constexpr int BK = 64;
  static constexpr bool B_MN_MAJOR = B_MN_MAJOR_;
  static constexpr bool V_F16 = V_F16_;
  static constexpr int STAGES = 6;
  static constexpr int GROUP_M = 8;             // row tiles per group of the tile order (grouped_tile)
  static constexpr int A_BYTES = HM * BK * 2;   // 16 KB
  static constexpr int B_BYTES = HN * BK * 2;   // 16 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_WARPS = 4;
  static constexpr int EPI_BUF = 32 * 128;
  static constexpr int EPI_BYTES = EPI_WARPS * 2 * EPI_BUF;
  static constexpr int NUM_BARS = 2 * STAGES + 4;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + NUM_BARS * 8 + 16;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr uint32_t TMEM_COLS = 512;   // two 256-column accumulators
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// A batch of independent GEMMs with the same M, N, K that differ only in
// where their operands sit in the three tensor maps: GEMM i reads A at
// column a_col0 + i * a_col_step, B at row b_row0 + i * b_row_step (rows are
// N for a K-major B, K for an N-major B) and writes C at column
// c_col0 + i * c_col_step. One plain GEMM is {1, 0, 0, 0, 0, 0, 0}.
struct GemmBatch {
  int count;
  int a_col0, a_col_step;
  int b_row0, b_row_step;
  int c_col0, c_col_step;
};

// K-split of the last, partial wave of tiles (one plain GEMM only). When the
// tile count T is not a multiple of the pair count P, the R = T mod P tiles
// of the last wave would run on R pairs while the others idle. Instead the
// T - R tiles of the whole waves run as usual and each of the R last tiles is
// cut into `split` contiguous K ranges: pair p < R * split takes tile
// T - R + p / split, range p % split, and writes its fp32 partial tile to
// slot p of `part` (SPLIT_SLOT_FLOATS floats per slot). gemm_split_sum_kernel
// then adds each tile's partials in range order into C. tail == 0: no split.
struct GemmSplit {
  float* part;
  int tail;   // R
  int split;  // K ranges per tile (>= 2 when tail > 0)
};
constexpr int SPLIT_SLOT_FLOATS = 256 * 256;  // one 256 x 256 tile
constexpr GemmSplit kNoSplit = {nullptr, 0, 0};

// Spin for about `ns` nanoseconds (used only to let in-flight copies land on
// the abort path, where this CTA cannot observe the leader's barrier).
__device__ __forceinline__ void spin_ns(uint64_t ns) {
  const uint64_t t0 = global_timer_ns();
  while (global_timer_ns() - t0 < ns) {
  }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
gemm_bf16_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, int M, int N, int K, const GemmBatch bt,
                     const GemmSplit sk, int* err) {
  constexpr int BK = Cfg::BK, S = Cfg::STAGES;
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
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf0 + 8 * a, 1);
      mbar_init(acce0 + 8 * a, 2 * Cfg::EPI_WARPS);  // epilogue warps of both CTAs
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
    tmem_alloc_pair(smem_u32(tmem_slot), Cfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Abort ab{abort_word, err};

  const int num_m = (M + Cfg::BM - 1) / Cfg::BM;
  const int num_n = N / Cfg::BN;
  const int num_tiles = num_m * num_n * bt.count;
  const int num_kb = K / BK;
  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const int num_pairs = static_cast<int>(gridDim.x) >> 1;
  // This pair's work items: its whole tiles of the full waves, then (with a
  // K-split tail) one K range of a last-wave tile. Item i gives the tile and
  // the K-block range [kb0, kb1); the result says whether it is a K range.
  const int full_end = num_tiles - sk.tail;
  const int n_whole = pair < full_end ? (full_end - 1 - pair) / num_pairs + 1 : 0;
  const int n_items = n_whole + (pair < sk.tail * sk.split ? 1 : 0);
  auto item = [&](int i, int& tile, int& kb0, int& kb1) {
    if (i < n_whole) {
      tile = pair + i * num_pairs;
      kb0 = 0;
      kb1 = num_kb;
      return false;
    }
    const int r = pair % sk.split;
    tile = full_end + pair / sk.split;
    kb0 = r * num_kb / sk.split;
    kb1 = (r + 1) * num_kb / sk.split;
    return true;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (this CTA's halves)
      int it = 0;
      bool ok = true;
      for (int i = 0; i < n_items && ok; ++i) {
        int tile, kb0, kb1;
        item(i, tile, kb0, kb1);
        const int bi = tile / (num_m * num_n);
        int mt, nt;
        grouped_tile(tile - bi * num_m * num_n, num_m, num_n, Cfg::GROUP_M, mt, nt);
        const int arow = mt * Cfg::BM + static_cast<int>(rank) * Cfg::HM;
        const int bcol = nt * Cfg::BN + static_cast<int>(rank) * Cfg::HN;
        const int acol0 = bt.a_col0 + bi * bt.a_col_step;
        const int brow0 = bt.b_row0 + bi * bt.b_row_step;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1, ab, kErrWaitConsumer)) {
            ok = false;
            break;
          }
          const uint32_t full_leader = mapa_shared(full0 + 8 * s, 0);
          if (leader) mbar_arrive_expect_tx(full0 + 8 * s, 2 * Cfg::STAGE_BYTES);
          const uint32_t sa = smem_u32(smem + s * Cfg::STAGE_BYTES);
          const uint32_t sb = sa + Cfg::A_BYTES;
          tma_load_2d_pair(sa, &tmA, full_leader, acol0 + kb * BK, arow);
          if constexpr (!Cfg::B_MN_MAJOR) {
            tma_load_2d_pair(sb, &tmB, full_leader, kb * BK, brow0 + bcol);
          } else {
#pragma unroll
            for (int h = 0; h < Cfg::HN / 64; ++h)
              tma_load_2d_pair(sb + h * BK * 128, &tmB, full_leader, bcol + 64 * h, brow0 + kb * BK);
          }
        }
      }
      if (!ok) spin_ns(2000000);  // let issued loads land before the CTA can exit
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- UMMA issuer (leader CTA only)
      constexpr uint32_t idesc = idesc_bf16_f32(Cfg::BM, Cfg::BN, 0, Cfg::B_MN_MAJOR ? 1 : 0);
      int it = 0, t = 0;
      bool ok = true;
      for (int i = 0; i < n_items && ok; ++i, ++t) {
        int tile, kb0, kb1;
        item(i, tile, kb0, kb1);
        const int a = t & 1;
        const uint32_t aph = (t >> 1) & 1;
        if (!mbar_wait(acce0 + 8 * a, aph ^ 1, ab, kErrWaitEpilogue)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + a * 256;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
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
            umma_ss_pair(d, adesc, bdesc, idesc, (kb != kb0 || k != 0) ? 1u : 0u);
          }
          umma_commit_pair(empty0 + 8 * s, 0x3);
        }
        if (!ok) break;
        umma_commit_pair(accf0 + 8 * a, 0x3);
      }
      if (!ok && it > 0) {
        const int i = it - 1;
        mbar_wait_drain(empty0 + 8 * (i % S), (i / S) & 1);
      }
    }
  } else {
    // ---------------- epilogue warps: this CTA's 128 rows of the tile
    const int q = warp & 3;
    uint8_t* bufs = epi + (warp - 2) * 2 * Cfg::EPI_BUF;
    int t = 0, nbuf = 0;
    float vmax = 0.f;  // largest |value| stored as f16 (V_F16)
    for (int i = 0; i < n_items; ++i, ++t) {
      int tile, kb0, kb1;
      const bool ranged = item(i, tile, kb0, kb1);
      const int bi = tile / (num_m * num_n);
      int mt, nt;
      grouped_tile(tile - bi * num_m * num_n, num_m, num_n, Cfg::GROUP_M, mt, nt);
      const int a = t & 1;
      const uint32_t aph = (t >> 1) & 1;
      if (!warp_wait(accf0 + 8 * a, aph, ab, kErrWaitMma)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * 256;
      const int row0 = mt * Cfg::BM + static_cast<int>(rank) * Cfg::HM + q * 32;
      if constexpr (Cfg::BN == 256 && !Cfg::V_F16) {
        if (ranged) {
          // fp32 partial of this warp's 32 rows in slot `pair`, laid out as
          // [64 column quads][32 rows][4] so that every store of the warp
          // covers 512 contiguous bytes.
          float* dst = sk.part + static_cast<size_t>(pair) * SPLIT_SLOT_FLOATS + (rank * 4 + q) * 8192;
#pragma unroll 1
          for (int c = 0; c < 4 && row0 < M; ++c) {
            uint32_t r0[32], r1[32];
            tmem_ld32x2(tb + c * 64, tb + c * 64 + 32, r0, r1);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              *reinterpret_cast<float4*>(dst + ((c * 16 + j) * 32 + lane) * 4) =
                  make_float4(__uint_as_float(r0[4 * j]), __uint_as_float(r0[4 * j + 1]),
                              __uint_as_float(r0[4 * j + 2]), __uint_as_float(r0[4 * j + 3]));
              *reinterpret_cast<float4*>(dst + ((c * 16 + 8 + j) * 32 + lane) * 4) =
                  make_float4(__uint_as_float(r1[4 * j]), __uint_as_float(r1[4 * j + 1]),
                              __uint_as_float(r1[4 * j + 2]), __uint_as_float(r1[4 * j + 3]));
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(mapa_shared(acce0 + 8 * a, 0));
          continue;
        }
      }
      // A warp whose 32 rows all lie past M has nothing to store. It must
      // then skip the staging too: the two staging buffers alternate per
      // issued store, and `wait_group.read 1` before a buffer is rewritten
      // only covers the store two issues back if every staged chunk was
      // stored (otherwise the previous tile's last store could still be
      // reading the buffer being overwritten).
#pragma unroll 1
      for (int c = 0; c < Cfg::BN / 64 && row0 < M; ++c) {
        uint32_t r0[32], r1[32];
        tmem_ld32x2(tb + c * 64, tb + c * 64 + 32, r0, r1);
        uint8_t* buf = bufs + (nbuf & 1) * Cfg::EPI_BUF;
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        uint8_t* rowp = buf + lane * 128;
        const bool f16 = Cfg::V_F16 && c >= 2;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float* f0 = reinterpret_cast<const float*>(r0) + 8 * j;
          const float* f1 = reinterpret_cast<const float*>(r1) + 8 * j;
          uint4 v0, v1;
          if (f16) {
#pragma unroll
            for (int i = 0; i < 8; ++i) vmax = max3(vmax, fabsf(f0[i]), fabsf(f1[i]));
            v0 = make_uint4(pack_f16x2(f0[0], f0[1]), pack_f16x2(f0[2], f0[3]), pack_f16x2(f0[4], f0[5]),
                            pack_f16x2(f0[6], f0[7]));
            v1 = make_uint4(pack_f16x2(f1[0], f1[1]), pack_f16x2(f1[2], f1[3]), pack_f16x2(f1[4], f1[5]),
                            pack_f16x2(f1[6], f1[7]));
          } else {
            v0 = make_uint4(pack_bf16x2(f0[0], f0[1]), pack_bf16x2(f0[2], f0[3]), pack_bf16x2(f0[4], f0[5]),
                            pack_bf16x2(f0[6], f0[7]));
            v1 = make_uint4(pack_bf16x2(f1[0], f1[1]), pack_bf16x2(f1[2], f1[3]), pack_bf16x2(f1[4], f1[5]),
                            pack_bf16x2(f1[6], f1[7]));
          }
          *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) = v0;
          *reinterpret_cast<uint4*>(rowp + (((j + 4) ^ (lane & 7)) << 4)) = v1;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmC, smem_u32(buf), bt.c_col0 + bi * bt.c_col_step + nt * Cfg::BN + c * 64, row0);
          bulk_commit_group();
        }
        ++nbuf;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(mapa_shared(acce0 + 8 * a, 0));
    }
    if (lane == 0) bulk_wait_group<0>();
    if (Cfg::V_F16 && __any_sync(0xffffffffu, vmax >= kF16Overflow) && lane == 0) atomicCAS(err, 0, kErrRangeF16);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the leader's UMMAs read the peer's shared memory until here
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
}

// Second half of the K-split tail (GemmSplit): one thread per 4 output
// columns of one row of a last-wave tile adds the tile's `split` partials in
// K-range order (the same order for every element and every run) and stores
// the bf16 result; rows past M are skipped. Thread e of the launch reads
// element e % 16384 of each of its tile's slots, so the loads of a warp are
// 512 contiguous bytes. C is row-major bf16 with row pitch ldc; the tile
// order is the GEMM's (grouped_tile with group_m row tiles).
__global__ void __launch_bounds__(256)
gemm_split_sum_kernel(const float* __restrict__ part, __nv_bfloat16* __restrict__ C, int M, int ldc, int num_m,
                      int num_n, int group_m, int first_tile, int tail, int split) {
  const int e = static_cast<int>(blockIdx.x) * 256 + static_cast<int>(threadIdx.x);
  if (e >= tail * (SPLIT_SLOT_FLOATS / 4)) return;
  const int t = e / (SPLIT_SLOT_FLOATS / 4);
  const int w = e - t * (SPLIT_SLOT_FLOATS / 4);  // [rank][warp][column quad][row] of the epilogue
  const int row = (w & 31) + 32 * ((w >> 11) & 3) + 128 * (w >> 13);
  const int quad = (w >> 5) & 63;
  int mt, nt;
  grouped_tile(first_tile + t, num_m, num_n, group_m, mt, nt);
  const int grow = mt * 256 + row;
  if (grow >= M) return;
  const float4* p = reinterpret_cast<const float4*>(part) + static_cast<size_t>(t) * split * (SPLIT_SLOT_FLOATS / 4) + w;
  float4 acc = p[0];
  for (int r = 1; r < split; ++r) {
    const float4 v = p[static_cast<size_t>(r) * (SPLIT_SLOT_FLOATS / 4)];
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  *reinterpret_cast<uint2*>(C + static_cast<size_t>(grow) * ldc + nt * 256 + quad * 4) =
      make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
}

}  // namespace mla
