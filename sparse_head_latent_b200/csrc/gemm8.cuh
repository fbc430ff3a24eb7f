// gemm8.cuh -- persistent tcgen05 GEMM on CTA pairs for e4m3 x e4m3 operands
// with fine-grained scales (sm_100a):
//
//   C[m, n] = sum_kb  sa[kb][m] * sw(kb, n / 128) * sum_{k in block kb} A[m, k] * B(k, n)
//
//   A  e4m3 activation codes [M, K] (K contiguous) with one fp32 scale per row
//      and 128-deep K block, stored sa[K / 128][M];
//   B  e4m3 weight codes with one fp32 scale per 128 x 128 block, stored
//      [N, K] (K contiguous) or [K, N] (N contiguous);
//   C  bf16 [M, N]; with V_F16 the odd 128-column tiles (the v half of every
//      head of the up-projection) are stored as f16.
//
// The scale changes with every 128-deep K block, so the tensor core cannot
// accumulate across blocks. It accumulates each K block (four K = 32 UMMAs)
// into its own BN-column fp32 buffer in tensor memory (512 / BN buffers: all
// 512 columns); eight "promotion" warps per CTA load each finished buffer,
// release it, and add it scaled by sa * sw into fp32 registers. After the
// last K block they convert and TMA-store the tile.
//
// Pair tile 256 x BN (BN = 128 or 256): CTA r of the cluster holds A rows
// [128r, 128r+128) and B columns [BN/2 r, BN/2 (r+1)) of the tile; one
// M = 256, N = BN UMMA per K step is issued by the leader; D rows
// [128r, 128r+128) land in CTA r's tensor memory. No load is multicast.
// Per SM and K step the tensor core reads A (4 KB) and its half of B from
// shared memory while TMA writes the next stages: with BN = 128 that is
// about 190 B/clk at the full e4m3 rate, more than shared memory delivers;
// BN = 256 halves the A reads per output and is the shape to use for large
// problems.
//
// Roles per CTA (320 threads; with three warps on two of the four SM
// sub-partitions the register file allows 168 per thread: 128 fp32
// accumulators, a 16-column load and the addressing):
//   warp 0      TMA producer for this CTA's halves (completion counted on the
//               leader's full barrier)
//   warp 1      tensor-memory allocator (pair); UMMA issuer in the leader
//   warps 2..9  promotion + epilogue: warp w reads tensor-memory lanes
//               [32 (w % 4), +32) (its 32 rows) and columns
//               [BN/2 ((w - 2) / 4), +BN/2) of the tile
#pragma once

#include "ptx.cuh"

namespace mla {

template <bool B_MN_MAJOR_, bool V_F16_ = false, int BN_ = 256>
struct Gemm8Cfg {
  static_assert(BN_ == 128 || BN_ == 256, "tile width");
  static constexpr int BM = 256;     // per CTA pair
  static constexpr int BN = BN_;     // per CTA pair
  static constexpr int HM = 128;     // A rows per CTA
  static constexpr int HN = BN_ / 2; // B columns per CTA
  static constexpr int BK = 128;     // e4m3 elements = bytes; one scale block
  static constexpr bool B_MN_MAJOR = B_MN_MAJOR_;
  static constexpr bool V_F16 = V_F16_;
  static constexpr int A_BYTES = HM * BK;   // 16 KB
  static constexpr int B_BYTES = HN * BK;   // 8 or 16 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN_ == 128 ? 6 : 5;
  static constexpr int GROUP_M = 8;          // row tiles per group of the tile order (grouped_tile)
  static constexpr int ACC_BUFS = 512 / BN_;  // BN-column partial buffers
  static constexpr int PROMO_WARPS = 8;
  static constexpr int CW = BN_ / 2;         // columns per promotion warp
  static constexpr int CH = 16;              // columns per tensor-memory load
  static constexpr int SCALE_DEPTH = 2;      // K blocks of scales loaded ahead
  static constexpr int EPI_BUF = 32 * 128;   // 32 rows x 64 bf16 columns
  static constexpr int EPI_BYTES = PROMO_WARPS * 2 * EPI_BUF;
  static constexpr int NUM_BARS = 2 * STAGES + 2 * ACC_BUFS;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + NUM_BARS * 8 + 16;
  static constexpr int THREADS = 64 + 32 * PROMO_WARPS;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Scales of one GEMM: activation scales sa[kb * M + m]; weight block scale
// of K block kb and 128-column block nb at sw[kb * sw_kb + nb * sw_nb].
struct Gemm8Scales {
  const float* sa;
  const float* sw;
  int sw_kb, sw_nb;
};

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
gemm_e4m3_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, int M, int N, int K, const Gemm8Scales sc, int* err) {
  constexpr int BK = Cfg::BK, S = Cfg::STAGES, NB = Cfg::ACC_BUFS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi = smem + S * Cfg::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi + Cfg::EPI_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
  int* abort_word = reinterpret_cast<int*>(tmem_slot + 1);

  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + S);
  const uint32_t pfull0 = smem_u32(bars + 2 * S);        // a K block's partial sum is in buffer b
  const uint32_t pempty0 = smem_u32(bars + 2 * S + NB);  // buffer b has been read (leader's copy counts)
  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(pfull0 + 8 * b, 1);
      mbar_init(pempty0 + 8 * b, 2 * Cfg::PROMO_WARPS);  // promotion warps of both CTAs
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
  const int num_tiles = num_m * num_n;
  const int num_kb = K / BK;
  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const int num_pairs = static_cast<int>(gridDim.x) >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (this CTA's halves)
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        int mt, nt;
        grouped_tile(tile, num_m, num_n, Cfg::GROUP_M, mt, nt);
        const int arow = mt * Cfg::BM + static_cast<int>(rank) * Cfg::HM;
        const int bcol = nt * Cfg::BN + static_cast<int>(rank) * Cfg::HN;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
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
          tma_load_2d_pair(sa, &tmA, full_leader, kb * BK, arow);
          if constexpr (!Cfg::B_MN_MAJOR)
            tma_load_2d_pair(sb, &tmB, full_leader, kb * BK, bcol);   // box 128 (K) x HN rows (N)
          else
            tma_load_2d_pair(sb, &tmB, full_leader, bcol, kb * BK);   // box HN (N) x 128 rows (K)
        }
      }
      if (!ok) spin_ns(2000000);  // let issued loads land before the CTA can exit
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- UMMA issuer (leader CTA only)
      constexpr uint32_t idesc = idesc_e4m3_f32(Cfg::BM, Cfg::BN, 0, Cfg::B_MN_MAJOR ? 1 : 0);
      int it = 0, pc = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        for (int kb = 0; kb < num_kb; ++kb, ++it, ++pc) {
          const int b = pc % NB;
          if (!mbar_wait(pempty0 + 8 * b, ((pc / NB) & 1) ^ 1, ab, kErrWaitEpilogue)) {
            ok = false;
            break;
          }
          const int s = it % S;
          if (!mbar_wait(full0 + 8 * s, (it / S) & 1, ab, kErrWaitTma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * Cfg::STAGE_BYTES);
          const uint32_t sb = sa + Cfg::A_BYTES;
          const uint32_t d = tmem_base + b * Cfg::BN;
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            const uint64_t adesc = smem_desc_sw128(sa + k * 32, 16, 1024);
            // N-major B: HN-byte rows along N (64-byte swizzle for HN = 64,
            // 128-byte for HN = 128), 32 K rows per UMMA; K-major B: 128-byte
            // rows along K, 32 bytes per UMMA.
            uint64_t bdesc;
            if constexpr (!Cfg::B_MN_MAJOR)
              bdesc = smem_desc_sw128(sb + k * 32, 16, 1024);
            else if constexpr (Cfg::HN == 64)
              bdesc = smem_desc_sw64(sb + k * 32 * 64, Cfg::B_BYTES, 512);
            else
              bdesc = smem_desc_sw128(sb + k * 32 * 128, Cfg::B_BYTES, 1024);
            umma_ss_pair_f8(d, adesc, bdesc, idesc, k != 0 ? 1u : 0u);
          }
          umma_commit_pair(empty0 + 8 * s, 0x3);
          umma_commit_pair(pfull0 + 8 * b, 0x3);
        }
      }
      if (!ok && it > 0) {
        const int i = it - 1;
        mbar_wait_drain(empty0 + 8 * (i % S), (i / S) & 1);
      }
    }
  } else {
    // ---------------- promotion + epilogue warps
    constexpr int CW = Cfg::CW, CH = Cfg::CH;
    const int q = warp & 3;
    const int hh = (warp - 2) >> 2;
    uint8_t* bufs = epi + (warp - 2) * 2 * Cfg::EPI_BUF;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + hh * CW;
    int pc = 0, nbuf = 0;
    bool ok = true;
    float vmax = 0.f;  // largest |value| stored as f16 (V_F16)
    for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
      int mt, nt;
      grouped_tile(tile, num_m, num_n, Cfg::GROUP_M, mt, nt);
      const int row0 = mt * Cfg::BM + static_cast<int>(rank) * Cfg::HM + q * 32;
      const int row = row0 + static_cast<int>(lane);
      const bool live = row < M;
      const int col0 = nt * Cfg::BN + hh * CW;   // this warp's columns: one 128-column weight block
      const float* sap = sc.sa + (live ? row : 0);
      const float* swp = sc.sw + static_cast<size_t>(col0 / 128) * sc.sw_nb;
      // The scales of K block kb sit in slot kb % SD, loaded SD blocks ahead
      // (the unrolled loop names the slots statically, so a pending load is
      // only waited for where it is used).
      constexpr int SD = Cfg::SCALE_DEPTH;
      auto sa_at = [&](int kb) { return (live && kb < num_kb) ? __ldg(sap + static_cast<size_t>(kb) * M) : 0.0f; };
      auto sw_at = [&](int kb) { return kb < num_kb ? __ldg(swp + static_cast<size_t>(kb) * sc.sw_kb) : 0.0f; };
      float as[SD], ws[SD];
#pragma unroll
      for (int j = 0; j < SD; ++j) {
        as[j] = sa_at(j);
        ws[j] = sw_at(j);
      }
      float acc[CW];
#pragma unroll
      for (int j = 0; j < CW; ++j) acc[j] = 0.0f;
#pragma unroll 1
      for (int kb0 = 0; kb0 < num_kb && ok; kb0 += SD) {
#pragma unroll
        for (int j = 0; j < SD; ++j) {
          const int kb = kb0 + j;
          if (kb < num_kb) {
            const int b = pc % NB;
            if (!warp_wait(pfull0 + 8 * b, (pc / NB) & 1, ab, kErrWaitMma)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const float f = as[j] * ws[j];
            as[j] = sa_at(kb + SD);
            ws[j] = sw_at(kb + SD);
#pragma unroll
            for (int c = 0; c < CW; c += CH) {
              uint32_t p[CH];
              tmem_ld16(lane_base + b * Cfg::BN + c, p);
#pragma unroll
              for (int i = 0; i < CH; i += 2)
                fma2_acc(acc[c + i], acc[c + i + 1], __uint_as_float(p[i]), __uint_as_float(p[i + 1]), f);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(mapa_shared(pempty0 + 8 * b, 0));
            ++pc;
          }
        }
      }
      if (!ok) break;
      // A warp whose 32 rows all lie past M has nothing to store and skips the
      // staging too (the two staging buffers alternate per issued store).
#pragma unroll
      for (int c = 0; c < CW / 64 && row0 < M; ++c) {
        uint8_t* buf = bufs + (nbuf & 1) * Cfg::EPI_BUF;
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        uint8_t* rowp = buf + lane * 128;
        const bool f16 = Cfg::V_F16 && (((col0 + 64 * c) / 128) & 1);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float* v = acc + 64 * c + 8 * j;
          uint4 u;
          if (f16) {
#pragma unroll
            for (int i = 0; i < 8; i += 2) vmax = max3(vmax, fabsf(v[i]), fabsf(v[i + 1]));
            u = make_uint4(pack_f16x2(v[0], v[1]), pack_f16x2(v[2], v[3]), pack_f16x2(v[4], v[5]),
                           pack_f16x2(v[6], v[7]));
          } else {
            u = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                           pack_bf16x2(v[6], v[7]));
          }
          *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) = u;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmC, smem_u32(buf), col0 + 64 * c, row0);
          bulk_commit_group();
        }
        ++nbuf;
      }
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

}  // namespace mla
