// gemm_w8t.cuh -- bf16 activations x block-scaled e4m3 weights on CTA pairs
// (tcgen05, sm_100a), computed transposed so that the converted weights are
// the tensor-memory A operand:
//
//   C[r, f] = sum_k X[r, k] * bf16(code(f, k) * s(f / 128, k / 128))
//
//   X     bf16 activations [R, K] (K contiguous)
//   code  e4m3 weight codes, stored [F, K] (K contiguous) or, with
//         W_F_MAJOR, [K, F] (F contiguous); one fp32 scale per 128 x 128
//         block (Kimi K2 "Down projection": fmt e4m3, weight_block_size
//         [128, 128])
//   C     bf16 [R, F]; with V_F16 the second 128 features of every 256 (the v
//         half of a head of the up-projection) are stored as f16
//
// The weight element is rounded to bf16 once, as code * scale in fp32: the
// same operand a dequantised bf16 copy would hold, so the products and
// the fp32 accumulation are those of the bf16 GEMM on that copy.
//
// The pair computes D = W_tile . X_tile^T with one M = 256 UMMA per K step:
// CTA r holds output features [128r, 128r+128) of the 256-feature tile as
// tensor-memory lanes and the tokens [HN r, HN r + HN) of the token tile as
// its half of the B operand (TMA, K-major, no multicast). Eight converter
// warps per CTA read the e4m3 codes of their 128 features from shared
// memory, scale, round to bf16 and store them into tensor memory (A operand,
// lane = feature, column c = k pair (2c, 2c+1)); they arrive on the leader's
// barrier as the attention's softmax warps do with P, so no converted data
// crosses between the two CTAs. Eight epilogue warps read D (lane = feature,
// column = token); lane pairs trade values so that each lane holds two
// adjacent features of one token, and the warp writes [token][feature] rows
// with plain 32-bit stores (two 64-byte row segments per instruction), so no
// staging buffer is needed.
//
// Two forms:
//   STATIONARY (K <= 512: the up-projection): a pair walks a contiguous range
//     of (feature tile, token tile) units, converts a feature tile's whole K
//     once into 8 x 32 tensor-memory columns and reuses it for every token
//     tile of that feature tile; 256-token units and one D buffer (a
//     128-token form with two D buffers, whose epilogue overlapped the next
//     unit, measured slower: 0.79 against 0.63 ms at 16384 x 32768 x 512).
//   streaming (large K: the output projection): a ring of four A stages
//     converted per K step, each used by the UMMAs of two 192-token tiles
//     (two D slots of 192 columns), which halves the conversion work per
//     FLOP: converting one 64-deep step for 128 features takes about as
//     many issue slots as a 256-token UMMA group lasts. 384-token units in
//     the grouped order of the bf16 GEMM; the epilogue costs ~1 % of a unit.
//
// Roles per CTA (576 threads):
//   warp 0      TMA producer (activation halves, counted on the leader's
//               barrier; weight codes, counted locally)
//   warp 1      tensor-memory allocator (pair); UMMA issuer in the leader
//   warps 2..9  converters: warp w converts lanes 32 (w % 4) .. +31 of
//               tensor memory, K values [32h, 32h+32) of each 64-deep step
//               with h = (w - 2) / 4 (two warps per SM sub-partition, so
//               one's loads overlap the other's arithmetic)
//   warps 10..17 epilogue: lanes 32 (w % 4) .. +31, alternate 32-token
//               chunks ((w - 10) / 4)
#pragma once

#include "gemm2.cuh"
#include "ptx.cuh"

namespace mla {

template <bool W_F_MAJOR_, bool STATIONARY_, bool V_F16_ = false>
struct GemmW8tCfg {
  static constexpr bool W_F_MAJOR = W_F_MAJOR_;
  static constexpr bool STATIONARY = STATIONARY_;
  static constexpr bool V_F16 = V_F16_;
  static constexpr int BM = 256;                    // output features per pair (UMMA M)
  static constexpr int HM = 128;                    // per CTA (tensor-memory lanes)
  static constexpr int BN = STATIONARY ? 256 : 192; // tokens per token tile (UMMA N)
  static constexpr int HN = BN / 2;                 // tokens of a tile whose activations one CTA loads
  static constexpr int NT = STATIONARY ? 1 : 2;     // token tiles per unit (each converted A stage feeds NT UMMA groups)
  static constexpr int BK = 64;
  static constexpr int MAX_K = 512;                 // STATIONARY: the whole K fits the A stages
  static constexpr int A_STAGES = STATIONARY ? MAX_K / BK : 4;  // 32 tensor-memory columns each
  static constexpr int NUM_D = STATIONARY ? 1 : 2;  // D slots of BN columns: one per token tile in flight
  static constexpr int A_COL0 = NUM_D * BN;         // D buffers first, then the A stages
  static_assert(A_COL0 + A_STAGES * 32 <= 512, "tensor-memory budget");
  static constexpr int B_STAGES = STATIONARY ? 8 : 6;  // 16 or 12 KB stages
  static constexpr int B_BYTES = HN * BK * 2;       // bf16 activations of one token tile half
  static constexpr int W_STAGES = 4;
  static constexpr int W_BYTES = HM * BK;           // 8 KB of codes
  static constexpr int CONV_WARPS = 8;               // two per tensor-memory lane quadrant
  static constexpr int EPI_WARPS = 8;               // two per lane quadrant, alternate 32-token chunks
  static constexpr int THREADS = 64 + 32 * (CONV_WARPS + EPI_WARPS);
  static constexpr int GROUP_RT = 8;                // streaming form: token super-tiles per group
  // shared memory: B ring | W ring | barriers
  static constexpr int OFF_W = B_STAGES * B_BYTES;
  static constexpr int OFF_BARS = OFF_W + W_STAGES * W_BYTES;
  static constexpr int NUM_BARS = 2 * B_STAGES + 2 * W_STAGES + 2 * A_STAGES + 2 * NUM_D;
  static constexpr int SMEM_BYTES = 1024 + OFF_BARS + NUM_BARS * 8 + 16;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Scale layout: the weight's block scales, row-major over (row block, column
// block) of the stored [F, K] or [K, F] matrix.
struct GemmW8tArgs {
  const float* scale;
  void* C;  // [R, F] 16-bit output, written with plain stores from the epilogue
  int R, F, K;
  int* err;
};

// warp_wait for the warps that wait long (converters between feature tiles,
// epilogue warps between units): lane 0 sleeps between polls so that the
// polling does not take issue slots from the UMMA issuer and the producer on
// the same SM sub-partitions. Bounded like warp_wait.
__device__ __forceinline__ bool w8t_warp_wait_idle(uint32_t bar, uint32_t parity, const Abort& ab, int code) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) {
    if (!mbar_try_wait(bar, parity)) {
      const uint64_t t0 = global_timer_ns();
      const uint64_t limit = wait_timeout_ns();
      while (true) {
        __nanosleep(256);
        if (mbar_try_wait(bar, parity)) break;
        if (ab.raised()) {
          ok = 0;
          break;
        }
        if (global_timer_ns() - t0 > limit) {
          ab.raise(code);
          ok = 0;
          break;
        }
      }
    }
  }
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

template <class Cfg>
__device__ __forceinline__ void w8t_unit(int u, int num_rt, int num_ft, int& ft, int& rt) {
  if constexpr (Cfg::STATIONARY) {
    ft = u / num_rt;
    rt = u - ft * num_rt;
  } else {
    grouped_tile(u, num_rt, num_ft, Cfg::GROUP_RT, rt, ft);
  }
}

// Units of pair `pair`: STATIONARY takes a contiguous range (so the feature
// tile, and its converted weights, change rarely), the streaming form every
// num_pairs-th unit.
template <class Cfg>
__device__ __forceinline__ void w8t_range(int pair, int num_pairs, int units, int& u0, int& u1, int& step) {
  if constexpr (Cfg::STATIONARY) {
    u0 = static_cast<int>((static_cast<int64_t>(units) * pair) / num_pairs);
    u1 = static_cast<int>((static_cast<int64_t>(units) * (pair + 1)) / num_pairs);
    step = 1;
  } else {
    u0 = pair;
    u1 = units;
    step = num_pairs;
  }
}

// 32 lanes x 16 columns in one store, then wait until it has completed.
__device__ __forceinline__ void w8t_tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// e4m3 -> fp32 with integer operations only (the conversion pipe is as
// slow as MUFU and would set the pace): the code's exponent and mantissa
// bits placed at fp32 bits 20..26, sign at 31, read as a float, equal the
// code's value times 2^-120 exactly, subnormal codes included. A packed
// multiply by 2^120 restores the value (exact), a second one applies the
// block scale (the one rounding of code * scale), and a packed convert
// rounds the pair to bf16. The format's NaN codes (0x7F, 0xFF), which a
// saturating quantizer never produces, come out as 480 * scale.
__device__ __forceinline__ uint32_t e4m3_lo_bits(uint32_t c) {  // code in bits 0..7
  return ((c & 0x80u) << 24) | ((c & 0x7Fu) << 20);
}

__device__ __forceinline__ uint32_t w8t_pair(uint32_t b0, uint32_t b1, float s) {
  float lo = __uint_as_float(b0), hi = __uint_as_float(b1);
  asm("{\n\t.reg .b64 t, u, v;\n\t"
      "mov.b64 t, {%0, %1};\n\t"
      "mov.b64 u, {%2, %2};\n\t"
      "mov.b64 v, {%3, %3};\n\t"
      "mul.rn.f32x2 t, t, u;\n\t"
      "mul.rn.f32x2 t, t, v;\n\t"
      "mov.b64 {%0, %1}, t;\n\t}"
      : "+f"(lo), "+f"(hi)
      : "f"(0x1p120f), "f"(s));
  return pack_bf16x2(lo, hi);
}

// Four codes of one 32-bit word (byte i = k + i) -> two bf16x2 words.
__device__ __forceinline__ void w8t_word(uint32_t w, float s, uint32_t& p01, uint32_t& p23) {
  const uint32_t b0 = ((w & 0x80u) << 24) | ((w & 0x7Fu) << 20);
  const uint32_t b1 = ((w & 0x8000u) << 16) | ((w & 0x7F00u) << 12);
  const uint32_t b2 = ((w & 0x800000u) << 8) | ((w & 0x7F0000u) << 4);
  const uint32_t b3 = (w & 0x80000000u) | ((w & 0x7F000000u) >> 4);
  p01 = w8t_pair(b0, b1, s);
  p23 = w8t_pair(b2, b3, s);
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
gemm_bf16_w8t_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const GemmW8tArgs g) {
  constexpr int BK = Cfg::BK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BARS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
  int* abort_word = reinterpret_cast<int*>(tmem_slot + 1);
  const uint32_t bar0 = smem_u32(bars);
  const uint32_t bfull0 = bar0;                                   // leader, per B stage
  const uint32_t bempty0 = bfull0 + 8 * Cfg::B_STAGES;            // local (UMMA commit)
  const uint32_t wfull0 = bempty0 + 8 * Cfg::B_STAGES;            // local (TMA of codes)
  const uint32_t wempty0 = wfull0 + 8 * Cfg::W_STAGES;            // local (converter warps)
  const uint32_t afull0 = wempty0 + 8 * Cfg::W_STAGES;            // leader (converters of both CTAs)
  const uint32_t aempty0 = afull0 + 8 * Cfg::A_STAGES;            // local (UMMA commit)
  const uint32_t dfull0 = aempty0 + 8 * Cfg::A_STAGES;            // local (UMMA commit)
  const uint32_t dempty0 = dfull0 + 8 * Cfg::NUM_D;               // leader (epilogue warps of both CTAs)

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  if (blockDim.x != Cfg::THREADS || (gridDim.x & 1u) != 0u || g.F % Cfg::BM != 0 || g.K % BK != 0 ||
      (Cfg::STATIONARY && g.K > Cfg::MAX_K)) {
    if (threadIdx.x == 0) atomicCAS(g.err, 0, kErrGeometry);
    return;
  }
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::B_STAGES; ++s) {
      mbar_init(bfull0 + 8 * s, 1);
      mbar_init(bempty0 + 8 * s, 1);
    }
    for (int s = 0; s < Cfg::W_STAGES; ++s) {
      mbar_init(wfull0 + 8 * s, 1);
      mbar_init(wempty0 + 8 * s, Cfg::CONV_WARPS);
    }
    for (int a = 0; a < Cfg::A_STAGES; ++a) {
      mbar_init(afull0 + 8 * a, 2 * Cfg::CONV_WARPS);
      mbar_init(aempty0 + 8 * a, 1);
    }
    for (int d = 0; d < Cfg::NUM_D; ++d) {
      mbar_init(dfull0 + 8 * d, 1);
      mbar_init(dempty0 + 8 * d, 2 * Cfg::EPI_WARPS);
    }
    *abort_word = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW);
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
  const Abort ab{abort_word, g.err};

  const int num_ft = g.F / Cfg::BM;
  constexpr int UT = Cfg::NT * Cfg::BN;  // tokens per unit
  const int num_rt = (g.R + UT - 1) / UT;
  const int units = num_ft * num_rt;
  const int nk = g.K / BK;
  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const int num_pairs = static_cast<int>(gridDim.x) >> 1;
  int u0, u1, ustep;
  w8t_range<Cfg>(pair, num_pairs, units, u0, u1, ustep);
  const int fcta = static_cast<int>(rank) * Cfg::HM;  // this CTA's first feature within a tile

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int itb = 0, itw = 0, prev_ft = -1;
      bool ok = true;
      for (int u = u0; u < u1 && ok; u += ustep) {
        int ft, rt;
        w8t_unit<Cfg>(u, num_rt, num_ft, ft, rt);
        const bool conv = !Cfg::STATIONARY || ft != prev_ft;
        prev_ft = ft;
        const int f0 = ft * Cfg::BM + fcta;
        for (int kb = 0; kb < nk; ++kb) {
          if (conv) {
            const int s = itw % Cfg::W_STAGES;
            if (!(ok = mbar_wait(wempty0 + 8 * s, ((itw / Cfg::W_STAGES) & 1) ^ 1, ab, kErrWaitConsumer))) break;
            const uint32_t dst = smem_u32(smem + Cfg::OFF_W + s * Cfg::W_BYTES);
            mbar_arrive_expect_tx(wfull0 + 8 * s, Cfg::W_BYTES);
            if constexpr (Cfg::W_F_MAJOR)
              tma_load_2d(dst, &tmW, wfull0 + 8 * s, f0, kb * BK);   // box 128 (F) x 64 rows (K)
            else
              tma_load_2d(dst, &tmW, wfull0 + 8 * s, kb * BK, f0);   // box 64 (K) x 128 rows (F)
            ++itw;
          }
          for (int i = 0; i < Cfg::NT && ok; ++i, ++itb) {
            const int s = itb % Cfg::B_STAGES;
            if (!(ok = mbar_wait(bempty0 + 8 * s, ((itb / Cfg::B_STAGES) & 1) ^ 1, ab, kErrWaitConsumer))) break;
            if (leader) mbar_arrive_expect_tx(bfull0 + 8 * s, 2 * Cfg::B_BYTES);
            tma_load_2d_pair(smem_u32(smem + s * Cfg::B_BYTES), &tmX, mapa_shared(bfull0 + 8 * s, 0), kb * BK,
                             rt * UT + i * Cfg::BN + static_cast<int>(rank) * Cfg::HN);
          }
          if (!ok) break;
        }
      }
      if (!ok) spin_ns(2000000);  // let issued loads land before the CTA can exit
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- UMMA issuer (leader CTA only)
      constexpr uint32_t idesc = idesc_bf16_f32(Cfg::BM, Cfg::BN, 0, 0);
      int itb = 0, ita = 0, gen = 0, t = 0, prev_ft = -1;
      bool ok = true;
      for (int u = u0; u < u1 && ok; u += ustep, ++t) {
        int ft, rt;
        w8t_unit<Cfg>(u, num_rt, num_ft, ft, rt);
        if constexpr (Cfg::STATIONARY) {
          if (ft != prev_ft && prev_ft >= 0) {
            // Every UMMA on the previous feature tile's weights is issued:
            // release its A stages to the converters.
            for (int a = 0; a < nk; ++a) umma_commit_pair(aempty0 + 8 * a, 0x3);
            ++gen;
          }
          prev_ft = ft;
        }
        // Token tile i of unit t accumulates in D slot (t NT + i) % NUM_D.
        for (int i = 0; i < Cfg::NT && ok; ++i) {
          const int n = t * Cfg::NT + i;
          ok = mbar_wait(dempty0 + 8 * (n % Cfg::NUM_D), ((n / Cfg::NUM_D) & 1) ^ 1, ab, kErrWaitEpilogue);
        }
        if (!ok) break;
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb, ++ita) {
          const int a = Cfg::STATIONARY ? kb : ita % Cfg::A_STAGES;
          const uint32_t aph = Cfg::STATIONARY ? static_cast<uint32_t>(gen & 1) : ((ita / Cfg::A_STAGES) & 1);
          if (!(ok = mbar_wait(afull0 + 8 * a, aph, ab, kErrWaitConsumer))) break;
          const uint32_t acol = tmem_base + static_cast<uint32_t>(Cfg::A_COL0 + a * 32);
          for (int i = 0; i < Cfg::NT && ok; ++i, ++itb) {
            const int s = itb % Cfg::B_STAGES;
            if (!(ok = mbar_wait(bfull0 + 8 * s, (itb / Cfg::B_STAGES) & 1, ab, kErrWaitTma))) break;
            tc_fence_after();
            const uint32_t sb = smem_u32(smem + s * Cfg::B_BYTES);
            const uint32_t dcol = tmem_base + static_cast<uint32_t>(((t * Cfg::NT + i) % Cfg::NUM_D) * Cfg::BN);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_ts_pair(dcol, acol + k * 8, smem_desc_sw128(sb + k * 32, 16, 1024), idesc, (kb | k) != 0 ? 1u : 0u);
            umma_commit_pair(bempty0 + 8 * s, 0x3);
          }
          if (!ok) break;
          if constexpr (!Cfg::STATIONARY) umma_commit_pair(aempty0 + 8 * a, 0x3);
        }
        if (!ok) break;
        for (int i = 0; i < Cfg::NT; ++i) umma_commit_pair(dfull0 + 8 * ((t * Cfg::NT + i) % Cfg::NUM_D), 0x3);
      }
      if (!ok && itb > 0) {
        const int i = itb - 1;
        mbar_wait_drain(bempty0 + 8 * (i % Cfg::B_STAGES), (i / Cfg::B_STAGES) & 1);
      }
    }
  } else if (warp < 2 + Cfg::CONV_WARPS) {
    // ---------------- converters: warp w converts features 32 (w % 4) + lane
    // of this CTA's 128 (its tensor-memory lanes), K values [32h, 32h+32)
    // of every step
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    const int fr = q * 32 + static_cast<int>(lane);
    const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int itw = 0, ita = 0, gen = 0, prev_ft = -1;
    bool ok = true;
    for (int u = u0; u < u1 && ok; u += ustep) {
      int ft, rt;
      w8t_unit<Cfg>(u, num_rt, num_ft, ft, rt);
      if (Cfg::STATIONARY && ft == prev_ft) continue;
      prev_ft = ft;
      const int fb = (ft * Cfg::BM + fcta) / 128;  // this CTA's feature block (scale index)
      // The block scale of K step kb (one per 128-deep K block), loaded two
      // steps ahead so that its latency stays off the conversion.
      auto scale_at = [&](int kk) -> float {
        if (kk >= nk) return 0.f;
        return Cfg::W_F_MAJOR ? __ldg(g.scale + static_cast<int64_t>((kk * BK) / 128) * (g.F / 128) + fb)
                              : __ldg(g.scale + static_cast<int64_t>(fb) * (g.K / 128) + (kk * BK) / 128);
      };
      float sc_next = scale_at(0), sc_next2 = scale_at(1);
      for (int kb = 0; kb < nk; ++kb, ++itw, ++ita) {
        const float sc = sc_next;
        sc_next = sc_next2;
        sc_next2 = scale_at(kb + 2);
        const int a = Cfg::STATIONARY ? kb : ita % Cfg::A_STAGES;
        const uint32_t eph = Cfg::STATIONARY ? static_cast<uint32_t>((gen & 1) ^ 1)
                                             : (((ita / Cfg::A_STAGES) & 1) ^ 1);
        if (!(ok = w8t_warp_wait_idle(aempty0 + 8 * a, eph, ab, kErrWaitMma))) break;
        const int s = itw % Cfg::W_STAGES;
        if (!(ok = warp_wait(wfull0 + 8 * s, (itw / Cfg::W_STAGES) & 1, ab, kErrWaitTma))) break;
        const uint8_t* ws = smem + Cfg::OFF_W + s * Cfg::W_BYTES;
        uint32_t pk[16];
        if constexpr (Cfg::W_F_MAJOR) {
          // [64 k][128 f] codes, 128-byte rows: a warp reads 32 consecutive
          // bytes of one row per load.
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int k = 32 * h + 2 * c;
            const uint32_t lo = ws[k * 128 + fr];
            const uint32_t hi = ws[(k + 1) * 128 + fr];
            pk[c] = w8t_pair(e4m3_lo_bits(lo), e4m3_lo_bits(hi), sc);
          }
        } else {
          // [128 f][64 k] codes in the 64-byte swizzle: 16-byte chunk j of
          // row f sits at chunk j ^ ((f >> 1) & 3).
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            const int j = 2 * h + jj;
            const uint4 v = *reinterpret_cast<const uint4*>(ws + fr * 64 + ((j ^ ((fr >> 1) & 3)) << 4));
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) w8t_word(w4[i], sc, pk[8 * jj + 2 * i], pk[8 * jj + 2 * i + 1]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(wempty0 + 8 * s);  // the codes are in registers
        w8t_tmem_st16(trow + static_cast<uint32_t>(Cfg::A_COL0 + a * 32 + 16 * h), pk);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(mapa_shared(afull0 + 8 * a, 0));
      }
      ++gen;
    }
  } else {
    // ---------------- epilogue: warp w turns features 32 (w % 4) + lane of D
    // into 16-bit values of [token][feature] staging rows (its own two
    // buffers of 32 tokens x 32 features) and stores them with TMA; the two
    // warps of a lane quadrant take alternate 32-token chunks
    const int q = warp & 3;
    const int e = (warp - 2 - Cfg::CONV_WARPS) >> 2;
    const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const bool f16 = Cfg::V_F16 && rank == 1;  // features 128..255 of the tile: v of one head
    float vmax = 0.f;
    int t = 0;
    bool ok = true;
    for (int u = u0; u < u1 && ok; u += ustep, ++t) {
      int ft, rt;
      w8t_unit<Cfg>(u, num_rt, num_ft, ft, rt);
      for (int i = 0; i < Cfg::NT && ok; ++i) {
        const int n = t * Cfg::NT + i;
        const int d = n % Cfg::NUM_D;
        if (!(ok = w8t_warp_wait_idle(dfull0 + 8 * d, (n / Cfg::NUM_D) & 1, ab, kErrWaitMma))) break;
        tc_fence_after();
        const int tok0 = rt * UT + i * Cfg::BN;
        // Chunks of tokens past R are skipped whole.
        const int chunks = min(Cfg::BN / 32, (g.R - tok0 + 31) / 32);
#pragma unroll 1
        for (int c = e; c < chunks; c += 2) {
          uint32_t v[32];
          tmem_ld32(trow + static_cast<uint32_t>(d * Cfg::BN + c * 32), v);
          // Lanes 2m and 2m+1 (features f, f+1) trade one value per two
          // tokens, so that the even lane holds token j of both features and
          // the odd lane token j+1; each store instruction of the warp then
          // writes two 64-byte row segments (32 features of tokens j, j+1).
          const bool odd = lane & 1u;
          const int tok = tok0 + c * 32 + (odd ? 1 : 0);
          uint32_t* dst = reinterpret_cast<uint32_t*>(g.C) + (static_cast<int64_t>(tok) * g.F + ft * Cfg::BM + fcta +
                                                              q * 32 + 2 * static_cast<int>(lane >> 1)) / 2;
          const int64_t row_words = g.F / 2;
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float mine_keep = __uint_as_float(odd ? v[j + 1] : v[j]);
            const float mine_give = __uint_as_float(odd ? v[j] : v[j + 1]);
            const float other = __shfl_xor_sync(0xffffffffu, mine_give, 1);
            const float lo = odd ? other : mine_keep;  // feature f (the even lane's)
            const float hi = odd ? mine_keep : other;  // feature f + 1
            if (f16) vmax = max3(vmax, fabsf(lo), fabsf(hi));
            if (tok + j < g.R) dst[j * row_words] = f16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(mapa_shared(dempty0 + 8 * d, 0));
      }
    }
    if (Cfg::V_F16 && __any_sync(0xffffffffu, vmax >= kF16Overflow) && lane == 0) atomicCAS(g.err, 0, kErrRangeF16);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the leader's UMMAs read the peer's shared and tensor memory until here
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
}

}  // namespace mla
