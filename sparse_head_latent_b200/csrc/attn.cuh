// attn.cuh -- fused sparse-causal MLA attention for sm_100a (tcgen05 on CTA
// pairs + TMA).
//
// For one batch b and one head h, over every 128-key block in which a query
// of the work item selected a key (DeepSeek-V3.2-Exp "Sparse attention",
// prefill):
//   S   = q_h . [k_nope_h | k_pe]^T             (UMMA, K = 192, S in tensor memory)
//   S   = -inf where bit(s, t) = 0               (top-k + causal selection)
//   m   = running max of S*scale*log2e per row  (fp32)
//   P   = exp2(S*scale*log2e - m)               (MUFU ex2, fp32; sums in fp32)
//   O  += P . v_h                               (UMMA, P f16 from tensor memory, v f16)
//   attn[b, s, h, :] = O / l                    (bf16)
// Neither the [T, T] scores nor a float mask is ever materialised: the
// selection arrives as one bit per causal (query, key) pair.
//
// Work item: a cluster of two CTAs (a CTA pair) and a group of four
// consecutive 128-query tiles 4g .. 4g+3 of one (b, h). The pair's UMMAs have
// M = 256: "super-tile" A is tiles 4g (rows in CTA 0) and 4g+1 (CTA 1),
// super-tile B is 4g+2 (CTA 0) and 4g+3 (CTA 1). Each CTA loads half of every
// operand the two SMs share: keys [64r, 64r+64) of each K block and value
// columns [64r, 64r+64) of each V block (r = rank in the pair), which halves
// the shared-memory traffic per SM against one CTA per 128 queries. With
// both operands of QK^T in shared memory that traffic, not the tensor core,
// was the bound.
//
// Super-tiles A and B share every K and V block and alternate on the tensor
// core: while the softmax warps of A work on block j, the tensor core runs
// PV of B's block j-1 and QK^T of B's block j, and vice versa ("ping-pong").
// A stops at its last causal block (tile 4g+1); B goes on alone to 4g+3.
//
// CTA = 320 threads:
//   warp 0      TMA producer: this CTA's two Q tiles once; its halves of K
//               (k_nope from the up-projected kv plus the shared k_pe) into
//               a 3-deep ring and of V into a 2-deep ring
//   warp 1      tensor-memory allocator; in CTA 0 also the UMMA issuer of
//               the pair
//   warps 2..5  softmax of this CTA's tile of A, warps 6..9 of its tile of
//               B: one query row per thread (tensor-memory lane = row)
// Tensor memory (each CTA, its own 128 rows): S_A [0,128), O_A [128,256),
// S_B [256,384), O_B [384,512). P (f16 pairs, 64 columns) overwrites the
// first half of S once the softmax has read S; PV reads it from there.
#pragma once

#include "prepass.cuh"
#include "ptx.cuh"

namespace mla {

struct AttnParams {
  int B, T, H, nq;
  int ngroups;                  // groups of four query tiles to run: groups 0 .. ngroups-1
  int gpitch;                   // ceil(nq / 4): groups per batch element in `blocks`
  int hgroup;                   // heads per scheduling group (divides H)
  float scale_log2;             // softmax scale * log2(e)
  const uint4* bitmap;          // selection bitmap, NULL = causal mask only
  const int32_t* blocks;        // active key blocks per tile group (with bitmap)
  __nv_bfloat16* attn;          // [B, T, H, 128]
  // When set, the output is written as dynamic e4m3 activations instead of
  // bf16 (the input of an e4m3 x e4m3 output projection): each (row, head)
  // is one 128-channel group; codes [B*T, H*128], scales [H, B*T].
  uint8_t* attn8;
  float* attn8_s;
  int* err;
};

struct AttnSmem {
  static constexpr int QA = 0;             // 3 x [128 x 64] bf16, 128B-swizzled
  static constexpr int QB = 49152;
  static constexpr int K0 = 98304;         // stage: k_nope 0-63, 64-127, k_pe, each [64 keys x 64]
  static constexpr int K_STAGE = 24576;
  static constexpr int K_STAGES = 3;
  static constexpr int V0 = K0 + K_STAGES * K_STAGE;  // stage: [128 keys x 64 dv] f16
  static constexpr int V_STAGE = 16384;
  static constexpr int V_STAGES = 2;
  static constexpr int BARS = V0 + V_STAGES * V_STAGE;
  static constexpr int NUM_BARS = 17;
  static constexpr int BYTES = 1024 + BARS + 256;
};
static_assert(AttnSmem::BARS % 1024 == 0, "stage alignment");
static_assert(AttnSmem::BYTES <= 232448, "shared memory per CTA");

constexpr int kAttnThreads = 320;

// Tensor-memory columns of super-tile t: S at 256t, O at 256t + 128.
__host__ __device__ constexpr uint32_t tmem_s(int t) { return 256u * t; }
__host__ __device__ constexpr uint32_t tmem_o(int t) { return 256u * t + 128u; }

// Barrier slots (the same offsets in both CTAs). "Leader" barriers live in
// CTA 0 and count both CTAs; the others are local and receive the pair's
// commits by multicast.
enum : int {
  kBarQFull = 0,    // leader: both CTAs' Q tiles landed
  kBarKFull0 = 1,   // leader, per K stage
  kBarKEmpty0 = 4,  // local, per K stage: the UMMAs reading it are done
  kBarVFull0 = 7,   // leader, per V stage
  kBarVEmpty0 = 9,  // local, per V stage
  kBarSFull0 = 11,  // local, per super-tile: S of the current block is in tensor memory
  kBarPFull0 = 13,  // leader, per super-tile: P written by all 8 softmax warps of the pair
  kBarODone = 15,   // local: every UMMA of the pair has completed
  kBarDrain = 16    // leader: drain after an abort
};

__global__ void __launch_bounds__(kAttnThreads, 1)
sparse_mla_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKpe,
                       const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnSmem::BARS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + AttnSmem::NUM_BARS);
  int* abort_word = reinterpret_cast<int*>(tmem_slot + 1);
  const uint32_t bar0 = smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  if (blockDim.x != kAttnThreads || (gridDim.x & 1u) != 0u) {  // every role below assumes this geometry
    if (threadIdx.x == 0) atomicCAS(p.err, 0, kErrGeometry);
    return;
  }
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  // Work item: (batch, head, group of four tiles). Pairs are ordered by
  // groups of `hgroup` heads, so that the pairs resident at any time read
  // the K/V of a few heads and those stay in L2; within a head group, heavy
  // (late) tile groups first.
  const int cl = static_cast<int>(blockIdx.x >> 1);
  const int per_group = p.ngroups * p.B * p.hgroup;
  const int hg = cl / per_group;
  const int rem0 = cl % per_group;
  const int grp = p.ngroups - 1 - rem0 / (p.B * p.hgroup);
  const int rem = rem0 % (p.B * p.hgroup);
  const int b = rem / p.hgroup, h = hg * p.hgroup + rem % p.hgroup;
  const int q0 = 4 * grp;
  // Super-tile t = tiles q0 + 2t (CTA 0) and q0 + 2t + 1 (CTA 1). It exists
  // if its first tile does and visits the blocks of the list up to its last
  // existing tile: a prefix of the list, which is ascending.
  const bool has_b = q0 + 2 < p.nq;
  const int32_t* blist = p.blocks ? p.blocks + (static_cast<int64_t>(b) * p.gpitch + grp) * (p.nq + 2) : nullptr;
  int nA, nB;
  if (blist) {
    nA = blist[1];
    nB = has_b ? blist[0] : 0;
  } else {
    nA = min(q0 + 1, p.nq - 1) + 1;
    nB = has_b ? min(q0 + 3, p.nq - 1) + 1 : 0;
  }
  const int n = max(nA, nB);
  auto kblock = [&](int j) { return blist ? blist[2 + j] : j; };

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQFull), 1);
    for (int i = 0; i < AttnSmem::K_STAGES; ++i) {
      mbar_init(bar(kBarKFull0 + i), 1);
      mbar_init(bar(kBarKEmpty0 + i), 1);
    }
    for (int i = 0; i < AttnSmem::V_STAGES; ++i) {
      mbar_init(bar(kBarVFull0 + i), 1);
      mbar_init(bar(kBarVEmpty0 + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarSFull0 + i), 1);
      mbar_init(bar(kBarPFull0 + i), 8);  // four softmax warps in each CTA of the pair
    }
    mbar_init(bar(kBarODone), 1);
    mbar_init(bar(kBarDrain), 1);
    *abort_word = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmKpe);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Abort ab{abort_word, p.err};

  if (warp == 0) {
    if (lane == 0 && n > 0 && *reinterpret_cast<volatile int*>(&g_mla_withhold_attn_loads) == 0) {
      // ---------------- TMA producer (this CTA's halves; completion is
      // counted on the leader's barriers, which expect both CTAs' bytes)
      int nk = 0, nv = 0;
      bool ok = true;
      const int ntq = has_b ? 2 : 1;
      if (leader) mbar_arrive_expect_tx(bar(kBarQFull), ntq * 2 * 3 * 16384);
      const uint32_t qfull = mapa_shared(bar(kBarQFull), 0);
      for (int t = 0; t < ntq; ++t) {
        const uint32_t sq = smem_u32(smem + (t ? AttnSmem::QB : AttnSmem::QA));
        const int row = (q0 + 2 * t + static_cast<int>(rank)) * 128;  // past T: zero-filled
        for (int c = 0; c < 3; ++c) tma_load_3d_pair(sq + c * 16384, &tmQ, qfull, h * 192 + 64 * c, row, b);
      }
      auto load_k = [&](int j) -> bool {
        const int s = j % AttnSmem::K_STAGES;
        if (!mbar_wait(bar(kBarKEmpty0 + s), ((j / AttnSmem::K_STAGES) & 1) ^ 1, ab, kErrWaitMma)) return false;
        const int r0 = kblock(j) * 128 + static_cast<int>(rank) * 64;
        const uint32_t dst = smem_u32(smem + AttnSmem::K0 + s * AttnSmem::K_STAGE);
        const uint32_t fb = bar(kBarKFull0 + s);
        if (leader) mbar_arrive_expect_tx(fb, 2 * AttnSmem::K_STAGE);
        const uint32_t fbl = mapa_shared(fb, 0);
        tma_load_3d_pair(dst, &tmK, fbl, h * 256, r0, b);
        tma_load_3d_pair(dst + 8192, &tmK, fbl, h * 256 + 64, r0, b);
        tma_load_3d_pair(dst + 16384, &tmKpe, fbl, 0, r0, b);
        ++nk;
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int s = j & 1;
        if (!mbar_wait(bar(kBarVEmpty0 + s), ((j >> 1) & 1) ^ 1, ab, kErrWaitMma)) return false;
        const uint32_t fb = bar(kBarVFull0 + s);
        if (leader) mbar_arrive_expect_tx(fb, 2 * AttnSmem::V_STAGE);
        tma_load_3d_pair(smem_u32(smem + AttnSmem::V0 + s * AttnSmem::V_STAGE), &tmV, mapa_shared(fb, 0),
                         h * 256 + 128 + static_cast<int>(rank) * 64, kblock(j) * 128, b);
        ++nv;
        return true;
      };
      // K runs two blocks ahead, V one: the issuer consumes K_{j+1} before V_j.
      ok = load_k(0) && (n < 2 || load_k(1));
      for (int j = 0; j < n && ok; ++j) {
        if (j + 2 < n && !(ok = load_k(j + 2))) break;
        if (!(ok = load_v(j))) break;
      }
      if (!ok && leader) {
        mbar_wait_drain(bar(kBarQFull), 0);
        for (int i = (nk > AttnSmem::K_STAGES ? nk - AttnSmem::K_STAGES : 0); i < nk; ++i)
          mbar_wait_drain(bar(kBarKFull0 + i % AttnSmem::K_STAGES), (i / AttnSmem::K_STAGES) & 1);
        for (int i = (nv > AttnSmem::V_STAGES ? nv - AttnSmem::V_STAGES : 0); i < nv; ++i)
          mbar_wait_drain(bar(kBarVFull0 + (i & 1)), (i >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0 && n > 0) {
      // ---------------- UMMA issuer of the pair
      // Order per key block j: for each super-tile t, O_t += P_t(j) . V_j as
      // soon as both CTAs' softmax warps have written P_t(j), then
      // S_t(j+1) = Q_t . K_{j+1}^T. The tensor core therefore runs B's
      // PV/QK^T while A's softmax works and vice versa. Every commit covers
      // all earlier UMMAs of this thread, so "S_t(j+1) is ready" also means
      // "PV_t(j) is done".
      constexpr uint32_t idesc_qk = idesc_bf16_f32(256, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_f16_f32(256, 128, 0, 1);
      // Shared-memory descriptors are built once; a K step or a stage only
      // moves the start address (bits 0-13, in 16-byte units), which never
      // carries.
      const uint64_t dQA = smem_desc_sw128(smem_u32(smem + AttnSmem::QA), 16, 1024);
      const uint64_t dQB = smem_desc_sw128(smem_u32(smem + AttnSmem::QB), 16, 1024);
      const uint64_t dK = smem_desc_sw128(smem_u32(smem + AttnSmem::K0), 16, 1024);
      const uint64_t dV = smem_desc_sw128(smem_u32(smem + AttnSmem::V0), 16384, 1024);
      int issued = 0;
      auto qk = [&](int t, int j) {
        const uint64_t q = t ? dQB : dQA;
        const uint64_t k = dK + static_cast<uint64_t>(((j % AttnSmem::K_STAGES) * AttnSmem::K_STAGE) >> 4);
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          const uint32_t oa = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          const uint32_t ob = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
          umma_ss_pair(tmem + tmem_s(t), q + oa, k + ob, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit_pair(bar(kBarSFull0 + t), 3);
        ++issued;
      };
      auto pv = [&](int t, int j) {
        const uint64_t v = dV + static_cast<uint64_t>(((j & 1) * AttnSmem::V_STAGE) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts_pair(tmem + tmem_o(t), tmem + tmem_s(t) + kk * 8, v + ((kk * 2048) >> 4), idesc_pv,
                       (j > 0 || kk > 0) ? 1u : 0u);
        ++issued;
      };
      bool ok = mbar_wait(bar(kBarQFull), 0, ab, kErrWaitTma) && mbar_wait(bar(kBarKFull0), 0, ab, kErrWaitTma);
      if (ok) {
        tc_fence_after();
        if (nA > 0) qk(0, 0);
        if (nB > 0) qk(1, 0);
        umma_commit_pair(bar(kBarKEmpty0), 3);
      }
      for (int j = 0; j < n && ok; ++j) {
        if (!(ok = mbar_wait(bar(kBarVFull0 + (j & 1)), (j >> 1) & 1, ab, kErrWaitTma))) break;
        bool k_ready = false;
        for (int t = 0; t < 2 && ok; ++t) {
          const int nt = t ? nB : nA;
          if (j >= nt) continue;
          if (!(ok = mbar_wait(bar(kBarPFull0 + t), j & 1, ab, kErrWaitSoftmax))) break;
          tc_fence_after();
          pv(t, j);
          if (t == 1 || j >= nB) umma_commit_pair(bar(kBarVEmpty0 + (j & 1)), 3);  // V_j no longer read
          if (j + 1 < nt) {
            if (!k_ready) {
              const int j1 = j + 1;
              if (!(ok = mbar_wait(bar(kBarKFull0 + j1 % AttnSmem::K_STAGES), (j1 / AttnSmem::K_STAGES) & 1, ab,
                                   kErrWaitTma)))
                break;
              k_ready = true;
            }
            tc_fence_after();
            qk(t, j + 1);
          }
        }
        if (ok && j + 1 < n) umma_commit_pair(bar(kBarKEmpty0 + (j + 1) % AttnSmem::K_STAGES), 3);
      }
      if (ok) umma_commit_pair(bar(kBarODone), 3);
      if (!ok && issued > 0) {
        umma_commit_pair(bar(kBarDrain), 1);
        mbar_wait_drain(bar(kBarDrain), 0);
      }
    }
  } else {
    // ---------------- softmax: warpgroup t = (warp - 2) / 4 owns this CTA's
    // tile of super-tile t; thread = query row r of the tile (tensor-memory
    // lane r)
    const int t = (warp - 2) >> 2;
    const int nt = t ? nB : nA;
    const bool exists = t ? has_b : true;
    if (exists) {
      const int q4 = warp & 3;
      const int r = q4 * 32 + static_cast<int>(lane);
      const int qt = q0 + 2 * t + static_cast<int>(rank);  // this CTA's tile
      const bool tile_ok = qt < p.nq;                       // a tile past T is computed and dropped
      const int s = qt * 128 + r;
      const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
      const uint32_t tS = trow + tmem_s(t), tO = trow + tmem_o(t);
      const int64_t tri_total = tri_index(p.nq, 0);
      const uint4* bm_row = (p.bitmap && tile_ok)
                                ? p.bitmap + (static_cast<int64_t>(b) * tri_total + tri_index(qt, 0)) * 128 + r
                                : nullptr;
      // Selection words of block j for this row; blocks past this tile's
      // causal range select nothing.
      auto bits_of = [&](int j) -> uint4 {
        const int kb = kblock(j);
        if (kb > qt || !tile_ok) return make_uint4(0u, 0u, 0u, 0u);
        if (!bm_row) return make_uint4(0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu);
        return __ldg(bm_row + static_cast<int64_t>(kb) * 128);
      };
      const float c = p.scale_log2;
      const uint32_t pfull = mapa_shared(bar(kBarPFull0 + t), 0);
      float m_run = -INFINITY, l_run = 0.f;  // running max (scaled log2 domain) and row sum
      bool ok = true;
      uint4 bits_next = nt > 0 ? bits_of(0) : make_uint4(0u, 0u, 0u, 0u);

      for (int j = 0; j < nt; ++j) {
        const int kb = kblock(j);
        const uint32_t bw[4] = {bits_next.x, bits_next.y, bits_next.z, bits_next.w};
        if (j + 1 < nt) bits_next = bits_of(j + 1);
        if (!(ok = warp_wait(bar(kBarSFull0 + t), j & 1, ab, kErrWaitMma))) break;
        tc_fence_after();
        uint32_t pk[64];
        float alpha = 1.f;
        bool resc = false;
        if (kb > qt || !tile_ok) {
          // Block beyond this tile's causal range (visited for the pair's
          // other tiles).
#pragma unroll
          for (int i = 0; i < 64; ++i) pk[i] = 0u;
        } else {
          float x[128];
          tmem_ld128(tS, *reinterpret_cast<uint32_t(*)[128]>(x));
          // Selection: unselected scores become -inf (raw domain; the scale is
          // positive, so the max commutes with it).
          const bool all_sel = (bw[0] & bw[1] & bw[2] & bw[3]) == 0xffffffffu;
          if (p.bitmap == nullptr && kb == qt) {
#pragma unroll
            for (int i = 0; i < 128; ++i) x[i] = (i <= r) ? x[i] : -INFINITY;
          } else if (!__all_sync(0xffffffffu, all_sel)) {
#pragma unroll
            for (int i = 0; i < 128; ++i) x[i] = ((bw[i >> 5] >> (i & 31)) & 1u) ? x[i] : -INFINITY;
          }
          // Row max: 8 independent chains of 3-input max.
          float mx[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = max3(x[i], x[8 + i], x[16 + i]);
#pragma unroll
          for (int k0 = 24; k0 < 120; k0 += 16) {
#pragma unroll
            for (int i = 0; i < 8; ++i) mx[i] = max3(mx[i], x[k0 + i], x[k0 + 8 + i]);
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], x[120 + i]);
          const float mblk = fmaxf(max3(mx[0], mx[1], mx[2]), max3(mx[3], max3(mx[4], mx[5], mx[6]), mx[7])) * c;
          // Lazy rescaling: keep the running max unless the block max exceeds
          // it by more than 8 (a factor of 256), so O is rarely touched and P
          // stays below 2^8 (well inside f16).
          const float m_new = fmaxf(m_run, mblk);
          resc = (m_new - m_run) > 8.f;
          if (resc) {
            alpha = ex2_approx(m_run - m_new);
            m_run = m_new;
          }
          const float nb = (m_run == -INFINITY) ? 0.f : -m_run;
          float sm[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) sm[i] = 0.f;
          // The argument and the row sums use packed f32x2 FMA/add (one issue
          // slot per two elements); the softmax is bound by issue slots.
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            fma2_scalar(x[2 * i], x[2 * i + 1], c, nb);
            const float p0 = ex2_approx(x[2 * i]);
            const float p1 = ex2_approx(x[2 * i + 1]);
            add2(sm[2 * (i & 3)], sm[2 * (i & 3) + 1], p0, p1);
            pk[i] = pack_f16x2(p0, p1);
          }
          l_run = l_run * alpha + (((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7])));
        }
        // O holds PV of blocks < j (complete: S(j) was committed after
        // them); rescale it before PV of block j is issued.
        if (j >= 1 && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c0, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + c0, o);
          }
        }
        // P (f16 pairs) over the first half of S, then one arrival per warp
        // on the leader's barrier.
        tmem_st64(tS, pk);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(pfull);
      }

      if (ok) {
        __nv_bfloat16* dst = p.attn + ((static_cast<int64_t>(b) * p.T + s) * p.H + h) * 128;
        if (nt > 0) {
          ok = warp_wait(bar(kBarODone), 0, ab, kErrWaitMma);
          if (ok) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            if (p.attn8 != nullptr) {
              // e4m3 output: the row's 128 values, rounded to bf16 as the
              // bf16 path stores them, quantized as one group (s = amax / 448,
              // code = e4m3(v / s), divisions rounded to nearest even).
              uint32_t a[128];
              tmem_ld128(tO, a);
              float amax = 0.f;
#pragma unroll
              for (int i = 0; i < 128; ++i) {
                const float v = __bfloat162float(__float2bfloat16_rn(__uint_as_float(a[i]) * inv));
                a[i] = __float_as_uint(v);
                amax = fmaxf(amax, fabsf(v));
              }
              const float sc = __fdiv_rn(amax, 448.0f);
              if (s < p.T) {
                const int64_t row = static_cast<int64_t>(b) * p.T + s;
                uint4* d4 = reinterpret_cast<uint4*>(p.attn8 + (row * p.H + h) * 128);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  uint32_t w[4];
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    const float* v = reinterpret_cast<const float*>(a) + 16 * i + 4 * k;
                    w[k] = sc == 0.f ? 0u
                                     : (static_cast<uint32_t>(pack_e4m3x2(__fdiv_rn(v[0], sc), __fdiv_rn(v[1], sc))) |
                                        (static_cast<uint32_t>(pack_e4m3x2(__fdiv_rn(v[2], sc), __fdiv_rn(v[3], sc)))
                                         << 16));
                  }
                  d4[i] = make_uint4(w[0], w[1], w[2], w[3]);
                }
                p.attn8_s[static_cast<int64_t>(h) * p.B * p.T + row] = sc;
              }
            } else {
#pragma unroll 1
            for (int c0 = 0; c0 < 128; c0 += 64) {
              uint32_t a0[32], a1[32];
              tmem_ld32x2(tO + c0, tO + c0 + 32, a0, a1);
              if (s < p.T) {
                uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  d4[i] = make_uint4(pack_bf16x2(__uint_as_float(a0[8 * i + 0]) * inv, __uint_as_float(a0[8 * i + 1]) * inv),
                                     pack_bf16x2(__uint_as_float(a0[8 * i + 2]) * inv, __uint_as_float(a0[8 * i + 3]) * inv),
                                     pack_bf16x2(__uint_as_float(a0[8 * i + 4]) * inv, __uint_as_float(a0[8 * i + 5]) * inv),
                                     pack_bf16x2(__uint_as_float(a0[8 * i + 6]) * inv, __uint_as_float(a0[8 * i + 7]) * inv));
                  d4[4 + i] = make_uint4(pack_bf16x2(__uint_as_float(a1[8 * i + 0]) * inv, __uint_as_float(a1[8 * i + 1]) * inv),
                                         pack_bf16x2(__uint_as_float(a1[8 * i + 2]) * inv, __uint_as_float(a1[8 * i + 3]) * inv),
                                         pack_bf16x2(__uint_as_float(a1[8 * i + 4]) * inv, __uint_as_float(a1[8 * i + 5]) * inv),
                                         pack_bf16x2(__uint_as_float(a1[8 * i + 6]) * inv, __uint_as_float(a1[8 * i + 7]) * inv));
                }
              }
            }
            }
          }
        } else if (s < p.T) {  // no surviving key
          if (p.attn8 != nullptr) {
            const int64_t row = static_cast<int64_t>(b) * p.T + s;
            uint4* d4 = reinterpret_cast<uint4*>(p.attn8 + (row * p.H + h) * 128);
            for (int i = 0; i < 8; ++i) d4[i] = make_uint4(0, 0, 0, 0);
            p.attn8_s[static_cast<int64_t>(h) * p.B * p.T + row] = 0.f;
          } else {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
            for (int i = 0; i < 16; ++i) d4[i] = make_uint4(0, 0, 0, 0);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's UMMAs into this CTA's tensor memory are complete
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

}  // namespace mla
