// attn_abs.cuh -- absorbed-form attention over gathered keys, for query rows
// whose causal prefix is much longer than their top-k selection (sm_100a).
//
// The block-dense kernel (attn.cuh) up-projects every key and visits every
// 128-key block that holds a selected key; for a row s with s + 1 >> k
// nearly all of that work is masked away. Here each row attends only its
// selected keys, in the latent space: the form the DeepSeek-V3.2-Exp "Sparse
// attention" page's Explanation names for a decoded token, which scores the
// cached latent directly (same per-head weights as the prefill path):
//   q_abs[h] = q_nope[h] . W_UK[h]            (absorb GEMM, before this kernel)
//   z_t      = [q_abs[h] | q_pe[h]] . [c_t | k_pe_t]     t in A_s, 576 wide
//   o_lat[h] = sum_t softmax(z * scale)_t c_t            (this kernel)
//   attn[h]  = W_UV[h] . o_lat[h]              (un-absorb GEMM, after it)
// which equals softmax(q_h . k_h) v_h up to rounding, since k_nope_t =
// W_UK c_t and v_t = W_UV c_t.
//
// Work item: one CTA per (query row, group of 64 heads): M = 64 heads
// against the row's selected keys, gathered in blocks of 64 from the latent
// rows by three warps of 16-byte cp.async copies (coalesced along each key's
// row, written into the 128-byte-swizzled operand layout; a TMA gather4
// moved only ~8 bytes per clock per SM for these 128-byte rows). The list
// of selected keys comes from the causal selection bitmap (ascending,
// duplicates and out-of-range entries already gone).
//
// Tensor memory (M = 64 accumulators occupy 16 of the 32 lanes of each
// sub-partition; the other 16 lanes are addressed with lane offset 16):
//   lanes +0   columns [0, 512)    O = o_lat accumulator, fp32, 64 heads x 512
//   lanes +16  columns [0, 288)    Q = [q_abs | q_pe] as bf16 pairs: the A
//                                  operand of QK^T read from tensor memory
//   lanes +16  columns [288, 416)  S, two 64-column buffers
// Shared memory: three 72 KB stages of gathered keys (nine [64 keys x 64]
// chunks: eight latent, one rope; 128-byte swizzle) and P (64 heads x 64
// keys, bf16).
//   QK^T: M=64, N=64, K=576, A from tensor memory, B = the key stage (K-major)
//   PV:   M=64, N=256 (twice), K=64, A = P, B = the key stage's latent chunks
//         read N-major (the same bytes: a key's 64 latent values per row)
//
// CTA = 256 threads: warps 0, 6, 7 gather, warp 1 allocates tensor memory
// and issues the UMMAs, warps 2..5 run the softmax (lanes 16..31 own the
// heads' S rows; lanes 0..15 own the same heads' O rows, for the rescale and
// the epilogue).
#pragma once

#include "ptx.cuh"

namespace mla {

struct AbsParams {
  int rows;                    // query rows of this launch
  int H;
  int kpad;                    // pitch of `lists`
  // Row of key t = 0 for query row r in the latent tensors: key_row0 +
  // (r / rows_per_seq) * seq_stride (prefill: the launch's rows share one
  // sequence; decode: one row per sequence, seq_stride = T).
  int key_row0, rows_per_seq, seq_stride;
  float scale_log2;            // softmax scale * log2(e)
  const int32_t* lists;        // [rows][kpad] selected keys, ascending, padded with 0
  const int32_t* counts;       // [rows]
  const __nv_bfloat16* qabs;   // [rows][H][512]
  const __nv_bfloat16* q;      // [rows][H][192] (rope at 128..191)
  const __nv_bfloat16* lat;    // kv_latent [B*T][512]
  const __nv_bfloat16* kpe;    // k_pe [B*T][64]
  __nv_bfloat16* olat;         // [rows][H][512]
  // Split of each row's key list into `parts` contiguous runs of blocks, one
  // CTA each (decode, where one CTA per row leaves most SMs idle). With
  // parts > 1 a CTA writes its normalised partial output and its running
  // max and sum instead of o_lat; absorbed_combine_kernel merges them.
  int parts;
  float2* part_ml;             // [rows][parts][H]: (max in the scaled log2 domain, sum)
  __nv_bfloat16* part_o;       // [rows][parts][H][512]
  int* err;
};

struct AbsSmem {
  static constexpr int CHUNK = 8192;                // [64 keys x 64] bf16
  static constexpr int K_STAGE = 9 * CHUNK;         // 72 KB
  static constexpr int K_STAGES = 3;
  static constexpr int P = K_STAGES * K_STAGE;      // [64 heads x 64 keys] bf16
  static constexpr int BARS = P + CHUNK;
  static constexpr int NUM_BARS = 13;
  static constexpr int BYTES = 1024 + BARS + 256;
};
static_assert(AbsSmem::BYTES <= 232448, "shared memory per CTA");

constexpr int kAbsThreads = 256;
constexpr int kAbsLoaders = 96;              // threads of the three gather warps
constexpr uint32_t kAbsLaneHi = 16u << 16;   // lane offset of Q and S
constexpr int kL_abs = 512;                  // latent width
constexpr uint32_t kAbsColS = 288;           // first S column (after Q's 288)

enum : int {
  kAbsKFull0 = 0,    // per stage: the gathered keys landed (every gather thread)
  kAbsKEmpty0 = 3,   // per stage: the UMMAs reading it are done
  kAbsQReady = 6,    // Q is in tensor memory (four softmax warps)
  kAbsSFull0 = 7,    // per S buffer
  kAbsPFull = 9,     // P of the current block is in shared memory (four softmax warps)
  kAbsPVDone = 10,   // PV of a block has completed (P buffer free, O stable)
  kAbsODone = 11,    // every UMMA has completed
  kAbsDrain = 12
};

__global__ void __launch_bounds__(kAbsThreads, 1)
absorbed_attn_kernel(const AbsParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AbsSmem::BARS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + AbsSmem::NUM_BARS);
  int* abort_word = reinterpret_cast<int*>(tmem_slot + 1);
  const uint32_t bar0 = smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  if (blockDim.x != kAbsThreads) {
    if (threadIdx.x == 0) atomicCAS(p.err, 0, kErrGeometry);
    return;
  }
  const int hgroups = (p.H + 63) >> 6;
  const int row = static_cast<int>(blockIdx.x) / (hgroups * p.parts);  // query row of this launch
  const int hh = static_cast<int>(blockIdx.x) / p.parts % hgroups;     // group of 64 heads (slots past H compute zeros)
  const int part = static_cast<int>(blockIdx.x) % p.parts;
  // This CTA's run of the row's 64-key blocks: [jb0, jb0 + n).
  const int count_row = p.counts[row];
  const int n_row = (count_row + 63) >> 6;
  const int per_part = (n_row + p.parts - 1) / p.parts;
  const int jb0 = part * per_part;
  const int n = max(0, min(per_part, n_row - jb0));
  const int count = n > 0 ? min(count_row - 64 * jb0, 64 * n) : 0;  // keys of this run
  const int32_t* keys = p.lists + static_cast<int64_t>(row) * p.kpad + 64 * jb0;
  const int key_base = p.key_row0 + (row / p.rows_per_seq) * p.seq_stride;

  if (threadIdx.x == 0) {
    for (int i = 0; i < AbsSmem::K_STAGES; ++i) {
      mbar_init(bar(kAbsKFull0 + i), kAbsLoaders);
      mbar_init(bar(kAbsKEmpty0 + i), 1);
    }
    mbar_init(bar(kAbsQReady), 4);
    mbar_init(bar(kAbsSFull0), 1);
    mbar_init(bar(kAbsSFull0 + 1), 1);
    mbar_init(bar(kAbsPFull), 4);
    mbar_init(bar(kAbsPVDone), 1);
    mbar_init(bar(kAbsODone), 1);
    mbar_init(bar(kAbsDrain), 1);
    *abort_word = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Abort ab{abort_word, p.err};

  if (warp == 0 || warp >= 6) {
    if (n > 0) {
      // ---------------- gather: block j = keys [64j, 64j + 64) of the row's
      // list into stage j % 3 as nine [64 keys x 64] chunks (eight latent,
      // one rope). Loader warp w (0..2) takes keys w, w + 3, ...; the lanes
      // copy a key's 72 16-byte pieces (1152 bytes: 1024 latent + 128 rope)
      // in three coalesced instructions. The block's 64 indices are read
      // once per warp (two per lane) and broadcast by shuffle. Each thread
      // waits for its own copies, makes them visible to the tensor core's
      // (async) proxy, and arrives on the stage's barrier.
      const int w = warp == 0 ? 0 : warp - 5;
      const uint8_t* lat = reinterpret_cast<const uint8_t*>(p.lat);
      const uint8_t* pe = reinterpret_cast<const uint8_t*>(p.kpe);
      bool ok = true;
      for (int j = 0; j < n && ok; ++j) {
        const int s = j % AbsSmem::K_STAGES;
        if (!(ok = warp_wait(bar(kAbsKEmpty0 + s), ((j / AbsSmem::K_STAGES) & 1) ^ 1, ab, kErrWaitMma))) break;
        const uint32_t stage = smem_u32(smem + s * AbsSmem::K_STAGE);
        const int2 kk = __ldg(reinterpret_cast<const int2*>(keys + 64 * j) + lane);  // keys 2l, 2l+1
#pragma unroll 2
        for (int i = w; i < 64; i += 3) {
          const int kx = __shfl_sync(0xffffffffu, kk.x, i >> 1);
          const int ky = __shfl_sync(0xffffffffu, kk.y, i >> 1);
          const int64_t krow = static_cast<int64_t>(key_base) + ((i & 1) ? ky : kx);
          const uint32_t drow = stage + i * 128;
#pragma unroll
          for (int r = 0; r < 3; ++r) {
            const int pc = static_cast<int>(lane) + 32 * r;  // piece of this key: chunk pc / 8, column pc % 8
            if (pc < 72) {
              const int c = pc >> 3, e = pc & 7;
              const uint8_t* src = c < 8 ? lat + krow * (kL_abs * 2) + pc * 16 : pe + krow * 128 + e * 16;
              cp_async16(drow + c * AbsSmem::CHUNK + ((e ^ (i & 7)) << 4), src);
            }
          }
        }
        cp_async_commit_wait_all();
        fence_proxy_async_smem();
        mbar_arrive(bar(kAbsKFull0 + s));
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && n > 0) {
      // ---------------- UMMA issuer: S(j) = Q K_j^T into S buffer j % 2, and
      // O += P(j) . C_j once the softmax has written P(j), then release
      // stage j (the scheduling rule is below).
      constexpr uint32_t idesc_qk = idesc_bf16_f32(64, 64, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(64, 256, 0, 1);
      const uint32_t stage0 = smem_u32(smem);
      const uint64_t dP = smem_desc_sw128(smem_u32(smem + AbsSmem::P), 16, 1024);
      int commits = 0;
      auto qk = [&](int j) -> bool {
        const int s = j % AbsSmem::K_STAGES;
        if (!mbar_wait(bar(kAbsKFull0 + s), (j / AbsSmem::K_STAGES) & 1, ab, kErrWaitTma)) return false;
        tc_fence_after();
        const uint64_t dk = smem_desc_sw128(stage0 + s * AbsSmem::K_STAGE, 16, 1024);
        const uint32_t ts = tmem + kAbsLaneHi + kAbsColS + 64u * static_cast<uint32_t>(j & 1);
#pragma unroll
        for (int ks = 0; ks < 36; ++ks) {
          const uint32_t off = ((ks >> 2) * AbsSmem::CHUNK + (ks & 3) * 32) >> 4;
          umma_ts(ts, tmem + kAbsLaneHi + static_cast<uint32_t>(ks) * 8u, dk + off, idesc_qk, ks > 0 ? 1u : 0u);
        }
        umma_commit(bar(kAbsSFull0 + (j & 1)));
        ++commits;
        return true;
      };
      auto pv = [&](int j) {
        const uint32_t st = stage0 + (j % AbsSmem::K_STAGES) * AbsSmem::K_STAGE;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint64_t dc = smem_desc_sw128(st + half * 4 * AbsSmem::CHUNK + kk * 2048, AbsSmem::CHUNK, 1024);
            umma_ss(tmem + 256u * half, dP + static_cast<uint64_t>((kk * 32) >> 4), dc, idesc_pv,
                    (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(bar(kAbsPVDone));
        umma_commit(bar(kAbsKEmpty0 + j % AbsSmem::K_STAGES));
        ++commits;
      };
      bool ok = mbar_wait(bar(kAbsQReady), 0, ab, kErrWaitSoftmax);
      if (ok) {
        tc_fence_after();
        ok = qk(0);
      }
      // Issue whichever is ready next: PV(next_pv) once the softmax has
      // written P(next_pv), or S(next_qk) = Q K^T once its keys have landed
      // and its S buffer is free (S(i-2)'s P handed over, i.e. PV(i-2)
      // issued). In a fixed order a slow gather of block j+2 would hold back
      // PV(j+1) behind it. Neither barrier can run two phases ahead: the
      // softmax writes P(j+1) only after PV(j) completed, and the gather
      // refills a stage only after the PV that read it.
      int next_pv = 0, next_qk = 1;
      uint64_t t_idle = 0;
      while (ok && next_pv < n) {
        if (next_qk < n && next_pv >= next_qk - 1 &&
            mbar_test_wait(bar(kAbsKFull0 + next_qk % AbsSmem::K_STAGES), (next_qk / AbsSmem::K_STAGES) & 1)) {
          ok = qk(next_qk);  // ready: returns at once
          ++next_qk;
          t_idle = 0;
        } else if (mbar_test_wait(bar(kAbsPFull), next_pv & 1)) {
          tc_fence_after();
          pv(next_pv);
          ++next_pv;
          t_idle = 0;
        } else {
          const uint64_t now = global_timer_ns();
          if (t_idle == 0) {
            t_idle = now;
          } else if (now - t_idle > wait_timeout_ns() || ab.raised()) {
            if (!ab.raised()) ab.raise(kErrWaitSoftmax);
            ok = false;
          }
        }
      }
      if (ok) umma_commit(bar(kAbsODone));
      if (!ok && commits > 0) {
        umma_commit(bar(kAbsDrain));
        mbar_wait_drain(bar(kAbsDrain), 0);
      }
    }
  } else {
    // ---------------- softmax warps (2..5). Warp w covers the tensor-memory lanes of
    // sub-partition q = w % 4: lanes 16..31 of it hold the S rows (and Q) of
    // heads 16q .. 16q+15 of this half, lanes 0..15 the O rows of the same
    // heads, so a lane and the lane 16 above it work on the same head.
    const int quad = warp & 3;
    const bool srow = lane >= 16;
    const int hl = 16 * quad + static_cast<int>(lane & 15);  // head within the half
    const int h = 64 * hh + hl;
    const bool hvalid = h < p.H;
    const int hp = hvalid ? h : 0;  // for addressing only
    const uint32_t tq = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    bool ok = true;
    float m_run = -INFINITY, l_run = 0.f;  // running max (scaled log2 domain) and row sum
    if (n > 0) {
      // Q = [q_abs | q_pe] (576 bf16 = 288 columns) into lanes 16..31. Lanes
      // 0..15 store zeros into O's columns, which PV(0) overwrites.
      const __nv_bfloat16* qa = p.qabs + (static_cast<int64_t>(row) * p.H + hp) * 512;
      const __nv_bfloat16* qr = p.q + (static_cast<int64_t>(row) * p.H + hp) * 192 + 128;
      // Software-pipelined: the loads of chunk cc + 1 are in flight while
      // chunk cc is stored (a load-then-store round trip per chunk would put
      // nine global-load latencies on every CTA's path to its first UMMA).
      const bool qload = srow && hvalid;
      auto load_chunk = [&](int cc, uint4 (&w)[8]) {
        const uint4* src = reinterpret_cast<const uint4*>(cc < 8 ? qa + 64 * cc : qr);
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = qload ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
      };
      uint4 cur[8], nxt[8];
      load_chunk(0, cur);
#pragma unroll 1
      for (int cc = 0; cc < 9; ++cc) {
        if (cc + 1 < 9) load_chunk(cc + 1, nxt);
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[4 * i] = cur[i].x;
          v[4 * i + 1] = cur[i].y;
          v[4 * i + 2] = cur[i].z;
          v[4 * i + 3] = cur[i].w;
        }
        tmem_st32(tq + 32u * cc, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) cur[i] = nxt[i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kAbsQReady));

      const float c = p.scale_log2;
      uint8_t* prow = smem + AbsSmem::P + hl * 128;
      for (int j = 0; j < n; ++j) {
        if (!(ok = warp_wait(bar(kAbsSFull0 + (j & 1)), (j >> 1) & 1, ab, kErrWaitMma))) break;
        tc_fence_after();
        float x[64];
        tmem_ld64(tq + kAbsColS + 64u * (j & 1), *reinterpret_cast<uint32_t(*)[64]>(x));
        float alpha = 1.f, bsum = 0.f;
        bool resc = false;
        uint32_t pk[32];
        if (srow) {
          const int valid = min(64, count - 64 * j);  // the last block is padded
          if (valid < 64) {
#pragma unroll
            for (int i = 0; i < 64; ++i) x[i] = i < valid ? x[i] : -INFINITY;
          }
          float mx[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) mx[i] = max3(x[i], x[4 + i], x[8 + i]);
#pragma unroll
          for (int k0 = 12; k0 < 60; k0 += 8) {
#pragma unroll
            for (int i = 0; i < 4; ++i) mx[i] = max3(mx[i], x[k0 + i], x[k0 + 4 + i]);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) mx[i] = fmaxf(mx[i], x[60 + i]);
          const float mblk = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c;
          // Lazy rescaling as in the block-dense kernel: the running max moves
          // only when a block's max exceeds it by more than 8, so P < 2^8.
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
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            fma2_scalar(x[2 * i], x[2 * i + 1], c, nb);
            const float p0 = ex2_approx(x[2 * i]);
            const float p1 = ex2_approx(x[2 * i + 1]);
            add2(sm[2 * (i & 3)], sm[2 * (i & 3) + 1], p0, p1);
            pk[i] = pack_bf16x2(p0, p1);
          }
          bsum = ((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7]));
        }
        // PV(j-1) must be done before P is overwritten and before O is rescaled.
        if (j >= 1 && !(ok = warp_wait(bar(kAbsPVDone), (j - 1) & 1, ab, kErrWaitMma))) break;
        if (j >= 1 && __any_sync(0xffffffffu, resc)) {
          // Rare. The rescale reads and writes whole 32-lane rows, so the
          // S/Q lanes of the same columns are written back unchanged; wait
          // for S(j+1), the only UMMA that can still be running, first.
          if (j + 1 < n && !(ok = warp_wait(bar(kAbsSFull0 + ((j + 1) & 1)), ((j + 1) >> 1) & 1, ab, kErrWaitMma)))
            break;
          tc_fence_after();
          const float a_o = __shfl_down_sync(0xffffffffu, alpha, 16);  // lanes 0..15: their head's alpha
          const float f = srow ? 1.f : a_o;
#pragma unroll 1
          for (int c0 = 0; c0 < 512; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tq + c0, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st32(tq + c0, o);
          }
          tc_fence_before();
        }
        if (srow) {
          // P row of this head: 64 bf16 = 128 bytes, 16-byte chunk cc at cc ^ (row & 7).
#pragma unroll
          for (int cc = 0; cc < 8; ++cc)
            *reinterpret_cast<uint4*>(prow + ((cc ^ (hl & 7)) << 4)) =
                make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
          l_run = l_run * alpha + bsum;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kAbsPFull));
      }
    }

    if (ok) {
      // lanes 0..15 write their head's o_lat row (512 bf16), or with a split
      // the run's normalised partial row; lanes 16..31 its (max, sum)
      const int64_t prow = (static_cast<int64_t>(row) * p.parts + part) * p.H + hp;
      __nv_bfloat16* dst = p.parts > 1 ? p.part_o + prow * 512 : p.olat + (static_cast<int64_t>(row) * p.H + hp) * 512;
      if (p.parts > 1 && srow && hvalid) p.part_ml[prow] = make_float2(m_run, l_run);
      if (n > 0) {
        ok = warp_wait(bar(kAbsODone), 0, ab, kErrWaitMma);
        if (ok) {
          tc_fence_after();
          const float l_o = __shfl_down_sync(0xffffffffu, l_run, 16);
          const float inv = l_o > 0.f ? 1.f / l_o : 0.f;
#pragma unroll 1
          for (int c0 = 0; c0 < 512; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tq + c0, o);
            if (!srow && hvalid) {
              uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                d4[i] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * i + 0]) * inv, __uint_as_float(o[8 * i + 1]) * inv),
                                   pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv),
                                   pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv),
                                   pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv));
            }
          }
        }
      } else if (!srow && hvalid) {
        uint4* d4 = reinterpret_cast<uint4*>(dst);
        for (int i = 0; i < 64; ++i) d4[i] = make_uint4(0, 0, 0, 0);  // no selected key (in this run)
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// Merges the parts of a split row: per (row, head), with M the largest
// part max, o_lat = sum_p w_p o_p / sum_p w_p where w_p = l_p 2^(m_p - M)
// and o_p is part p's normalised output. One warp per (row, head), 16 of
// the 512 values per lane. A head whose parts saw no key gets 0.
constexpr int kCombineWarps = 8;

__global__ void __launch_bounds__(32 * kCombineWarps)
absorbed_combine_kernel(const AbsParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t item = static_cast<int64_t>(blockIdx.x) * kCombineWarps + (threadIdx.x >> 5);  // row * H + h
  if (item >= static_cast<int64_t>(p.rows) * p.H) return;
  const int64_t row = item / p.H, h = item % p.H;
  float M = -INFINITY;
  for (int q = 0; q < p.parts; ++q) M = fmaxf(M, p.part_ml[(row * p.parts + q) * p.H + h].x);
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  for (int q = 0; q < p.parts; ++q) {
    const int64_t pr = (row * p.parts + q) * p.H + h;
    const float2 ml = p.part_ml[pr];
    const float w = ml.y > 0.f ? ml.y * ex2_approx(ml.x - M) : 0.f;
    if (w == 0.f) continue;
    wsum += w;
    const uint4* src = reinterpret_cast<const uint4*>(p.part_o + pr * 512 + lane * 16);
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const uint4 u = __ldg(src + v);
      const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wd[e]));
        acc[8 * v + 2 * e] = fmaf(w, f.x, acc[8 * v + 2 * e]);
        acc[8 * v + 2 * e + 1] = fmaf(w, f.y, acc[8 * v + 2 * e + 1]);
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint4* dst = reinterpret_cast<uint4*>(p.olat + item * 512 + lane * 16);
#pragma unroll
  for (int v = 0; v < 2; ++v)
    dst[v] = make_uint4(pack_bf16x2(acc[8 * v] * inv, acc[8 * v + 1] * inv),
                        pack_bf16x2(acc[8 * v + 2] * inv, acc[8 * v + 3] * inv),
                        pack_bf16x2(acc[8 * v + 4] * inv, acc[8 * v + 5] * inv),
                        pack_bf16x2(acc[8 * v + 6] * inv, acc[8 * v + 7] * inv));
}

}  // namespace mla
