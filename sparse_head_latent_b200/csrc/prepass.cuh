// prepass.cuh -- top-k indices -> causal selection bitmap + active key blocks.
//
// The pages build a [B, T, T] float mask: -inf everywhere, 0 at the top-k
// keys of each query, plus the causal mask (DeepSeek-V3.2-Exp "Sparse
// attention": full(-inf).scatter_(-1, topk_indices, 0), += mask). Here the
// same selection is one bit per causal (query, key) pair:
//   bit(s, t) = [t appears in topk_idx[b, s, :]] and 0 <= t <= s
// Duplicates set the same bit once; entries outside [0, T) are dropped.
//
// Layout (per batch b, 128-query tile qt, 128-key block kb <= qt):
//   bitmap[b][qt*(qt+1)/2 + kb][row 0..127][4 x u32]   (bit c of the 128 = key kb*128 + c)
//   blocks[b][g][0] = number of key blocks with any bit set for a query
//   tile of group g (tiles 4g .. 4g+3, which one CTA pair of the attention
//   kernel processes together), blocks[b][g][1] = how many of those lie at
//   or below tile 4g+1 (the blocks the group's first two tiles can see),
//   blocks[b][g][2 + i] = the indices, ascending. Row pitch nq + 2.
//
// Two launches:
//   topk_bitmap_rows_kernel   one warp per query row (B * tiles * 128 rows):
//                             shared-memory atomics build the row's bits,
//                             then the row's words are written for every
//                             causal block (rows past T get zeros)
//   topk_block_list_kernel    one CTA per (tile group, batch), a warp per key
//                             block: OR of each
//                             block's bits over the group's tiles,
//                             ballot-compacted into the group's list
// No global atomics; the result is deterministic.
#pragma once

#include "mla.h"
#include "ptx.cuh"

namespace mla {

constexpr int kPrepassWarps = 8;

__host__ __device__ inline int64_t tri_index(int qt, int kb) {
  return static_cast<int64_t>(qt) * (qt + 1) / 2 + kb;
}

__global__ void __launch_bounds__(32 * kPrepassWarps)
topk_bitmap_rows_kernel(const int32_t* __restrict__ topk_idx, int B, int T, int k, int nq,
                        uint4* __restrict__ bitmap) {
  extern __shared__ uint32_t psmem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kPrepassWarps + warp;  // over B * nq * 128
  const int64_t rows_per_batch = static_cast<int64_t>(nq) * 128;
  if (row >= static_cast<int64_t>(B) * rows_per_batch) return;
  const int b = static_cast<int>(row / rows_per_batch);
  const int s = static_cast<int>(row % rows_per_batch);
  const int qt = s >> 7, r = s & 127;
  const int nwords = (qt + 1) * 4;  // bits for keys [0, (qt+1)*128)
  uint32_t* bits = psmem + warp * nq * 4;

  for (int w = lane; w < nwords; w += 32) bits[w] = 0u;
  __syncwarp();
  if (s < T) {
    const int32_t* idx = topk_idx + (static_cast<int64_t>(b) * T + s) * k;
    int i0 = 0;
    if ((k & 3) == 0 && (reinterpret_cast<uintptr_t>(topk_idx) & 15u) == 0) {
      // 16-byte loads, two per lane per round, issued before the atomics so
      // that several are in flight (the row is 4k bytes).
      for (; i0 + 256 <= k; i0 += 256) {
        const int4 u = __ldg(reinterpret_cast<const int4*>(idx + i0) + lane);
        const int4 v = __ldg(reinterpret_cast<const int4*>(idx + i0 + 128) + lane);
        const int32_t t[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (t[j] >= 0 && t[j] <= s) atomicOr(&bits[t[j] >> 5], 1u << (t[j] & 31));
      }
    }
    for (int i = i0 + lane; i < k; i += 32) {
      const int32_t t = __ldg(idx + i);
      if (t >= 0 && t <= s) atomicOr(&bits[t >> 5], 1u << (t & 31));
    }
  }
  __syncwarp();
  uint32_t* bm = reinterpret_cast<uint32_t*>(bitmap + (b * tri_index(nq, 0) + tri_index(qt, 0)) * 128);
  for (int w = lane; w < nwords; w += 32) bm[(static_cast<int64_t>(w >> 2) * 128 + r) * 4 + (w & 3)] = bits[w];
}

constexpr int kBlockListWarps = 16;

__global__ void __launch_bounds__(32 * kBlockListWarps)
topk_block_list_kernel(const uint4* __restrict__ bitmap, int nq, int32_t* __restrict__ blocks) {
  __shared__ uint32_t flags[MLA_MAX_T / 128];
  const int g = blockIdx.x, b = blockIdx.y;
  const int q0 = 4 * g;
  const int last = min(q0 + 3, nq - 1);     // highest key block a tile of the group can see
  const int last_a = min(q0 + 1, nq - 1);   // highest one of the group's first two tiles
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int kb = warp; kb <= last; kb += kBlockListWarps) {
    uint32_t acc = 0;
    for (int qt = q0; qt <= last; ++qt) {
      if (kb > qt) continue;  // outside this tile's causal triangle
      const uint4* blk = bitmap + (b * tri_index(nq, 0) + tri_index(qt, kb)) * 128;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = __ldg(blk + lane + 32 * i);
        acc |= v.x | v.y | v.z | v.w;
      }
    }
    const bool any = __any_sync(0xffffffffu, acc != 0u);
    if (lane == 0) flags[kb] = any ? 1u : 0u;
  }
  __syncthreads();
  if (warp == 0) {
    const int ngroups = (nq + 3) / 4;
    int32_t* out = blocks + (static_cast<int64_t>(b) * ngroups + g) * (nq + 2);
    int count = 0, count_a = 0;
    for (int base = 0; base <= last; base += 32) {
      const int kb = base + lane;
      const bool on = kb <= last && flags[kb] != 0u;
      const uint32_t m = __ballot_sync(0xffffffffu, on);
      const uint32_t ma = __ballot_sync(0xffffffffu, on && kb <= last_a);
      if (on) out[2 + count + __popc(m & ((1u << lane) - 1u))] = kb;
      count += __popc(m);
      count_a += __popc(ma);
    }
    if (lane == 0) {
      out[0] = count;
      out[1] = count_a;
    }
  }
}

// Selected keys of query rows, ascending, for the absorbed path: row i of
// the launch is query s = s0 + i of batch b (s < T). One warp per row reads
// the row's bitmap words block by block, counts the set bits per 128-key
// block, scans the counts across the warp and writes each block's keys at
// its offset. lists[i][0 .. count) are the keys, padded with key 0 up to the
// next multiple of 64 (the gather loads whole 64-key blocks; the padding is
// masked by the count). Row pitch kpad >= count, a multiple of 64.
__global__ void __launch_bounds__(32 * kPrepassWarps)
topk_row_lists_kernel(const uint4* __restrict__ bitmap, int nq, int T, int b, int s0, int rows, int kpad,
                      int32_t* __restrict__ lists, int32_t* __restrict__ counts) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = static_cast<int>(blockIdx.x) * kPrepassWarps + warp;
  if (i >= rows) return;
  const int s = s0 + i;
  int32_t* out = lists + static_cast<int64_t>(i) * kpad;
  int count = 0;
  if (s < T) {
    const int qt = s >> 7, r = s & 127;
    const uint4* row = bitmap + (static_cast<int64_t>(b) * tri_index(nq, 0) + tri_index(qt, 0)) * 128 + r;
    for (int base = 0; base <= qt; base += 32) {
      const int kb = base + lane;
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (kb <= qt) w = __ldg(row + static_cast<int64_t>(kb) * 128);
      const int c = __popc(w.x) + __popc(w.y) + __popc(w.z) + __popc(w.w);
      int incl = c;  // inclusive scan of the per-block counts
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
      }
      int pos = count + incl - c;
      const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t m = words[q];
        while (m) {
          const int bit = __ffs(m) - 1;
          m &= m - 1;
          if (pos < kpad) out[pos] = kb * 128 + q * 32 + bit;
          ++pos;
        }
      }
      count += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  if (count > kpad) count = kpad;
  const int padded = (count + 63) & ~63;
  for (int j = count + lane; j < padded; j += 32) out[j] = 0;
  if (lane == 0) counts[i] = count;
}

// Decode: the selected cache positions of the one new query of sequence b
// (topk_idx[b][0 .. k)), deduplicated and ascending, padded with 0 up to a
// multiple of 64 (row pitch kpad); a NULL topk_idx selects every position
// [0, T). One CTA per sequence sets the positions' bits in a T-bit set in
// shared memory (entries outside [0, T) are dropped), then each thread
// compacts a run of words at the offset a block-wide scan of the bit counts
// gives it.
constexpr int kDecodeListThreads = 256;

__global__ void __launch_bounds__(kDecodeListThreads)
decode_row_lists_kernel(const int32_t* __restrict__ topk_idx, int T, int k, int kpad, int32_t* __restrict__ lists,
                        int32_t* __restrict__ counts) {
  __shared__ uint32_t bits[MLA_MAX_T / 32];
  __shared__ int warp_total[kDecodeListThreads / 32];
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = (T + 31) / 32;
  for (int w = tid; w < nw; w += kDecodeListThreads) {
    uint32_t v = 0u;
    if (topk_idx == nullptr) v = (w + 1) * 32 <= T ? 0xffffffffu : ((1u << (T - 32 * w)) - 1u);
    bits[w] = v;
  }
  __syncthreads();
  if (topk_idx != nullptr) {
    const int32_t* idx = topk_idx + static_cast<int64_t>(b) * k;
    for (int i = tid; i < k; i += kDecodeListThreads) {
      const int32_t t = __ldg(idx + i);
      if (t >= 0 && t < T) atomicOr(&bits[t >> 5], 1u << (t & 31));
    }
  }
  __syncthreads();
  const int wpt = (nw + kDecodeListThreads - 1) / kDecodeListThreads;  // words per thread
  const int w0 = tid * wpt, w1 = min(w0 + wpt, nw);
  int c = 0;
  for (int w = w0; w < w1; ++w) c += __popc(bits[w]);
  int incl = c;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  if (lane == 31) warp_total[warp] = incl;
  __syncthreads();
  int before = 0, total = 0;
  for (int i = 0; i < kDecodeListThreads / 32; ++i) {
    if (i < warp) before += warp_total[i];
    total += warp_total[i];
  }
  int32_t* out = lists + static_cast<int64_t>(b) * kpad;
  int pos = before + incl - c;
  for (int w = w0; w < w1; ++w) {
    uint32_t m = bits[w];
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1;
      if (pos < kpad) out[pos] = w * 32 + bit;
      ++pos;
    }
  }
  const int count = total < kpad ? total : kpad;
  const int padded = (count + 63) & ~63;
  for (int j = count + tid; j < padded; j += kDecodeListThreads) out[j] = 0;
  if (tid == 0) counts[b] = count;
}

}  // namespace mla
