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
//   blocks[b][qt][0] = number of key blocks with any bit set for the tile,
//   blocks[b][qt][1 + i] = their indices, ascending.
// One CTA per (tile, batch); each warp builds the bits of 16 query rows in
// shared memory with shared atomics, then writes them out.
#pragma once

#include "ptx.cuh"

namespace mla {

constexpr int kPrepassWarps = 8;

__host__ __device__ inline int64_t tri_index(int qt, int kb) {
  return static_cast<int64_t>(qt) * (qt + 1) / 2 + kb;
}

__global__ void __launch_bounds__(32 * kPrepassWarps)
topk_bitmap_kernel(const int32_t* __restrict__ topk_idx, int T, int k, int nq,
                   uint4* __restrict__ bitmap, int32_t* __restrict__ blocks) {
  extern __shared__ uint32_t psmem[];
  const int qt = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwords = (qt + 1) * 4;  // bits for keys [0, (qt+1)*128)
  uint32_t* flags = psmem;                       // [nq] any-bit flag per key block
  uint32_t* rowbits = psmem + nq + warp * nq * 4;  // this warp's row, [nq*4] words
  for (int i = threadIdx.x; i < nq; i += blockDim.x) flags[i] = 0;
  __syncthreads();

  const int64_t tri_total = tri_index(nq, 0);
  uint32_t* bm = reinterpret_cast<uint32_t*>(bitmap + (b * tri_total + tri_index(qt, 0)) * 128);

  for (int r = warp; r < 128; r += kPrepassWarps) {
    const int s = qt * 128 + r;
    for (int w = lane; w < nwords; w += 32) rowbits[w] = 0u;
    __syncwarp();
    if (s < T) {
      const int32_t* idx = topk_idx + (static_cast<int64_t>(b) * T + s) * k;
      for (int i = lane; i < k; i += 32) {
        const int32_t t = __ldg(idx + i);
        if (t >= 0 && t <= s) atomicOr(&rowbits[t >> 5], 1u << (t & 31));
      }
    }
    __syncwarp();
    for (int w = lane; w < nwords; w += 32) {
      const uint32_t v = rowbits[w];
      const int kb = w >> 2;
      bm[(static_cast<int64_t>(kb) * 128 + r) * 4 + (w & 3)] = v;
      if (v) flags[kb] = 1u;
    }
    __syncwarp();
  }
  __syncthreads();

  if (warp == 0) {
    int32_t* out = blocks + (static_cast<int64_t>(b) * nq + qt) * (nq + 1);
    int count = 0;
    for (int base = 0; base <= qt; base += 32) {
      const int kb = base + lane;
      const bool on = kb <= qt && flags[kb] != 0u;
      const uint32_t m = __ballot_sync(0xffffffffu, on);
      if (on) out[1 + count + __popc(m & ((1u << lane) - 1u))] = kb;
      count += __popc(m);
    }
    if (lane == 0) out[0] = count;
  }
}

}  // namespace mla
