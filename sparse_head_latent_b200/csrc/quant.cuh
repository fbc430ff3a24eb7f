// quant.cuh -- dynamic per-token e4m3 quantization of bf16 activations for
// sm_100a.
//
// Kimi K2 "Down projection" page (config.json quantization_config:
// activation_scheme "dynamic", fmt "e4m3", 128 x 128 weight blocks): the
// input of an FP8 linear layer is quantized on the fly. Per row and group of
// 128 consecutive channels:
//   s    = amax / 448               (fp32, round to nearest even)
//   code = e4m3(x / s)              (fp32 division, nearest even, saturating at +-448)
// and a group of zeros gets s = 0 and zero codes. The layer then computes
// with code * s.
#pragma once

#include "ptx.cuh"

namespace mla {

constexpr int kQuantWarps = 8;
constexpr int kQuantItemsPerHalfWarp = 4;   // (row, group) items per half-warp, loads issued together

// x bf16 [rows, cols] (row pitch cols) -> codes u8 [rows, cols] and scales
// fp32 [cols / 128, rows] (one row of scales per 128-column group, so that
// consecutive rows' scales are adjacent). Items are (row, group) pairs taken
// group-major (item i = group i / rows, row i % rows). A half-warp handles
// one item at a time, lane l of it columns 8l .. 8l+7 of the group; each
// half-warp issues the loads of its kQuantItemsPerHalfWarp items before it
// quantizes them, so that several 16-byte loads per lane are in flight.
__global__ void __launch_bounds__(32 * kQuantWarps)
quant_e4m3_1x128_kernel(const __nv_bfloat16* __restrict__ x, int rows, int cols, uint8_t* __restrict__ codes,
                        float* __restrict__ scales) {
  constexpr int IT = kQuantItemsPerHalfWarp;
  const int lane = threadIdx.x & 31;
  const int hl = lane & 15;
  const int64_t half = (static_cast<int64_t>(blockIdx.x) * kQuantWarps + (threadIdx.x >> 5)) * 2 + (lane >> 4);
  const int64_t total = static_cast<int64_t>(rows) * (cols / 128);
  uint4 raw[IT];
  size_t off[IT];
#pragma unroll
  for (int i = 0; i < IT; ++i) {
    const int64_t item = half * IT + i;
    const int64_t it = item < total ? item : total - 1;   // past the end: reload the last item, store nothing
    const int64_t r = it % rows, g = it / rows;
    off[i] = static_cast<size_t>(r) * cols + static_cast<size_t>(g) * 128 + 8 * hl;
    raw[i] = *reinterpret_cast<const uint4*>(x + off[i]);
  }
#pragma unroll
  for (int i = 0; i < IT; ++i) {
    const int64_t item = half * IT + i;
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[i]);
    float v[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(h2[j]);
      v[2 * j] = f.x;
      v[2 * j + 1] = f.y;
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = __fdiv_rn(amax, 448.0f);
    uint2 packed = make_uint2(0u, 0u);
    if (s != 0.0f) {
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = pack_e4m3x2(__fdiv_rn(v[2 * j], s), __fdiv_rn(v[2 * j + 1], s));
      packed = make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
    }
    if (item < total) {
      *reinterpret_cast<uint2*>(codes + off[i]) = packed;
      if (hl == 0) {
        const int64_t r = item % rows, g = item / rows;
        scales[static_cast<size_t>(g) * rows + r] = s;
      }
    }
  }
}

}  // namespace mla
