// dequant.cuh -- block-scaled e4m3 weights -> bf16 (HBM-bound elementwise).
//
// The stored weight is W[r][c] = e4m3(code[r][c]) * scale[r/128][c/128]
// (Kimi K2 "Down projection" page: fmt e4m3, weight_block_size [128, 128]).
// The tensor-core GEMMs run on bf16 operands, so the product is rounded to
// bf16 once here; e4m3 -> f16 is exact and the scale multiply is fp32.
#pragma once

#include <cuda_fp8.h>

#include "ptx.cuh"

namespace mla {

// Each thread converts 16 consecutive codes of one row (cols % 16 == 0).
__global__ void __launch_bounds__(256)
dequant_e4m3_block128_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ scale,
                             __nv_bfloat16* __restrict__ out, int rows, int cols) {
  const int64_t groups_per_row = cols / 16;
  const int64_t total = static_cast<int64_t>(rows) * groups_per_row;
  const int sc_cols = cols / 128;
  for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < total;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = g / groups_per_row;
    const int64_t c0 = (g % groups_per_row) * 16;
    const float s = __ldg(scale + (r / 128) * sc_cols + c0 / 128);
    const uint4 in = __ldg(reinterpret_cast<const uint4*>(codes + r * cols + c0));
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[i] & 0xFFFF), __NV_E4M3);
      const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[i] >> 16), __NV_E4M3);
      const float2 flo = __half22float2(*reinterpret_cast<const __half2*>(&lo));
      const float2 fhi = __half22float2(*reinterpret_cast<const __half2*>(&hi));
      o[2 * i] = pack_bf16x2(flo.x * s, flo.y * s);
      o[2 * i + 1] = pack_bf16x2(fhi.x * s, fhi.y * s);
    }
    uint4* dst = reinterpret_cast<uint4*>(out + r * cols + c0);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace mla
