// mla_api.cu -- host side of the C ABI declared in include/mla.h:
// argument validation, workspace carving, TMA tensor-map encoding, launch
// sequencing on the caller's stream, device error word and per-kernel
// event timing. All kernels live in the headers included below (one
// translation unit, so no relocatable device code is needed).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <vector>

#include "../../include/mla.h"
#include "attn.cuh"
#include "attn_abs.cuh"
#include "dequant.cuh"
#include "gemm2.cuh"
#include "gemm_w8t.cuh"
#include "gemm8.cuh"
#include "gemm_m64.cuh"
#include "prepass.cuh"
#include "quant.cuh"
#include "ptx.cuh"

// Device error word: kernels record the first error code here.
__device__ int g_mla_device_error;

namespace {

constexpr int kDn = 128, kDr = 64, kDv = 128, kL = 512, kD = 7168;
using Gemm2Kvb = mla::Gemm2Cfg<false>;  // latent x W_kvb^T  (B stored [N, K])
using Gemm2KvbAttn = mla::Gemm2Cfg<false, true>;  // same, v columns written as f16 for the attention
using Gemm2Wo = mla::Gemm2Cfg<true>;    // attn x W_o         (B stored [K, N]); also q_nope x W_UK
using Gemm2Unabs = mla::Gemm2Cfg<false, false, 128>;  // o_lat x W_UV^T (B stored [N, K], 128 wide)
using Gemm2WoNarrow = mla::Gemm2Cfg<true, false, 128>;
using GemmW8tKvb = mla::GemmW8tCfg<false, true>;            // latent x e4m3 W_kvb^T, weights converted on chip
using GemmW8tKvbAttn = mla::GemmW8tCfg<false, true, true>;  // same, v columns written as f16 for the attention
using GemmW8tWo = mla::GemmW8tCfg<true, false>;             // attn x e4m3 W_o, weights converted on chip  // attn x W_o with one row tile (decode): twice the pairs
using GemmM64 = mla::GemmM64Cfg<64>;     // decode's output projection (stream-K), M <= 64
using GemmM128 = mla::GemmM64Cfg<128>;   // and 64 < M <= 256 (128-row tiles)
using GemmM64Abs = mla::GemmM64Cfg<64, true, true>;     // decode's q_nope x W_UK per head, bf16 out
using GemmM128Abs = mla::GemmM64Cfg<128, true, true>;
using GemmM64Unabs = mla::GemmM64Cfg<64, false, true>;  // decode's o_lat x W_UV^T per head, bf16 out
using GemmM128Unabs = mla::GemmM64Cfg<128, false, true>;
using Gemm8Kvb = mla::Gemm8Cfg<false>;              // e4m3 latent x e4m3 W_kvb^T
using Gemm8KvbAttn = mla::Gemm8Cfg<false, true>;    // same, v tiles written as f16 for the attention
using Gemm8Wo = mla::Gemm8Cfg<true>;           // e4m3 attn x e4m3 W_o (B stored [K, N])

// ------------------------------------------------------------------ device state

struct DeviceState {
  bool ready = false;
  int status = MLA_OK;
  int sms = 0;
  int pairs_kvb = 0;   // CTA pairs of the pair GEMMs that fit on the device at once
  int pairs_wo = 0;
  int pairs_w8t_kvb = 0;  // CTA pairs of the e4m3-weight GEMMs with on-chip conversion
  int pairs_w8t_wo = 0;
  int pairs_unabs = 0;
  int pairs_wo_narrow = 0;
  int pairs8_kvb = 0;  // CTA pairs of the e4m3 GEMMs
  int pairs8_wo = 0;
  int* err = nullptr;  // address of g_mla_device_error on this device
};

template <class Kernel>
int max_pairs(Kernel k, int smem, int threads = 192) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess) return 0;
  return n;
}

std::mutex g_mutex;
std::vector<DeviceState> g_devices;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// One-time set-up per device: device checks, kernel attributes, address of
// the error word. Returns an mla_status.
int device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (static_cast<int>(g_devices.size()) <= dev) g_devices.resize(dev + 1);
  DeviceState& st = g_devices[dev];
  if (!st.ready) {
    st.ready = true;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
      st.status = MLA_ERR_CUDA;
    } else if (prop.major != 10) {
      st.status = MLA_ERR_UNSUPPORTED;  // built for sm_100a only
    } else {
      st.sms = prop.multiProcessorCount;
      bool ok = cudaGetSymbolAddress(reinterpret_cast<void**>(&st.err), g_mla_device_error) == cudaSuccess;
      ok = ok && cudaMemset(st.err, 0, sizeof(int)) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::gemm_bf16_tc2_kernel<Gemm2Kvb>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      Gemm2Kvb::SMEM_BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::gemm_bf16_tc2_kernel<Gemm2Wo>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      Gemm2Wo::SMEM_BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::gemm_bf16_tc2_kernel<Gemm2KvbAttn>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, Gemm2KvbAttn::SMEM_BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::gemm_bf16_tc2_kernel<Gemm2Unabs>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, Gemm2Unabs::SMEM_BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::gemm_bf16_tc2_kernel<Gemm2WoNarrow>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, Gemm2WoNarrow::SMEM_BYTES) == cudaSuccess;
      if (ok) {
        st.pairs_kvb = max_pairs(mla::gemm_bf16_tc2_kernel<Gemm2Kvb>, Gemm2Kvb::SMEM_BYTES);
        st.pairs_wo = max_pairs(mla::gemm_bf16_tc2_kernel<Gemm2Wo>, Gemm2Wo::SMEM_BYTES);
        ok = ok && cudaFuncSetAttribute(mla::gemm_bf16_w8t_kernel<GemmW8tKvb>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, GemmW8tKvb::SMEM_BYTES) == cudaSuccess;
        ok = ok && cudaFuncSetAttribute(mla::gemm_bf16_w8t_kernel<GemmW8tKvbAttn>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, GemmW8tKvbAttn::SMEM_BYTES) == cudaSuccess;
        ok = ok && cudaFuncSetAttribute(mla::gemm_bf16_w8t_kernel<GemmW8tWo>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, GemmW8tWo::SMEM_BYTES) == cudaSuccess;
        st.pairs_w8t_kvb = max_pairs(mla::gemm_bf16_w8t_kernel<GemmW8tKvb>, GemmW8tKvb::SMEM_BYTES, GemmW8tKvb::THREADS);
        st.pairs_w8t_wo = max_pairs(mla::gemm_bf16_w8t_kernel<GemmW8tWo>, GemmW8tWo::SMEM_BYTES, GemmW8tWo::THREADS);
        st.pairs_unabs = max_pairs(mla::gemm_bf16_tc2_kernel<Gemm2Unabs>, Gemm2Unabs::SMEM_BYTES);
        st.pairs_wo_narrow = max_pairs(mla::gemm_bf16_tc2_kernel<Gemm2WoNarrow>, Gemm2WoNarrow::SMEM_BYTES);
        ok = ok && st.pairs_kvb > 0 && st.pairs_wo > 0 && st.pairs_w8t_kvb > 0 && st.pairs_w8t_wo > 0 && st.pairs_unabs > 0 && st.pairs_wo_narrow > 0;
      }
      ok = ok && cudaFuncSetAttribute(mla::gemm_e4m3_tc2_kernel<Gemm8Kvb>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      Gemm8Kvb::SMEM_BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::gemm_e4m3_tc2_kernel<Gemm8KvbAttn>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, Gemm8KvbAttn::SMEM_BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::gemm_e4m3_tc2_kernel<Gemm8Wo>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      Gemm8Wo::SMEM_BYTES) == cudaSuccess;
      if (ok) {
        st.pairs8_kvb = max_pairs(mla::gemm_e4m3_tc2_kernel<Gemm8Kvb>, Gemm8Kvb::SMEM_BYTES, Gemm8Kvb::THREADS);
        st.pairs8_wo = max_pairs(mla::gemm_e4m3_tc2_kernel<Gemm8Wo>, Gemm8Wo::SMEM_BYTES, Gemm8Wo::THREADS);
        ok = st.pairs8_kvb > 0 && st.pairs8_wo > 0;
      }
      ok = ok && cudaFuncSetAttribute(mla::gemm_m64_kernel<GemmM64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      GemmM64::SMEM_BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::gemm_m64_kernel<GemmM128>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, GemmM128::SMEM_BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::gemm_m64_kernel<GemmM64Abs>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, GemmM64Abs::SMEM_BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::gemm_m64_kernel<GemmM128Abs>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, GemmM128Abs::SMEM_BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::gemm_m64_kernel<GemmM64Unabs>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, GemmM64Unabs::SMEM_BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::gemm_m64_kernel<GemmM128Unabs>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      GemmM128Unabs::SMEM_BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::absorbed_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      mla::AbsSmem::BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::sparse_mla_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      mla::AttnSmem::BYTES) == cudaSuccess;
      ok = ok && cudaFuncSetAttribute(mla::topk_bitmap_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      mla::kPrepassWarps * (MLA_MAX_T / 128) * 16) == cudaSuccess;
      if (ok && g_encode == nullptr) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        ok = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
             q == cudaDriverEntryPointSuccess && fn != nullptr;
        if (ok) g_encode = reinterpret_cast<EncodeTiledFn>(fn);
      }
      st.status = ok ? MLA_OK : MLA_ERR_CUDA;
    }
  }
  *out = &st;
  return st.status;
}

// ------------------------------------------------------------------ tensor maps

// Row-major bf16/u8 matrix [outer, inner] with a row pitch; box
// [box_outer, box_inner]; 128-byte swizzle; out-of-range rows read as zero.
bool map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
            uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer,
            CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t es[2] = {1, 1};
  return g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 tensor [B, T, inner] (row pitch inner*2 bytes), box [1, box_rows, 64];
// rows past T read as zero.
bool map_3d_bt(CUtensorMap* m, const void* base, uint64_t inner, uint64_t T, uint64_t B, uint32_t box_rows = 128) {
  const cuuint64_t dims[3] = {inner, T, B};
  const cuuint64_t strides[2] = {inner * 2, inner * 2 * T};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// How e4m3 weights meet bf16 activations (mla_set_e4m3_weight_conversion):
// 0 = dequantised into a bf16 workspace copy per call, 1 = converted on chip
// by the projection GEMMs.
int g_e4m3_onchip = 0;

// ------------------------------------------------------------------ profiling

struct ProfRecord {
  int cls;
  cudaEvent_t start, stop;
};

struct Profiler {
  bool on = false;
  std::vector<ProfRecord> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};
thread_local Profiler t_prof;

// Runs `launch` on `stream`, bracketed by events when profiling is on.
template <class F>
int timed_launch(int cls, cudaStream_t stream, F&& launch) {
  ProfRecord r{cls, nullptr, nullptr};
  if (t_prof.on) {
    r.start = t_prof.get();
    r.stop = t_prof.get();
    cudaEventRecord(r.start, stream);
  }
  launch();
  const cudaError_t e = cudaGetLastError();
  if (t_prof.on) {
    cudaEventRecord(r.stop, stream);
    t_prof.recs.push_back(r);
  }
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace

// ------------------------------------------------------------------ validation and workspace

namespace {

constexpr size_t kNone = ~size_t(0);
constexpr int64_t kMaxRows = int64_t(1) << 24;  // B*T limit (int32 tile coordinates with margin)

struct WsLayout {
  size_t kvh = kNone, attn = kNone, bitmap = kNone, blocks = kNone, wkvb = kNone, wo = kNone;
  size_t qabs = kNone, olat = kNone, lists = kNone, counts = kNone;  // absorbed path, one chunk of rows
  size_t part_ml = kNone, part_o = kNone;  // decode: partial results of split rows
  size_t lat8 = kNone, lat8_s = kNone;    // e4m3 activations: quantized latent and its scales
  size_t attn8 = kNone, attn8_s = kNone;  // e4m3 activations: quantized attention rows and scales
  int parts = 1;                          // decode: CTAs per (sequence, 64-head group)
  size_t wo_part = kNone;                 // decode: stream-K partial tiles of the output projection
  size_t wo_split = kNone;                // prefill: partial tiles of the output projection's K-split last wave
  int g_abs = 0;       // first tile group on the absorbed path (groups of 4 x 128 query rows)
  int abs_chunk = 0;   // absorbed rows processed per pass
  int kpad = 0;        // pitch of the per-row key lists
  size_t total = 0;
};

// Absorbed rows are processed in passes of at most this many rows of one
// batch element, which bounds the workspace (q_abs and o_lat are
// rows x H x 1 KB each).
constexpr int kAbsChunkRows = 2048;
// SM count the decode split is planned for (the workspace size cannot depend
// on the device; a different count only changes how full the waves are).
constexpr int kSmsForSplit = 148;
constexpr int kStreamKCtas = 256;  // upper bound on the stream-K grid (the SM count)
// K-split last wave of the prefill output projection (wo_split_plan): only
// for K of at least kSplitMinTileKb 64-deep blocks (H >= 32; a shorter tile's
// last wave ends before the partial sums would pay), each K range keeps at
// least kSplitMinKb blocks, and the workspace holds kSplitSlots partial tiles
// (the pair count of a 148-SM part; with more pairs the split only gets
// coarser).
constexpr int kSplitMinTileKb = 64;
constexpr int kSplitMinKb = 8;
constexpr int kSplitSlots = 74;
// Cost model for MLA_PATH_AUTO: a tile group goes absorbed when its middle
// row's causal prefix exceeds this many times the selection size. Measured
// on B200 at T = 32768, H = 128, top-k 2048: the block-dense kernel costs
// about 80 ps per (row, prefix key) for all heads, the absorbed kernel about
// 870 ps per (row, selected key) (2176 instead of 640 FLOP per head and key,
// M = 64 UMMAs, and every 64-head group gathers the row's keys from L2).
constexpr int kAbsorbRatio = 11;

// First tile group that runs on the absorbed path (== number of groups when
// none does).
int absorbed_first_group(const mla_dims& d, bool has_topk) {
  const int nq = (d.T + 127) / 128;
  const int ng = (nq + 3) / 4;
  if (!has_topk || d.path == MLA_PATH_BLOCK_DENSE || d.act == MLA_ACT_E4M3_DYNAMIC) return ng;
  if (d.path == MLA_PATH_ABSORBED) return 0;
  const int64_t k = d.topk < d.T ? d.topk : d.T;
  for (int g = 0; g < ng; ++g)
    if (int64_t(512) * g + 256 > int64_t(kAbsorbRatio) * k) return g;
  return ng;
}

int check_dims(const mla_dims* d) {
  if (d == nullptr) return MLA_ERR_NULL;
  if (d->d_nope != kDn || d->d_rope != kDr || d->d_v != kDv || d->d_latent != kL || d->d_model != kD)
    return MLA_ERR_UNSUPPORTED;
  if (d->wdtype != MLA_W_BF16 && d->wdtype != MLA_W_E4M3_BLOCK128) return MLA_ERR_UNSUPPORTED;
  if (d->B < 0 || d->T < 0 || d->H < 1 || d->T > MLA_MAX_T) return MLA_ERR_SHAPE;
  if (static_cast<int64_t>(d->B) * d->T > kMaxRows) return MLA_ERR_SHAPE;
  if (d->path != MLA_PATH_AUTO && d->path != MLA_PATH_BLOCK_DENSE && d->path != MLA_PATH_ABSORBED)
    return MLA_ERR_UNSUPPORTED;
  if (d->act != MLA_ACT_BF16 && d->act != MLA_ACT_E4M3_DYNAMIC) return MLA_ERR_UNSUPPORTED;
  if (d->act == MLA_ACT_E4M3_DYNAMIC && (d->wdtype != MLA_W_E4M3_BLOCK128 || d->path == MLA_PATH_ABSORBED))
    return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

WsLayout ws_layout(const mla_dims& d, int entry, bool has_topk) {
  WsLayout w;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = (off + bytes + 255) & ~size_t(255);
    return o;
  };
  const size_t rows = static_cast<size_t>(d.B) * d.T;
  const size_t H = d.H;
  const size_t nq = (static_cast<size_t>(d.T) + 127) / 128;
  const bool fp8 = d.wdtype == MLA_W_E4M3_BLOCK128;
  const bool attend = entry == MLA_ENTRY_ATTEND || entry == MLA_ENTRY_PREFILL;
  if (attend) {
    w.g_abs = absorbed_first_group(d, has_topk);
    if (w.g_abs > 0) w.kvh = take(rows * H * (kDn + kDv) * 2);  // block-dense rows only
    // The whole block keeps the attention rows in the workspace (as e4m3
    // codes + scales when the activations are quantized, see below).
    if (entry == MLA_ENTRY_PREFILL && d.act != MLA_ACT_E4M3_DYNAMIC) w.attn = take(rows * H * kDv * 2);
    if (has_topk) {
      w.bitmap = take(static_cast<size_t>(d.B) * (nq * (nq + 1) / 2) * 128 * 16);
      w.blocks = take(static_cast<size_t>(d.B) * ((nq + 3) / 4) * (nq + 2) * 4);
    }
    const int64_t abs_rows = int64_t(d.T) - int64_t(512) * w.g_abs;
    if (abs_rows > 0 && d.B > 0) {
      w.abs_chunk = static_cast<int>(abs_rows < kAbsChunkRows ? abs_rows : kAbsChunkRows);
      const int k = d.topk < d.T ? d.topk : d.T;
      w.kpad = (k + 63) / 64 * 64;
      const size_t ch = static_cast<size_t>(w.abs_chunk);
      w.qabs = take(ch * H * kL * 2);
      w.olat = take(ch * H * kL * 2);
      w.lists = take(ch * static_cast<size_t>(w.kpad) * 4);
      w.counts = take(ch * 4);
    }
  }
  if (entry == MLA_ENTRY_DECODE && d.B > 0) {
    const size_t B = d.B;
    const int k = has_topk ? (d.topk < d.T ? d.topk : d.T) : d.T;
    w.kpad = (k + 63) / 64 * 64;
    w.qabs = take(B * H * kL * 2);
    w.olat = take(B * H * kL * 2);
    w.lists = take(B * static_cast<size_t>(w.kpad) * 4);
    w.counts = take(B * 4);
    w.attn = take(B * H * kDv * 2);
    // Split each sequence's keys over several CTAs when B alone cannot fill
    // the device: about two waves of CTAs, at least four 64-key blocks each.
    const int hgroups = (d.H + 63) / 64;
    const int want = (2 * kSmsForSplit + d.B * hgroups - 1) / (d.B * hgroups);
    const int most = w.kpad / 64 / 4;
    w.parts = want < most ? want : most;
    if (w.parts > 16) w.parts = 16;
    if (w.parts < 1) w.parts = 1;
    if (w.parts > 1) {
      w.part_ml = take(B * w.parts * H * 8);
      w.part_o = take(B * w.parts * H * kL * 2);
    }
    // The output projection of up to 256 rows runs as a stream-K GEMM with
    // 64- or 128-row tiles: one fp32 partial tile per (CTA, tile) segment.
    if (d.B <= 256) {
      const int bm = d.B <= 64 ? 64 : 128;
      const size_t tiles = static_cast<size_t>((d.B + bm - 1) / bm) * (kD / 128);
      w.wo_part = take((kStreamKCtas + tiles) * bm * 128 * 4);
    }
  }
  const bool dec = entry == MLA_ENTRY_DECODE;
  const bool act8 = d.act == MLA_ACT_E4M3_DYNAMIC;
  if (act8) {
    if (attend || entry == MLA_ENTRY_KV_UPPROJECT) {
      w.lat8 = take(rows * kL);
      w.lat8_s = take(rows * (kL / 128) * 4);
    }
    if (entry == MLA_ENTRY_PREFILL || entry == MLA_ENTRY_OUT_PROJECT) {
      w.attn8 = take(rows * H * kDv);
      w.attn8_s = take(rows * H * 4);
    }
  } else {
    // bf16 W_o over more than one row tile with a long K: partial tiles of
    // the K-split last wave.
    if (!fp8 && (entry == MLA_ENTRY_PREFILL || entry == MLA_ENTRY_OUT_PROJECT) && rows > 256 &&
        static_cast<int>(H * kDv / 64) >= kSplitMinTileKb)
      w.wo_split = take(static_cast<size_t>(kSplitSlots) * mla::SPLIT_SLOT_FLOATS * 4);
    if (!g_e4m3_onchip) {
      if (fp8 && (attend || dec || entry == MLA_ENTRY_KV_UPPROJECT)) w.wkvb = take(H * (kDn + kDv) * kL * 2);
      if (fp8 && (entry == MLA_ENTRY_PREFILL || dec || entry == MLA_ENTRY_OUT_PROJECT)) w.wo = take(H * kDv * kD * 2);
    } else {
      // On-chip conversion: only the absorbed rows' GEMMs and decode read a
      // bf16 copy of W_kvb (and decode one of W_o).
      const int ng = (static_cast<int>(nq) + 3) / 4;
      if (fp8 && ((attend && w.g_abs < ng) || dec)) w.wkvb = take(H * (kDn + kDv) * kL * 2);
      if (fp8 && dec) w.wo = take(H * kDv * kD * 2);
    }
  }
  w.total = off;
  return w;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

uint8_t* ws_at(void* ws, size_t off) { return static_cast<uint8_t*>(ws) + off; }

// ------------------------------------------------------------------ stage launchers

int launch_dequant(const DeviceState* ds, const void* codes, const float* scale, void* out, int rows, int cols,
                   cudaStream_t st) {
  const int64_t groups = static_cast<int64_t>(rows) * (cols / 16);
  const int64_t want = (groups + 255) / 256;
  const int grid = static_cast<int>(want < int64_t(ds->sms) * 8 ? want : int64_t(ds->sms) * 8);
  return timed_launch(1, st, [&] {
    mla::dequant_e4m3_block128_kernel<<<grid, 256, 0, st>>>(static_cast<const uint8_t*>(codes), scale,
                                                            static_cast<__nv_bfloat16*>(out), rows, cols);
  });
}

constexpr mla::GemmBatch kOneGemm = {1, 0, 0, 0, 0, 0, 0};

template <class Cfg>
int launch_gemm_pair(int pairs_max, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, int M,
                     int N, int K, int* err, int cls, cudaStream_t st, const mla::GemmBatch& bt = kOneGemm,
                     const mla::GemmSplit& sk = mla::kNoSplit) {
  const int tiles = ((M + Cfg::BM - 1) / Cfg::BM) * (N / Cfg::BN) * bt.count;
  const int pairs = tiles < pairs_max ? tiles : pairs_max;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t le = cudaSuccess;
  const int rc = timed_launch(
      cls, st, [&] { le = cudaLaunchKernelEx(&cfg, mla::gemm_bf16_tc2_kernel<Cfg>, ta, tb, tc, M, N, K, bt, sk, err); });
  return le != cudaSuccess ? MLA_ERR_CUDA : rc;
}

// v_f16: store the v half of every head as f16 (the attention path's kvh).
int launch_gemm_kvb(const DeviceState* ds, int M, int H, const void* lat, const void* wkvb, void* kvh, bool v_f16,
                    cudaStream_t st) {
  const int N = H * (kDn + kDv), K = kL;
  CUtensorMap ta, tb, tc;
  if (!map_2d(&ta, lat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, M, K * 2, 64, 128) ||
      !map_2d(&tb, wkvb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, N, K * 2, 64, Gemm2Kvb::HN) ||
      !map_2d(&tc, kvh, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, static_cast<uint64_t>(N) * 2, 64, 32))
    return MLA_ERR_CUDA;
  if (v_f16) return launch_gemm_pair<Gemm2KvbAttn>(ds->pairs_kvb, ta, tb, tc, M, N, K, ds->err, 2, st);
  return launch_gemm_pair<Gemm2Kvb>(ds->pairs_kvb, ta, tb, tc, M, N, K, ds->err, 2, st);
}

// K-split of the output projection's last wave (mla::GemmSplit): how many
// last-wave tiles are split (tail) and into how many K ranges (split), for a
// grid of `pairs` CTA pairs. Each range keeps at least kSplitMinKb 64-deep K
// blocks, and tail * split stays within the kSplitSlots partial tiles the
// workspace holds; no split (tail 0) when K is short, the waves are whole or
// fewer than two ranges would result.
mla::GemmSplit wo_split_plan(int tiles, int pairs, int num_kb, float* part) {
  mla::GemmSplit sk = mla::kNoSplit;
  if (part == nullptr || pairs <= 0 || num_kb < kSplitMinTileKb) return sk;
  const int tail = tiles % pairs;
  if (tail == 0) return sk;
  int split = pairs / tail;
  if (split > num_kb / kSplitMinKb) split = num_kb / kSplitMinKb;
  if (split > kSplitSlots / tail) split = kSplitSlots / tail;
  if (split < 2) return sk;
  sk.part = part;
  sk.tail = tail;
  sk.split = split;
  return sk;
}

// split_part: kSplitSlots * SPLIT_SLOT_FLOATS fp32 of workspace for the
// K-split last wave, or nullptr (every tile whole, e.g. so that the result
// matches another kernel's whole-K tiles bit for bit).
int launch_gemm_wo(const DeviceState* ds, int M, int H, const void* attn, const void* wo, void* out,
                   cudaStream_t st, float* split_part = nullptr) {
  const int N = kD, K = H * kDv;
  CUtensorMap ta, tb, tc;
  if (!map_2d(&ta, attn, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, M, static_cast<uint64_t>(K) * 2, 64, 128) ||
      !map_2d(&tb, wo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, K, static_cast<uint64_t>(N) * 2, 64, 64) ||
      !map_2d(&tc, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, static_cast<uint64_t>(N) * 2, 64, 32))
    return MLA_ERR_CUDA;
  // With a single row tile (decode) the 256-wide tiles would leave most SMs
  // idle while W_o streams through; 128-wide tiles double the pairs.
  if (M <= Gemm2WoNarrow::BM)
    return launch_gemm_pair<Gemm2WoNarrow>(ds->pairs_wo_narrow, ta, tb, tc, M, N, K, ds->err, 4, st);
  const int num_m = (M + Gemm2Wo::BM - 1) / Gemm2Wo::BM, num_n = N / Gemm2Wo::BN;
  const int tiles = num_m * num_n;
  const int pairs = tiles < ds->pairs_wo ? tiles : ds->pairs_wo;
  const mla::GemmSplit sk = wo_split_plan(tiles, pairs, K / Gemm2Wo::BK, split_part);
  int rc = launch_gemm_pair<Gemm2Wo>(ds->pairs_wo, ta, tb, tc, M, N, K, ds->err, 4, st, kOneGemm, sk);
  if (rc != MLA_OK || sk.tail == 0) return rc;
  const int threads = sk.tail * (mla::SPLIT_SLOT_FLOATS / 4);
  return timed_launch(9, st, [&] {
    mla::gemm_split_sum_kernel<<<(threads + 255) / 256, 256, 0, st>>>(
        sk.part, static_cast<__nv_bfloat16*>(out), M, N, num_m, num_n, Gemm2Wo::GROUP_M, tiles - sk.tail, sk.tail,
        sk.split);
  });
}

template <class Cfg>
int launch_gemm_w8t(int pairs_max, const CUtensorMap& tx, const CUtensorMap& tw, const mla::GemmW8tArgs& g, int cls,
                    cudaStream_t st) {
  const int64_t ut = static_cast<int64_t>(Cfg::NT) * Cfg::BN;  // tokens per unit
  const int64_t units = static_cast<int64_t>(g.F / Cfg::BM) * ((g.R + ut - 1) / ut);
  const int pairs = units < pairs_max ? static_cast<int>(units) : pairs_max;
  if (pairs <= 0) return MLA_OK;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t le = cudaSuccess;
  const int rc = timed_launch(cls, st, [&] { le = cudaLaunchKernelEx(&cfg, mla::gemm_bf16_w8t_kernel<Cfg>, tx, tw, g); });
  return le != cudaSuccess ? MLA_ERR_CUDA : rc;
}

// kvh = latent . W_kvb^T with W_kvb as e4m3 codes [H*256, 512] and 128 x 128
// block scales, converted on chip (no dequantised copy).
int launch_gemm_w8t_kvb(const DeviceState* ds, int M, int H, const void* lat, const void* wkvb, const float* wkvb_s,
                        void* kvh, bool v_f16, cudaStream_t st) {
  const int N = H * (kDn + kDv), K = kL;
  CUtensorMap tx, tw;
  if (!map_2d(&tx, lat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, M, K * 2, 64, GemmW8tKvb::HN) ||
      !map_2d(&tw, wkvb, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, N, K, 64, 128, CU_TENSOR_MAP_SWIZZLE_64B))
    return MLA_ERR_CUDA;
  const mla::GemmW8tArgs g = {wkvb_s, kvh, M, N, K, ds->err};
  if (v_f16) return launch_gemm_w8t<GemmW8tKvbAttn>(ds->pairs_w8t_kvb, tx, tw, g, 2, st);
  return launch_gemm_w8t<GemmW8tKvb>(ds->pairs_w8t_kvb, tx, tw, g, 2, st);
}

// out = attn . W_o with W_o as e4m3 codes [H*128, 7168] and block scales,
// converted on chip.
int launch_gemm_w8t_wo(const DeviceState* ds, int M, int H, const void* attn, const void* wo, const float* wo_s,
                       void* out, cudaStream_t st) {
  const int N = kD, K = H * kDv;
  CUtensorMap tx, tw;
  if (!map_2d(&tx, attn, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, M, static_cast<uint64_t>(K) * 2, 64, GemmW8tWo::HN) ||
      !map_2d(&tw, wo, CU_TENSOR_MAP_DATA_TYPE_UINT8, N, K, N, 128, 64, CU_TENSOR_MAP_SWIZZLE_NONE))
    return MLA_ERR_CUDA;
  const mla::GemmW8tArgs g = {wo_s, out, M, N, K, ds->err};
  return launch_gemm_w8t<GemmW8tWo>(ds->pairs_w8t_wo, tx, tw, g, 4, st);
}

// Dynamic e4m3 quantization of a bf16 [rows, cols] matrix: codes [rows, cols],
// scales [cols / 128, rows].
int launch_quant(const void* x, int rows, int cols, void* codes, float* scales, cudaStream_t st) {
  const int64_t items = static_cast<int64_t>(rows) * (cols / 128);
  const int64_t per_block = int64_t(2) * mla::kQuantWarps * mla::kQuantItemsPerHalfWarp;
  const unsigned grid = static_cast<unsigned>((items + per_block - 1) / per_block);
  if (grid == 0) return MLA_OK;
  return timed_launch(8, st, [&] {
    mla::quant_e4m3_1x128_kernel<<<grid, 32 * mla::kQuantWarps, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), rows, cols, static_cast<uint8_t*>(codes), scales);
  });
}

template <class Cfg>
int launch_gemm8_pair(int pairs_max, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, int M,
                      int N, int K, const mla::Gemm8Scales& sc, int* err, int cls, cudaStream_t st) {
  const int tiles = ((M + Cfg::BM - 1) / Cfg::BM) * (N / Cfg::BN);
  const int pairs = tiles < pairs_max ? tiles : pairs_max;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t le = cudaSuccess;
  const int rc = timed_launch(
      cls, st, [&] { le = cudaLaunchKernelEx(&cfg, mla::gemm_e4m3_tc2_kernel<Cfg>, ta, tb, tc, M, N, K, sc, err); });
  return le != cudaSuccess ? MLA_ERR_CUDA : rc;
}

// e4m3 up-projection: lat8 codes [M, 512] with scales [4, M] times the e4m3
// W_kvb [H*256, 512] with block scales [2H, 4].
int launch_gemm8_kvb(const DeviceState* ds, int M, int H, const void* lat8, const float* lat_s, const void* wkvb,
                     const float* wkvb_s, void* kvh, bool v_f16, cudaStream_t st) {
  const int N = H * (kDn + kDv), K = kL;
  CUtensorMap ta, tb, tc;
  if (!map_2d(&ta, lat8, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, M, K, 128, 128) ||
      !map_2d(&tb, wkvb, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, N, K, 128, Gemm8Kvb::HN) ||
      !map_2d(&tc, kvh, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, static_cast<uint64_t>(N) * 2, 64, 32))
    return MLA_ERR_CUDA;
  const mla::Gemm8Scales sc{lat_s, wkvb_s, 1, K / 128};
  if (v_f16) return launch_gemm8_pair<Gemm8KvbAttn>(ds->pairs8_kvb, ta, tb, tc, M, N, K, sc, ds->err, 2, st);
  return launch_gemm8_pair<Gemm8Kvb>(ds->pairs8_kvb, ta, tb, tc, M, N, K, sc, ds->err, 2, st);
}

// e4m3 output projection: attn8 codes [M, H*128] with scales [H, M] times
// the e4m3 W_o [H*128, 7168] with block scales [H, 56].
int launch_gemm8_wo(const DeviceState* ds, int M, int H, const void* attn8, const float* attn_s, const void* wo,
                    const float* wo_s, void* out, cudaStream_t st) {
  const int N = kD, K = H * kDv;
  CUtensorMap ta, tb, tc;
  if (!map_2d(&ta, attn8, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, M, K, 128, 128) ||
      !map_2d(&tb, wo, CU_TENSOR_MAP_DATA_TYPE_UINT8, N, K, N, Gemm8Wo::HN, 128,
              Gemm8Wo::HN == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map_2d(&tc, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, static_cast<uint64_t>(N) * 2, 64, 32))
    return MLA_ERR_CUDA;
  const mla::Gemm8Scales sc{attn_s, wo_s, N / 128, 1};
  return launch_gemm8_pair<Gemm8Wo>(ds->pairs8_wo, ta, tb, tc, M, N, K, sc, ds->err, 4, st);
}

// One launch of the few-row GEMM: 64-row tiles for M <= 64, else 128-row
// tiles (Cfg64 / Cfg128); K columns of A per batch item, or the stream-K
// split of one GEMM over `grid` CTAs.
template <class Cfg64, class Cfg128>
int launch_m64(const DeviceState* ds, const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K,
               const mla::M64Batch& bt, int grid, float* part, void* out, int cls, cudaStream_t st) {
  const int bm = M <= 64 ? 64 : 128;
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
  return timed_launch(cls, st, [&] {
    if (bm == 64)
      mla::gemm_m64_kernel<Cfg64><<<grid, Cfg64::THREADS, Cfg64::SMEM_BYTES, st>>>(ta, tb, M, N, K, bt, part,
                                                                                         o, ds->err);
    else
      mla::gemm_m64_kernel<Cfg128><<<grid, Cfg128::THREADS, Cfg128::SMEM_BYTES, st>>>(ta, tb, M, N, K, bt,
                                                                                            part, o, ds->err);
  });
}

// Output projection of M <= 256 rows as a stream-K GEMM (M = 64 or 128 UMMA
// tiles): every CTA takes an equal share of the tiles' k-blocks and writes
// one fp32 partial tile per tile it touches into `part` (room for
// kStreamKCtas + tiles of them); a second kernel sums them into `out`.
int launch_gemm_wo_m64(const DeviceState* ds, int M, int H, const void* attn, const void* wo, float* part,
                       void* out, cudaStream_t st) {
  const int N = kD, K = H * kDv;
  const int bm = M <= 64 ? 64 : 128;
  CUtensorMap ta, tb;
  if (!map_2d(&ta, attn, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, M, static_cast<uint64_t>(K) * 2, 64, bm) ||
      !map_2d(&tb, wo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, K, static_cast<uint64_t>(N) * 2, 64, 64))
    return MLA_ERR_CUDA;
  const int64_t units = static_cast<int64_t>((M + bm - 1) / bm) * (N / GemmM64::BN) * (K / GemmM64::BK);
  int grid = ds->sms < kStreamKCtas ? ds->sms : kStreamKCtas;
  if (units < grid) grid = static_cast<int>(units);
  const mla::M64Batch bt = {1, 0, 0, 0, 0, 0};
  int rc = launch_m64<GemmM64, GemmM128>(ds, ta, tb, M, N, K, bt, grid, part, nullptr, 4, st);
  if (rc != MLA_OK) return rc;
  const int blocks = ((M + bm - 1) / bm) * (N / GemmM64::BN) * (bm / mla::kSumRows);
  return timed_launch(4, st, [&] {
    mla::sum_segments_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(part, M, N, K, bm, grid,
                                                                            static_cast<__nv_bfloat16*>(out), ds->err);
  });
}

int launch_prepass(const DeviceState* ds, const mla_dims& d, const int32_t* topk, void* bitmap, void* blocks,
                   cudaStream_t st) {
  (void)ds;
  const int nq = (d.T + 127) / 128;
  const int64_t rows = static_cast<int64_t>(d.B) * nq * 128;
  const unsigned grid_rows = static_cast<unsigned>((rows + mla::kPrepassWarps - 1) / mla::kPrepassWarps);
  const size_t smem = static_cast<size_t>(mla::kPrepassWarps) * nq * 4 * 4;
  int rc = timed_launch(0, st, [&] {
    mla::topk_bitmap_rows_kernel<<<grid_rows, 32 * mla::kPrepassWarps, smem, st>>>(
        topk, d.B, d.T, d.topk, nq, static_cast<uint4*>(bitmap));
  });
  if (rc != MLA_OK) return rc;
  dim3 grid((nq + 3) / 4, d.B);
  return timed_launch(0, st, [&] {
    mla::topk_block_list_kernel<<<grid, 32 * mla::kBlockListWarps, 0, st>>>(static_cast<const uint4*>(bitmap), nq,
                                                      static_cast<int32_t*>(blocks));
  });
}

// Block-dense attention for tile groups [0, ngroups_run).
// attn8 / attn8_s set: the output is written as e4m3 codes + scales (the
// input of the e4m3 output projection) instead of bf16.
int launch_attention(const DeviceState* ds, const mla_dims& d, const void* q, const void* kvh, const void* k_pe,
                     const void* bitmap, const void* blocks, float scale, void* attn, int ngroups_run,
                     cudaStream_t st, void* attn8 = nullptr, float* attn8_s = nullptr) {
  // Q tiles and V blocks are 128 rows; each CTA of a pair loads 64 keys of K.
  CUtensorMap tq, tk, tv, tpe;
  const uint64_t kv_inner = static_cast<uint64_t>(d.H) * (kDn + kDv);
  if (!map_3d_bt(&tq, q, static_cast<uint64_t>(d.H) * (kDn + kDr), d.T, d.B) ||
      !map_3d_bt(&tk, kvh, kv_inner, d.T, d.B, 64) || !map_3d_bt(&tv, kvh, kv_inner, d.T, d.B) ||
      !map_3d_bt(&tpe, k_pe, kDr, d.T, d.B, 64))
    return MLA_ERR_CUDA;
  mla::AttnParams p;
  p.B = d.B;
  p.T = d.T;
  p.H = d.H;
  p.nq = (d.T + 127) / 128;
  p.gpitch = (p.nq + 3) / 4;
  p.ngroups = ngroups_run;
  // Heads per scheduling group: the largest of 8, 4, 2, 1 that divides H and
  // keeps the group's K/V (T x 512 bytes per head and batch) near 48 MB or less.
  p.hgroup = 1;
  for (int g = 8; g > 1; g /= 2) {
    if (d.H % g == 0 && static_cast<int64_t>(g) * d.B * d.T * 512 <= (int64_t(48) << 20)) {
      p.hgroup = g;
      break;
    }
  }
  p.scale_log2 = scale * 1.4426950408889634f;
  p.bitmap = static_cast<const uint4*>(bitmap);
  p.blocks = static_cast<const int32_t*>(blocks);
  p.attn = static_cast<__nv_bfloat16*>(attn);
  p.attn8 = static_cast<uint8_t*>(attn8);
  p.attn8_s = attn8_s;
  p.err = ds->err;
  const int64_t pairs = static_cast<int64_t>(d.B) * p.ngroups * d.H;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
  cfg.blockDim = dim3(mla::kAttnThreads, 1, 1);
  cfg.dynamicSmemBytes = mla::AttnSmem::BYTES;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t le = cudaSuccess;
  const int rc = timed_launch(3, st, [&] { le = cudaLaunchKernelEx(&cfg, mla::sparse_mla_attn_kernel, tq, tk, tv, tpe, p); });
  return le != cudaSuccess ? MLA_ERR_CUDA : rc;
}

// Selected keys of rows s0 .. s0+rows-1 of batch element b, from the bitmap.
int launch_row_lists(const mla_dims& d, const void* bitmap, int b, int s0, int rows, int kpad, int32_t* lists,
                     int32_t* counts, cudaStream_t st) {
  const int nq = (d.T + 127) / 128;
  const unsigned grid = static_cast<unsigned>((rows + mla::kPrepassWarps - 1) / mla::kPrepassWarps);
  return timed_launch(5, st, [&] {
    mla::topk_row_lists_kernel<<<grid, 32 * mla::kPrepassWarps, 0, st>>>(static_cast<const uint4*>(bitmap), nq, d.T,
                                                                          b, s0, rows, kpad, lists, counts);
  });
}

// Decode: selected cache positions of each sequence's new query.
int launch_decode_lists(const mla_dims& d, const int32_t* topk, int kpad, int32_t* lists, int32_t* counts,
                        cudaStream_t st) {
  return timed_launch(5, st, [&] {
    mla::decode_row_lists_kernel<<<static_cast<unsigned>(d.B), mla::kDecodeListThreads, 0, st>>>(
        topk, d.T, topk ? d.topk : 0, kpad, lists, counts);
  });
}

// Up to this many rows the per-head GEMMs run on the few-row kernel (64- or
// 128-row UMMA tiles, one CTA per item), beyond it on the CTA-pair GEMM.
constexpr int kFewRows = 256;

// q_abs[r, h, :] = q[r, h, 0:128] . W_kvb[h*256 + (0..127), :] for `rows`
// consecutive rows: one GEMM per head (M = rows, N = 512, K = 128).
int launch_gemm_absorb(const DeviceState* ds, int H, int rows, const void* q_rows, const void* wk, void* qabs,
                       cudaStream_t st) {
  CUtensorMap ta, tb, tc;
  const uint64_t qw = static_cast<uint64_t>(H) * (kDn + kDr);
  if (rows <= kFewRows) {
    if (!map_2d(&ta, q_rows, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, qw, rows, qw * 2, 64, rows <= 64 ? 64 : 128) ||
        !map_2d(&tb, wk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kL, static_cast<uint64_t>(H) * (kDn + kDv), kL * 2, 64, 64))
      return MLA_ERR_CUDA;
    const mla::M64Batch bt = {H, kDn + kDr, 0, kDn + kDv, kL, H * kL};
    const int items = (rows <= 64 ? 1 : (rows + 127) / 128) * (kL / 128) * H;
    return launch_m64<GemmM64Abs, GemmM128Abs>(ds, ta, tb, rows, kL, kDn, bt, items < ds->sms ? items : ds->sms,
                                               nullptr, qabs, 6, st);
  }
  if (!map_2d(&ta, q_rows, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, qw, rows, qw * 2, 64, 128) ||
      !map_2d(&tb, wk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kL, static_cast<uint64_t>(H) * (kDn + kDv), kL * 2, 64, 64) ||
      !map_2d(&tc, qabs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<uint64_t>(H) * kL, rows,
              static_cast<uint64_t>(H) * kL * 2, 64, 32))
    return MLA_ERR_CUDA;
  const mla::GemmBatch bt = {H, 0, kDn + kDr, 0, kDn + kDv, 0, kL};
  return launch_gemm_pair<Gemm2Wo>(ds->pairs_wo, ta, tb, tc, rows, kL, kDn, ds->err, 6, st, bt);
}

// attn[r, h, :] = o_lat[r, h, :] . W_kvb[h*256 + 128 + (0..127), :]^T: one
// GEMM per head (M = rows, N = 128, K = 512).
int launch_gemm_unabsorb(const DeviceState* ds, int H, int rows, const void* olat, const void* wk, void* attn_rows,
                         cudaStream_t st) {
  CUtensorMap ta, tb, tc;
  if (rows <= kFewRows) {
    if (!map_2d(&ta, olat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<uint64_t>(H) * kL, rows,
                static_cast<uint64_t>(H) * kL * 2, 64, rows <= 64 ? 64 : 128) ||
        !map_2d(&tb, wk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kL, static_cast<uint64_t>(H) * (kDn + kDv), kL * 2, 64,
                128))
      return MLA_ERR_CUDA;
    const mla::M64Batch bt = {H, kL, kDn, kDn + kDv, kDv, H * kDv};
    const int items = (rows <= 64 ? 1 : (rows + 127) / 128) * H;
    return launch_m64<GemmM64Unabs, GemmM128Unabs>(ds, ta, tb, rows, kDv, kL, bt, items < ds->sms ? items : ds->sms,
                                                   nullptr, attn_rows, 6, st);
  }
  if (!map_2d(&ta, olat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<uint64_t>(H) * kL, rows,
              static_cast<uint64_t>(H) * kL * 2, 64, 128) ||
      !map_2d(&tb, wk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kL, static_cast<uint64_t>(H) * (kDn + kDv), kL * 2, 64,
              Gemm2Unabs::HN) ||
      !map_2d(&tc, attn_rows, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<uint64_t>(H) * kDv, rows,
              static_cast<uint64_t>(H) * kDv * 2, 64, 32))
    return MLA_ERR_CUDA;
  const mla::GemmBatch bt = {H, 0, kL, kDn, kDn + kDv, 0, kDv};
  return launch_gemm_pair<Gemm2Unabs>(ds->pairs_unabs, ta, tb, tc, rows, kDv, kL, ds->err, 6, st, bt);
}

// Absorbed attention for `rows` rows (one CTA per row and group of 64 heads).
int launch_attention_absorbed(const DeviceState* ds, const mla_dims& d, const void* lat, const void* k_pe, int rows,
                              int key_row0, int rows_per_seq, int seq_stride, int kpad, const int32_t* lists,
                              const int32_t* counts, const void* qabs,
                              const void* q_rows, void* olat, float scale, cudaStream_t st, int parts = 1,
                              void* part_ml = nullptr, void* part_o = nullptr) {
  mla::AbsParams p;
  p.rows = rows;
  p.H = d.H;
  p.kpad = kpad;
  p.key_row0 = key_row0;
  p.rows_per_seq = rows_per_seq;
  p.seq_stride = seq_stride;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.lists = lists;
  p.counts = counts;
  p.qabs = static_cast<const __nv_bfloat16*>(qabs);
  p.q = static_cast<const __nv_bfloat16*>(q_rows);
  p.lat = static_cast<const __nv_bfloat16*>(lat);
  p.kpe = static_cast<const __nv_bfloat16*>(k_pe);
  p.olat = static_cast<__nv_bfloat16*>(olat);
  p.parts = parts;
  p.part_ml = static_cast<float2*>(part_ml);
  p.part_o = static_cast<__nv_bfloat16*>(part_o);
  p.err = ds->err;
  int rc = timed_launch(7, st, [&] {
    mla::absorbed_attn_kernel<<<static_cast<unsigned>(rows * ((d.H + 63) / 64) * parts), mla::kAbsThreads,
                                 mla::AbsSmem::BYTES, st>>>(p);
  });
  if (rc != MLA_OK || parts == 1) return rc;
  const int64_t items = static_cast<int64_t>(rows) * d.H;
  return timed_launch(7, st, [&] {
    mla::absorbed_combine_kernel<<<static_cast<unsigned>((items + mla::kCombineWarps - 1) / mla::kCombineWarps),
                                    32 * mla::kCombineWarps, 0, st>>>(p);
  });
}

}  // namespace

// ------------------------------------------------------------------ C ABI

namespace {

int begin_call(const mla_dims* dims, int entry, bool has_topk, void* ws, size_t ws_bytes, DeviceState** ds,
               WsLayout* lay) {
  int rc = check_dims(dims);
  if (rc != MLA_OK) return rc;
  *lay = ws_layout(*dims, entry, has_topk);
  if (lay->total > 0 && (ws == nullptr || ws_bytes < lay->total)) return MLA_ERR_WORKSPACE;
  if (ws != nullptr && !aligned16(ws)) return MLA_ERR_ALIGN;
  return device_state(ds);
}

// Up-projection into kvh; dequantises W_kvb into the workspace first when
// it is stored as e4m3.
int run_upproject(const DeviceState* ds, const mla_dims& d, const WsLayout& lay, void* ws, const void* lat,
                  const void* W_kvb, const float* W_kvb_scale, void* kvh, bool v_f16, cudaStream_t st) {
  if (d.act == MLA_ACT_E4M3_DYNAMIC) {
    const int M = d.B * d.T;
    void* lat8 = ws_at(ws, lay.lat8);
    float* lat_s = reinterpret_cast<float*>(ws_at(ws, lay.lat8_s));
    int rc = launch_quant(lat, M, kL, lat8, lat_s, st);
    if (rc != MLA_OK) return rc;
    return launch_gemm8_kvb(ds, M, d.H, lat8, lat_s, W_kvb, W_kvb_scale, kvh, v_f16, st);
  }
  const void* wk = W_kvb;
  if (d.wdtype == MLA_W_E4M3_BLOCK128) {
    if (g_e4m3_onchip) return launch_gemm_w8t_kvb(ds, d.B * d.T, d.H, lat, W_kvb, W_kvb_scale, kvh, v_f16, st);
    void* dq = ws_at(ws, lay.wkvb);
    int rc = launch_dequant(ds, W_kvb, W_kvb_scale, dq, d.H * (kDn + kDv), kL, st);
    if (rc != MLA_OK) return rc;
    wk = dq;
  }
  return launch_gemm_kvb(ds, d.B * d.T, d.H, lat, wk, kvh, v_f16, st);
}

int run_attend(const DeviceState* ds, const mla_dims& d, const WsLayout& lay, void* ws, const void* q,
               const void* lat, const void* k_pe, const void* W_kvb, const float* W_kvb_scale,
               const int32_t* topk_idx, float scale, void* attn, cudaStream_t st, void* attn8 = nullptr,
               float* attn8_s = nullptr) {
  const int nq = (d.T + 127) / 128;
  const int ng = (nq + 3) / 4;
  const void* wk = W_kvb;
  int rc = MLA_OK;
  const bool act8 = d.act == MLA_ACT_E4M3_DYNAMIC;  // every row block-dense (absorbed_first_group)
  // e4m3 W_kvb with bf16 activations: dequantised once into the workspace for
  // every GEMM of the call, or, with on-chip conversion, only for the
  // absorbed rows' absorb / un-absorb GEMMs (which read it as bf16).
  const bool onchip = d.wdtype == MLA_W_E4M3_BLOCK128 && !act8 && g_e4m3_onchip;
  if (d.wdtype == MLA_W_E4M3_BLOCK128 && !act8 && (!onchip || lay.g_abs < ng)) {
    void* dq = ws_at(ws, lay.wkvb);
    rc = launch_dequant(ds, W_kvb, W_kvb_scale, dq, d.H * (kDn + kDv), kL, st);
    if (rc != MLA_OK) return rc;
    wk = dq;
  }
  void* kvh = nullptr;
  if (lay.g_abs > 0) {  // up-projected keys, for the block-dense rows only
    kvh = ws_at(ws, lay.kvh);
    rc = (act8 || onchip) ? run_upproject(ds, d, lay, ws, lat, W_kvb, W_kvb_scale, kvh, /*v_f16=*/true, st)
                          : launch_gemm_kvb(ds, d.B * d.T, d.H, lat, wk, kvh, /*v_f16=*/true, st);
    if (rc != MLA_OK) return rc;
  }
  void* bitmap = nullptr;
  void* blocks = nullptr;
  if (topk_idx != nullptr) {
    bitmap = ws_at(ws, lay.bitmap);
    blocks = ws_at(ws, lay.blocks);
    rc = launch_prepass(ds, d, topk_idx, bitmap, blocks, st);
    if (rc != MLA_OK) return rc;
  }
  if (lay.g_abs > 0) {
    rc = launch_attention(ds, d, q, kvh, k_pe, bitmap, blocks, scale, attn, lay.g_abs, st, attn8, attn8_s);
    if (rc != MLA_OK) return rc;
  }
  if (lay.g_abs >= ng) return MLA_OK;
  // Absorbed rows [512 * g_abs, T) of every batch element, in passes.
  void* qabs = ws_at(ws, lay.qabs);
  void* olat = ws_at(ws, lay.olat);
  int32_t* lists = reinterpret_cast<int32_t*>(ws_at(ws, lay.lists));
  int32_t* counts = reinterpret_cast<int32_t*>(ws_at(ws, lay.counts));
  const size_t qrow = static_cast<size_t>(d.H) * (kDn + kDr) * 2, arow = static_cast<size_t>(d.H) * kDv * 2;
  for (int b = 0; b < d.B; ++b) {
    for (int s0 = 512 * lay.g_abs; s0 < d.T; s0 += lay.abs_chunk) {
      const int rows = d.T - s0 < lay.abs_chunk ? d.T - s0 : lay.abs_chunk;
      const size_t r0 = static_cast<size_t>(b) * d.T + s0;
      const void* q_rows = static_cast<const uint8_t*>(q) + r0 * qrow;
      void* attn_rows = static_cast<uint8_t*>(attn) + r0 * arow;
      if ((rc = launch_row_lists(d, bitmap, b, s0, rows, lay.kpad, lists, counts, st)) != MLA_OK) return rc;
      if ((rc = launch_gemm_absorb(ds, d.H, rows, q_rows, wk, qabs, st)) != MLA_OK) return rc;
      if ((rc = launch_attention_absorbed(ds, d, lat, k_pe, rows, b * d.T, rows, 0, lay.kpad, lists, counts, qabs,
                                          q_rows, olat, scale, st)) != MLA_OK)
        return rc;
      if ((rc = launch_gemm_unabsorb(ds, d.H, rows, olat, wk, attn_rows, st)) != MLA_OK) return rc;
    }
  }
  return MLA_OK;
}

int run_out_project(const DeviceState* ds, const mla_dims& d, const WsLayout& lay, void* ws, const void* attn,
                    const void* W_o, const float* W_o_scale, void* out, cudaStream_t st) {
  if (d.act == MLA_ACT_E4M3_DYNAMIC) {
    const int M = d.B * d.T;
    void* attn8 = ws_at(ws, lay.attn8);
    float* attn_s = reinterpret_cast<float*>(ws_at(ws, lay.attn8_s));
    int rc = launch_quant(attn, M, d.H * kDv, attn8, attn_s, st);
    if (rc != MLA_OK) return rc;
    return launch_gemm8_wo(ds, M, d.H, attn8, attn_s, W_o, W_o_scale, out, st);
  }
  const void* wo = W_o;
  if (d.wdtype == MLA_W_E4M3_BLOCK128 && g_e4m3_onchip)
    return launch_gemm_w8t_wo(ds, d.B * d.T, d.H, attn, W_o, W_o_scale, out, st);
  if (d.wdtype == MLA_W_E4M3_BLOCK128) {
    // Whole-K tiles only, so that both e4m3 conversion modes give the same bits.
    void* dq = ws_at(ws, lay.wo);
    int rc = launch_dequant(ds, W_o, W_o_scale, dq, d.H * kDv, kD, st);
    if (rc != MLA_OK) return rc;
    return launch_gemm_wo(ds, d.B * d.T, d.H, attn, dq, out, st);
  }
  float* split = lay.wo_split == kNone ? nullptr : reinterpret_cast<float*>(ws_at(ws, lay.wo_split));
  return launch_gemm_wo(ds, d.B * d.T, d.H, attn, wo, out, st, split);
}

// Decode: one new query per sequence (row s = T-1) against the cache, in the
// absorbed form.
int run_decode(const DeviceState* ds, const mla_dims& d, const WsLayout& lay, void* ws, const void* q,
               const void* lat, const void* k_pe, const void* W_kvb, const float* W_kvb_scale, const void* W_o,
               const float* W_o_scale, const int32_t* topk_idx, float scale, void* out, cudaStream_t st) {
  const void* wk = W_kvb;
  int rc = MLA_OK;
  if (d.wdtype == MLA_W_E4M3_BLOCK128) {
    void* dq = ws_at(ws, lay.wkvb);
    if ((rc = launch_dequant(ds, W_kvb, W_kvb_scale, dq, d.H * (kDn + kDv), kL, st)) != MLA_OK) return rc;
    wk = dq;
  }
  void* qabs = ws_at(ws, lay.qabs);
  void* olat = ws_at(ws, lay.olat);
  void* attn = ws_at(ws, lay.attn);
  int32_t* lists = reinterpret_cast<int32_t*>(ws_at(ws, lay.lists));
  int32_t* counts = reinterpret_cast<int32_t*>(ws_at(ws, lay.counts));
  if ((rc = launch_decode_lists(d, topk_idx, lay.kpad, lists, counts, st)) != MLA_OK) return rc;
  if ((rc = launch_gemm_absorb(ds, d.H, d.B, q, wk, qabs, st)) != MLA_OK) return rc;
  if ((rc = launch_attention_absorbed(ds, d, lat, k_pe, d.B, 0, 1, d.T, lay.kpad, lists, counts, qabs, q, olat, scale,
                                      st, lay.parts, lay.parts > 1 ? ws_at(ws, lay.part_ml) : nullptr,
                                      lay.parts > 1 ? ws_at(ws, lay.part_o) : nullptr)) != MLA_OK)
    return rc;
  if ((rc = launch_gemm_unabsorb(ds, d.H, d.B, olat, wk, attn, st)) != MLA_OK) return rc;
  const void* wo = W_o;
  if (d.wdtype == MLA_W_E4M3_BLOCK128) {
    void* dq = ws_at(ws, lay.wo);
    if ((rc = launch_dequant(ds, W_o, W_o_scale, dq, d.H * kDv, kD, st)) != MLA_OK) return rc;
    wo = dq;
  }
  if (lay.wo_part != kNone)
    return launch_gemm_wo_m64(ds, d.B, d.H, attn, wo, reinterpret_cast<float*>(ws_at(ws, lay.wo_part)), out, st);
  return launch_gemm_wo(ds, d.B, d.H, attn, wo, out, st);
}

bool fp8_scales_ok(const mla_dims* d, const float* s) { return d->wdtype != MLA_W_E4M3_BLOCK128 || s != nullptr; }

}  // namespace

extern "C" {

size_t mla_workspace_bytes(const mla_dims* dims, int entry, int has_topk) {
  if (check_dims(dims) != MLA_OK || entry < MLA_ENTRY_KV_UPPROJECT || entry > MLA_ENTRY_DECODE) return 0;
  if (entry == MLA_ENTRY_DECODE && dims->act != MLA_ACT_BF16) return 0;
  return ws_layout(*dims, entry, has_topk != 0).total;
}

int mla_kv_upproject(const mla_dims* dims, const void* kv_latent, const void* W_kvb, const float* W_kvb_scale,
                     void* kvh_out, void* workspace, size_t ws_bytes, mla_stream_t stream) {
  DeviceState* ds = nullptr;
  WsLayout lay;
  int rc = check_dims(dims);
  if (rc != MLA_OK) return rc;
  if (static_cast<int64_t>(dims->B) * dims->T == 0) return MLA_OK;
  if (!kv_latent || !W_kvb || !kvh_out || !fp8_scales_ok(dims, W_kvb_scale)) return MLA_ERR_NULL;
  if (!aligned16(kv_latent) || !aligned16(W_kvb) || !aligned16(kvh_out) || !aligned16(W_kvb_scale))
    return MLA_ERR_ALIGN;
  rc = begin_call(dims, MLA_ENTRY_KV_UPPROJECT, false, workspace, ws_bytes, &ds, &lay);
  if (rc != MLA_OK) return rc;
  if (static_cast<int64_t>(dims->B) * dims->T == 0) return MLA_OK;
  return run_upproject(ds, *dims, lay, workspace, kv_latent, W_kvb, W_kvb_scale, kvh_out, /*v_f16=*/false,
                       reinterpret_cast<cudaStream_t>(stream));
}

int mla_attend(const mla_dims* dims, const void* q, const void* kv_latent, const void* k_pe, const void* W_kvb,
               const float* W_kvb_scale, const int32_t* topk_idx, float scale, void* attn_out, void* workspace,
               size_t ws_bytes, mla_stream_t stream) {
  DeviceState* ds = nullptr;
  WsLayout lay;
  int rc = check_dims(dims);
  if (rc != MLA_OK) return rc;
  if (static_cast<int64_t>(dims->B) * dims->T == 0) return MLA_OK;
  if (!q || !kv_latent || !k_pe || !W_kvb || !attn_out || !fp8_scales_ok(dims, W_kvb_scale)) return MLA_ERR_NULL;
  if (topk_idx != nullptr && dims->topk < 1) return MLA_ERR_SHAPE;
  if (!std::isfinite(scale) || !(scale > 0.f)) return MLA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(kv_latent) || !aligned16(k_pe) || !aligned16(W_kvb) || !aligned16(attn_out) ||
      !aligned16(W_kvb_scale) || !aligned16(topk_idx))
    return MLA_ERR_ALIGN;
  rc = begin_call(dims, MLA_ENTRY_ATTEND, topk_idx != nullptr, workspace, ws_bytes, &ds, &lay);
  if (rc != MLA_OK) return rc;
  if (static_cast<int64_t>(dims->B) * dims->T == 0) return MLA_OK;
  return run_attend(ds, *dims, lay, workspace, q, kv_latent, k_pe, W_kvb, W_kvb_scale, topk_idx, scale, attn_out,
                    reinterpret_cast<cudaStream_t>(stream));
}

int mla_out_project(const mla_dims* dims, const void* attn, const void* W_o, const float* W_o_scale, void* out,
                    void* workspace, size_t ws_bytes, mla_stream_t stream) {
  DeviceState* ds = nullptr;
  WsLayout lay;
  int rc = check_dims(dims);
  if (rc != MLA_OK) return rc;
  if (static_cast<int64_t>(dims->B) * dims->T == 0) return MLA_OK;
  if (!attn || !W_o || !out || !fp8_scales_ok(dims, W_o_scale)) return MLA_ERR_NULL;
  if (!aligned16(attn) || !aligned16(W_o) || !aligned16(out) || !aligned16(W_o_scale)) return MLA_ERR_ALIGN;
  rc = begin_call(dims, MLA_ENTRY_OUT_PROJECT, false, workspace, ws_bytes, &ds, &lay);
  if (rc != MLA_OK) return rc;
  if (static_cast<int64_t>(dims->B) * dims->T == 0) return MLA_OK;
  return run_out_project(ds, *dims, lay, workspace, attn, W_o, W_o_scale, out,
                         reinterpret_cast<cudaStream_t>(stream));
}

int mla_prefill(const mla_dims* dims, const void* q, const void* kv_latent, const void* k_pe, const void* W_kvb,
                const float* W_kvb_scale, const void* W_o, const float* W_o_scale, const int32_t* topk_idx,
                float scale, void* out, void* workspace, size_t ws_bytes, mla_stream_t stream) {
  DeviceState* ds = nullptr;
  WsLayout lay;
  int rc = check_dims(dims);
  if (rc != MLA_OK) return rc;
  if (static_cast<int64_t>(dims->B) * dims->T == 0) return MLA_OK;
  if (!q || !kv_latent || !k_pe || !W_kvb || !W_o || !out || !fp8_scales_ok(dims, W_kvb_scale) ||
      !fp8_scales_ok(dims, W_o_scale))
    return MLA_ERR_NULL;
  if (topk_idx != nullptr && dims->topk < 1) return MLA_ERR_SHAPE;
  if (!std::isfinite(scale) || !(scale > 0.f)) return MLA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(kv_latent) || !aligned16(k_pe) || !aligned16(W_kvb) || !aligned16(W_o) ||
      !aligned16(out) || !aligned16(W_kvb_scale) || !aligned16(W_o_scale) || !aligned16(topk_idx))
    return MLA_ERR_ALIGN;
  rc = begin_call(dims, MLA_ENTRY_PREFILL, topk_idx != nullptr, workspace, ws_bytes, &ds, &lay);
  if (rc != MLA_OK) return rc;
  if (static_cast<int64_t>(dims->B) * dims->T == 0) return MLA_OK;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims->act == MLA_ACT_E4M3_DYNAMIC) {
    // The attention kernel writes its output already quantized (every row
    // is block-dense with e4m3 activations), so W_o reads the codes directly.
    void* attn8 = ws_at(workspace, lay.attn8);
    float* attn8_s = reinterpret_cast<float*>(ws_at(workspace, lay.attn8_s));
    rc = run_attend(ds, *dims, lay, workspace, q, kv_latent, k_pe, W_kvb, W_kvb_scale, topk_idx, scale, nullptr, st,
                    attn8, attn8_s);
    if (rc != MLA_OK) return rc;
    return launch_gemm8_wo(ds, dims->B * dims->T, dims->H, attn8, attn8_s, W_o, W_o_scale, out, st);
  }
  void* attn = ws_at(workspace, lay.attn);
  rc = run_attend(ds, *dims, lay, workspace, q, kv_latent, k_pe, W_kvb, W_kvb_scale, topk_idx, scale, attn, st);
  if (rc != MLA_OK) return rc;
  return run_out_project(ds, *dims, lay, workspace, attn, W_o, W_o_scale, out, st);
}

int mla_decode(const mla_dims* dims, const void* q, const void* kv_latent, const void* k_pe, const void* W_kvb,
               const float* W_kvb_scale, const void* W_o, const float* W_o_scale, const int32_t* topk_idx,
               float scale, void* out, void* workspace, size_t ws_bytes, mla_stream_t stream) {
  DeviceState* ds = nullptr;
  WsLayout lay;
  int rc = check_dims(dims);
  if (rc != MLA_OK) return rc;
  if (static_cast<int64_t>(dims->B) * dims->T == 0) return MLA_OK;
  if (!q || !kv_latent || !k_pe || !W_kvb || !W_o || !out || !fp8_scales_ok(dims, W_kvb_scale) ||
      !fp8_scales_ok(dims, W_o_scale))
    return MLA_ERR_NULL;
  if (topk_idx != nullptr && dims->topk < 1) return MLA_ERR_SHAPE;
  if (!std::isfinite(scale) || !(scale > 0.f)) return MLA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(kv_latent) || !aligned16(k_pe) || !aligned16(W_kvb) || !aligned16(W_o) ||
      !aligned16(out) || !aligned16(W_kvb_scale) || !aligned16(W_o_scale) || !aligned16(topk_idx))
    return MLA_ERR_ALIGN;
  if (dims->act != MLA_ACT_BF16) return MLA_ERR_UNSUPPORTED;
  rc = begin_call(dims, MLA_ENTRY_DECODE, topk_idx != nullptr, workspace, ws_bytes, &ds, &lay);
  if (rc != MLA_OK) return rc;
  return run_decode(ds, *dims, lay, workspace, q, kv_latent, k_pe, W_kvb, W_kvb_scale, W_o, W_o_scale, topk_idx,
                    scale, out, reinterpret_cast<cudaStream_t>(stream));
}

int mla_quantize_act(const void* x, int rows, int cols, void* codes, float* scales, mla_stream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 128 != 0) return MLA_ERR_SHAPE;
  if (static_cast<int64_t>(rows) * cols >= (int64_t(1) << 40)) return MLA_ERR_SHAPE;
  if (rows == 0) return MLA_OK;
  if (!x || !codes || !scales) return MLA_ERR_NULL;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return MLA_ERR_ALIGN;
  DeviceState* ds = nullptr;
  const int rc = device_state(&ds);
  if (rc != MLA_OK) return rc;
  return launch_quant(x, rows, cols, codes, scales, reinterpret_cast<cudaStream_t>(stream));
}

const char* mla_status_str(int status) {
  switch (status) {
    case MLA_OK: return "ok";
    case MLA_ERR_NULL: return "a required pointer is NULL";
    case MLA_ERR_SHAPE: return "a size is out of range";
    case MLA_ERR_UNSUPPORTED: return "unsupported head geometry, weight type or device";
    case MLA_ERR_WORKSPACE: return "workspace missing or too small";
    case MLA_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case MLA_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case MLA_ERR_DEVICE: return "a kernel recorded a device-side error";
    case MLA_ERR_TOO_LARGE: return "problem needs more scratch than the built-in MLA_STATIC_SCRATCH_BYTES";
    default: return "unknown status";
  }
}

int mla_device_status(mla_stream_t stream, int* device_error) {
  if (device_error == nullptr) return MLA_ERR_NULL;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != MLA_OK) return rc;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MLA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ds->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MLA_ERR_CUDA;
  if (v != 0 && cudaMemset(ds->err, 0, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  *device_error = v;
  return MLA_OK;
}

int mla_set_e4m3_weight_conversion(int onchip) {
  if (onchip != 0 && onchip != 1) return MLA_ERR_SHAPE;
  g_e4m3_onchip = onchip;
  return MLA_OK;
}

int mla_set_wait_timeout_ns(unsigned long long ns) {
  const unsigned long long v = ns == 0 ? mla::kWaitTimeoutNs : ns;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  return cudaMemcpyToSymbol(mla::g_mla_wait_timeout_ns, &v, sizeof v) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_test_withhold_attention_loads(int on) {
  const int v = on != 0 ? 1 : 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  return cudaMemcpyToSymbol(mla::g_mla_withhold_attn_loads, &v, sizeof v) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_test_wo_split_plan(int tiles, int pairs, int num_kb, int* tail, int* split) {
  if (tail == nullptr || split == nullptr) return MLA_ERR_NULL;
  if (tiles < 0 || pairs < 0 || num_kb < 0) return MLA_ERR_SHAPE;
  float dummy = 0.f;  // any non-null workspace pointer: the plan only tests it for null
  const mla::GemmSplit sk = wo_split_plan(tiles, pairs, num_kb, &dummy);
  *tail = sk.tail;
  *split = sk.split;
  return MLA_OK;
}

int mla_profile_begin(void) {
  for (auto& r : t_prof.recs) {
    t_prof.pool.push_back(r.start);
    t_prof.pool.push_back(r.stop);
  }
  t_prof.recs.clear();
  t_prof.on = true;
  return MLA_OK;
}

int mla_profile_end(float* ms_total, int* launches) {
  if (ms_total == nullptr || launches == nullptr) return MLA_ERR_NULL;
  for (int i = 0; i < MLA_PROFILE_CLASSES; ++i) {
    ms_total[i] = 0.f;
    launches[i] = 0;
  }
  int rc = MLA_OK;
  for (auto& r : t_prof.recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) {
      rc = MLA_ERR_CUDA;
      continue;
    }
    ms_total[r.cls] += ms;
    launches[r.cls] += 1;
  }
  for (auto& r : t_prof.recs) {
    t_prof.pool.push_back(r.start);
    t_prof.pool.push_back(r.stop);
  }
  t_prof.recs.clear();
  t_prof.on = false;
  return rc;
}

}  // extern "C"

// ------------------------------------------------------------------ built-in scratch entry point

// Scratch of mla_attend_static for callers that cannot allocate device
// memory. The module holds it on every GPU that loads the library.
__device__ __align__(256) uint8_t g_mla_static_scratch[MLA_STATIC_SCRATCH_BYTES];

namespace {

std::mutex g_static_mutex;
std::vector<uint8_t*> g_static_scratch;  // device address of the array, per device (NULL: not looked up)

// Device address of g_mla_static_scratch on the current device, looked up
// once per device. In host code the array's name is only a host-side
// stand-in, so kernels must be given this address instead.
int static_scratch(uint8_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (static_cast<int>(g_static_scratch.size()) <= dev) g_static_scratch.resize(dev + 1, nullptr);
  if (g_static_scratch[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mla_static_scratch) != cudaSuccess || p == nullptr) return MLA_ERR_CUDA;
    g_static_scratch[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_static_scratch[dev];
  return MLA_OK;
}

}  // namespace

extern "C" int mla_attend_static(const mla_dims* dims, const void* q, const void* kv_latent, const void* k_pe,
                                 const void* W_kvb, const float* W_kvb_scale, const int32_t* topk_idx, float scale,
                                 void* attn_out, mla_stream_t stream) {
  int rc = check_dims(dims);
  if (rc != MLA_OK) return rc;
  if (static_cast<int64_t>(dims->B) * dims->T == 0) return MLA_OK;
  if (!q || !kv_latent || !k_pe || !W_kvb || !attn_out || !fp8_scales_ok(dims, W_kvb_scale)) return MLA_ERR_NULL;
  if (topk_idx != nullptr && dims->topk < 1) return MLA_ERR_SHAPE;
  if (!std::isfinite(scale) || !(scale > 0.f)) return MLA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(kv_latent) || !aligned16(k_pe) || !aligned16(W_kvb) || !aligned16(attn_out) ||
      !aligned16(W_kvb_scale) || !aligned16(topk_idx))
    return MLA_ERR_ALIGN;
  const WsLayout lay = ws_layout(*dims, MLA_ENTRY_ATTEND, topk_idx != nullptr);
  if (lay.total > MLA_STATIC_SCRATCH_BYTES) return MLA_ERR_TOO_LARGE;
  DeviceState* ds = nullptr;
  rc = device_state(&ds);
  if (rc != MLA_OK) return rc;
  uint8_t* scratch = nullptr;
  rc = static_scratch(&scratch);
  if (rc != MLA_OK) return rc;
  return run_attend(ds, *dims, lay, scratch, q, kv_latent, k_pe, W_kvb, W_kvb_scale, topk_idx, scale, attn_out,
                    reinterpret_cast<cudaStream_t>(stream));
}
