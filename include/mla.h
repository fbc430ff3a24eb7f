/*
 * mla.h -- C ABI of the B200 (sm_100a) sparse MLA prefill attend block.
 *
 * The block is the full-sequence (prefill) path of multi-head latent
 * attention as given on the DeepSeek-V3.2-Exp "Sparse attention" page
 * (its prefill code) and the Kimi K2 "Output projection" page:
 *
 *   [k_nope_h | v_h][t] = W_kvb,h . kv_latent[t]              (wkv_b, view, split)
 *   k_h[t]              = k_nope_h[t] ++ k_pe[t]                (rotary key shared by heads)
 *   z[s,h,t]            = scale * <q[s,h], k_h[t]>              (scores)
 *   keep(s,t)           = t in topk_idx[s,:] and t <= s          (index mask + causal mask)
 *   attn[s,h]           = sum_t softmax_t(z | keep) v_h[t]      (softmax, value mix)
 *   out[s]              = flatten_h(attn[s]) . W_o              (wo(x.flatten(2)), Delta = o W_O)
 *
 * Conventions (all calls):
 *  - Every pointer argument except `workspace`'s host-side size is a DEVICE
 *    pointer owned by the caller, 16-byte aligned, on the current device.
 *    The library allocates no device memory; scratch lives in `workspace`.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and never synchronise. Host-side argument checks
 *    return a status synchronously, before anything is launched.
 *  - bf16 is IEEE binary16-bfloat (1-8-7); e4m3 is OCP FP8 E4M3FN.
 *  - Fixed head geometry: d_nope = 128, d_rope = 64, d_v = 128,
 *    d_latent = 512, d_model = 7168 (any other value: MLA_ERR_UNSUPPORTED).
 *    Any H >= 1, B >= 0, 0 <= T <= MLA_MAX_T. B*T == 0 is a no-op that
 *    returns MLA_OK right after the geometry check (NULL pointers allowed).
 *  - Inputs are read-only; outputs must not alias inputs or the workspace.
 *  - Kernels that wait on on-chip barriers give up after a bounded time and
 *    record an error word on the device instead of hanging; read it with
 *    mla_device_status().
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* mla_stream_t;

#define MLA_MAX_T 65536

typedef enum {
  MLA_OK = 0,
  MLA_ERR_NULL = 1,         /* a required pointer is NULL */
  MLA_ERR_SHAPE = 2,        /* a size is out of range (negative, T > MLA_MAX_T, topk < 1) */
  MLA_ERR_UNSUPPORTED = 3,  /* head geometry other than 128/64/128/512/7168, or no sm_100 device */
  MLA_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than mla_workspace_bytes() */
  MLA_ERR_CUDA = 5,         /* a CUDA runtime/driver call or a launch failed */
  MLA_ERR_ALIGN = 6,        /* a pointer is not 16-byte aligned */
  MLA_ERR_DEVICE = 7,       /* a kernel recorded a device-side error (see mla_device_status) */
  MLA_ERR_TOO_LARGE = 8     /* the problem needs more scratch than mla_attend_static's built-in
                               MLA_STATIC_SCRATCH_BYTES */
} mla_status;

typedef enum {
  MLA_W_BF16 = 0,          /* weights stored as bf16 */
  MLA_W_E4M3_BLOCK128 = 1  /* e4m3 codes, one fp32 scale per 128 x 128 block (Kimi K2
                              "Down projection" page: fmt e4m3, weight_block_size [128, 128]) */
} mla_wdtype;

/* How the attention rows are computed (same result up to rounding; see
 * mla_attend). AUTO picks per group of 512 query rows by a cost model. */
typedef enum {
  MLA_PATH_AUTO = 0,
  MLA_PATH_BLOCK_DENSE = 1,  /* every row: up-projected keys, 128-key blocks */
  MLA_PATH_ABSORBED = 2      /* every row with a topk_idx: absorbed form over the gathered keys */
} mla_path;

/* Activations entering the two projections (W_kvb, W_o).
 * MLA_ACT_E4M3_DYNAMIC follows the Kimi K2 "Down projection" page's
 * quantization_config (activation_scheme "dynamic", fmt "e4m3", 128 x 128
 * weight blocks): the latent rows entering W_kvb and the attention rows
 * entering W_o are quantized on the fly per row and group of 128 channels
 * (see mla_quantize_act) and the projections run as e4m3 x e4m3 tensor-core
 * GEMMs with the activation and weight block scales applied per 128-deep K
 * block. Needs wdtype MLA_W_E4M3_BLOCK128 and the block-dense attention path
 * (MLA_PATH_AUTO then means block-dense; MLA_PATH_ABSORBED and mla_decode
 * return MLA_ERR_UNSUPPORTED). */
typedef enum {
  MLA_ACT_BF16 = 0,          /* bf16 activations (weights dequantized for e4m3) */
  MLA_ACT_E4M3_DYNAMIC = 1   /* dynamic per-token 1 x 128 e4m3 activations */
} mla_act;

typedef struct {
  int B, T, H;
  int d_nope, d_rope, d_v, d_latent, d_model;
  int topk;          /* entries per row of topk_idx (ignored when topk_idx == NULL) */
  mla_wdtype wdtype; /* storage of W_kvb and W_o */
  mla_path path;     /* MLA_PATH_AUTO (0) unless a caller forces one path */
  mla_act act;       /* MLA_ACT_BF16 (0) unless the activations are quantized */
} mla_dims;

/* Entry points, for mla_workspace_bytes(). */
#define MLA_ENTRY_KV_UPPROJECT 0
#define MLA_ENTRY_ATTEND 1
#define MLA_ENTRY_OUT_PROJECT 2
#define MLA_ENTRY_PREFILL 3
#define MLA_ENTRY_DECODE 4

/* Device workspace bytes that `entry` needs for these dims (has_topk = 1
 * if a topk_idx will be passed). 0 when nothing is needed or the dims are
 * invalid. The library never allocates; the caller passes this much. */
size_t mla_workspace_bytes(const mla_dims* dims, int entry, int has_topk);

/* Step A2 -- W_kvb up-projection (DeepSeek-V3.2-Exp "Sparse attention",
 * `kv = self.wkv_b(kv)`; W_kvb shape from the MLA init, kv_b_proj
 * [H*(128+128), 512] stored [out, in]).
 *   kv_latent : bf16 [B*T, 512] (post-RMSNorm latent)
 *   W_kvb     : bf16 or e4m3 [H*256, 512]; row h*256+i is k_nope_h[i] for
 *               i < 128 and v_h[i-128] otherwise
 *   W_kvb_scale: fp32 [2H, 4] (block scales) for e4m3, else ignored
 *   kvh_out   : bf16 [B*T, H*256], same column order as W_kvb's rows
 * Uses the tcgen05 tensor-core GEMM; fp32 accumulation, bf16 rounding.
 * With dims->act = MLA_ACT_E4M3_DYNAMIC the latent is quantized first and
 * the GEMM is e4m3 x e4m3 (kind::f8f6f4) with per-block scales. */
int mla_kv_upproject(const mla_dims* dims, const void* kv_latent, const void* W_kvb,
                     const float* W_kvb_scale, void* kvh_out, void* workspace,
                     size_t ws_bytes, mla_stream_t stream);

/* Steps A0-A5 -- up-projection, then sparse-causal attention
 * (DeepSeek-V3.2-Exp "Sparse attention": scores, index mask + causal mask,
 * softmax, value mix). Stops before W_o.
 *   q        : bf16 [B, T, H, 192]: 128 non-rotary dims then 64 rotary dims
 *   kv_latent: bf16 [B, T, 512]
 *   k_pe     : bf16 [B, T, 64], rotated, shared by all heads
 *   W_kvb, W_kvb_scale: as for mla_kv_upproject
 *   topk_idx : int32 [B, T, topk] key indices per query, any order; NULL =
 *              causal mask only (top-k >= T). Duplicates select once;
 *              entries outside [0, T) select nothing; entries > s are
 *              removed by the causal mask.
 *   scale    : softmax scale applied to q.k, finite and > 0 (192^-0.5 for
 *              these models)
 *   attn_out : bf16 [B, T, H, 128]. A query with no surviving key gets 0.
 * Softmax in fp32 (exp2 form). On the block-dense path the softmax weights
 * P and the up-projected values v enter the PV product as f16 (three more
 * mantissa bits than bf16): every |v| must stay below 65504 (the f16
 * range). A larger v (|v| >= 65520 rounds to infinity) is detected in the
 * up-projection's epilogue and recorded as device error 301 (see
 * mla_device_status); the attention rows that read it are then undefined.
 * RMS-normalised latents with trained weights give |v| of order 10.
 * Two ways to the same result (dims->path):
 *   block-dense: up-project every key (k_nope_h, v_h = W_kvb rows applied to
 *     kv_latent), then per (query tile, 128-key block holding a selected key)
 *     scores, mask, softmax, value mix;
 *   absorbed (the generation-time form of the DeepSeek-V3.2-Exp "Sparse
 *     attention" page's Explanation, where a decoded token scores the cached
 *     latent directly, applied to prefill rows): per query row, q_nope of each head is
 *     multiplied into W_kvb's k_nope rows (q_abs, 512 wide), scored against
 *     the row's selected latent rows [kv_latent | k_pe] only, the softmax
 *     weights mix the latent rows, and W_kvb's v rows map the 512-wide
 *     result to the head's 128 values. It costs 2176 instead of 640 FLOP
 *     per (head, key) but visits only the selected keys, so it wins for rows
 *     whose causal prefix is several times longer than topk.
 * The absorbed path needs topk_idx; without it every row is block-dense. */
int mla_attend(const mla_dims* dims, const void* q, const void* kv_latent,
               const void* k_pe, const void* W_kvb, const float* W_kvb_scale,
               const int32_t* topk_idx, float scale, void* attn_out,
               void* workspace, size_t ws_bytes, mla_stream_t stream);

/* Step A6 -- output projection (Kimi K2 / DeepSeek-V3.2-Exp "Output
 * projection": Delta_attn = o W_O, no bias).
 *   attn : bf16 [B*T, H*128] (heads flattened, h*128 + d)
 *   W_o  : bf16 or e4m3 [H*128, 7168] (math orientation [in, out]; a
 *          checkpoint's [out, in] weight is transposed once at load)
 *   W_o_scale: fp32 [H, 56] block scales for e4m3, else ignored
 *   out  : bf16 [B*T, 7168]
 * With bf16 weights, more than 256 rows and K = H*128 >= 4096, the tiles of
 * a last wave that would leave CTA pairs idle are split along K: their fp32
 * partial tiles go to the workspace and a second kernel adds them in a
 * fixed order. The result is deterministic for a given device and row
 * count, but the rows of those tiles may round differently from a call
 * with another row count. e4m3 weights keep whole-K tiles. */
int mla_out_project(const mla_dims* dims, const void* attn, const void* W_o,
                    const float* W_o_scale, void* out, void* workspace,
                    size_t ws_bytes, mla_stream_t stream);

/* The whole block: mla_attend followed by mla_out_project, with the
 * attention output kept in the workspace. out: bf16 [B, T, 7168]. */
int mla_prefill(const mla_dims* dims, const void* q, const void* kv_latent,
                const void* k_pe, const void* W_kvb, const float* W_kvb_scale,
                const void* W_o, const float* W_o_scale, const int32_t* topk_idx,
                float scale, void* out, void* workspace, size_t ws_bytes,
                mla_stream_t stream);

/* Decode: one new position per sequence against its cache (DeepSeek-V3.2-
 * Exp "Sparse attention" page, Explanation: at generation time a single
 * decoded token scores the cached latent directly, i.e. the absorbed form
 * with W_UK folded into the query and W_UV applied after the value mix).
 * Equals row s = T-1 of mla_prefill for a sequence whose
 * first T-1 positions are the cache, up to rounding.
 *   dims     : B sequences, T = cache length including the new position
 *              (the query sits at s = T-1), H, topk, wdtype; path ignored
 *   q        : bf16 [B, H, 192] of the new position (nope then rope)
 *   kv_latent: bf16 [B, T, 512] latent cache, the new position's row last
 *   k_pe     : bf16 [B, T, 64] rotated rope keys of the cache
 *   W_kvb, W_kvb_scale, W_o, W_o_scale: as for mla_prefill
 *   topk_idx : int32 [B, topk] selected cache positions of the new query,
 *              any order; duplicates select once, entries outside [0, T)
 *              select nothing. NULL = every position.
 *   out      : bf16 [B, 7168]. A sequence with no selected key gets 0 before
 *              W_o (so 0).
 * Steps: per-sequence key lists, q_abs = q_nope . W_UK per head (tcgen05
 * GEMM), attention over the gathered latent keys (the absorbed kernel),
 * attn = W_UV . o_lat per head, then W_o. Workspace: mla_workspace_bytes(
 * dims, MLA_ENTRY_DECODE, topk_idx != NULL). Errors as for mla_prefill. */
int mla_decode(const mla_dims* dims, const void* q, const void* kv_latent,
               const void* k_pe, const void* W_kvb, const float* W_kvb_scale,
               const void* W_o, const float* W_o_scale, const int32_t* topk_idx,
               float scale, void* out, void* workspace, size_t ws_bytes,
               mla_stream_t stream);

/* mla_attend without a caller-supplied workspace (no counterpart on the
 * pages: it exists for callers that cannot hand the library device memory).
 *
 * Some callers cannot call cudaMalloc: a plugin running inside a host
 * framework that owns all device memory through its own pool and hands out
 * no raw allocations, or a latency-critical path where cudaMalloc's implicit
 * device synchronisation is not acceptable. This entry runs exactly the
 * mla_attend computation, but its scratch (up-projected kv, selection
 * bitmap, block lists) lives in one file-scope device array of
 * MLA_STATIC_SCRATCH_BYTES that the library module holds on every GPU that
 * loads it, from load until process exit. It allocates nothing: no
 * cudaMalloc, cudaFree or allocating library routine.
 *   - Arguments and layouts: as for mla_attend (minus workspace/ws_bytes).
 *   - Limit: returns MLA_ERR_TOO_LARGE, before launching anything, when
 *     mla_workspace_bytes(dims, MLA_ENTRY_ATTEND, topk_idx != NULL) exceeds
 *     MLA_STATIC_SCRATCH_BYTES (e.g. B*T*H*512 bytes of kv alone).
 *   - Set-up: the first call on a device (with that device current) looks
 *     up the array's device address once (cudaGetSymbolAddress); make that
 *     first call before any stream capture.
 *   - Sharing: every call on a device uses the same array, which keeps the
 *     previous call's contents; each call writes every scratch word it reads,
 *     so nothing has to start at zero. Calls that overlap on the GPU (other
 *     streams, other host threads) race on the array: order them. */
#define MLA_STATIC_SCRATCH_BYTES (32u << 20)
int mla_attend_static(const mla_dims* dims, const void* q, const void* kv_latent,
                      const void* k_pe, const void* W_kvb, const float* W_kvb_scale,
                      const int32_t* topk_idx, float scale, void* attn_out,
                      mla_stream_t stream);

/* Dynamic activation quantization (the step MLA_ACT_E4M3_DYNAMIC runs in
 * front of each projection), exposed on its own.
 *   x      : bf16 [rows, cols], cols a multiple of 128 (row pitch cols)
 *   codes  : e4m3 [rows, cols]: code = e4m3(x / s), the division in fp32 and
 *            the conversion rounding to nearest even, saturating at +-448
 *   scales : fp32 [cols / 128, rows]: s = amax / 448 (fp32, nearest even) of
 *            each row's group of 128 columns; an all-zero group gets s = 0
 *            and zero codes. Group-major so that one group's row scales are
 *            contiguous.
 * x, codes and scales must be 16-byte aligned. Stream-ordered, no
 * workspace. Errors: MLA_ERR_NULL, MLA_ERR_SHAPE (rows < 0, cols not a
 * positive multiple of 128), MLA_ERR_ALIGN, MLA_ERR_CUDA. */
int mla_quantize_act(const void* x, int rows, int cols, void* codes, float* scales, mla_stream_t stream);

/* Human-readable text of a status code (static storage). */
const char* mla_status_str(int status);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device. *device_error receives 0 (none) or the first code a
 * kernel recorded: 1xx a pipeline wait timed out (101 TMA load, 102
 * tensor-core commit, 103 consumer release, 104 epilogue, 105 softmax
 * hand-off); 201 bad launch geometry; 301 an up-projected value v exceeded
 * the f16 range (|v| >= 65520) on the attention path (see mla_attend).
 * Returns MLA_ERR_CUDA if synchronisation fails, else MLA_OK. */
int mla_device_status(mla_stream_t stream, int* device_error);

/* How e4m3 weights (MLA_W_E4M3_BLOCK128) meet bf16 activations (MLA_ACT_BF16)
 * in the projections, process-wide for calls made afterwards (Kimi K2 page,
 * "Down projection": weights stored as e4m3 codes with one fp32 scale per
 * 128 x 128 block; here each weight becomes bf16(code * scale), the fp32
 * product rounded once, and meets the bf16 activations on the tensor cores).
 *   onchip = 0 (default): each call dequantises W_kvb / W_o into a bf16 copy
 *     in its workspace, then runs the bf16 GEMMs.
 *   onchip = 1: the W_kvb and W_o GEMMs of prefill read the e4m3 codes and
 *     their scales directly: converter warps turn each code tile into bf16
 *     in tensor memory (the UMMA A operand of a transposed GEMM), so no copy
 *     is written. Bit-identical to mode 0; measured slower on B200 at the
 *     batched workload (B 16, T 1024, H 128): W_kvb 0.63 against 0.45 ms,
 *     W_o 3.6 against 2.7 ms, because the conversion is repeated for every
 *     token tile. The absorbed rows' GEMMs and mla_decode keep a bf16 copy of
 *     W_kvb (and decode one of W_o) in both modes.
 * mla_workspace_bytes() follows the mode in force when it is called: query
 * it after switching. Host-only (no device work); returns MLA_ERR_SHAPE for
 * an onchip value other than 0 or 1. */
int mla_set_e4m3_weight_conversion(int onchip);

/* Failure detection. Every on-chip wait of the kernels (mbarrier waits on
 * TMA loads, tensor-core commits and hand-offs between warps) gives up after
 * a time limit, records a 1xx code in the device error word, lets its
 * in-flight copies and tensor-core work land (again bounded), releases its
 * tensor memory and returns, so that a lost arrival ends as an error status
 * instead of a hung GPU.
 * mla_set_wait_timeout_ns sets that limit, in nanoseconds of the GPU's
 * global timer, for kernels launched afterwards on the current device (0
 * restores the default of 1 s). Synchronous with the host (a copy to a
 * device variable); call it between launches, not during stream capture.
 * Returns MLA_ERR_CUDA if no device is usable. */
int mla_set_wait_timeout_ns(unsigned long long ns);

/* Test hook for the failure path above, off by default: while on (on != 0)
 * the producer warp of the block-dense attention kernel issues none of its
 * loads on the current device, so that the kernel's waits for them (and for
 * the tensor-core work that would follow) run into the time limit. The
 * kernel then records a 1xx code and exits cleanly; its output is
 * undefined. Nothing faults or hangs: every wait is bounded. Synchronous
 * like mla_set_wait_timeout_ns; switch it off again before normal use. */
int mla_test_withhold_attention_loads(int on);

/* Test hook, host only (no device work): the plan mla_out_project and
 * mla_prefill use for a W_o GEMM of `tiles` 256 x 256 tiles on `pairs` CTA
 * pairs with K of `num_kb` 64-deep blocks (bf16 weights, more than 256
 * rows): *tail tiles of the last wave, each cut into *split contiguous K
 * ranges, one per pair, the partial tiles in the first tail * split of the
 * workspace's 74 slots; 0 and 0 for no split. tail and split are HOST
 * pointers. Returns MLA_ERR_NULL if one is NULL, MLA_ERR_SHAPE if an
 * argument is negative. */
int mla_test_wo_split_plan(int tiles, int pairs, int num_kb, int* tail, int* split);

/* Per-kernel device timing (CUDA events on the launching stream).
 * mla_profile_begin() starts recording events around every launch made by
 * the calls above on this host thread's library instance; mla_profile_end()
 * synchronises those events and writes, per kernel class, the total
 * milliseconds and launch count, then stops recording.
 * Classes: 0 topk prepass, 1 weight dequant, 2 W_kvb GEMM, 3 attention
 * (block-dense), 4 W_o GEMM, 5 per-row key lists (prefill and decode),
 * 6 absorb and un-absorb GEMMs, 7 attention (absorbed), 8 activation
 * quantization, 9 sums of the W_o GEMM's K-split last-wave tiles. Arrays
 * must hold MLA_PROFILE_CLASSES entries. */
#define MLA_PROFILE_CLASSES 10
int mla_profile_begin(void);
int mla_profile_end(float* ms_total, int* launches);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
