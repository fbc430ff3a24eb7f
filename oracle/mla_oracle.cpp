// mla_oracle.cpp -- plain single-threaded fp64 CPU oracle for the sparse MLA
// prefill attend block.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path may call, link or
// load this file's library; only the test suite, the smoke check and the
// CPU-baseline leg of the benchmark do. It shares no code, header or table
// with the CUDA library.
//
// What it computes (DeepSeek-V3.2-Exp "Sparse attention" page, its prefill
// code; Kimi K2 "Output projection" page):
//   kv            = W_kvb applied to the 512-wide latent, viewed per head as
//                   [k_nope (128) | v (128)]                     (wkv_b, view, split)
//   k_h[t]        = k_nope_h[t] ++ k_pe[t]  (rotary key shared by all heads)
//   z[s,h,t]      = scale * <q[s,h], k_h[t]>                     (einsum bshd,bthd->bsht)
//   mask          = -inf except at the top-k keys of query s, plus the causal
//                   mask (-inf for t > s)                         (scatter_, += mask)
//   attn[s,h]     = softmax_t(z[s,h,:] + mask[s,:]) . v_h        (softmax, einsum bsht,bthd->bshd)
//   out[s]        = flatten_h(attn[s]) . W_o                     (wo(x.flatten(2)), Delta = o W_O)
// All arithmetic is fp64 on the exact values of the stored bf16 / e4m3 bytes,
// with no intermediate rounding. Sums run in ascending index order.
//
// Readings where the pages are silent (each is a convention, stated here):
//   * Causal mask value: -inf for t > s, 0 otherwise (start_pos = 0, empty cache).
//   * Duplicate top-k entries select a key once (scatter_ writes the same 0).
//   * Top-k entries outside [0, T) select nothing.
//   * A query with no surviving key gets attn = 0 (torch would give NaN).
//   * FP8 weights: OCP E4M3FN codes (bias 7, max 448, S.1111.111 = NaN), one
//     fp32 scale per 128 x 128 block of the stored [rows, cols] matrix.
//   * W_kvb is stored [H*(dn+dv), L] (module [out, in]); W_o is stored
//     [H*dv, D] (the math form o W_O).
//   * Dynamic FP8 activations (Kimi K2 "Down projection" page, config.json
//     quantization_config: activation_scheme "dynamic", fmt "e4m3", 128 x 128
//     weight blocks), when act_e4m3 is set: the input of each FP8 linear layer
//     -- the latent entering W_kvb and the attention output entering W_o -- is
//     quantized per row in groups of 128 consecutive channels, s = amax / 448
//     and code = e4m3(x / s), both divisions in fp32 rounding to nearest even,
//     the conversion rounding to nearest even and saturating at +-448; an
//     all-zero group gets s = 0. The layer then sees code * s. The attention
//     output is a bf16 tensor in the pages' model, so it is rounded to bf16
//     (nearest even) before it is quantized.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

namespace {

double bf16_value(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

// OCP 8-bit floating point, E4M3FN variant: 1 sign, 4 exponent (bias 7),
// 3 mantissa bits; exponent 0 is subnormal; no infinities; S.1111.111 is NaN.
double e4m3_value(uint8_t code) {
  const int sign = code >> 7;
  const int ex = (code >> 3) & 0xF;
  const int man = code & 0x7;
  double mag;
  if (ex == 0xF && man == 0x7) {
    mag = std::numeric_limits<double>::quiet_NaN();
  } else if (ex == 0) {
    mag = std::ldexp(static_cast<double>(man) / 8.0, -6);
  } else {
    mag = std::ldexp(1.0 + static_cast<double>(man) / 8.0, ex - 7);
  }
  return sign ? -mag : mag;
}

// bf16 value nearest to v (ties to an even last mantissa bit), as bits.
// bf16 keeps fp32's 8 exponent bits and 7 of its mantissa bits.
uint16_t bf16_bits_nearest(double v) {
  double a = std::fabs(v);
  double r = 0.0;
  if (a != 0.0) {
    int E = 0;
    std::frexp(a, &E);        // a = f * 2^E, f in [0.5, 1)
    int e = E - 1;            // a in [2^e, 2^(e+1))
    if (e < -126) e = -126;   // subnormal range: fixed quantum
    const double quantum = std::ldexp(1.0, e - 7);
    r = std::nearbyint(a / quantum) * quantum;   // ties to even
  }
  const float f = static_cast<float>(std::signbit(v) ? -r : r);   // exact
  uint32_t u;
  std::memcpy(&u, &f, sizeof u);
  return static_cast<uint16_t>(u >> 16);
}

// E4M3FN code nearest to x (ties to an even code), saturating at +-448.
uint8_t e4m3_code_nearest(float x) {
  const uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  const double a = std::fabs(static_cast<double>(x));
  if (a == 0.0) return sign;
  int E = 0;
  std::frexp(a, &E);
  int e = E - 1;
  if (e < -6) e = -6;   // subnormals share the quantum of the smallest binade
  const double quantum = std::ldexp(1.0, e - 3);
  double v = std::nearbyint(a / quantum) * quantum;
  if (v > 448.0) v = 448.0;
  if (v == 0.0) return sign;
  if (v < std::ldexp(1.0, -6)) return sign | static_cast<uint8_t>(v / std::ldexp(1.0, -9));
  std::frexp(v, &E);
  e = E - 1;
  const int man = static_cast<int>((v / std::ldexp(1.0, e) - 1.0) * 8.0);
  return sign | static_cast<uint8_t>(((e + 7) << 3) | man);
}

// One group of a row: codes[i] and the group's scale from x[0..n).
void quantize_group(const float* x, int n, uint8_t* codes, float* scale) {
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) amax = std::fabs(x[i]) > amax ? std::fabs(x[i]) : amax;
  const float s = amax / 448.0f;
  *scale = s;
  for (int i = 0; i < n; ++i) codes[i] = s == 0.0f ? 0 : e4m3_code_nearest(x[i] / s);
}

// Values a layer sees for an activation row under dynamic FP8: quantize the
// row's groups of 128 channels and decode code * s.
void fake_quantize_row(const float* x, int n, double* out) {
  uint8_t codes[128];
  float s = 0.0f;
  for (int g = 0; g < n; g += 128) {
    const int w = n - g < 128 ? n - g : 128;
    quantize_group(x + g, w, codes, &s);
    for (int i = 0; i < w; ++i) out[g + i] = e4m3_value(codes[i]) * static_cast<double>(s);
  }
}

}  // namespace

extern "C" {

// Problem description. Pointers are host memory owned by the caller.
struct mlao_problem {
  int B, T, H;
  int d_nope, d_rope, d_v, d_latent, d_model;
  int topk;                   // entries per query row; ignored when topk_idx == NULL
  int w_fp8;                  // 0: bf16 weights; 1: e4m3 codes + fp32 block scales
  const uint16_t* q;          // bf16 [B,T,H,d_nope+d_rope], nope then rope
  const uint16_t* kv_latent;  // bf16 [B,T,d_latent]
  const uint16_t* k_pe;       // bf16 [B,T,d_rope]
  const void* W_kvb;          // [H*(d_nope+d_v), d_latent]
  const float* W_kvb_scale;   // [H*(d_nope+d_v)/128, d_latent/128] when w_fp8
  const void* W_o;            // [H*d_v, d_model]
  const float* W_o_scale;     // [H*d_v/128, d_model/128] when w_fp8
  const int32_t* topk_idx;    // [B,T,topk] or NULL (causal mask only)
  double scale;               // softmax scale
  int act_e4m3;               // 1: dynamic per-token e4m3 activations into W_kvb and W_o
};

double mlao_bf16_to_double(uint16_t bits) { return bf16_value(bits); }
double mlao_e4m3_to_double(uint8_t code) { return e4m3_value(code); }
uint16_t mlao_bf16_from_double(double v) { return bf16_bits_nearest(v); }
uint8_t mlao_e4m3_from_float(float x) { return e4m3_code_nearest(x); }

// Dynamic activation quantization of x [rows][cols] (cols a multiple of 128):
// codes [rows][cols], scales [rows][cols / 128].
int mlao_quantize_act(const float* x, int rows, int cols, uint8_t* codes, float* scales) {
  if (cols % 128 != 0) return 1;
  for (int r = 0; r < rows; ++r)
    for (int g = 0; g < cols / 128; ++g)
      quantize_group(x + static_cast<size_t>(r) * cols + 128 * g, 128, codes + static_cast<size_t>(r) * cols + 128 * g,
                     scales + static_cast<size_t>(r) * (cols / 128) + g);
  return 0;
}

// Latent row at flattened position pos as the up-projection sees it.
static void latent_row(const mlao_problem* p, int64_t pos, double* out) {
  const int L = p->d_latent;
  const uint16_t* lat = p->kv_latent + pos * L;
  if (!p->act_e4m3) {
    for (int j = 0; j < L; ++j) out[j] = bf16_value(lat[j]);
    return;
  }
  std::vector<float> x(L);
  for (int j = 0; j < L; ++j) x[j] = static_cast<float>(bf16_value(lat[j]));
  fake_quantize_row(x.data(), L, out);
}

// Exact stored value of W_kvb[r][c] or W_o[r][c].
static double weight_value(const void* w, const float* sc, int w_fp8, int cols,
                           int64_t r, int64_t c) {
  if (!w_fp8) return bf16_value(static_cast<const uint16_t*>(w)[r * cols + c]);
  const int sc_cols = cols / 128;
  return e4m3_value(static_cast<const uint8_t*>(w)[r * cols + c]) *
         static_cast<double>(sc[(r / 128) * sc_cols + (c / 128)]);
}

// Up-projection of the latent at the given flattened positions (b*T + t):
//   kvh[n][r] = sum_j kv_latent[pos][j] * W_kvb[r][j]   for r < H*(dn+dv).
// Output is [n_rows][H*(dn+dv)] in the stored row order of W_kvb
// (head-major, k_nope then v within a head).
int mlao_upproject_rows(const mlao_problem* p, int n_rows, const int64_t* rows, double* kvh) {
  const int L = p->d_latent;
  const int R = p->H * (p->d_nope + p->d_v);
  // Decoded weight, transposed to [L][R] so that the loop below walks r
  // contiguously; each output still sums over j in ascending order.
  std::vector<double> wt(static_cast<size_t>(L) * R);
  for (int r = 0; r < R; ++r)
    for (int j = 0; j < L; ++j)
      wt[static_cast<size_t>(j) * R + r] = weight_value(p->W_kvb, p->W_kvb_scale, p->w_fp8, L, r, j);
  std::vector<double> lat(L);
  for (int n = 0; n < n_rows; ++n) {
    latent_row(p, rows[n], lat.data());
    double* acc = kvh + static_cast<size_t>(n) * R;
    for (int r = 0; r < R; ++r) acc[r] = 0.0;
    for (int j = 0; j < L; ++j) {
      const double a = lat[j];
      const double* w = wt.data() + static_cast<size_t>(j) * R;
      for (int r = 0; r < R; ++r) acc[r] += a * w[r];
    }
  }
  return 0;
}

// Attention output for the given query rows (flattened b*T + s) and heads:
// attn[n][i][d] for head heads[i] (all heads 0..H-1 when heads == NULL).
int mlao_attend_rows(const mlao_problem* p, int n_rows, const int64_t* rows,
                     int n_heads, const int32_t* heads, double* attn) {
  const int T = p->T, H = p->H, dn = p->d_nope, dr = p->d_rope, dv = p->d_v, L = p->d_latent;
  const int dqk = dn + dr;
  const int per_head = dn + dv;
  if (heads == nullptr) n_heads = H;

  // Selected keys A_s of each row, in ascending key order.
  std::vector<std::vector<int>> sel(n_rows);
  std::vector<char> mark(T);
  for (int n = 0; n < n_rows; ++n) {
    const int64_t bs = rows[n];
    const int s = static_cast<int>(bs % T);
    if (p->topk_idx == nullptr) {
      for (int t = 0; t <= s; ++t) sel[n].push_back(t);
      continue;
    }
    std::fill(mark.begin(), mark.end(), 0);
    const int32_t* idx = p->topk_idx + bs * p->topk;
    for (int i = 0; i < p->topk; ++i) {
      const int32_t t = idx[i];
      if (t >= 0 && t < T && t <= s) mark[t] = 1;  // index mask + causal mask
    }
    for (int t = 0; t <= s; ++t)
      if (mark[t]) sel[n].push_back(t);
  }

  std::vector<double> wt(static_cast<size_t>(L) * per_head);
  std::vector<double> kv_cache;              // [B*T][per_head], filled lazily per head
  std::vector<char> have;
  kv_cache.resize(static_cast<size_t>(p->B) * T * per_head);
  have.resize(static_cast<size_t>(p->B) * T);
  std::vector<double> z, w, lat(L);

  for (int hi = 0; hi < n_heads; ++hi) {
    const int h = heads ? heads[hi] : hi;
    if (h < 0 || h >= H) return 1;
    // This head's rows of W_kvb, decoded and transposed to [L][per_head].
    for (int r = 0; r < per_head; ++r)
      for (int j = 0; j < L; ++j)
        wt[static_cast<size_t>(j) * per_head + r] =
            weight_value(p->W_kvb, p->W_kvb_scale, p->w_fp8, L, static_cast<int64_t>(h) * per_head + r, j);
    std::fill(have.begin(), have.end(), 0);

    for (int n = 0; n < n_rows; ++n) {
      const int64_t bs = rows[n];
      const int64_t b = bs / T;
      double* o = attn + (static_cast<size_t>(n) * n_heads + hi) * dv;
      for (int d = 0; d < dv; ++d) o[d] = 0.0;
      const std::vector<int>& A = sel[n];
      if (A.empty()) continue;  // no surviving key: attn = 0
      const uint16_t* qv = p->q + (bs * H + h) * dqk;
      z.assign(A.size(), 0.0);
      for (size_t a = 0; a < A.size(); ++a) {
        const int64_t bt = b * T + A[a];
        double* kv = kv_cache.data() + static_cast<size_t>(bt) * per_head;
        if (!have[bt]) {  // k_nope_h[t] and v_h[t]
          latent_row(p, bt, lat.data());
          for (int r = 0; r < per_head; ++r) kv[r] = 0.0;
          for (int j = 0; j < L; ++j) {
            const double x = lat[j];
            const double* wr = wt.data() + static_cast<size_t>(j) * per_head;
            for (int r = 0; r < per_head; ++r) kv[r] += x * wr[r];
          }
          have[bt] = 1;
        }
        const uint16_t* kpe = p->k_pe + bt * dr;
        double dot = 0.0;
        for (int i = 0; i < dn; ++i) dot += bf16_value(qv[i]) * kv[i];
        for (int i = 0; i < dr; ++i) dot += bf16_value(qv[dn + i]) * bf16_value(kpe[i]);
        z[a] = p->scale * dot;
      }
      double m = -std::numeric_limits<double>::infinity();
      for (double x : z) m = x > m ? x : m;
      w.assign(A.size(), 0.0);
      double l = 0.0;
      for (size_t a = 0; a < A.size(); ++a) {
        w[a] = std::exp(z[a] - m);
        l += w[a];
      }
      for (size_t a = 0; a < A.size(); ++a) {
        const double* v = kv_cache.data() + static_cast<size_t>(b * T + A[a]) * per_head + dn;
        for (int d = 0; d < dv; ++d) o[d] += w[a] * v[d];
      }
      for (int d = 0; d < dv; ++d) o[d] /= l;
    }
  }
  return 0;
}

// Output projection of full-width attention rows:
//   out[n][c] = sum_k attn[n][k] * W_o[k][c],  k = h*d_v + d ascending.
// With act_e4m3 the row is first rounded to bf16 and quantized.
int mlao_project_rows(const mlao_problem* p, int n_rows, const double* attn, double* out) {
  const int K = p->H * p->d_v, D = p->d_model;
  // The rows as W_o sees them (quantized when act_e4m3).
  std::vector<double> rows_in(static_cast<size_t>(n_rows) * K);
  std::vector<float> xb(K);
  for (int n = 0; n < n_rows; ++n) {
    const double* a = attn + static_cast<size_t>(n) * K;
    double* r = rows_in.data() + static_cast<size_t>(n) * K;
    if (p->act_e4m3) {
      for (int k = 0; k < K; ++k) xb[k] = static_cast<float>(bf16_value(bf16_bits_nearest(a[k])));
      fake_quantize_row(xb.data(), K, r);
    } else {
      for (int k = 0; k < K; ++k) r[k] = a[k];
    }
  }
  for (size_t i = 0; i < static_cast<size_t>(n_rows) * D; ++i) out[i] = 0.0;
  // Each W_o row is decoded once and applied to every row; every output
  // still sums over k in ascending order.
  std::vector<double> w(D);
  for (int k = 0; k < K; ++k) {
    for (int c = 0; c < D; ++c) w[c] = weight_value(p->W_o, p->W_o_scale, p->w_fp8, D, k, c);
    for (int n = 0; n < n_rows; ++n) {
      const double ak = rows_in[static_cast<size_t>(n) * K + k];
      double* o = out + static_cast<size_t>(n) * D;
      for (int c = 0; c < D; ++c) o[c] += ak * w[c];
    }
  }
  return 0;
}

// The whole block for the given rows: attn over all heads, then W_o.
// attn_out (may be NULL) receives [n_rows][H*d_v]; out receives [n_rows][d_model].
int mlao_prefill_rows(const mlao_problem* p, int n_rows, const int64_t* rows,
                      double* attn_out, double* out) {
  std::vector<double> attn(static_cast<size_t>(n_rows) * p->H * p->d_v);
  int rc = mlao_attend_rows(p, n_rows, rows, p->H, nullptr, attn.data());
  if (rc) return rc;
  if (attn_out) std::memcpy(attn_out, attn.data(), attn.size() * sizeof(double));
  return mlao_project_rows(p, n_rows, attn.data(), out);
}

}  // extern "C"
