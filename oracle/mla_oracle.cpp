// mla_oracle.cpp -- plain single-threaded fp64 CPU oracle for the sparse MLA
// prefill attend block.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path may call, link or
// load this file's library; only the test suite, the smoke check and the
// CPU-baseline leg of the benchmark do. It shares no code, header or table
// with the CUDA library.
//
// What it computes (DeepSeek-V3.2-Exp "Sparse attention" page, prefill code
// of model.py 574-589 and 607-608; Kimi K2 "Output projection" page):
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
};

double mlao_bf16_to_double(uint16_t bits) { return bf16_value(bits); }
double mlao_e4m3_to_double(uint8_t code) { return e4m3_value(code); }

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
  for (int n = 0; n < n_rows; ++n) {
    const uint16_t* lat = p->kv_latent + rows[n] * L;
    double* acc = kvh + static_cast<size_t>(n) * R;
    for (int r = 0; r < R; ++r) acc[r] = 0.0;
    for (int j = 0; j < L; ++j) {
      const double a = bf16_value(lat[j]);
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
  std::vector<double> z, w;

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
          const uint16_t* lat = p->kv_latent + bt * L;
          for (int r = 0; r < per_head; ++r) kv[r] = 0.0;
          for (int j = 0; j < L; ++j) {
            const double x = bf16_value(lat[j]);
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
int mlao_project_rows(const mlao_problem* p, int n_rows, const double* attn, double* out) {
  const int K = p->H * p->d_v, D = p->d_model;
  for (int n = 0; n < n_rows; ++n) {
    double* o = out + static_cast<size_t>(n) * D;
    for (int c = 0; c < D; ++c) o[c] = 0.0;
    const double* a = attn + static_cast<size_t>(n) * K;
    for (int k = 0; k < K; ++k) {
      const double ak = a[k];
      if (!p->w_fp8) {
        const uint16_t* wr = static_cast<const uint16_t*>(p->W_o) + static_cast<size_t>(k) * D;
        for (int c = 0; c < D; ++c) o[c] += ak * bf16_value(wr[c]);
      } else {
        for (int c = 0; c < D; ++c) o[c] += ak * weight_value(p->W_o, p->W_o_scale, 1, D, k, c);
      }
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
