/*
 * Float64 CPU oracle for the GPT-OSS MXFP4 mixture-of-experts feed-forward layer.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the plain, slow definition the CUDA
 * path is checked against. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the product library never links,
 * includes or calls it, and it shares no code, header or table with the
 * CUDA sources.
 *
 * What it computes, per token t (x[t] is bf16, widened exactly to double):
 *   1. router logits  l_e = sum_h x_h * W_r[e,h] + b_r[e]
 *      ("a top-num_experts_per_tok router", ZeroModels GPT-OSS docs, GPT-OSS
 *      section, mixture-of-experts bullet; the router bias is part of the
 *      reading that the layer takes).
 *   2. S = the k largest logits, descending; an exact tie goes to the lower
 *      expert index (the pages are silent on ties; reading).
 *   3. w_s = softmax over the k selected logits only (reading: the pages say
 *      the experts' "softmax weights combine per-expert outputs").
 *   4. For each selected expert e (in slot order s = 0..k-1):
 *        W_gu = dequant(gate_up_blocks[e], gate_up_scales[e])   [2I, H]
 *        h_r  = sum_c x_c * W_gu[r,c] + b_gu[e,r]                r < 2I
 *        gate_i = h[2i], up_i = h[2i+1]   (the ::2 / 1::2 split of the
 *          interleaved gate_up rows: MaxText PR 2647, section "1 Support
 *          many-to-one transform"; Megatron-Bridge GPT-OSS bridge,
 *          GPTOSSMLPGateUpProjMapping, "alternating row interleaving")
 *        g_i = min(gate_i, 7); u_i = min(max(up_i, -7), 7)   (the docs'
 *          "clamp 7"; reading: the gate is clamped from above only, up on
 *          both sides, after the bias)
 *        a_i = (u_i + 1) * g_i * sigmoid(1.702 * g_i)   (ZeroModels GPT-OSS
 *          docs, mixture-of-experts bullet)
 *        W_d = dequant(down_blocks[e], down_scales[e])   [H, I]  (the
 *          MXFP4-dequantised down_proj is [E, hidden, intermediate]:
 *          Megatron-Bridge bridge, maybe_modify_loaded_hf_weight)
 *        y_j = sum_i a_i * W_d[j,i] + b_d[e,j]
 *   5. out[t] = sum_s w_s * y^(s), summed in slot order.
 *
 * MXFP4 storage (ZeroModels GPT-OSS docs, "MXFP4 experts" bullet: uint8
 * nibble blocks plus e8m0 scales): blocks are uint8 [R, C/32, 16]; byte j
 * of block b holds column b*32+2j in its low nibble and b*32+2j+1 in its
 * high nibble (reading: low nibble first). Each nibble is an FP4 E2M1 code
 * (OCP Microscaling Formats v1.0, FP4 E2M1: sign bit, two exponent bits,
 * one mantissa bit) and each block has one E8M0 scale byte s meaning
 * 2^(s-127) (same spec, E8M0).
 *
 * Sums run in double, in index order, one term at a time. OpenMP (when
 * compiled in) only splits the token loop; each token's arithmetic is the
 * same sequential code whatever the thread count, so results are
 * bit-identical for any thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* FP4 E2M1 code -> value, codes 0..15 (bit 3 is the sign; code 8 is -0). */
static const double kE2M1[16] = {
    0.0,  0.5,  1.0,  1.5,  2.0,  3.0,  4.0,  6.0,
    -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0,
};

static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

double oracle_e2m1_value(int code) { return kE2M1[code & 15]; }

double oracle_e8m0_value(int s) { return ldexp(1.0, s - 127); }

/* Element (r, c) of an MXFP4 tensor with C columns. */
static double mx_element(const uint8_t* blocks, const uint8_t* scales, int64_t C, int64_t r, int64_t c) {
  const int64_t nb = C / 32;
  const int64_t b = c / 32;
  const uint8_t byte = blocks[(r * nb + b) * 16 + (c % 32) / 2];
  const int code = (c % 2) ? (byte >> 4) : (byte & 15);
  return kE2M1[code] * ldexp(1.0, (int)scales[r * nb + b] - 127);
}

/* Dequantise an MXFP4 tensor [rows, cols] to double. */
void oracle_dequant(const uint8_t* blocks, const uint8_t* scales, int64_t rows, int64_t cols, double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) out[r * cols + c] = mx_element(blocks, scales, cols, r, c);
}

/* Dequantise to bf16 bit patterns. Every value with 2 <= s <= 252 is exactly
 * representable in bf16 (at most two significant bits, normal exponent); the
 * return value counts elements that are not, whose bits are then those of the
 * nearest float32 truncated (they are out of contract). */
int64_t oracle_dequant_bf16(const uint8_t* blocks, const uint8_t* scales, int64_t rows, int64_t cols,
                            uint16_t* out) {
  int64_t inexact = 0;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      const double v = mx_element(blocks, scales, cols, r, c);
      const float f = (float)v;
      uint32_t u;
      memcpy(&u, &f, sizeof u);
      if ((double)f != v || (u & 0xFFFFu) != 0 || (v != 0.0 && fabs(v) < 0x1p-126) || isinf(f)) ++inexact;
      out[r * cols + c] = (uint16_t)(u >> 16);
    }
  return inexact;
}

/* Router logits for one token. */
static void router_row(const uint16_t* xrow, const float* rw, const float* rb, int64_t H, int64_t E,
                       double* logits) {
  for (int64_t e = 0; e < E; ++e) {
    double acc = 0.0;
    for (int64_t h = 0; h < H; ++h) acc += bf16_bits_to_double(xrow[h]) * (double)rw[e * H + h];
    logits[e] = acc + (double)rb[e];
  }
}

void oracle_router_logits(const uint16_t* x, const float* rw, const float* rb, int64_t T, int64_t H, int64_t E,
                          double* logits) {
  for (int64_t t = 0; t < T; ++t) router_row(x + t * H, rw, rb, H, E, logits + t * E);
}

/* Top-k by repeated selection of the largest remaining logit (ties: lower
 * index), then softmax over the k selected logits. */
static void topk_row(const double* l, int64_t E, int k, int32_t* idx, double* w) {
  unsigned char* taken = (unsigned char*)calloc((size_t)E, 1);
  for (int s = 0; s < k; ++s) {
    int64_t best = -1;
    for (int64_t e = 0; e < E; ++e) {
      if (taken[e]) continue;
      if (best < 0 || l[e] > l[best]) best = e;
    }
    taken[best] = 1;
    idx[s] = (int32_t)best;
  }
  free(taken);
  const double lmax = l[idx[0]];
  double z = 0.0;
  for (int s = 0; s < k; ++s) z += exp(l[idx[s]] - lmax);
  for (int s = 0; s < k; ++s) w[s] = exp(l[idx[s]] - lmax) / z;
}

void oracle_topk_softmax(const double* logits, int64_t T, int64_t E, int k, int32_t* idx, double* w) {
  for (int64_t t = 0; t < T; ++t) topk_row(logits + t * E, E, k, idx + t * k, w + t * k);
}

/* Smallest gap between adjacent logits among the k+1 largest (only the k
 * largest when k == E), per token. */
void oracle_router_margins(const uint16_t* x, const float* rw, const float* rb, int64_t T, int64_t H, int64_t E,
                           int k, int threads, double* margins) {
  (void)threads;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads > 0 ? threads : 1)
#endif
  for (int64_t t = 0; t < T; ++t) {
    double* l = (double*)malloc(sizeof(double) * (size_t)E);
    router_row(x + t * H, rw, rb, H, E, l);
    const int n = (k + 1 <= E) ? k + 1 : k;
    int32_t* id = (int32_t*)malloc(sizeof(int32_t) * (size_t)n);
    double* ww = (double*)malloc(sizeof(double) * (size_t)n);
    topk_row(l, E, n, id, ww);
    double m = INFINITY;
    for (int s = 0; s + 1 < n; ++s) {
      const double g = l[id[s]] - l[id[s + 1]];
      if (g < m) m = g;
    }
    margins[t] = m;
    free(l);
    free(id);
    free(ww);
  }
}

double oracle_sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* Clamped gated SiLU on interleaved pre-activations h[2I] -> act[I]. */
void oracle_swiglu(const double* h, int64_t I, double* act) {
  for (int64_t i = 0; i < I; ++i) {
    double g = h[2 * i];
    double u = h[2 * i + 1];
    if (g > 7.0) g = 7.0;
    if (u > 7.0) u = 7.0;
    if (u < -7.0) u = -7.0;
    act[i] = (u + 1.0) * g * oracle_sigmoid(1.702 * g);
  }
}

/* One expert on one token. Pointers are already offset to the expert.
 * h_out (2I), act_out (I) may be NULL; y_out (H) receives the expert output. */
void oracle_expert(const double* x, const uint8_t* gu_blocks, const uint8_t* gu_scales, const uint16_t* gu_bias,
                   const uint8_t* d_blocks, const uint8_t* d_scales, const uint16_t* d_bias, int64_t H, int64_t I,
                   double* h_out, double* act_out, double* y_out) {
  double* h = (double*)malloc(sizeof(double) * (size_t)(2 * I));
  double* a = (double*)malloc(sizeof(double) * (size_t)I);
  for (int64_t r = 0; r < 2 * I; ++r) {
    double acc = 0.0;
    for (int64_t c = 0; c < H; ++c) acc += x[c] * mx_element(gu_blocks, gu_scales, H, r, c);
    h[r] = acc + bf16_bits_to_double(gu_bias[r]);
  }
  oracle_swiglu(h, I, a);
  for (int64_t j = 0; j < H; ++j) {
    double acc = 0.0;
    for (int64_t i = 0; i < I; ++i) acc += a[i] * mx_element(d_blocks, d_scales, I, j, i);
    y_out[j] = acc + bf16_bits_to_double(d_bias[j]);
  }
  if (h_out) memcpy(h_out, h, sizeof(double) * (size_t)(2 * I));
  if (act_out) memcpy(act_out, a, sizeof(double) * (size_t)I);
  free(h);
  free(a);
}

/* The whole layer on a list of tokens (all tokens when token_list is NULL).
 * out: [n, H] double; idx_out: [n, k] (may be NULL); w_out: [n, k] (may be NULL). */
int oracle_moe_forward(const uint16_t* x, const float* router_w, const float* router_b, const uint8_t* gu_blocks,
                       const uint8_t* gu_scales, const uint16_t* gu_bias, const uint8_t* d_blocks,
                       const uint8_t* d_scales, const uint16_t* d_bias, int64_t T, int64_t H, int64_t I, int64_t E,
                       int k, const int64_t* token_list, int64_t n, int threads, double* out, int32_t* idx_out,
                       double* w_out) {
  if (k < 1 || k > E || H % 32 || I % 32) return 1;
  if (!token_list) n = T;
  const int64_t gu_rows = 2 * I, nbh = H / 32, nbi = I / 32;
  (void)threads;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads > 0 ? threads : 1)
#endif
  for (int64_t j = 0; j < n; ++j) {
    const int64_t t = token_list ? token_list[j] : j;
    double* xf = (double*)malloc(sizeof(double) * (size_t)H);
    double* l = (double*)malloc(sizeof(double) * (size_t)E);
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    int32_t* id = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    double* w = (double*)malloc(sizeof(double) * (size_t)k);
    for (int64_t h = 0; h < H; ++h) xf[h] = bf16_bits_to_double(x[t * H + h]);
    router_row(x + t * H, router_w, router_b, H, E, l);
    topk_row(l, E, k, id, w);
    double* o = out + j * H;
    for (int64_t h = 0; h < H; ++h) o[h] = 0.0;
    for (int s = 0; s < k; ++s) {
      const int64_t e = id[s];
      oracle_expert(xf, gu_blocks + e * gu_rows * nbh * 16, gu_scales + e * gu_rows * nbh, gu_bias + e * gu_rows,
                    d_blocks + e * H * nbi * 16, d_scales + e * H * nbi, d_bias + e * H, H, I, NULL, NULL, y);
      for (int64_t h = 0; h < H; ++h) o[h] += w[s] * y[h];
    }
    if (idx_out)
      for (int s = 0; s < k; ++s) idx_out[j * k + s] = id[s];
    if (w_out)
      for (int s = 0; s < k; ++s) w_out[j * k + s] = w[s];
    free(xf);
    free(l);
    free(y);
    free(id);
    free(w);
  }
  return 0;
}

int oracle_has_openmp(void) {
#ifdef _OPENMP
  return 1;
#else
  return 0;
#endif
}
