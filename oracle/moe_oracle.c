/*
 * moe_oracle.c -- plain, slow, single-threaded CPU oracle for the MoE
 * token-routing pipeline (mask -> create_indices -> MXFP4 dispatch ->
 * NVFP4 grouped GEMV -> combine).
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path and must never be used by it.
 *
 * Floating-point references are computed in double precision.  Where a step
 * is defined by a rounding (an fp32 quotient, an E2M1 / E4M3 code) the step
 * is written out exactly as defined, in the stated precision, so that codes
 * and scales can be compared bit for bit.  Each function names the page and
 * section whose behaviour it restates.
 *
 * Format definitions used (not printed on the pages, standard formats):
 *   E2M1 (FP4):  sign | 2-bit exponent (bias 1) | 1-bit mantissa; magnitudes
 *                0, 0.5, 1, 1.5, 2, 3, 4, 6; no Inf/NaN.
 *   E4M3 (FP8):  sign | 4-bit exponent (bias 7) | 3-bit mantissa; max 448;
 *                magnitude code 0x7F is NaN; subnormals m * 2^-9.
 *   E8M0:        unsigned power of two, value 2^(v - 127).
 *   bf16:        upper half of an IEEE binary32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------ */
/* scalar format helpers                                               */
/* ------------------------------------------------------------------ */

static float bf16_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* Value of an E2M1 code: (-1)^s * 2^(e-1) * (1 + m/2) for e > 0, and
 * (-1)^s * m/2 for e == 0. */
EXPORT double oracle_e2m1_value(uint8_t code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = e ? ldexp(1.0 + 0.5 * m, e - 1) : 0.5 * m;
  return s ? -mag : mag;
}

/* E2M1 encode: round to the nearest of the eight magnitudes, ties to the
 * even code, saturate to 6 above the range, keep the sign (also when the
 * result is zero).  Input is exact (a double holding the rounded quotient). */
EXPORT uint8_t oracle_e2m1_encode(double v) {
  int neg = signbit(v) ? 1 : 0;
  double a = fabs(v);
  int best = 7;
  if (!(a >= 6.0)) {
    double bestd = INFINITY;
    for (int c = 0; c < 8; ++c) {
      double d = fabs(a - oracle_e2m1_value((uint8_t)c));
      if (d < bestd || (d == bestd && (c & 1) == 0)) {
        best = c;
        bestd = d;
      }
    }
  }
  return (uint8_t)((neg << 3) | best);
}

/* Value of an E4M3 code (0x7F / 0xFF are NaN). */
EXPORT double oracle_e4m3_value(uint8_t code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  double mag;
  if ((code & 0x7F) == 0x7F) return NAN;
  mag = e ? ldexp(1.0 + m / 8.0, e - 7) : ldexp((double)m, -9);
  return s ? -mag : mag;
}

/* E4M3 encode with round-to-nearest-even and saturation to the largest
 * finite value (448); subnormals kept.  Magnitude codes 0..126 are monotone
 * in value, so the two neighbours are found by bisection. */
EXPORT uint8_t oracle_e4m3_encode_satfinite(double v) {
  int neg = signbit(v) ? 1 : 0;
  double a = fabs(v);
  int lo = 0, hi = 126, c;
  if (a >= 448.0) return (uint8_t)((neg << 7) | 126);
  /* largest code with value <= a */
  while (lo < hi) {
    int mid = (lo + hi + 1) / 2;
    if (oracle_e4m3_value((uint8_t)mid) <= a) lo = mid; else hi = mid - 1;
  }
  c = lo;
  if (c < 126) {
    double dl = a - oracle_e4m3_value((uint8_t)c);
    double du = oracle_e4m3_value((uint8_t)(c + 1)) - a;
    if (du < dl || (du == dl && ((c + 1) & 1) == 0)) c = c + 1;
  }
  return (uint8_t)((neg << 7) | c);
}

/* ------------------------------------------------------------------ */
/* step 1: mask routing padding                                        */
/* Megatron-Core "core.transformer.moe.inference_routing_mask_kernel", */
/* mask_routing_padding: rows r with r + tp_rank*N >= real_token_count */
/* get -1 in every top_k slot; other rows are untouched.               */
/* ------------------------------------------------------------------ */
EXPORT void oracle_mask_padding(int64_t *routing_map, int32_t N, int32_t top_k,
                                int32_t real_token_count, int32_t tp_rank) {
  for (int64_t r = 0; r < N; ++r) {
    if (r + (int64_t)tp_rank * N >= (int64_t)real_token_count) {
      for (int32_t j = 0; j < top_k; ++j) routing_map[r * top_k + j] = -1;
    }
  }
}

/* ------------------------------------------------------------------ */
/* step 2: create indices                                              */
/* MAX "moe_create_indices": group the flattened (token, slot) pairs   */
/* by expert (histogram -> CSR offsets -> scatter), with:              */
/*   token_expert_order  pair indices grouped by expert, stable in     */
/*                       ascending pair order; tail = 0xFFFFFFFF       */
/*   expert_start_indices CSR offsets over the active experts;         */
/*                       tail = total routed pairs                     */
/*   restore_token_order position of each pair in token_expert_order;  */
/*                       unrouted pairs = 0xFFFFFFFF                   */
/*   expert_ids          active experts in ascending id; tail = -1     */
/*   expert_usage_stats  {max pairs on one expert, active experts}     */
/*   scales_offset       (optional) offset of each active expert when  */
/*                       every expert's rows are padded to a multiple  */
/*                       of 128 ("aligned scale offsets for block-     */
/*                       scaled grouped matmul"); tail = padded total  */
/* Ids outside [0, E) (the -1 padding sentinel included) route nowhere.*/
/* ------------------------------------------------------------------ */
EXPORT void oracle_create_indices(const int64_t *topk_ids, int64_t S, int32_t E,
                                  uint32_t *token_expert_order, uint32_t *expert_start_indices,
                                  uint32_t *restore_token_order, int32_t *expert_ids,
                                  uint32_t *expert_usage_stats, uint32_t *scales_offset) {
  uint32_t *cnt = (uint32_t *)calloc((size_t)E, sizeof(uint32_t));
  int32_t A = 0;
  uint32_t maxc = 0, pos = 0;
  for (int64_t p = 0; p < S; ++p) {
    int64_t id = topk_ids[p];
    if (id >= 0 && id < E) cnt[id] += 1;
  }
  for (int32_t e = 0; e < E; ++e) {
    if (cnt[e] > 0) expert_ids[A++] = e;
    if (cnt[e] > maxc) maxc = cnt[e];
  }
  for (int32_t i = A; i < E; ++i) expert_ids[i] = -1;
  expert_start_indices[0] = 0;
  for (int32_t i = 0; i < A; ++i)
    expert_start_indices[i + 1] = expert_start_indices[i] + cnt[expert_ids[i]];
  for (int32_t i = A + 1; i <= E; ++i) expert_start_indices[i] = expert_start_indices[A];
  for (int64_t p = 0; p < S; ++p) {
    token_expert_order[p] = 0xFFFFFFFFu;
    restore_token_order[p] = 0xFFFFFFFFu;
  }
  /* stable grouping: experts in ascending id, pairs in ascending index */
  for (int32_t i = 0; i < A; ++i) {
    int32_t e = expert_ids[i];
    for (int64_t p = 0; p < S; ++p) {
      if (topk_ids[p] == e) {
        token_expert_order[pos] = (uint32_t)p;
        restore_token_order[p] = pos;
        ++pos;
      }
    }
  }
  expert_usage_stats[0] = maxc;
  expert_usage_stats[1] = (uint32_t)A;
  if (scales_offset) {
    scales_offset[0] = 0;
    for (int32_t i = 0; i < A; ++i)
      scales_offset[i + 1] = scales_offset[i] + (cnt[expert_ids[i]] + 127u) / 128u * 128u;
    for (int32_t i = A + 1; i <= E; ++i) scales_offset[i] = scales_offset[A];
  }
  free(cnt);
}

/* ------------------------------------------------------------------ */
/* step 3: MXFP4 dispatch                                              */
/* MAX "Struct_ep_dispatch_async_mxfp4", execute(): tokens travel as   */
/* MXFP4 with their block scales packed next to the FP4 quants in the  */
/* send buffer.  One row of the buffer for K hidden values:            */
/*   K/2 bytes of E2M1 codes (element 2i in the low nibble of byte i), */
/*   K/32 E8M0 block scales, zero padding up to a 16-byte stride.      */
/* Block scale: X = 2^(floor(log2(amax)) - 2), the largest power of two */
/* not above amax / 4 (4 = largest power of two in E2M1), exponent     */
/* clamped to [-127, 127]; amax == 0 gives the minimum code 0.         */
/* ------------------------------------------------------------------ */
EXPORT int32_t oracle_mxfp4_row_stride(int32_t K) {
  int32_t raw = K / 2 + K / 32;
  return (raw + 15) / 16 * 16;
}

EXPORT void oracle_mxfp4_encode_row(const uint16_t *x_bf16, int32_t K, uint8_t *row) {
  int32_t stride = oracle_mxfp4_row_stride(K);
  memset(row, 0, (size_t)stride);
  for (int32_t b = 0; b < K / 32; ++b) {
    double amax = 0.0;
    int se, ex;
    for (int32_t i = 0; i < 32; ++i) {
      double v = fabs((double)bf16_to_float(x_bf16[b * 32 + i]));
      if (v > amax) amax = v;
    }
    if (amax == 0.0) {
      se = -127;
    } else {
      frexp(amax, &ex); /* amax = f * 2^ex, f in [0.5, 1) => floor(log2 amax) = ex - 1 */
      se = (ex - 1) - 2;
      if (se < -127) se = -127;
      if (se > 127) se = 127;
    }
    row[K / 2 + b] = (uint8_t)(se + 127);
    for (int32_t i = 0; i < 32; ++i) {
      int32_t k = b * 32 + i;
      double v = (double)bf16_to_float(x_bf16[k]);
      uint8_t q = oracle_e2m1_encode(ldexp(v, -se));
      if (k & 1) row[k / 2] |= (uint8_t)(q << 4);
      else row[k / 2] |= q;
    }
  }
}

/* Row i of the expert-grouped buffer (i < routed pairs) holds the MXFP4
 * encoding of token token_expert_order[i] / top_k; recv_counts[e] is the
 * number of pairs routed to expert e.  Rows >= routed pairs are untouched. */
EXPORT void oracle_dispatch_mxfp4(const uint16_t *input_tokens, int32_t K, int32_t top_k,
                                  int32_t E, const uint32_t *token_expert_order,
                                  const uint32_t *expert_start_indices, const int32_t *expert_ids,
                                  const uint32_t *expert_usage_stats, uint8_t *recv_buf,
                                  uint32_t *recv_counts) {
  int32_t stride = oracle_mxfp4_row_stride(K);
  uint32_t A = expert_usage_stats[1];
  uint32_t R = expert_start_indices[A];
  for (int32_t e = 0; e < E; ++e) recv_counts[e] = 0;
  for (uint32_t a = 0; a < A; ++a)
    recv_counts[expert_ids[a]] = expert_start_indices[a + 1] - expert_start_indices[a];
  for (uint32_t i = 0; i < R; ++i) {
    uint32_t t = token_expert_order[i] / (uint32_t)top_k;
    oracle_mxfp4_encode_row(input_tokens + (size_t)t * K, K, recv_buf + (size_t)i * stride);
  }
}

/* ------------------------------------------------------------------ */
/* NVFP4 encode (FlashRT "grouped-moe-gemv" card, Available functions:  */
/* quantize_activations_nvfp4_bf16 / quantize_weights_nvfp4_bf16).     */
/* One 16-element block with fp32 global scale g > 0:                  */
/*   s32  = fl32( fl32(amax / 6) / g )            two IEEE divisions    */
/*   sc   = E4M3_RNE_SATFINITE(s32)                                    */
/*   sdec = fl32( e4m3(sc) * g )                                        */
/*   q_i  = E2M1_RNE_SAT( fl32(x_i / sdec) ),  or signed zeros if sdec==0 */
/* Codes: element 2i in the low nibble of byte i.                      */
/* ------------------------------------------------------------------ */
static void nvfp4_block(const float *x, float g, uint8_t *q8, uint8_t *sc_out) {
  float amax = 0.0f;
  volatile float t, s32, sdec;
  uint8_t sc;
  for (int i = 0; i < 16; ++i) {
    float v = fabsf(x[i]);
    if (v > amax) amax = v;
  }
  t = amax / 6.0f;
  s32 = t / g;
  sc = oracle_e4m3_encode_satfinite((double)s32);
  sdec = (float)oracle_e4m3_value(sc) * g;
  *sc_out = sc;
  for (int i = 0; i < 8; ++i) q8[i] = 0;
  for (int i = 0; i < 16; ++i) {
    uint8_t q;
    if (sdec == 0.0f) {
      q = signbit(x[i]) ? 8 : 0;
    } else {
      volatile float quot = x[i] / sdec;
      q = oracle_e2m1_encode((double)quot);
    }
    q8[i / 2] |= (uint8_t)((i & 1) ? (q << 4) : q);
  }
}

/* Quantise rows x[rows, K] (fp32 values) with one global scale g:
 * q[rows, K/2], sf[rows, K/16]. */
EXPORT void oracle_nvfp4_quantize(const float *x, int64_t rows, int32_t K, float g, uint8_t *q,
                                  uint8_t *sf) {
  for (int64_t r = 0; r < rows; ++r)
    for (int32_t b = 0; b < K / 16; ++b)
      nvfp4_block(x + r * K + b * 16, g, q + r * (K / 2) + b * 8, sf + r * (K / 16) + b);
}

/* Same, reading bf16 activations. */
EXPORT void oracle_nvfp4_quantize_bf16(const uint16_t *x, int64_t rows, int32_t K, float g,
                                       uint8_t *q, uint8_t *sf) {
  float blk[16];
  for (int64_t r = 0; r < rows; ++r)
    for (int32_t b = 0; b < K / 16; ++b) {
      for (int i = 0; i < 16; ++i) blk[i] = bf16_to_float(x[r * K + b * 16 + i]);
      nvfp4_block(blk, g, q + r * (K / 2) + b * 8, sf + r * (K / 16) + b);
    }
}

/* Per-expert weight global scale: fl32(amax(W_e) / (6 * 448)), 1 when W_e == 0. */
EXPORT float oracle_nvfp4_weight_global(const float *w, int64_t n) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    float v = fabsf(w[i]);
    if (v > amax) amax = v;
  }
  if (amax == 0.0f) return 1.0f;
  {
    volatile float g = amax / 2688.0f;
    return g;
  }
}

/* Expert library quantisation: w[E, N, K] fp32 -> wq[E, N, K/2],
 * sfw[E, N, K/16], w_global[E]. */
EXPORT void oracle_quantize_weights_nvfp4(const float *w, int32_t E, int32_t N, int32_t K,
                                          uint8_t *wq, uint8_t *sfw, float *w_global) {
  for (int32_t e = 0; e < E; ++e) {
    const float *we = w + (int64_t)e * N * K;
    float g = oracle_nvfp4_weight_global(we, (int64_t)N * K);
    w_global[e] = g;
    oracle_nvfp4_quantize(we, N, K, g, wq + (int64_t)e * N * (K / 2),
                          sfw + (int64_t)e * N * (K / 16));
  }
}

/* ------------------------------------------------------------------ */
/* step 4: grouped GEMV (FlashRT "grouped-moe-gemv" card: W4A4 routing */
/* is token-major -- activations [M, K], indices [M, top_k], library   */
/* [E, N, K/2], output [M, top_k, N]).                                 */
/*   y[m,j,n] = g_w[e] * g_a * sum_K a(m,K) * w(e,n,K),  e = idx[m,j]   */
/* a = bf16 x (mode 0, W4A16) or e2m1(xq)*e4m3(sfa) (mode 1, W4A4);    */
/* w = e2m1(wq) * e4m3(sfw).  Slots with e outside [0, E) are skipped  */
/* (not written).  Double-precision accumulation.                      */
/* ------------------------------------------------------------------ */
static double act_value(int32_t mode, const uint16_t *act_bf16, const uint8_t *xq,
                        const uint8_t *sfa, int64_t m, int32_t K, int32_t k) {
  if (mode == 0) return (double)bf16_to_float(act_bf16[m * K + k]);
  {
    uint8_t byte = xq[m * (K / 2) + k / 2];
    uint8_t code = (k & 1) ? (byte >> 4) : (byte & 15);
    return oracle_e2m1_value(code) * oracle_e4m3_value(sfa[m * (K / 16) + k / 16]);
  }
}

static double weight_value(const uint8_t *w, const uint8_t *sfw, int64_t e, int64_t n, int32_t N,
                           int32_t K, int32_t k) {
  int64_t row = e * N + n;
  uint8_t byte = w[row * (K / 2) + k / 2];
  uint8_t code = (k & 1) ? (byte >> 4) : (byte & 15);
  return oracle_e2m1_value(code) * oracle_e4m3_value(sfw[row * (K / 16) + k / 16]);
}

/* one output element; returns 0 and leaves *y untouched for an unrouted slot */
EXPORT int oracle_gemv_element(int32_t mode, const uint16_t *act_bf16, const uint8_t *xq,
                               const uint8_t *sfa, float g_a, const int64_t *indices,
                               int32_t top_k, const uint8_t *w, const uint8_t *sfw,
                               const float *w_global, int32_t E, int32_t N, int32_t K, int64_t m,
                               int32_t j, int32_t n, double *y) {
  int64_t e = indices[m * top_k + j];
  double acc = 0.0;
  if (e < 0 || e >= E) return 0;
  for (int32_t k = 0; k < K; ++k)
    acc += act_value(mode, act_bf16, xq, sfa, m, K, k) * weight_value(w, sfw, e, n, N, K, k);
  *y = acc * (w_global ? (double)w_global[e] : 1.0) * (double)g_a;
  return 1;
}

EXPORT void oracle_grouped_gemv(int32_t mode, const uint16_t *act_bf16, const uint8_t *xq,
                                const uint8_t *sfa, float g_a, const int64_t *indices, int32_t M,
                                int32_t top_k, const uint8_t *w, const uint8_t *sfw,
                                const float *w_global, int32_t E, int32_t N, int32_t K,
                                double *y) {
  for (int64_t m = 0; m < M; ++m)
    for (int32_t j = 0; j < top_k; ++j)
      for (int32_t n = 0; n < N; ++n)
        oracle_gemv_element(mode, act_bf16, xq, sfa, g_a, indices, top_k, w, sfw, w_global, E, N,
                            K, m, j, n, y + (m * top_k + j) * N + n);
}

/* ------------------------------------------------------------------ */
/* step 5: combine                                                     */
/* MAX "Struct_ep_combine_wait", execute(): weighted sum of each       */
/* token's routed expert outputs with the router weights, then the     */
/* optional elementwise epilogue (has_epilogue_fusion).                */
/*   out[t,h] = epi( sum_{j: id in [0,E)} w[t,j] * y[t,j,h] )           */
/* epi: 0 none, 1 identity, 2 scale by alpha.  A row with no routed     */
/* slot gives epi(0).                                                  */
/* ------------------------------------------------------------------ */
EXPORT void oracle_combine(const uint16_t *expert_out, const float *router_weights,
                           const int64_t *topk_ids, int32_t M, int32_t top_k, int32_t H,
                           int32_t E, int32_t epi, float alpha, double *out) {
  for (int64_t t = 0; t < M; ++t) {
    for (int32_t h = 0; h < H; ++h) {
      double acc = 0.0;
      for (int32_t j = 0; j < top_k; ++j) {
        int64_t id = topk_ids[t * top_k + j];
        if (id < 0 || id >= E) continue;
        acc += (double)router_weights[t * top_k + j] *
               (double)bf16_to_float(expert_out[(t * top_k + j) * H + h]);
      }
      if (epi == 2) acc *= (double)alpha;
      out[t * H + h] = acc;
    }
  }
}
