/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU oracle of the routed
 * Mixture-of-Experts layer forward.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library. The product path (the
 * CUDA library) never calls it, and the two share no code, header, table or
 * helper.
 *
 * What it computes (the layer as served by vLLM-Moet, topairepos.com page,
 * "DeepSeek-V4.1-Flash ... MoET hybrid" row and the hybrid results table: 384
 * routed experts per layer, top-k routing, bit-identical resident/non-resident
 * experts). The formulas are the standard routed-MoE layer:
 *   1. router logits  l[t,e] = <x[t,:], Wr[e,:]> (+ bias[e])        (fp32)
 *   2. top-k          the K experts with the largest logits, ties -> lower e,
 *                     listed by (logit desc, e asc)
 *      weights        w[t,k] = exp(l_k - l_0) / sum_j exp(l_j - l_0)
 *                     (softmax over all experts, renormalised over the top-k)
 *   3. permutation    pairs (t,k) sorted by (expert asc, token asc)
 *   4. gate/up+SwiGLU g = Wg[e] x, u = Wu[e] x, h = bf16(silu(g) * u)
 *   5. down           y_pair[p] = w[t,k] * (Wd[e] h)
 *   6. combine        out[t] = bf16(sum_k y_pair[inv[t,k]]), k ascending
 *   7. FP8 variant    e4m3 weights with 128x128 block scales, activations
 *                     quantised per token per 128 columns, per-block
 *                     promotion acc = fma(P_kb, sx*sw, acc)
 *   8. MXFP4 variant  OCP MX block scaling along K: e2m1 weights and e4m3
 *                     activations, one E8M0 (power-of-two) scale per 32
 *                     consecutive elements of a row, per-block promotion
 *                     acc = fma(P_b, 2^(ew + ea), acc)
 *
 * Reading of the layer where the definition leaves a step open (each one is
 * listed with its reason in the design notes):
 *   - Logit reduction order (needed for bit-exact top-k across two
 *     implementations): lane j of 32 accumulates
 *     fmaf(f32(x[h]), Wr[e][h], acc) from +0 over h = j, j+32, j+64, ... in
 *     increasing h; the 32 partials are then summed pairwise,
 *     p[j] += p[j+o] for o = 16, 8, 4, 2, 1 (j < o) -- what an xor butterfly
 *     over a warp leaves in lane 0; the logit is p[0], then + bias[e] (one
 *     fp32 add) when a bias is given.
 *   - Top-k runs on the logits (softmax is monotone, so the set is the same
 *     in exact arithmetic, and no exp() rounding can flip an index).
 *   - Within one expert, pairs are ordered by token; no padding.
 *   - Rounding points: h is rounded once to bf16; y_pair stays fp32; the
 *     combined output is rounded once to bf16 (RNE). Accumulation is fp32 in
 *     increasing index order (the tensor cores' internal order differs, so
 *     FFN outputs are compared within a tolerance, not bit for bit).
 *   - The combine starts from the k = 0 term (not from 0.0f), then adds
 *     k = 1 .. K-1 left to right.
 *   - FP8: s = amax / 448 (IEEE fp32 divide; amax == 0 -> s = 1),
 *     q = e4m3_rne_satfinite(v / s); x is quantised before gate/up, the
 *     bf16 h before down.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (no fast-math:
 * every fp32 operation here must be the IEEE one it names).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- bf16 -- */

static float bf16_to_f32(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* IEEE round-to-nearest-even from fp32 to bfloat16 (1-8-7). */
static uint16_t f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u); /* quiet NaN */
  uint32_t rounding_bias = 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)((u + rounding_bias) >> 16);
}

uint16_t oracle_f32_to_bf16(float f) { return f32_to_bf16(f); }
float oracle_bf16_to_f32(uint16_t b) { return bf16_to_f32(b); }

/* ---------------------------------------------------------------- e4m3 -- */
/* OCP 8-bit floating point, E4M3 ("fn" variant): sign, 4 exponent bits with
 * bias 7, 3 mantissa bits; no infinities; S.1111.111 is NaN; the largest
 * finite magnitude is 1.75 * 2^8 = 448; subnormals are m/8 * 2^-6. */

float oracle_e4m3_to_f32(uint8_t c) {
  int sign = (c >> 7) & 1;
  int ex = (c >> 3) & 0xf;
  int man = c & 7;
  double v;
  if (ex == 0xf && man == 7) return NAN;
  if (ex == 0)
    v = ldexp((double)man, -9); /* man/8 * 2^-6 */
  else
    v = ldexp(1.0 + man / 8.0, ex - 7);
  return (float)(sign ? -v : v);
}

/* fp32 -> e4m3, round to nearest even, saturating to +-448 (finite inputs). */
uint8_t oracle_f32_to_e4m3(float f) {
  uint8_t sign = signbit(f) ? 0x80 : 0x00;
  double a = fabs((double)f);
  if (isnan(f)) return 0x7f;
  if (a >= 448.0) return sign | 0x7e;
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: multiples of 2^-9; q = 8 is the smallest normal */
    double q = nearbyint(a * 512.0); /* exact scaling; default mode = RNE */
    return sign | (uint8_t)q;
  }
  int e;
  double m = frexp(a, &e); /* a = m * 2^e, m in [0.5, 1) */
  m *= 2.0;
  e -= 1; /* a = m * 2^e, m in [1, 2) */
  double q = nearbyint((m - 1.0) * 8.0);
  if (q == 8.0) {
    q = 0.0;
    e += 1;
  }
  int biased = e + 7;
  if (biased > 15 || (biased == 15 && q == 7.0)) return sign | 0x7e;
  return sign | (uint8_t)((biased << 3) | (int)q);
}

/* Quantise a [rows, cols] bf16 matrix in blocks of br x 128 (br = 1 for
 * activations, 128 for weights): s = amax / 448 (amax == 0 -> 1),
 * q = e4m3(v / s). scales is [ceil(rows/br), cols/128] row-major. */
void oracle_quant_e4m3(const uint16_t* src, int rows, int cols, int br, uint8_t* q, float* scales) {
  int nbr = (rows + br - 1) / br, nbc = cols / 128;
  for (int rb = 0; rb < nbr; ++rb)
    for (int cb = 0; cb < nbc; ++cb) {
      float amax = 0.0f;
      for (int r = rb * br; r < rows && r < (rb + 1) * br; ++r)
        for (int c = cb * 128; c < (cb + 1) * 128; ++c) {
          float v = fabsf(bf16_to_f32(src[(size_t)r * cols + c]));
          if (v > amax) amax = v;
        }
      float s = (amax == 0.0f) ? 1.0f : amax / 448.0f;
      scales[(size_t)rb * nbc + cb] = s;
      for (int r = rb * br; r < rows && r < (rb + 1) * br; ++r)
        for (int c = cb * 128; c < (cb + 1) * 128; ++c) {
          float v = bf16_to_f32(src[(size_t)r * cols + c]);
          float t = v / s;
          q[(size_t)r * cols + c] = oracle_f32_to_e4m3(t);
        }
    }
}

/* ------------------------------------------------------------- router -- */

#define LANES 32

/* One logit in the specified order (see the header comment). */
static float logit_one(const uint16_t* xrow, const float* wrow, int H) {
  float p[LANES];
  for (int j = 0; j < LANES; ++j) {
    float acc = 0.0f;
    for (int h = j; h < H; h += LANES) acc = fmaf(bf16_to_f32(xrow[h]), wrow[h], acc);
    p[j] = acc;
  }
  for (int o = LANES / 2; o >= 1; o /= 2)
    for (int j = 0; j < o; ++j) p[j] = p[j] + p[j + o];
  return p[0];
}

/* logits [T, E] fp32. bias may be NULL. */
void oracle_router_logits(const uint16_t* x, const float* wr, const float* bias, int T, int H, int E,
                          float* logits, int threads) {
#ifdef _OPENMP
  if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel for schedule(static)
#endif
  for (long te = 0; te < (long)T * E; ++te) {
    int t = (int)(te / E), e = (int)(te % E);
    float l = logit_one(x + (size_t)t * H, wr + (size_t)e * H, H);
    if (bias) l = l + bias[e];
    logits[te] = l;
  }
}

/* Top-k by (logit desc, e asc) via a full stable selection of all E experts,
 * then weights renormalised over the chosen K, computed in double. */
void oracle_topk(const float* logits, int T, int E, int K, int32_t* idx, double* w) {
  int* order = (int*)malloc(sizeof(int) * (size_t)E);
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    for (int e = 0; e < E; ++e) order[e] = e;
    /* insertion sort = full stable sort by logit descending (ties keep index order) */
    for (int i = 1; i < E; ++i) {
      int v = order[i], j = i - 1;
      while (j >= 0 && l[order[j]] < l[v]) {
        order[j + 1] = order[j];
        --j;
      }
      order[j + 1] = v;
    }
    double l0 = (double)l[order[0]], den = 0.0;
    for (int k = 0; k < K; ++k) den += exp((double)l[order[k]] - l0);
    for (int k = 0; k < K; ++k) {
      idx[(size_t)t * K + k] = order[k];
      w[(size_t)t * K + k] = exp((double)l[order[k]] - l0) / den;
    }
  }
  free(order);
}

/* -------------------------------------------------------- permutation -- */

/* Counting sort of the T*K pairs by (expert asc, token asc).
 * counts [E], offsets [E+1], perm_src/perm_k [T*K], inv [T*K]. */
void oracle_permute(const int32_t* idx, int T, int K, int E, int32_t* counts, int32_t* offsets,
                    int32_t* perm_src, int32_t* perm_k, int32_t* inv) {
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (long i = 0; i < (long)T * K; ++i) counts[idx[i]]++;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
  for (int t = 0; t < T; ++t) /* tokens in order, so each expert's rows come out token-ascending */
    for (int k = 0; k < K; ++k) {
      int e = idx[(size_t)t * K + k];
      int p = cursor[e]++;
      perm_src[p] = t;
      perm_k[p] = k;
      inv[(size_t)t * K + k] = p;
    }
  free(cursor);
}

/* ---------------------------------------------------------------- FFN -- */

static float silu_f32(float g) { return g / (1.0f + expf(-g)); }

/* One (token, expert) pair, bf16 weights.
 *   xrow  [H] bf16, wgu [2I, H] bf16 (gate rows 0..I-1, up rows I..2I-1),
 *   wdn [H, I] bf16, weight = routing weight, y [H] fp32 out, hrow [I] bf16 out
 * acc64 != 0 accumulates the dot products in double instead of fp32 (a second
 * reference for error bounds). */
static void pair_bf16(const uint16_t* xrow, const uint16_t* wgu, const uint16_t* wdn, int H, int I,
                      float weight, float* y, uint16_t* hrow, int acc64) {
  for (int j = 0; j < I; ++j) {
    const uint16_t* wg = wgu + (size_t)j * H;
    const uint16_t* wu = wgu + (size_t)(I + j) * H;
    float g, u;
    if (acc64) {
      double gd = 0, ud = 0;
      for (int h = 0; h < H; ++h) {
        double xv = bf16_to_f32(xrow[h]);
        gd += (double)bf16_to_f32(wg[h]) * xv;
        ud += (double)bf16_to_f32(wu[h]) * xv;
      }
      g = (float)gd;
      u = (float)ud;
    } else {
      g = 0.0f;
      u = 0.0f;
      for (int h = 0; h < H; ++h) {
        float xv = bf16_to_f32(xrow[h]);
        g = fmaf(bf16_to_f32(wg[h]), xv, g);
        u = fmaf(bf16_to_f32(wu[h]), xv, u);
      }
    }
    hrow[j] = f32_to_bf16(silu_f32(g) * u);
  }
  for (int o = 0; o < H; ++o) {
    const uint16_t* wd = wdn + (size_t)o * I;
    float acc;
    if (acc64) {
      double a = 0;
      for (int j = 0; j < I; ++j) a += (double)bf16_to_f32(wd[j]) * bf16_to_f32(hrow[j]);
      acc = (float)a;
    } else {
      acc = 0.0f;
      for (int j = 0; j < I; ++j) acc = fmaf(bf16_to_f32(wd[j]), bf16_to_f32(hrow[j]), acc);
    }
    y[o] = weight * acc;
  }
}

/* FFN for a list of pairs.
 *   x [T, H] bf16; pair_token/pair_expert [npairs]; pair_weight [npairs] fp32;
 *   w_gu[e] / w_dn[e] = per-expert host pointers (NULL for experts not needed);
 *   y [npairs, H] fp32 out; h [npairs, I] bf16 out (may be NULL).
 * Returns 0, or -1 if a needed expert pointer is NULL. */
int oracle_ffn_bf16(const uint16_t* x, int H, int I, int npairs, const int32_t* pair_token,
                    const int32_t* pair_expert, const float* pair_weight, const uint16_t* const* w_gu,
                    const uint16_t* const* w_dn, float* y, uint16_t* h, int acc64, int threads) {
  for (int p = 0; p < npairs; ++p)
    if (!w_gu[pair_expert[p]] || !w_dn[pair_expert[p]]) return -1;
#ifdef _OPENMP
  if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel
#endif
  {
    uint16_t* htmp = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)I);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
    for (int p = 0; p < npairs; ++p) {
      int e = pair_expert[p];
      pair_bf16(x + (size_t)pair_token[p] * H, w_gu[e], w_dn[e], H, I, pair_weight[p], y + (size_t)p * H,
                htmp, acc64);
      if (h) memcpy(h + (size_t)p * I, htmp, sizeof(uint16_t) * (size_t)I);
    }
    free(htmp);
  }
  return 0;
}

/* FP8 block-scaled dot product of one weight row with one activation row:
 *   qw [n] e4m3, sw [n/128] fp32 (the row's block scales), qa [n] e4m3,
 *   sa [n/128]; P_kb = sum over the block of f32(qw)*f32(qa) (fp32),
 *   acc = fmaf(P_kb, sa[kb] * sw[kb], acc) for kb ascending. */
static float dot_fp8(const uint8_t* qw, const float* sw, const uint8_t* qa, const float* sa, int n,
                     const float* lut) {
  float acc = 0.0f;
  for (int kb = 0; kb < n / 128; ++kb) {
    float part = 0.0f;
    for (int i = kb * 128; i < (kb + 1) * 128; ++i) part = fmaf(lut[qw[i]], lut[qa[i]], part);
    acc = fmaf(part, sa[kb] * sw[kb], acc);
  }
  return acc;
}

/* FP8 FFN for a list of pairs.
 *   x [T, H] bf16 (quantised here per token per 128 columns);
 *   qgu[e] [2I, H] e4m3 + sgu[e] [2I/128, H/128]; qdn[e] [H, I] e4m3 + sdn[e] [H/128, I/128].
 *   y [npairs, H] fp32; h [npairs, I] bf16 (may be NULL). */
int oracle_ffn_fp8(const uint16_t* x, int H, int I, int npairs, const int32_t* pair_token,
                   const int32_t* pair_expert, const float* pair_weight, const uint8_t* const* qgu,
                   const float* const* sgu, const uint8_t* const* qdn, const float* const* sdn, float* y,
                   uint16_t* h, int threads) {
  for (int p = 0; p < npairs; ++p) {
    int e = pair_expert[p];
    if (!qgu[e] || !sgu[e] || !qdn[e] || !sdn[e]) return -1;
  }
  float lut[256];
  for (int c = 0; c < 256; ++c) lut[c] = oracle_e4m3_to_f32((uint8_t)c);
#ifdef _OPENMP
  if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel
#endif
  {
    uint8_t* qx = (uint8_t*)malloc((size_t)H);
    float* sx = (float*)malloc(sizeof(float) * (size_t)(H / 128));
    uint16_t* hb = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)I);
    uint8_t* qh = (uint8_t*)malloc((size_t)I);
    float* shh = (float*)malloc(sizeof(float) * (size_t)(I / 128));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
    for (int p = 0; p < npairs; ++p) {
      int e = pair_expert[p];
      const uint16_t* xrow = x + (size_t)pair_token[p] * H;
      oracle_quant_e4m3(xrow, 1, H, 1, qx, sx);
      for (int j = 0; j < I; ++j) {
        int rg = j, ru = I + j;
        float g = dot_fp8(qgu[e] + (size_t)rg * H, sgu[e] + (size_t)(rg / 128) * (H / 128), qx, sx, H, lut);
        float u = dot_fp8(qgu[e] + (size_t)ru * H, sgu[e] + (size_t)(ru / 128) * (H / 128), qx, sx, H, lut);
        hb[j] = f32_to_bf16(silu_f32(g) * u);
      }
      if (h) memcpy(h + (size_t)p * I, hb, sizeof(uint16_t) * (size_t)I);
      oracle_quant_e4m3(hb, 1, I, 1, qh, shh);
      for (int o = 0; o < H; ++o) {
        float acc = dot_fp8(qdn[e] + (size_t)o * I, sdn[e] + (size_t)(o / 128) * (I / 128), qh, shh, I, lut);
        y[(size_t)p * H + o] = pair_weight[p] * acc;
      }
    }
    free(qx);
    free(sx);
    free(hb);
    free(qh);
    free(shh);
  }
  return 0;
}

/* ---------------------------------------------------------- MX (e2m1) -- */
/* OCP Microscaling formats: E2M1 elements (sign, 2 exponent bits with bias
 * 1, 1 mantissa bit; no infinities or NaN; magnitudes 0, 0.5, 1, 1.5, 2, 3,
 * 4, 6) and E4M3 elements (above), with one E8M0 scale -- a power of two,
 * stored as its exponent + 127 -- per block of 32 consecutive elements. */

float oracle_e2m1_to_f32(uint8_t c) {
  int sign = (c >> 3) & 1;
  int ex = (c >> 1) & 3;
  int man = c & 1;
  double v = (ex == 0) ? 0.5 * man : ldexp(1.0 + 0.5 * man, ex - 1);
  return (float)(sign ? -v : v);
}

/* fp32 -> e2m1, round to nearest even, saturating to +-6 (finite inputs). */
uint8_t oracle_f32_to_e2m1(float f) {
  uint8_t sign = signbit(f) ? 0x8 : 0x0;
  double a = fabs((double)f);
  if (a >= 6.0) return sign | 0x7;
  if (a < 1.0) {
    /* subnormal step 0.5: codes 0 (0), 1 (0.5) and 2 (1.0, the smallest normal) */
    double q = nearbyint(a * 2.0); /* exact scaling; default mode = RNE */
    return sign | (uint8_t)q;
  }
  int e;
  double m = frexp(a, &e); /* a = m * 2^e, m in [0.5, 1) */
  m *= 2.0;
  e -= 1; /* a = m * 2^e, m in [1, 2), e in {0, 1, 2} */
  double q = nearbyint((m - 1.0) * 2.0);
  if (q == 2.0) {
    q = 0.0;
    e += 1;
  }
  if (e > 2) return sign | 0x7; /* only from rounding just below 6 up: 6 itself */
  return sign | (uint8_t)(((e + 1) << 1) | (int)q);
}

/* MX quantiser of a [rows, cols] bf16 matrix along its rows: for each run of
 * 32 elements, X = 2^(floor(log2 amax) - emax) with emax = 2 for E2M1
 * (6 = 1.5 * 2^2) and 8 for E4M3 (448 = 1.75 * 2^8), clamped to 2^-127 ..
 * 2^127 (an all-zero block takes 2^-127); q = encode(v / X), round to
 * nearest even, saturating (the block's largest element can exceed the
 * element format's maximum after scaling and is then clamped to it).
 * q [rows, cols] one code per byte; scales [rows, cols/32] E8M0 bytes.
 * elem: 0 = E2M1, 1 = E4M3. */
void oracle_quant_mx(const uint16_t* src, int rows, int cols, int elem, uint8_t* q, uint8_t* scales) {
  const int emax = elem == 0 ? 2 : 8;
  const int nb = cols / 32;
  for (int r = 0; r < rows; ++r)
    for (int b = 0; b < nb; ++b) {
      const uint16_t* v = src + (size_t)r * cols + (size_t)b * 32;
      float amax = 0.0f;
      for (int i = 0; i < 32; ++i) {
        float a = fabsf(bf16_to_f32(v[i]));
        if (a > amax) amax = a;
      }
      int sexp = -127;
      if (amax > 0.0f) {
        int e;
        frexpf(amax, &e); /* amax = m * 2^e, m in [0.5, 1): floor(log2 amax) = e - 1 */
        sexp = (e - 1) - emax;
        if (sexp < -127) sexp = -127;
        if (sexp > 127) sexp = 127;
      }
      scales[(size_t)r * nb + b] = (uint8_t)(sexp + 127);
      for (int i = 0; i < 32; ++i) {
        float t = (float)ldexp((double)bf16_to_f32(v[i]), -sexp);
        q[(size_t)r * cols + (size_t)b * 32 + i] = elem == 0 ? oracle_f32_to_e2m1(t) : oracle_f32_to_e4m3(t);
      }
    }
}

/* MX dot product of a weight row (e2m1 codes, E8M0 scales) with an
 * activation row (e4m3 codes, E8M0 scales): P_b = sum over the 32-element
 * block of f32(w)*f32(a) (fp32), acc = fmaf(P_b, 2^(ew_b + ea_b), acc) for
 * blocks in increasing order. */
static float dot_mx(const uint8_t* qw, const uint8_t* sw, const uint8_t* qa, const uint8_t* sa, int n,
                    const float* lw, const float* la) {
  float acc = 0.0f;
  for (int b = 0; b < n / 32; ++b) {
    float part = 0.0f;
    for (int i = b * 32; i < (b + 1) * 32; ++i) part = fmaf(lw[qw[i]], la[qa[i]], part);
    acc = fmaf(part, (float)ldexp(1.0, (int)sw[b] + (int)sa[b] - 254), acc);
  }
  return acc;
}

/* MXFP4 FFN for a list of pairs.
 *   x [T, H] bf16 (quantised here to MX e4m3 per token);
 *   qgu[e] [2I, H] e2m1 codes + sgu[e] [2I, H/32] E8M0; qdn[e] [H, I] + sdn[e] [H, I/32].
 *   y [npairs, H] fp32; h [npairs, I] bf16 (may be NULL). */
int oracle_ffn_mxfp4(const uint16_t* x, int H, int I, int npairs, const int32_t* pair_token,
                     const int32_t* pair_expert, const float* pair_weight, const uint8_t* const* qgu,
                     const uint8_t* const* sgu, const uint8_t* const* qdn, const uint8_t* const* sdn, float* y,
                     uint16_t* h, int threads) {
  for (int p = 0; p < npairs; ++p) {
    int e = pair_expert[p];
    if (!qgu[e] || !sgu[e] || !qdn[e] || !sdn[e]) return -1;
  }
  float lw[16], la[256];
  for (int c = 0; c < 16; ++c) lw[c] = oracle_e2m1_to_f32((uint8_t)c);
  for (int c = 0; c < 256; ++c) la[c] = oracle_e4m3_to_f32((uint8_t)c);
#ifdef _OPENMP
  if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel
#endif
  {
    uint8_t* qx = (uint8_t*)malloc((size_t)H);
    uint8_t* sx = (uint8_t*)malloc((size_t)(H / 32));
    uint16_t* hb = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)I);
    uint8_t* qh = (uint8_t*)malloc((size_t)I);
    uint8_t* shh = (uint8_t*)malloc((size_t)(I / 32));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
    for (int p = 0; p < npairs; ++p) {
      int e = pair_expert[p];
      oracle_quant_mx(x + (size_t)pair_token[p] * H, 1, H, 1, qx, sx);
      for (int j = 0; j < I; ++j) {
        int rg = j, ru = I + j;
        float g = dot_mx(qgu[e] + (size_t)rg * H, sgu[e] + (size_t)rg * (H / 32), qx, sx, H, lw, la);
        float u = dot_mx(qgu[e] + (size_t)ru * H, sgu[e] + (size_t)ru * (H / 32), qx, sx, H, lw, la);
        hb[j] = f32_to_bf16(silu_f32(g) * u);
      }
      if (h) memcpy(h + (size_t)p * I, hb, sizeof(uint16_t) * (size_t)I);
      oracle_quant_mx(hb, 1, I, 1, qh, shh);
      for (int o = 0; o < H; ++o) {
        float acc = dot_mx(qdn[e] + (size_t)o * I, sdn[e] + (size_t)o * (I / 32), qh, shh, I, lw, la);
        y[(size_t)p * H + o] = pair_weight[p] * acc;
      }
    }
    free(qx);
    free(sx);
    free(hb);
    free(qh);
    free(shh);
  }
  return 0;
}

/* ------------------------------------------------------------ combine -- */

/* out[t, o] = bf16(((y[inv[t,0]] + y[inv[t,1]]) + ...) + y[inv[t,K-1]]). */
void oracle_combine(const float* y_pair, const int32_t* inv, int T, int K, int H, uint16_t* out) {
  for (int t = 0; t < T; ++t)
    for (int o = 0; o < H; ++o) {
      float acc = y_pair[(size_t)inv[(size_t)t * K] * H + o];
      for (int k = 1; k < K; ++k) acc = acc + y_pair[(size_t)inv[(size_t)t * K + k] * H + o];
      out[(size_t)t * H + o] = f32_to_bf16(acc);
    }
}
