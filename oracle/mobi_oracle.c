/*
 * mobi_oracle.c — TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * A plain, slow, obviously correct CPU implementation of the MoBiQuant
 * token-routed mixed-bit linear layer, used only by the tests, by the smoke
 * check and by the benchmark's CPU-baseline leg. The CUDA library never links,
 * loads or calls this file, and this file shares no code with it.
 *
 * Sources (explainer pages of "MoBiQuant: Mixture-of-Bits Quantization for
 * Token-Adaptive Elastic LLMs"):
 *   [ja] gist.science/ja/paper/2602.20191 — §2.1 MoBiSlice (recursive residual
 *        quantisation R_1 = W, W_e = Q(R_e), R_{e+1} = R_e - W_e; W^(b) = sum W_e),
 *        §2.2 MoBiRoute (per-token score decides how many residual slices are
 *        active).
 *   [en] gist.science/paper/2602.20191 — §2.A MoBiSlice ("Recursive
 *        Decomposition", "Process", "Elasticity": a 6-bit weight is the 2-bit
 *        base plus two 2-bit residuals), §2.B MoBiRoute ("Routing Mechanism",
 *        "Dynamic Adjustment").
 *
 * Precision: the quantiser runs in IEEE fp32 with round-to-nearest-even
 * (compiled with -ffp-contract=off, no fast-math); routing logits and the GEMM
 * run in fp64 on exact operands.
 *
 * Readings where the pages are silent (the quantiser Q is named, not defined):
 *   asymmetric min-max round-to-nearest over groups of G = 128 along K, with an
 *   integer zero-point z = clamp(rint(-min/s), 0, 3), the scale s = (max-min)/3
 *   floored at 2^-14 and rounded to fp16 BEFORE it is used, deq = (q - z) * s,
 *   and the reconstruction W^(k) = sum_{s<k} deq_s kept exact (no rounding to
 *   a 16-bit type). Routing: a linear router, k_t = 1 + argmax (lowest index on
 *   an exact tie). Bucketing: stable ascending sort by k_t. Threshold routing
 *   (oracle_route_mlp): a ReLU two-layer MLP gives one score per residual
 *   slice, a slice is active iff sigmoid(score / tau) > delta, and
 *   k_t = 1 + the number of active residual slices. Generic slicing
 *   (oracle_pack_bits): the same quantiser with b-bit codes, L = 2^b - 1 steps
 *   (s = (max-min)/L, z and q clamped to [0, L]) over G-wide groups; 1-bit
 *   slices give 1..S bits per weight ([en] §2.A lists 3-bit precision, which
 *   2-bit slices cannot reach) and are stored at 1 bit per weight ([en] §3,
 *   "Specialized Kernel Implementation": the bytes fetched follow the bits
 *   used), 32 codes per word in the library's documented bit order. Slices of
 *   different widths in one layer (oracle_pack_slices): round s quantises the
 *   residual with its own width, and the slices are stored one after another,
 *   each in the layout of its width; widths (2, 1, 1, 2) give 2, 3, 4 and 6
 *   bits, the precisions [en] §2.A lists.
 *
 * Parity pins: every function here is pinned by tests/test_oracle.py against
 * closed-form groups, hand-derived packed words, invariants (non-increasing
 * reconstruction error, half-step rounding bound, fewer slices for a larger
 * threshold), brute force (numpy fp64 matmul and Python loops on tiny shapes,
 * one-hot inputs), library routines (torch's fp64 linear layers) and special
 * cases; see that file.
 * Whether the quantiser reading matches the MoBiQuant authors' own Q cannot be
 * pinned from the pages ("parity unpinned" for that reading, not for the code).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- scalar conversions (IEEE, round-to-nearest-even) ------------------- */

static float half_bits_to_float(uint16_t h) {
  _Float16 v;
  memcpy(&v, &h, sizeof v);
  return (float)v;
}

static uint16_t float_to_half_bits(float f) {
  _Float16 v = (_Float16)f; /* IEEE conversion, round to nearest even */
  uint16_t h;
  memcpy(&h, &v, sizeof h);
  return h;
}

static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ---- MoBiSlice ---------------------------------------------------------- */

/*
 * One group of G weights of one row through S rounds of the recursion
 * R_1 = W, W_s = Q(R_s), R_{s+1} = R_s - W_s   ([ja] §2.1, [en] §2.A), with Q
 * the asymmetric min-max round-to-nearest of widths[s]-bit codes in round s:
 * L = 2^widths[s] - 1 steps between the group's minimum and maximum.
 * q_out[s*G + i] receives the code of element i in slice s; scale_out[s] and
 * zero_out[s] the fp16 bit patterns of that slice's scale and zero.
 */
static void quantise_group(const uint16_t* w, int G, int S, const int* widths, uint8_t* q_out,
                           uint16_t* scale_out, uint16_t* zero_out) {
  float R[1024];
  for (int i = 0; i < G; ++i) R[i] = half_bits_to_float(w[i]);
  for (int s = 0; s < S; ++s) {
    const float L = (float)((1 << widths[s]) - 1); /* 2 bits: 4 levels, 3 steps; 1 bit: 1 step */
    float mn = R[0], mx = R[0];
    for (int i = 1; i < G; ++i) {
      if (R[i] < mn) mn = R[i];
      if (R[i] > mx) mx = R[i];
    }
    float sc = (mx - mn) / L;
    if (sc < 0x1p-14f) sc = 0x1p-14f;      /* degenerate group: smallest normal fp16 */
    uint16_t scale_bits = float_to_half_bits(sc);
    float step = half_bits_to_float(scale_bits); /* the stored scale is the one used */
    float zf = rintf(-mn / step);
    if (zf < 0.0f) zf = 0.0f;
    if (zf > L) zf = L;
    int z = (int)zf;
    for (int i = 0; i < G; ++i) {
      float qf = rintf(R[i] / step) + (float)z;
      if (qf < 0.0f) qf = 0.0f;
      if (qf > L) qf = L;
      int q = (int)qf;
      q_out[s * G + i] = (uint8_t)q;
      float deq = (float)(q - z) * step; /* exact: |q-z| <= 3 times an fp16 */
      R[i] = R[i] - deq;                 /* the residual of the next round */
    }
    scale_out[s] = scale_bits;
    zero_out[s] = float_to_half_bits((float)z);
  }
}

/*
 * The documented word layouts. 2-bit codes: words [S][N][K/16]; word (s, n, w)
 * holds q(s, n, 16w + i) in bits [2i+1 : 2i]. 1-bit codes: words [S][N][K/32];
 * word (s, n, w) holds q(s, n, 32w + i) in bit 2i for i < 16 and
 * q(s, n, 32w + 16 + i) in bit 2i + 1 (the first 16 codes on the even bits,
 * the next 16 on the odd bits).
 */
static int64_t words_per_row(int64_t K, int bits) { return bits == 1 ? K / 32 : K / 16; }

/* Word offset of slice s when the slices (widths[0..s-1]) are stored one after
 * another, each [N][K * width / 32]. */
static int64_t slice_offset(const int* widths, int64_t N, int64_t K, int64_t s) {
  int64_t off = 0;
  for (int64_t j = 0; j < s; ++j) off += N * words_per_row(K, widths[j]);
  return off;
}

static int code_of(const uint32_t* codes, int64_t N, int64_t K, const int* widths, int64_t s, int64_t n,
                   int64_t k) {
  const int bits = widths[s];
  const uint32_t word =
      codes[slice_offset(widths, N, K, s) + n * words_per_row(K, bits) + (bits == 1 ? k / 32 : k / 16)];
  if (bits == 1) {
    const int i = (int)(k % 32);
    return (int)((word >> (i < 16 ? 2 * i : 2 * (i - 16) + 1)) & 1u);
  }
  return (int)((word >> (2 * (k % 16))) & 3u);
}

static int uniform_widths(int* widths, int S, int bits) {
  if (S < 1 || S > 8) return -1;
  for (int j = 0; j < S; ++j) widths[j] = bits;
  return 0;
}

/*
 * oracle_pack_slices: W fp16 [N][K] -> codes and sz for S slices over G-wide
 * groups, slice s of widths[s]-bit codes (1 or 2) in the word layout of its
 * width (above), the slices one after another. sz is [S][K/G][N] (fp16 scale
 * in bits [15:0], fp16 zero in bits [31:16]). If q_out is not NULL it
 * receives the unpacked codes uint8 [S][N][K].
 * Returns 0, or -1 on an unsupported argument.
 */
int oracle_pack_slices(const uint16_t* W, int64_t N, int64_t K, int G, int S, const int* widths,
                       uint32_t* codes, uint32_t* sz, uint8_t* q_out, int nthreads) {
  if (G <= 0 || G > 1024 || K % G != 0 || K % 16 != 0 || S < 1 || S > 8) return -1;
  for (int j = 0; j < S; ++j) {
    if (widths[j] < 1 || widths[j] > 2) return -1;
    if (widths[j] == 1 && K % 32 != 0) return -1;
  }
  set_threads(nthreads);
  const int64_t ngroups = K / G;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t n = 0; n < N; ++n) {
    uint8_t q[8 * 1024];
    uint16_t sc[8], zr[8];
    uint8_t* row_codes = (uint8_t*)malloc((size_t)S * (size_t)K);
    for (int64_t g = 0; g < ngroups; ++g) {
      quantise_group(W + n * K + g * G, G, S, widths, q, sc, zr);
      for (int s = 0; s < S; ++s) {
        sz[((int64_t)s * ngroups + g) * N + n] = (uint32_t)sc[s] | ((uint32_t)zr[s] << 16);
        for (int i = 0; i < G; ++i) row_codes[(int64_t)s * K + g * G + i] = q[s * G + i];
      }
    }
    for (int s = 0; s < S; ++s) {
      const int bits = widths[s];
      const int64_t nwords = words_per_row(K, bits);
      uint32_t* slice = codes + slice_offset(widths, N, K, s);
      for (int64_t w = 0; w < nwords; ++w) {
        uint32_t word = 0;
        if (bits == 1) {
          for (int i = 0; i < 16; ++i) {
            word |= (uint32_t)row_codes[(int64_t)s * K + 32 * w + i] << (2 * i);
            word |= (uint32_t)row_codes[(int64_t)s * K + 32 * w + 16 + i] << (2 * i + 1);
          }
        } else {
          for (int i = 0; i < 16; ++i)
            word |= (uint32_t)row_codes[(int64_t)s * K + 16 * w + i] << (2 * i);
        }
        slice[n * nwords + w] = word;
      }
      if (q_out)
        memcpy(q_out + ((int64_t)s * N + n) * K, row_codes + (int64_t)s * K, (size_t)K);
    }
    free(row_codes);
  }
  return 0;
}

/* oracle_pack_bits: every slice `bits`-bit (1 or 2). */
int oracle_pack_bits(const uint16_t* W, int64_t N, int64_t K, int G, int S, int bits,
                     uint32_t* codes, uint32_t* sz, uint8_t* q_out, int nthreads) {
  int widths[8];
  if (uniform_widths(widths, S, bits) != 0) return -1;
  return oracle_pack_slices(W, N, K, G, S, widths, codes, sz, q_out, nthreads);
}

/*
 * oracle_pack: the 2-bit slicing (the method's configuration): oracle_pack_bits
 * with bits = 2.
 */
int oracle_pack(const uint16_t* W, int64_t N, int64_t K, int G, int S,
                uint32_t* codes, uint32_t* sz, uint8_t* q_out, int nthreads) {
  return oracle_pack_bits(W, N, K, G, S, 2, codes, sz, q_out, nthreads);
}

/* oracle_unpack_slices: the documented word layouts (slice s of widths[s]-bit
 * codes) back to codes uint8 [S][N][K]; oracle_unpack_bits has one width for
 * every slice and oracle_unpack is the 2-bit case. */
void oracle_unpack_slices(const uint32_t* codes, int64_t N, int64_t K, int S, const int* widths, uint8_t* q_out) {
  for (int64_t s = 0; s < S; ++s)
    for (int64_t n = 0; n < N; ++n)
      for (int64_t k = 0; k < K; ++k) q_out[(s * N + n) * K + k] = (uint8_t)code_of(codes, N, K, widths, s, n, k);
}

void oracle_unpack_bits(const uint32_t* codes, int64_t N, int64_t K, int S, int bits, uint8_t* q_out) {
  int widths[8];
  if (uniform_widths(widths, S, bits) == 0) oracle_unpack_slices(codes, N, K, S, widths, q_out);
}

void oracle_unpack(const uint32_t* codes, int64_t N, int64_t K, int S, uint8_t* q_out) {
  oracle_unpack_bits(codes, N, K, S, 2, q_out);
}

/*
 * oracle_reconstruct: the k-slice weight W^(k)[n][j] = sum_{s<k} (q - z) * scale
 * in fp64 (exact: every term is a small integer times an fp16 value)
 * ([ja] §2.1 W^(b) = sum W_e; [en] §2.A "Elasticity").
 */
void oracle_reconstruct_slices(const uint32_t* codes, const uint32_t* sz, int64_t N, int64_t K, int G, int S,
                               const int* widths, int k, double* W_hat) {
  const int64_t ngroups = K / G;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K; ++j) {
      double acc = 0.0;
      for (int s = 0; s < k && s < S; ++s) {
        int q = code_of(codes, N, K, widths, s, n, j);
        uint32_t e = sz[((int64_t)s * ngroups + j / G) * N + n];
        double scale = (double)half_bits_to_float((uint16_t)(e & 0xffffu));
        double zero = (double)half_bits_to_float((uint16_t)(e >> 16));
        acc += ((double)q - zero) * scale;
      }
      W_hat[n * K + j] = acc;
    }
}

void oracle_reconstruct_bits(const uint32_t* codes, const uint32_t* sz, int64_t N, int64_t K, int G, int S,
                             int bits, int k, double* W_hat) {
  int widths[8];
  if (uniform_widths(widths, S, bits) == 0) oracle_reconstruct_slices(codes, sz, N, K, G, S, widths, k, W_hat);
}

void oracle_reconstruct(const uint32_t* codes, const uint32_t* sz, int64_t N, int64_t K,
                        int G, int S, int k, double* W_hat) {
  oracle_reconstruct_bits(codes, sz, N, K, G, S, 2, k, W_hat);
}

/* ---- MoBiRoute ---------------------------------------------------------- */

/*
 * oracle_route: logit_j(t) = sum_k x[t,k] Wr[k,j] + bias_j in fp64 and
 * k_t = 1 + argmax_j (the first maximum wins) ([ja] §2.2, [en] §2.B).
 * gap[t] = best logit minus the runner-up (+inf when S == 1), so that callers
 * can tell near-ties apart. logits (fp64 [T][S]) may be NULL.
 */
void oracle_route(const uint16_t* X, int64_t T, int64_t K, const float* Wr, const float* bias,
                  int S, int32_t* k_out, double* gap, double* logits, int nthreads) {
  set_threads(nthreads);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    double l[8];
    for (int j = 0; j < S; ++j) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += bf16_bits_to_double(X[t * K + k]) * (double)Wr[k * S + j];
      l[j] = acc + (bias ? (double)bias[j] : 0.0);
    }
    int best = 0;
    for (int j = 1; j < S; ++j)
      if (l[j] > l[best]) best = j;
    double second = -INFINITY;
    for (int j = 0; j < S; ++j)
      if (j != best && l[j] > second) second = l[j];
    k_out[t] = best + 1;
    if (gap) gap[t] = l[best] - second;
    if (logits)
      for (int j = 0; j < S; ++j) logits[t * S + j] = l[j];
  }
}

/*
 * oracle_route_mlp: threshold routing with a two-layer MLP scorer
 * ([ja] §2.2: a 2-layer MLP scores each token; a threshold turns the gate
 * into a binary mask and moving it sets how many slices are active;
 * [en] §2.B "Differentiable Gating" (temperature-scaled sigmoid, a binary
 * mask at inference) and "Dynamic Adjustment" (raising delta activates fewer
 * slices)). Readings where the pages are silent: ReLU hidden layer, one score
 * per residual slice (S - 1 of them), slice j+1 active iff
 * sigmoid(score_j / tau) > delta, and k_t = 1 + the number of active residual
 * slices (the leading k_t slices are the ones summed).
 *   h_i    = max(0, sum_k x[t,k] W1[k,i] + b1[i])          i < H   (fp64)
 *   s_j    = sum_i h_i W2[i,j] + b2[j]                     j < S-1 (fp64)
 *   active = 1 / (1 + exp(-s_j / tau)) > delta
 * margin[t] = min_j |s_j - tau * log(delta / (1 - delta))| (the score's
 * distance from the threshold; +inf when S == 1), scores (fp64 [T][S-1]) may
 * be NULL. Returns -1 for tau <= 0 or delta outside (0, 1).
 */
int oracle_route_mlp(const uint16_t* X, int64_t T, int64_t K, const float* W1, const float* b1, int64_t H,
                     const float* W2, const float* b2, int S, double tau, double delta, int32_t* k_out,
                     double* margin, double* scores, int nthreads) {
  if (!(tau > 0.0) || !(delta > 0.0 && delta < 1.0) || S < 1 || S > 8 || H < 1) return -1;
  const double thr = tau * log(delta / (1.0 - delta));
  set_threads(nthreads);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    double* h = (double*)malloc((size_t)H * sizeof(double));
    for (int64_t i = 0; i < H; ++i) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += bf16_bits_to_double(X[t * K + k]) * (double)W1[k * H + i];
      acc += (double)b1[i];
      h[i] = acc > 0.0 ? acc : 0.0;
    }
    int active = 0;
    double m = INFINITY;
    for (int j = 0; j < S - 1; ++j) {
      double s = 0.0;
      for (int64_t i = 0; i < H; ++i) s += h[i] * (double)W2[i * (S - 1) + j];
      s += (double)b2[j];
      if (1.0 / (1.0 + exp(-s / tau)) > delta) ++active;
      const double d = fabs(s - thr);
      if (d < m) m = d;
      if (scores) scores[t * (S - 1) + j] = s;
    }
    free(h);
    k_out[t] = 1 + active;
    if (margin) margin[t] = m;
  }
  return 0;
}

/*
 * oracle_bucket: stable counting sort of the tokens by k_t ascending.
 * perm[i] = original index of the i-th token; bucket j (k_t = j+1) is
 * perm[offsets[j] .. offsets[j+1]). Returns -1 if a k_t is outside 1..S.
 */
int oracle_bucket(const int32_t* k_t, int64_t T, int S, int32_t* perm, int32_t* offsets) {
  int64_t count[9] = {0};
  for (int64_t t = 0; t < T; ++t) {
    if (k_t[t] < 1 || k_t[t] > S) return -1;
    count[k_t[t] - 1]++;
  }
  int64_t next[9];
  offsets[0] = 0;
  for (int j = 0; j < S; ++j) {
    next[j] = offsets[j];
    offsets[j + 1] = (int32_t)(offsets[j] + count[j]);
  }
  for (int64_t t = 0; t < T; ++t) perm[next[k_t[t] - 1]++] = (int32_t)t;
  return 0;
}

/* ---- mixed-bit GEMM ----------------------------------------------------- */

/*
 * oracle_gemm_slices: for each listed token t = tokens[i] (all tokens when
 * tokens is NULL, i = t), Y[i][n] = sum_k x[t,k] * W^(k_t)[n,k] in fp64, with
 * W^(k) = sum_{s<k} (q - z) * scale built exactly ([ja] §2.1; [en] §2.A) from
 * slices of widths[s]-bit codes. Y is fp64 [n_tokens][N]. The sum over k runs
 * in index order. oracle_gemm_bits has one width for every slice, and
 * oracle_gemm is the 2-bit case.
 */
void oracle_gemm_slices(const uint16_t* X, int64_t T, int64_t K, const int32_t* k_t,
                        const uint32_t* codes, const uint32_t* sz, int64_t N, int G, int S, const int* widths,
                        const int32_t* tokens, int64_t n_tokens, double* Y, int nthreads) {
  (void)T;
  set_threads(nthreads);
  const int64_t ngroups = K / G;
  if (!tokens) n_tokens = T;
#pragma omp parallel for schedule(dynamic, 8)
  for (int64_t n = 0; n < N; ++n) {
    /* the S reconstructions of row n: W^(1), ..., W^(S) */
    double* wk = (double*)malloc(sizeof(double) * (size_t)S * (size_t)K);
    for (int64_t j = 0; j < K; ++j) {
      double acc = 0.0;
      for (int s = 0; s < S; ++s) {
        int q = code_of(codes, N, K, widths, s, n, j);
        uint32_t e = sz[((int64_t)s * ngroups + j / G) * N + n];
        double scale = (double)half_bits_to_float((uint16_t)(e & 0xffffu));
        double zero = (double)half_bits_to_float((uint16_t)(e >> 16));
        acc += ((double)q - zero) * scale;
        wk[(int64_t)s * K + j] = acc;
      }
    }
    for (int64_t i = 0; i < n_tokens; ++i) {
      int64_t t = tokens ? tokens[i] : i;
      const double* w = wk + (int64_t)(k_t[t] - 1) * K;
      double acc = 0.0;
      for (int64_t j = 0; j < K; ++j) acc += bf16_bits_to_double(X[t * K + j]) * w[j];
      Y[i * N + n] = acc;
    }
    free(wk);
  }
}

void oracle_gemm_bits(const uint16_t* X, int64_t T, int64_t K, const int32_t* k_t,
                      const uint32_t* codes, const uint32_t* sz, int64_t N, int G, int S, int bits,
                      const int32_t* tokens, int64_t n_tokens, double* Y, int nthreads) {
  int widths[8];
  if (uniform_widths(widths, S, bits) == 0)
    oracle_gemm_slices(X, T, K, k_t, codes, sz, N, G, S, widths, tokens, n_tokens, Y, nthreads);
}

void oracle_gemm(const uint16_t* X, int64_t T, int64_t K, const int32_t* k_t,
                 const uint32_t* codes, const uint32_t* sz, int64_t N, int G, int S,
                 const int32_t* tokens, int64_t n_tokens, double* Y, int nthreads) {
  oracle_gemm_bits(X, T, K, k_t, codes, sz, N, G, S, 2, tokens, n_tokens, Y, nthreads);
}
