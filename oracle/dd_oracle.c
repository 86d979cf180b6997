/*
 * dd_oracle.c -- the ORACLE for one denoising step of block discrete-diffusion
 * decoding.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg load it; the product library never does.  It
 * shares no code, header, table or constant generator with the CUDA library.
 *
 * Plain, slow, float64.  Every function follows the definition it cites and
 * does nothing clever: no blocking, no fusion, no reordering beyond one
 * OpenMP loop over independent output rows.
 *
 * Sources (web pages on the method):
 *   [DG-mech]  "DiffusionGemma Technical Report" (paperfeed review),
 *              section "The mechanism: an AR model turned inside out":
 *              causal encoder -> KV cache; 256-token canvas refined with full
 *              bidirectional attention inside the canvas while attending to
 *              the cache; multinomial (uniform-token) noise instead of [MASK];
 *              per-position entropies from temperature-scaled logits.
 *   [DG-train] same review, section "Training": every canvas token is
 *              corrupted independently with probability t.
 *   [DG-samp]  same review, section "The mechanism", the paragraph on the
 *              sampler: temperature annealed 0.8 -> 0.4; positions accepted
 *              greedily from lowest to highest entropy until a cumulative
 *              entropy budget (b = 0.1) is exhausted, the rest re-noised to
 *              uniform random tokens; early halt when the mean canvas entropy
 *              is below 0.005 and the prediction is stable across two steps.
 *   [Philox]   Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
 *              as 1, 2, 3", SC'11: the Philox-4x32 bijection, 10 rounds.
 *
 * Readings taken where the pages are silent:
 *   - one softmax over the union [prefix keys || canvas keys], no mask;
 *   - query head h reads kv head h / (Hq / Hkv);
 *   - Gumbel noise g = -ln(-ln U) with U = (2*(x >> 9) + 1) * 2^-24 from a
 *     32-bit Philox word x, counter (v >> 2, row, step, stream), key = seed,
 *     word v & 3; streams 0 Gumbel, 1 re-noise decision, 2 replacement,
 *     3 canvas initialisation (streams 1-3 use counter word 0 = 0, output 0);
 *   - re-noise each position independently when U(stream 1) < rate (fp32);
 *   - replacement token = (x(stream 2) * V) >> 32; canvas init the same with
 *     stream 3 and step 0;
 *   - entropy-budget acceptance: entropies in increasing order, equal values
 *     by increasing position; the running sum is float64, summed in that
 *     order, and a position is accepted while the sum including it stays
 *     <= b, so the accepted set is a prefix of that order;
 *   - the early-halt "argmax prediction" is the sampler's prediction (the
 *     argmax of the Gumbel-perturbed scores); a canvas halts at a step whose
 *     float64 mean entropy is below the threshold and whose predictions all
 *     equal the previous step's.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BF16 0
#define ORACLE_F32 1
#define ORACLE_E4M3 2

/* ---------------------------------------------------------------- Philox */

/* One Philox-4x32 round [Philox]: two 32x32->64 products of words 0 and 2
 * with the round multipliers; the high halves are xor-ed with the other two
 * words and the round key; the words are permuted. */
static void philox_round(uint32_t x[4], const uint32_t k[2]) {
  const uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)x[0];
  const uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)x[2];
  const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
  const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
  const uint32_t y0 = hi1 ^ x[1] ^ k[0];
  const uint32_t y2 = hi0 ^ x[3] ^ k[1];
  x[0] = y0;
  x[1] = lo1;
  x[2] = y2;
  x[3] = lo0;
}

/* Philox4x32-10 [Philox]: ten rounds; the key is bumped by the Weyl
 * constants (golden ratio, sqrt(3)-1) between rounds. */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t x[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
  uint32_t k[2] = {key[0], key[1]};
  for (int r = 0; r < 10; ++r) {
    philox_round(x, k);
    k[0] += 0x9E3779B9u;
    k[1] += 0xBB67AE85u;
  }
  out[0] = x[0]; out[1] = x[1]; out[2] = x[2]; out[3] = x[3];
}

/* The 32-bit word for (stream, step, row, vocab index v). */
uint32_t oracle_word(uint64_t seed, uint32_t stream, uint32_t step, uint32_t row, uint32_t v) {
  const uint32_t ctr[4] = {v >> 2, row, step, stream};
  const uint32_t key[2] = {(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
  uint32_t out[4];
  oracle_philox4x32_10(ctr, key, out);
  return out[v & 3u];
}

/* Uniform in (0,1) from the top 23 bits of a word: an odd multiple of 2^-24,
 * exactly representable in float32 and float64. */
double oracle_uniform(uint32_t x) {
  return (2.0 * (double)(x >> 9) + 1.0) * ldexp(1.0, -24);
}

/* Vectorised helpers for the tests. */
void oracle_words(uint64_t seed, uint32_t stream, uint32_t step, const uint32_t* rows,
                  const uint32_t* vs, int64_t n, uint32_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_word(seed, stream, step, rows[i], vs[i]);
}

void oracle_philox_blocks(const uint32_t* ctrs, const uint32_t* keys, int64_t n, uint32_t* out) {
  for (int64_t i = 0; i < n; ++i) oracle_philox4x32_10(ctrs + 4 * i, keys + 2 * i, out + 4 * i);
}

/* ------------------------------------------------------------ input upcast */

/*
 * The 8-bit E4M3 floating-point format (OCP "8-bit Floating Point
 * Specification (OFP8)", rev. 1.0, the E4M3 encoding): one sign bit, four
 * exponent bits with bias 7, three mantissa bits.  An exponent field of 0
 * encodes the subnormals m * 2^-9; S.1111.111 is NaN; there are no
 * infinities, so the largest finite magnitude is 1.75 * 2^8 = 448.
 */
double oracle_e4m3_value(uint8_t x) {
  const int sign = x >> 7, e = (x >> 3) & 15, m = x & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

/* bf16 -> float64 is exact: the bf16 bits are the top half of a float32.
 * E4M3 -> float64 is exact too (four significant bits). */
static double load_elem(const void* base, int dtype, int64_t idx) {
  if (dtype == ORACLE_BF16) {
    const uint16_t h = ((const uint16_t*)base)[idx];
    const uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
  }
  if (dtype == ORACLE_E4M3) return oracle_e4m3_value(((const uint8_t*)base)[idx]);
  return (double)((const float*)base)[idx];
}

static void set_threads(int n_threads) {
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
}

/* ------------------------------------------------------- canvas attention */

/*
 * Bidirectional canvas attention over the cache [DG-mech]: for batch row b,
 * canvas position i and query head h, the keys are the L_b prefix rows of
 * batch row b followed by the C canvas rows of batch row b, all of kv head
 * g = h / (Hq / Hkv), with no mask:
 *   s_j = scale * <q, k_j>,  p = softmax(s),  O = sum_j p_j v_j,
 *   LSE = max_j s_j + ln sum_j exp(s_j - max s).
 * Layouts: q [B,C,Hq,D]; kc, vc [B,C,Hkv,D]; kp, vp [sum L_b, Hkv, D] packed
 * with cu_prefix[B+1]; out [B,C,Hq,D]; lse [B,Hq,C] (may be NULL).
 * pos_sel (n_pos entries) restricts the canvas positions computed; rows not
 * selected are left untouched.  n_pos < 0 means every position.
 * qkv_scale (NULL = all 1) holds per-tensor factors (q, k, v): the value of
 * an element is its stored value times its tensor's factor (the per-tensor
 * scaling of 8-bit inputs); K's factor covers Kp and Kc, V's Vp and Vc.
 * Returns 0, or -1 on bad arguments.
 */
int oracle_canvas_attn(int B, int C, int Hq, int Hkv, int D, double scale, int dtype,
                       const double* qkv_scale,
                       const void* q, const void* kc, const void* vc, const void* kp,
                       const void* vp, const int32_t* cu_prefix, const int32_t* pos_sel,
                       int n_pos, double* out, double* lse, int n_threads) {
  if (B < 0 || C < 1 || Hq < 1 || Hkv < 1 || D < 1 || Hq % Hkv != 0) return -1;
  for (int b = 0; b < B; ++b)
    if (cu_prefix[b + 1] < cu_prefix[b] || cu_prefix[0] != 0) return -1;
  const int group = Hq / Hkv;
  const double sq = qkv_scale ? qkv_scale[0] : 1.0;
  const double sk = qkv_scale ? qkv_scale[1] : 1.0;
  const double sv = qkv_scale ? qkv_scale[2] : 1.0;
  const int npos = n_pos < 0 ? C : n_pos;
  const int64_t n_rows = (int64_t)B * npos * Hq;
  set_threads(n_threads);

#pragma omp parallel
  {
    int max_keys = 0;
    for (int b = 0; b < B; ++b) {
      const int nk = cu_prefix[b + 1] - cu_prefix[b] + C;
      if (nk > max_keys) max_keys = nk;
    }
    double* s = (double*)malloc(sizeof(double) * (size_t)max_keys);
    double* qv = (double*)malloc(sizeof(double) * (size_t)D);
    double* acc = (double*)malloc(sizeof(double) * (size_t)D);

#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < n_rows; ++r) {
      const int h = (int)(r % Hq);
      const int pi = (int)((r / Hq) % npos);
      const int b = (int)(r / ((int64_t)Hq * npos));
      const int i = n_pos < 0 ? pi : pos_sel[pi];
      const int g = h / group;
      const int L = cu_prefix[b + 1] - cu_prefix[b];
      const int nk = L + C;

      for (int d = 0; d < D; ++d)
        qv[d] = sq * load_elem(q, dtype, (((int64_t)b * C + i) * Hq + h) * D + d);

      /* scores over [prefix || canvas] */
      for (int j = 0; j < nk; ++j) {
        const void* kb;
        int64_t krow;
        if (j < L) { kb = kp; krow = (int64_t)cu_prefix[b] + j; }
        else       { kb = kc; krow = (int64_t)b * C + (j - L); }
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
          dot += qv[d] * (sk * load_elem(kb, dtype, (krow * Hkv + g) * D + d));
        s[j] = scale * dot;
      }
      double m = -INFINITY;
      for (int j = 0; j < nk; ++j) if (s[j] > m) m = s[j];
      double sum = 0.0;
      for (int j = 0; j < nk; ++j) sum += exp(s[j] - m);

      for (int d = 0; d < D; ++d) acc[d] = 0.0;
      for (int j = 0; j < nk; ++j) {
        const double p = exp(s[j] - m) / sum;
        const void* vb;
        int64_t vrow;
        if (j < L) { vb = vp; vrow = (int64_t)cu_prefix[b] + j; }
        else       { vb = vc; vrow = (int64_t)b * C + (j - L); }
        for (int d = 0; d < D; ++d)
          acc[d] += p * (sv * load_elem(vb, dtype, (vrow * Hkv + g) * D + d));
      }
      double* o = out + (((int64_t)b * C + i) * Hq + h) * D;
      for (int d = 0; d < D; ++d) o[d] = acc[d];
      if (lse) lse[((int64_t)b * Hq + h) * C + i] = m + log(sum);
    }
    free(s);
    free(qv);
    free(acc);
  }
  return 0;
}

/* ------------------------------------------------ sampler and re-noising */

/*
 * One sampler step for the rows listed in row_sel (n_sel entries; n_sel < 0:
 * rows 0..rows-1).  Local row r has global row index row_offset + r, which
 * keys the random numbers.  With z_v = logit_v / tau [DG-mech, the sampler
 * paragraph]:
 *   pred     = argmax_v (z_v + g_v), lowest v on an exact tie, with Gumbel
 *              noise g_v from stream 0 (Gumbel-max sampling of softmax(z));
 *   conf     = softmax(z)[pred];
 *   entropy  = -sum_v p_v ln p_v,  p = softmax(z);
 *   renoised = U(stream 1) < rate, compared in float32 [DG-train, DG-mech];
 *   tokens   = renoised ? (x(stream 2) * V) >> 32 : pred  (uniform vocabulary
 *              token, multinomial noise [DG-mech]);
 *   gap      = best score - second best score (for the near-tie rule).
 * logits: [rows, V] with row_stride elements between rows (0 broadcasts one
 * row).  Outputs are indexed by position in row_sel.  Any output may be NULL.
 */
int oracle_sample_renoise(const void* logits, int dtype, int64_t rows, int64_t vocab,
                          int64_t row_stride, const int64_t* row_sel, int64_t n_sel,
                          double tau, float rate, uint64_t seed, uint32_t step,
                          uint32_t row_offset, int32_t* tokens, int32_t* pred, double* conf,
                          double* entropy, uint8_t* renoised, double* gap, double* best,
                          int n_threads) {
  if (rows < 0 || vocab < 1 || !(tau > 0.0)) return -1;
  const int64_t n = n_sel < 0 ? rows : n_sel;
  set_threads(n_threads);

#pragma omp parallel
  {
    double* z = (double*)malloc(sizeof(double) * (size_t)vocab);
#pragma omp for schedule(dynamic, 1)
    for (int64_t k = 0; k < n; ++k) {
      const int64_t r = n_sel < 0 ? k : row_sel[k];
      const uint32_t grow = row_offset + (uint32_t)r;
      for (int64_t v = 0; v < vocab; ++v) z[v] = load_elem(logits, dtype, r * row_stride + v) / tau;

      /* Gumbel-max */
      double s1 = -INFINITY, s2 = -INFINITY;
      int64_t arg = 0;
      for (int64_t v = 0; v < vocab; ++v) {
        const double u = oracle_uniform(oracle_word(seed, 0, step, grow, (uint32_t)v));
        const double g = -log(-log(u));
        const double sc = z[v] + g;
        if (sc > s1) { s2 = s1; s1 = sc; arg = v; }
        else if (sc > s2) { s2 = sc; }
      }

      /* softmax statistics */
      double m = -INFINITY;
      for (int64_t v = 0; v < vocab; ++v) if (z[v] > m) m = z[v];
      double sum = 0.0;
      for (int64_t v = 0; v < vocab; ++v) sum += exp(z[v] - m);
      const double lse = m + log(sum);
      double ent = 0.0;
      for (int64_t v = 0; v < vocab; ++v) {
        const double lp = z[v] - lse;
        const double p = exp(lp);
        if (p > 0.0) ent -= p * lp; /* 0 ln 0 = 0 (entries with logit -inf) */
      }

      /* re-noise */
      const float u1 = (float)oracle_uniform(oracle_word(seed, 1, step, grow, 0));
      const int rn = u1 < rate;
      const uint32_t x2 = oracle_word(seed, 2, step, grow, 0);
      const int32_t repl = (int32_t)(((uint64_t)x2 * (uint64_t)vocab) >> 32);

      if (pred) pred[k] = (int32_t)arg;
      if (conf) conf[k] = exp(z[arg] - lse);
      if (entropy) entropy[k] = ent;
      if (renoised) renoised[k] = (uint8_t)rn;
      if (tokens) tokens[k] = rn ? repl : (int32_t)arg;
      if (gap) gap[k] = s1 - s2;
      if (best) best[k] = s1;
    }
    free(z);
  }
  return 0;
}

/* Canvas initialisation: uniformly random vocabulary tokens [DG-mech]. */
void oracle_init_canvas(int32_t* out, int64_t rows, int64_t vocab, uint64_t seed,
                        uint32_t row_offset) {
  for (int64_t r = 0; r < rows; ++r) {
    const uint32_t x = oracle_word(seed, 3, 0, row_offset + (uint32_t)r, 0);
    out[r] = (int32_t)(((uint64_t)x * (uint64_t)vocab) >> 32);
  }
}

/* ------------------------------------------------ the pages' sampler policy */

typedef struct {
  float h;
  int64_t pos;
} ent_pos;

static int cmp_ent_pos(const void* a, const void* b) {
  const ent_pos* x = (const ent_pos*)a;
  const ent_pos* y = (const ent_pos*)b;
  if (x->h < y->h) return -1;
  if (x->h > y->h) return 1;
  return x->pos < y->pos ? -1 : (x->pos > y->pos ? 1 : 0);
}

/* Entropy-budget acceptance [DG-samp].  For each canvas b of C positions
 * (rows b*C .. b*C+C-1): sort the positions by entropy (ties by position),
 * accept them in that order while the float64 running sum of accepted
 * entropies stays <= budget, stop at the first that would exceed it.
 * Accepted positions keep pred; the others are re-noised to the uniform
 * replacement token x(stream 2) * V >> 32 of their row (as [DG-mech]).
 * entropy is float32, the precision the sampler outputs.  n_accepted[b] is
 * the count and sum_accepted[b] the float64 sum of the accepted entropies. */
void oracle_entropy_accept(const float* entropy, const int32_t* pred, int64_t B, int64_t C,
                           double budget, uint64_t seed, uint32_t step, uint32_t row_offset,
                           int64_t vocab, int32_t* tokens, uint8_t* accepted,
                           int32_t* n_accepted, double* sum_accepted) {
  ent_pos* order = (ent_pos*)malloc(sizeof(ent_pos) * (size_t)(C > 0 ? C : 1));
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t i = 0; i < C; ++i) {
      order[i].h = entropy[b * C + i];
      order[i].pos = i;
    }
    qsort(order, (size_t)C, sizeof(ent_pos), cmp_ent_pos);
    for (int64_t i = 0; i < C; ++i) accepted[b * C + i] = 0;
    double sum = 0.0;
    int64_t k = 0;
    for (; k < C; ++k) {
      const double next = sum + (double)order[k].h;
      if (!(next <= budget)) break;
      sum = next;
      accepted[b * C + order[k].pos] = 1;
    }
    if (n_accepted) n_accepted[b] = (int32_t)k;
    if (sum_accepted) sum_accepted[b] = sum;
    for (int64_t i = 0; i < C; ++i) {
      const int64_t r = b * C + i;
      const uint32_t x2 = oracle_word(seed, 2, step, row_offset + (uint32_t)r, 0);
      const int32_t repl = (int32_t)(((uint64_t)x2 * (uint64_t)vocab) >> 32);
      tokens[r] = accepted[r] ? pred[r] : repl;
    }
  }
  free(order);
}

/* Early-halt test [DG-samp]: done[b] = 1 when the float64 mean of canvas b's
 * entropies is below `threshold` and pred equals pred_prev at every position
 * (pred_prev NULL: no previous step, never done). */
void oracle_stop_check(const float* entropy, const int32_t* pred, const int32_t* pred_prev,
                       int64_t B, int64_t C, double threshold, uint8_t* done) {
  for (int64_t b = 0; b < B; ++b) {
    double sum = 0.0;
    int same = pred_prev != NULL;
    for (int64_t i = 0; i < C; ++i) {
      sum += (double)entropy[b * C + i];
      if (pred_prev && pred[b * C + i] != pred_prev[b * C + i]) same = 0;
    }
    done[b] = (uint8_t)(same && sum / (double)C < threshold);
  }
}
