/*
 * Plain fp64 CPU oracle for gpt-oss-style causal grouped-query attention with
 * learned sinks. TEST INFRASTRUCTURE ONLY: the tests, the package's smoke check
 * and the bench's CPU-baseline leg call it; the product path never does.
 *
 * What it computes is the plain definition, written out loop by loop:
 *
 *   q' = R(pos_i) q[b,i,h],  k'_j = R(pos_j) k[b,j,g],  g = floor(h / 8)
 *   s_j = (q' . k'_j) / sqrt(64)                       for visible keys j
 *   p_j = exp(s_j) / (exp(sigma_h) + sum_j' exp(s_j'))
 *   out[b,i,h,:] = sum_j p_j v[b,j,g,:]
 *
 * Sources (the gpt-oss pages):
 *  - grouped-query attention, 64 query heads over 8 key/value heads, grouping
 *    by num_attention_heads // num_key_value_heads: inteligile "gpt-oss-120b"
 *    techniques map, row "Grouped-query attention"; llm-atlas gpt-oss-20b
 *    field table (num_attention_heads, num_key_value_heads, head_dim).
 *  - half-split rotary embedding (first half * cos - second half * sin;
 *    second half * cos + first half * sin), on every layer, to q and k:
 *    techniques map rows "Partial RoPE" and "Layers without positional
 *    encoding (NoPE)"; rope_theta = 150000 from the llm-atlas field table.
 *  - learned per-head sink logit concatenated as an extra column of the
 *    scaled, masked scores before the softmax; its probability is dropped:
 *    techniques map row "Learnable attention sink".
 *  - causal mask on full layers, a 128-token sliding-window causal mask on
 *    sliding layers: techniques map rows "Sliding-window attention" and
 *    "Interleaved sliding-window and global attention"; sliding_window = 128
 *    in the llm-atlas field tables.
 *
 * Readings where the pages are silent: the scale is 1/sqrt(64); the sink is
 * not scaled; the rotation frequency of pair k (elements k and k+32) is
 * theta^(-2k/64); a window W > 0 makes key j visible to query i iff
 * i - W < j <= i (W keys including the query itself); W <= 0 means full
 * causal; masking is by token index, positions feed only the rotation.
 * Decode: the query sits at position len-1 and is rotated there, the cache
 * already holds rotated keys, the visible keys are max(0, len-W) <= j < len;
 * len = 0 gives a zero output.
 *
 * YaRN variant (rope = 1): the techniques map row "YaRN RoPE scaling" gives
 * rope_type yarn with factor 32 and "beta parameters" applied through the
 * transformers rope-initialisation functions; initial_context_length = 4096 is
 * in the llm-atlas field tables. The pages omit the betas, the attention
 * factor and the ramp's form. Reading taken: the transformers yarn
 * initialisation with beta_fast = 32, beta_slow = 1 (its defaults, and the
 * values of the published gpt-oss rope_scaling block, which also turns
 * truncation of the correction range off), attention factor 0.1 ln(s) + 1
 * (YaRN paper, Peng et al. 2023, section 3.4) multiplying cos and sin, i.e.
 * both rotated q and k. Pair k blends the original frequency theta_k with
 * theta_k / s by a ramp that is linear in the pair index between the pairs
 * whose wavelength fits beta_fast and beta_slow times into the original
 * context: 0 (original) below, 1 (interpolated) above.
 *
 * Exponentials subtract the maximum over the row's logits, the sink included,
 * which leaves every value unchanged. No blocking, no online rescaling.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define NQ 64
#define NKV 8
#define GROUP (NQ / NKV)
#define D 64
#define HALF (D / 2)
#define ROPE_THETA 150000.0
#define TWO_PI 6.283185307179586476925286766559
#define YARN_FACTOR 32.0
#define YARN_ORIGINAL_CONTEXT 4096.0
#define YARN_BETA_FAST 32.0
#define YARN_BETA_SLOW 1.0

int oracle_abi(void) { return 1; }

/* Rotation angle frequency of pair k: theta^(-2k/d). */
static double inv_freq(int k) { return pow(ROPE_THETA, -2.0 * (double)k / (double)D); }

/* y = scale * R x for one head vector of 64 elements (half-split pairing):
 * pair k = (element k, element k+32) turns by the angle p * freq[k]. */
static void rotate_by(const double* x, double p, const double* freq, double scale, double* y) {
  for (int k = 0; k < HALF; ++k) {
    double a = p * freq[k];
    double c = cos(a) * scale, s = sin(a) * scale;
    double x1 = x[k], x2 = x[k + HALF];
    y[k] = x1 * c - x2 * s;
    y[k + HALF] = x2 * c + x1 * s;
  }
}

/* y = R(p) x for one head vector of 64 elements (plain RoPE). */
void oracle_rope(const double* x, double p, double* y) {
  double f[HALF];
  for (int k = 0; k < HALF; ++k) f[k] = inv_freq(k);
  rotate_by(x, p, f, 1.0, y);
}

/* Fractional pair index whose wavelength 2 pi / theta_k fits `turns` times
 * into the original context: solves original * theta_k / (2 pi) = turns. */
static double yarn_pair_for_turns(double turns, double original) {
  return (double)D * log(original / (turns * TWO_PI)) / (2.0 * log(ROPE_THETA));
}

/* y = YaRN-scaled R(p) x: frequencies blended between theta_k (ramp 0) and
 * theta_k / factor (ramp 1), result scaled by the attention factor. */
void oracle_rope_yarn(const double* x, double p, double factor, double original,
                      double beta_fast, double beta_slow, double* y) {
  double lo = yarn_pair_for_turns(beta_fast, original);
  double hi = yarn_pair_for_turns(beta_slow, original);
  if (lo < 0.0) lo = 0.0;
  if (hi > (double)(D - 1)) hi = (double)(D - 1);
  if (hi == lo) hi += 0.001;
  const double mscale = factor <= 1.0 ? 1.0 : 0.1 * log(factor) + 1.0;
  double f[HALF];
  for (int k = 0; k < HALF; ++k) {
    double ramp = ((double)k - lo) / (hi - lo);
    if (ramp < 0.0) ramp = 0.0;
    if (ramp > 1.0) ramp = 1.0;
    f[k] = inv_freq(k) / factor * ramp + inv_freq(k) * (1.0 - ramp);
  }
  rotate_by(x, p, f, mscale, y);
}

/* The rotation a call uses: rope 0 plain, 1 YaRN with the gpt-oss constants. */
static void rotate(const double* x, double p, int rope, double* y) {
  if (rope)
    oracle_rope_yarn(x, p, YARN_FACTOR, YARN_ORIGINAL_CONTEXT, YARN_BETA_FAST, YARN_BETA_SLOW, y);
  else
    oracle_rope(x, p, y);
}

/* Rotate n head vectors stored contiguously (n x 64), one position each. */
void oracle_rope_rows(const double* x, const double* pos, int64_t n, int rope, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n; ++r) rotate(x + r * D, pos[r], rope, y + r * D);
}

/*
 * Attention output of one query row of one head, over keys [lo, hi] of one
 * sequence. kr: rotated keys of this sequence and KV head, laid out
 * [S][64]; v: values, laid out with row stride vstride (elements).
 * s: caller-provided scratch of at least hi-lo+1 doubles.
 */
static void attend_row(const double* qr, const double* kr, const double* v, int64_t vstride,
                       int64_t lo, int64_t hi, double sink, double* s, double* out) {
  const double scale = 1.0 / sqrt((double)D);
  double m = sink;
  for (int64_t j = lo; j <= hi; ++j) {
    double dot = 0.0;
    for (int e = 0; e < D; ++e) dot += qr[e] * kr[j * D + e];
    s[j - lo] = dot * scale;
    if (s[j - lo] > m) m = s[j - lo];
  }
  double acc[D];
  for (int e = 0; e < D; ++e) acc[e] = 0.0;
  /* sigma = -inf: the sink contributes nothing and m is the largest score */
  double den = isinf(sink) && sink < 0 ? 0.0 : exp(sink - m);
  for (int64_t j = lo; j <= hi; ++j) {
    double w = exp(s[j - lo] - m);
    den += w;
    for (int e = 0; e < D; ++e) acc[e] += w * v[j * vstride + e];
  }
  for (int e = 0; e < D; ++e) out[e] = den > 0.0 ? acc[e] / den : 0.0;
}

/*
 * Prefill oracle on selected query rows.
 *   q_rows [nrows][64][64]: the query vectors of the selected rows
 *   k, v [B][S][8][64], sinks [64], pos [B][S] (fp64 values)
 *   window: <= 0 full causal, else W; rope: 0 plain, 1 YaRN
 *   rows: nrows pairs (b, i) of query rows to compute; out [nrows][64][64]
 * Every head of each selected row is computed.
 */
void oracle_prefill_rows(const double* q_rows, const double* k, const double* v, const double* sinks,
                         const double* pos, int B, int S, int window, int rope,
                         const int64_t* rows, int64_t nrows, double* out) {
  double* kr = (double*)malloc((size_t)S * D * sizeof(double));
  for (int b = 0; b < B; ++b) {
    int any = 0;
    for (int64_t r = 0; r < nrows; ++r) any |= (rows[2 * r] == b);
    if (!any) continue;
    for (int g = 0; g < NKV; ++g) {
      /* rotated keys of sequence b, KV head g */
#pragma omp parallel for schedule(static)
      for (int64_t j = 0; j < S; ++j)
        rotate(k + (((int64_t)b * S + j) * NKV + g) * D, pos[(int64_t)b * S + j], rope, kr + j * D);
      const double* vg = v + ((int64_t)b * S * NKV + g) * D;
#pragma omp parallel
      {
        double* s = (double*)malloc((size_t)S * sizeof(double));
        double qr[D];
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
          if (rows[2 * r] != b) continue;
          int64_t i = rows[2 * r + 1];
          int64_t lo = window > 0 ? (i - window + 1 > 0 ? i - window + 1 : 0) : 0;
          for (int hh = 0; hh < GROUP; ++hh) {
            int h = g * GROUP + hh;
            rotate(q_rows + (r * NQ + h) * D, pos[(int64_t)b * S + i], rope, qr);
            attend_row(qr, kr, vg, (int64_t)NKV * D, lo, i, sinks[h], s, out + (r * NQ + h) * D);
          }
        }
        free(s);
      }
    }
  }
  free(kr);
}

/* Prefill oracle on every query row: out [B][S][64][64]. Row r = b*S + i of q
 * is query row (b, i), so q serves directly as the row list. */
void oracle_prefill(const double* q, const double* k, const double* v, const double* sinks,
                    const double* pos, int B, int S, int window, int rope, double* out) {
  int64_t n = (int64_t)B * S;
  int64_t* rows = (int64_t*)malloc((size_t)n * 2 * sizeof(int64_t));
  for (int64_t r = 0; r < n; ++r) {
    rows[2 * r] = r / S;
    rows[2 * r + 1] = r % S;
  }
  oracle_prefill_rows(q, k, v, sinks, pos, B, S, window, rope, rows, n, out);
  free(rows);
}

/*
 * Decode oracle: one new query token per sequence.
 *   q [B][64][64] un-rotated, rotated here at position len[b]-1
 *   kcache, vcache [B][max_len][8][64]; kcache rows are already rotated
 *   len [B]; visible keys max(0, len-W) <= j < len (all j < len if W <= 0)
 *   rope: 0 plain, 1 YaRN (the cache holds keys rotated the same way)
 *   out [B][64][64]
 */
void oracle_decode(const double* q, const double* kcache, const double* vcache,
                   const double* sinks, const int64_t* len, int B, int max_len, int window,
                   int rope, double* out) {
#pragma omp parallel
  {
    double* s = (double*)malloc((size_t)(max_len > 0 ? max_len : 1) * sizeof(double));
    double* kr = (double*)malloc((size_t)(max_len > 0 ? max_len : 1) * D * sizeof(double));
    double qr[D];
#pragma omp for schedule(dynamic, 1)
    for (int64_t bg = 0; bg < (int64_t)B * NKV; ++bg) {
      int b = (int)(bg / NKV), g = (int)(bg % NKV);
      int64_t L = len[b];
      int64_t lo = window > 0 ? (L - window > 0 ? L - window : 0) : 0;
      /* the cache rows of this sequence and KV head, gathered to [L][64] */
      for (int64_t j = lo; j < L; ++j)
        memcpy(kr + j * D, kcache + (((int64_t)b * max_len + j) * NKV + g) * D, D * sizeof(double));
      const double* vg = vcache + ((int64_t)b * max_len * NKV + g) * D;
      for (int hh = 0; hh < GROUP; ++hh) {
        int h = g * GROUP + hh;
        double* o = out + ((int64_t)b * NQ + h) * D;
        if (L <= 0) {
          for (int e = 0; e < D; ++e) o[e] = 0.0;
          continue;
        }
        rotate(q + ((int64_t)b * NQ + h) * D, (double)(L - 1), rope, qr);
        attend_row(qr, kr, vg, (int64_t)NKV * D, lo, L - 1, sinks[h], s, o);
      }
    }
    free(s);
    free(kr);
  }
}
