/*
 * CommVQ CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, single-threaded C that states what the CommVQ hot path computes.
 * (The Python face may run several calls at once on disjoint rows or heads; each call
 * is the same single-threaded code.)
 * Only the tests, the smoke check and the bench's CPU-baseline leg may load it;
 * the library's product path never does. It shares no code, header, table or
 * constant with the CUDA library.
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared (no fast-math), so every float
 * operation below is exactly the IEEE operation written.
 *
 * Sources (CommVQ: Commutative Vector Quantization for KV Cache Compression):
 *  - abstract: additive quantization decoded by a matrix multiply; a codebook that
 *    commutes with RoPE; EM fitting.
 *  - machine review, "What carries the argument": 2x2 key codebook blocks
 *    [[x, y], [-y, x]] commute with the RoPE rotation R_m (Property 1, Eq. 7/8);
 *    g consecutive scalars share one index; R residual rounds; R*log2(Nc')/g bits
 *    per scalar (Eq. 21); the codebook is fit by EM (Algorithm 1, Eq. 20).
 *  - machine review, "If this is right": softmax weights multiply the value codes
 *    before the codebook multiply.
 *  - machine review, "Assumptions & free parameters" and referee minor comment 4: the
 *    paper's own value code is a bit vector s in {0,1}^Nc over a codebook of Nc rows
 *    (Nc / d bits per scalar), decoded as s^T C (oracle_decode_bits).
 * Readings where the pages are silent (each is listed in the design notes):
 *  - a stored key pair (a, b) is the reconstructed 2-vector; its block is
 *    [[a, -b], [b, a]] (the pages' form with x = a, y = -b), so every stored pair
 *    commutes with R_m and the M-step is a plain mean;
 *  - RoPE pairs are interleaved channels (2p, 2p+1), theta_p = base^(-2p/d), keys sit
 *    at positions 0..T_b-1 of their own sequence, the query is already rotated;
 *  - scale 1/sqrt(d), no mask;
 *  - encoding is greedy residual nearest-codeword (the learned encoder needs trained
 *    weights); distances are fp32 with one subtract and one fused multiply-add per
 *    scalar in index order, ties go to the lowest index.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEM 2

static int valid_shape(int d, int g, int R, int n_codes) {
  return d > 0 && g > 0 && (d % g) == 0 && (g % 2) == 0 && R >= 1 && n_codes >= 1;
}

/* Nearest entry of one (round, group) sub-codebook to the residual sub-vector res[0..g).
 * Distances: e = res_k - c_k (fp32), dist = fmaf(e, e, dist), k = 0..g-1 in order.
 * Scan c = 0..Nc'-1, keep the first strict minimum (ties -> lowest index).
 * Also returns the two smallest distances seen (d1 <= d2), used for near-tie counts. */
static int32_t nearest(const float* res, const float* sub_cb, int g, int n_codes,
                       float* d1_out, float* d2_out) {
  float best = INFINITY, second = INFINITY;
  int32_t idx = 0;
  for (int c = 0; c < n_codes; ++c) {
    const float* e_c = sub_cb + (int64_t)c * g;
    float dist = 0.0f;
    for (int k = 0; k < g; ++k) {
      float e = res[k] - e_c[k];
      dist = fmaf(e, e, dist);
    }
    if (dist < best) {
      second = best;
      best = dist;
      idx = c;
    } else if (dist < second) {
      second = dist;
    }
  }
  *d1_out = best;
  *d2_out = second;
  return idx;
}

/* A near tie: at least two entries and (d2 - d1) <= 1e-5 * d2, evaluated in fp32. */
static int is_near_tie(float d1, float d2, int n_codes) {
  if (n_codes < 2) return 0;
  float gap = d2 - d1;
  float lim = 1e-5f * d2;
  return gap <= lim;
}

/* Residual additive encoder (the abstract's additive quantization; R rounds and
 * index sharing as in "What carries the argument").
 * x        [n_rows, d] fp32 (pre-RoPE keys or values, widened exactly from storage)
 * cb       [R, d/g, Nc', g] fp32
 * codes    [n_rows, R, d/g] int32 out
 * res_out  [n_rows, d] fp32 out, residual after the last round (nullable)
 * near_ties  out, number of (row, round, group) decisions that were near ties (nullable) */
int oracle_encode(const float* x, int64_t n_rows, int d, int g, int R, int n_codes,
                  const float* cb, int32_t* codes, float* res_out, int64_t* near_ties) {
  if (!valid_shape(d, g, R, n_codes) || n_rows < 0 || !x || !cb || !codes) return ORACLE_BAD_ARG;
  const int G = d / g;
  int64_t ties = 0;
  float* res = (float*)malloc(sizeof(float) * (size_t)g);
  if (!res) return ORACLE_NO_MEM;
  for (int64_t n = 0; n < n_rows; ++n) {
    for (int j = 0; j < G; ++j) {
      for (int k = 0; k < g; ++k) res[k] = x[n * d + (int64_t)j * g + k];
      for (int r = 0; r < R; ++r) {
        const float* sub_cb = cb + ((int64_t)r * G + j) * n_codes * g;
        float d1, d2;
        int32_t c = nearest(res, sub_cb, g, n_codes, &d1, &d2);
        ties += is_near_tie(d1, d2, n_codes);
        codes[(n * R + r) * G + j] = c;
        for (int k = 0; k < g; ++k) res[k] = res[k] - sub_cb[(int64_t)c * g + k];
      }
      if (res_out)
        for (int k = 0; k < g; ++k) res_out[n * d + (int64_t)j * g + k] = res[k];
    }
  }
  free(res);
  if (near_ties) *near_ties = ties;
  return ORACLE_OK;
}

/* Decoding is a sum of the selected codewords (the abstract's "simple matrix
 * multiplication" with one-hot codes), in fp64.
 * codes [n_rows, R, d/g] int32, cb [R, d/g, Nc', g] fp32 -> out [n_rows, d] fp64. */
int oracle_decode(const int32_t* codes, int64_t n_rows, int d, int g, int R, int n_codes,
                  const float* cb, double* out) {
  if (!valid_shape(d, g, R, n_codes) || n_rows < 0 || !codes || !cb || !out) return ORACLE_BAD_ARG;
  const int G = d / g;
  for (int64_t n = 0; n < n_rows; ++n)
    for (int j = 0; j < G; ++j)
      for (int k = 0; k < g; ++k) {
        double s = 0.0;
        for (int r = 0; r < R; ++r) {
          int32_t c = codes[(n * R + r) * G + j];
          if (c < 0 || c >= n_codes) return ORACLE_BAD_ARG;
          s += (double)cb[(((int64_t)r * G + j) * n_codes + c) * g + k];
        }
        out[n * d + (int64_t)j * g + k] = s;
      }
  return ORACLE_OK;
}

/* RoPE angle of pair p at position m: m * base^(-2p/d), fp64. */
static double rope_angle(int64_t m, int p, int d, double base) {
  double theta = pow(base, -2.0 * (double)p / (double)d);
  return (double)m * theta;
}

/* Plain attention scores of one query against T decompressed keys:
 * k~_t = R_{m=t} k^_t (pair p rotated by angle t*theta_p), s_t = q . k~_t / sqrt(d).
 * q [d] fp64; keys [T] rows of d fp64 with row stride key_stride; scores [T] out. */
int oracle_scores_plain(const double* q, const double* keys, int64_t key_stride, int64_t T,
                        int d, double base, double* scores) {
  if (d <= 0 || (d % 2) || T < 0 || !q || (T > 0 && (!keys || !scores))) return ORACLE_BAD_ARG;
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
  for (int64_t t = 0; t < T; ++t) {
    const double* k = keys + t * key_stride;
    double s = 0.0;
    for (int p = 0; p < d / 2; ++p) {
      double phi = rope_angle(t, p, d, base);
      double c = cos(phi), sn = sin(phi);
      double a = k[2 * p], b = k[2 * p + 1];
      double kr0 = a * c - b * sn;   /* R_m = [[cos, -sin], [sin, cos]] */
      double kr1 = a * sn + b * c;
      s += q[2 * p] * kr0 + q[2 * p + 1] * kr1;
    }
    scores[t] = s * inv_sqrt_d;
  }
  return ORACLE_OK;
}

/* RoPE applied to whole rows: out[n] = R_{pos[n]} x[n], pair p rotated by angle pos[n]*theta_p
 * in fp64 with R = [[cos, -sin], [sin, cos]] (the rotation of oracle_scores_plain, written out as
 * rows: this is what a decompress-then-attend implementation stores as its key cache).
 * x, out [n, d] fp64 (may alias); pos [n] int64, any sign (a negative position undoes one). */
int oracle_rope(const double* x, const int64_t* pos, int64_t n, int d, double base, double* out) {
  if (d <= 0 || (d % 2) || n < 0 || (n > 0 && (!x || !pos || !out))) return ORACLE_BAD_ARG;
  for (int64_t r = 0; r < n; ++r)
    for (int p = 0; p < d / 2; ++p) {
      const double phi = rope_angle(pos[r], p, d, base);
      const double c = cos(phi), sn = sin(phi);
      const double a = x[r * d + 2 * p], b = x[r * d + 2 * p + 1];
      out[r * d + 2 * p] = a * c - b * sn;
      out[r * d + 2 * p + 1] = a * sn + b * c;
    }
  return ORACLE_OK;
}

/* Scores through the query x codebook table ("What carries the argument": the
 * query-dependent and codebook-dependent factors are formed once and reused for
 * every cached position; the rotation is applied afterwards by commutation).
 * For pair p in group j (p = j*g/2 + i) and entry c of round r with stored pair (a, b):
 *   table[r][j][c][i] = conj(q_p) * (a + i b) = (q0 a + q1 b) + i (q0 b - q1 a),
 *   s_t = (1/sqrt d) * sum_p Re( e^{i t theta_p} * sum_r table[r][j][code[t][r][j]][i] ).
 * q [d] fp64, codes [T, R, d/g] int32 for one kv head with row stride code_stride
 * (in int32 elements), cb [R, d/g, Nc', g] fp32 -> scores [T] fp64. */
int oracle_scores_table(const double* q, const int32_t* codes, int64_t code_stride, int64_t T,
                        int d, int g, int R, int n_codes, const float* cb, double base,
                        double* scores) {
  if (!valid_shape(d, g, R, n_codes) || T < 0 || !q || !cb || (T > 0 && (!codes || !scores)))
    return ORACLE_BAD_ARG;
  const int G = d / g, P = g / 2;
  const int64_t n_entries = (int64_t)R * G * n_codes * P;
  double* tab = (double*)malloc(sizeof(double) * 2 * (size_t)n_entries);
  if (!tab) return ORACLE_NO_MEM;
  for (int r = 0; r < R; ++r)
    for (int j = 0; j < G; ++j)
      for (int c = 0; c < n_codes; ++c)
        for (int i = 0; i < P; ++i) {
          int p = j * P + i;
          double q0 = q[2 * p], q1 = q[2 * p + 1];
          const float* e = cb + (((int64_t)r * G + j) * n_codes + c) * g + 2 * i;
          double a = (double)e[0], b = (double)e[1];
          int64_t at = (((int64_t)r * G + j) * n_codes + c) * P + i;
          tab[2 * at] = q0 * a + q1 * b;
          tab[2 * at + 1] = q0 * b - q1 * a;
        }
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
  for (int64_t t = 0; t < T; ++t) {
    const int32_t* ct = codes + t * code_stride;
    double s = 0.0;
    for (int j = 0; j < G; ++j)
      for (int i = 0; i < P; ++i) {
        double U = 0.0, W = 0.0;
        for (int r = 0; r < R; ++r) {
          int32_t c = ct[r * G + j];
          if (c < 0 || c >= n_codes) { free(tab); return ORACLE_BAD_ARG; }
          int64_t at = (((int64_t)r * G + j) * n_codes + c) * P + i;
          U += tab[2 * at];
          W += tab[2 * at + 1];
        }
        double phi = rope_angle(t, j * P + i, d, base);
        s += U * cos(phi) - W * sin(phi);  /* Re((U + iW)(cos + i sin)) */
      }
    scores[t] = s * inv_sqrt_d;
  }
  free(tab);
  return ORACLE_OK;
}

/* Decode-step attention, the plain definition on the decompressed cache, in fp64.
 * q     [B, Hq, d] fp64 (post-RoPE decode queries, exact values of their storage type)
 * khat  [total_T, Hkv, d] fp64 pre-RoPE decoded keys; vhat likewise for values
 * offsets [B+1] int64: sequence b owns rows offsets[b]..offsets[b+1]-1, positions 0..T_b-1
 * Query head h reads kv head h / (Hq / Hkv).
 * out   [B, Hq, d] fp64 = sum_t softmax(s)_t v^_t ; lse [B, Hq] = log sum_t e^{s_t}
 * (nullable). An empty sequence gives out = 0 and lse = -inf. */
int oracle_attend(const double* q, const double* khat, const double* vhat, const int64_t* offsets,
                  int B, int Hq, int Hkv, int d, double base, double* out, double* lse) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) || d <= 0 || (d % 2) || !offsets || !out)
    return ORACLE_BAD_ARG;
  const int group = Hq / Hkv;
  for (int b = 0; b < B; ++b) {
    const int64_t t0 = offsets[b], T = offsets[b + 1] - offsets[b];
    if (T < 0) return ORACLE_BAD_ARG;
    double* s = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    if (!s) return ORACLE_NO_MEM;
    for (int h = 0; h < Hq; ++h) {
      const int kvh = h / group;
      const double* qh = q + ((int64_t)b * Hq + h) * d;
      double* o = out + ((int64_t)b * Hq + h) * d;
      for (int i = 0; i < d; ++i) o[i] = 0.0;
      if (T == 0) {
        if (lse) lse[(int64_t)b * Hq + h] = -INFINITY;
        continue;
      }
      int rc = oracle_scores_plain(qh, khat + (t0 * Hkv + kvh) * d, (int64_t)Hkv * d, T, d,
                                   base, s);
      if (rc) { free(s); return rc; }
      double M = -INFINITY;
      for (int64_t t = 0; t < T; ++t) M = s[t] > M ? s[t] : M;
      double Z = 0.0;
      for (int64_t t = 0; t < T; ++t) Z += exp(s[t] - M);
      for (int64_t t = 0; t < T; ++t) {
        const double p = exp(s[t] - M) / Z;
        const double* v = vhat + ((t0 + t) * Hkv + kvh) * d;
        for (int i = 0; i < d; ++i) o[i] += p * v[i];
      }
      if (lse) lse[(int64_t)b * Hq + h] = M + log(Z);
    }
    free(s);
  }
  return ORACLE_OK;
}

/* The paper's binary value code (review, "Assumptions & free parameters": value codebook of
 * Nc rows over the whole KV dimension, Nc/d bits per scalar): position t stores bits
 * s_t in {0,1}^Nc and decodes to v_t = sum_n s_{t,n} C[n, :], the row of all KV heads.
 * bits [T, Nc/8] uint8, bit n of a row = byte n/8, bit n%8 (little-endian);
 * C [Nc, dkv] fp32; out [T, dkv] fp64. Sums in fp64 in index order. */
int oracle_decode_bits(const uint8_t* bits, int64_t T, int Nc, const float* C, int dkv, double* out) {
  if (T < 0 || Nc <= 0 || (Nc % 8) || dkv <= 0 || (T > 0 && (!bits || !C || !out))) return ORACLE_BAD_ARG;
  for (int64_t t = 0; t < T; ++t) {
    double* o = out + t * dkv;
    for (int i = 0; i < dkv; ++i) o[i] = 0.0;
    const uint8_t* row = bits + t * (Nc / 8);
    for (int n = 0; n < Nc; ++n) {
      if (!((row[n >> 3] >> (n & 7)) & 1)) continue;
      const float* c = C + (int64_t)n * dkv;
      for (int i = 0; i < dkv; ++i) o[i] += (double)c[i];
    }
  }
  return ORACLE_OK;
}

/* Dense decode attention over keys that already carry their rotation (the second half of a
 * decompress-then-attend implementation): s_t = q . k_t / sqrt(d), out = softmax(s) . v,
 * lse = log sum e^{s_t}; shapes, GQA mapping, offsets and the empty case as oracle_attend. */
int oracle_attend_dense(const double* q, const double* k, const double* v, const int64_t* offsets,
                        int B, int Hq, int Hkv, int d, double* out, double* lse) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) || d <= 0 || !offsets || !out) return ORACLE_BAD_ARG;
  const int group = Hq / Hkv;
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
  for (int b = 0; b < B; ++b) {
    const int64_t t0 = offsets[b], T = offsets[b + 1] - offsets[b];
    if (T < 0) return ORACLE_BAD_ARG;
    double* s = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    if (!s) return ORACLE_NO_MEM;
    for (int h = 0; h < Hq; ++h) {
      const int kvh = h / group;
      const double* qh = q + ((int64_t)b * Hq + h) * d;
      double* o = out + ((int64_t)b * Hq + h) * d;
      for (int i = 0; i < d; ++i) o[i] = 0.0;
      if (T == 0) {
        if (lse) lse[(int64_t)b * Hq + h] = -INFINITY;
        continue;
      }
      double M = -INFINITY;
      for (int64_t t = 0; t < T; ++t) {
        const double* kt = k + ((t0 + t) * Hkv + kvh) * d;
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += qh[i] * kt[i];
        s[t] = acc * inv_sqrt_d;
        M = s[t] > M ? s[t] : M;
      }
      double Z = 0.0;
      for (int64_t t = 0; t < T; ++t) Z += exp(s[t] - M);
      for (int64_t t = 0; t < T; ++t) {
        const double p = exp(s[t] - M) / Z;
        const double* vt = v + ((t0 + t) * Hkv + kvh) * d;
        for (int i = 0; i < d; ++i) o[i] += p * vt[i];
      }
      if (lse) lse[(int64_t)b * Hq + h] = M + log(Z);
    }
    free(s);
  }
  return ORACLE_OK;
}

/* One EM step of one residual round's codebook (Algorithm 1 / Eq. 20 as the review
 * describes it: hard assignment, then the closed-form centroid update).
 * rows     [N, d] fp32 residual rows of this round
 * cb       [d/g, Nc', g] fp32, read as the current codebook and overwritten
 * codes_out [N, d/g] int32 assignments against the input codebook (nullable)
 * sse_out  sum over (row, group) of the assignment distance, accumulated in fp64
 *          in (row, group) order (nullable)
 * Update: entry = (float)(sum of assigned fp32 sub-vectors in fp64 / count); an entry
 * with no rows keeps its value. Every stored pair commutes with RoPE, so the key
 * codebook's commuting-block form needs no projection. */
int oracle_em_step(const float* rows, int64_t N, int d, int g, int n_codes, float* cb,
                   int32_t* codes_out, double* sse_out) {
  if (!valid_shape(d, g, 1, n_codes) || N < 0 || !rows || !cb) return ORACLE_BAD_ARG;
  const int G = d / g;
  double* sum = (double*)calloc((size_t)G * n_codes * g, sizeof(double));
  int64_t* cnt = (int64_t*)calloc((size_t)G * n_codes, sizeof(int64_t));
  if (!sum || !cnt) { free(sum); free(cnt); return ORACLE_NO_MEM; }
  double sse = 0.0;
  for (int64_t n = 0; n < N; ++n)
    for (int j = 0; j < G; ++j) {
      const float* x = rows + n * d + (int64_t)j * g;
      float d1, d2;
      int32_t c = nearest(x, cb + (int64_t)j * n_codes * g, g, n_codes, &d1, &d2);
      if (codes_out) codes_out[n * G + j] = c;
      sse += (double)d1;
      cnt[(int64_t)j * n_codes + c] += 1;
      for (int k = 0; k < g; ++k) sum[((int64_t)j * n_codes + c) * g + k] += (double)x[k];
    }
  for (int j = 0; j < G; ++j)
    for (int c = 0; c < n_codes; ++c) {
      int64_t m = cnt[(int64_t)j * n_codes + c];
      if (m == 0) continue;
      for (int k = 0; k < g; ++k) {
        int64_t at = ((int64_t)j * n_codes + c) * g + k;
        cb[at] = (float)(sum[at] / (double)m);
      }
    }
  free(sum);
  free(cnt);
  if (sse_out) *sse_out = sse;
  return ORACLE_OK;
}

/* The M-step of oracle_em_step on given assignments (Algorithm 1 / Eq. 20's closed-form
 * update): entry (j, c) becomes (float)(S / m), S the fp64 sum of the m fp32 sub-vectors
 * assigned to it, summed in (row, group) order; an entry with m = 0 keeps its value.
 * codes [N, d/g] int32 in [0, Nc'). With the assignments oracle_em_step makes (the encoder's
 * rule against the same codebook) the result is oracle_em_step's, bit for bit: the same sums
 * in the same order. */
int oracle_em_update(const float* rows, int64_t N, int d, int g, int n_codes, const int32_t* codes,
                     float* cb) {
  if (!valid_shape(d, g, 1, n_codes) || N < 0 || !rows || !cb || (N > 0 && !codes)) return ORACLE_BAD_ARG;
  const int G = d / g;
  double* sum = (double*)calloc((size_t)G * n_codes * g, sizeof(double));
  int64_t* cnt = (int64_t*)calloc((size_t)G * n_codes, sizeof(int64_t));
  if (!sum || !cnt) { free(sum); free(cnt); return ORACLE_NO_MEM; }
  for (int64_t n = 0; n < N; ++n)
    for (int j = 0; j < G; ++j) {
      const float* x = rows + n * d + (int64_t)j * g;
      const int32_t c = codes[n * G + j];
      if (c < 0 || c >= n_codes) { free(sum); free(cnt); return ORACLE_BAD_ARG; }
      cnt[(int64_t)j * n_codes + c] += 1;
      for (int k = 0; k < g; ++k) sum[((int64_t)j * n_codes + c) * g + k] += (double)x[k];
    }
  for (int j = 0; j < G; ++j)
    for (int c = 0; c < n_codes; ++c) {
      int64_t m = cnt[(int64_t)j * n_codes + c];
      if (m == 0) continue;
      for (int k = 0; k < g; ++k) {
        int64_t at = ((int64_t)j * n_codes + c) * g + k;
        cb[at] = (float)(sum[at] / (double)m);
      }
    }
  free(sum);
  free(cnt);
  return ORACLE_OK;
}

/* Value side through softmax-weight histograms (the review's "If this is right":
 * softmax weights multiply the value codes before the codebook multiply).
 * H[r][j][c] = sum_t p_t [code[t][r][j] == c]; o[j*g + k] = sum_r sum_c H[r][j][c] cb[r][j][c][k].
 * p [T] fp64 weights, codes [T, R, d/g] int32 with row stride code_stride,
 * cb [R, d/g, Nc', g] fp32 -> hist [R, d/g, Nc'] fp64 (nullable), o [d] fp64. */
int oracle_values_hist(const double* p, const int32_t* codes, int64_t code_stride, int64_t T,
                       int d, int g, int R, int n_codes, const float* cb, double* hist,
                       double* o) {
  if (!valid_shape(d, g, R, n_codes) || T < 0 || !o || (T > 0 && (!p || !codes))) return ORACLE_BAD_ARG;
  const int G = d / g;
  double* H = (double*)calloc((size_t)R * G * n_codes, sizeof(double));
  if (!H) return ORACLE_NO_MEM;
  for (int64_t t = 0; t < T; ++t)
    for (int r = 0; r < R; ++r)
      for (int j = 0; j < G; ++j) {
        int32_t c = codes[t * code_stride + r * G + j];
        if (c < 0 || c >= n_codes) { free(H); return ORACLE_BAD_ARG; }
        H[((int64_t)r * G + j) * n_codes + c] += p[t];
      }
  for (int j = 0; j < G; ++j)
    for (int k = 0; k < g; ++k) {
      double s = 0.0;
      for (int r = 0; r < R; ++r)
        for (int c = 0; c < n_codes; ++c)
          s += H[((int64_t)r * G + j) * n_codes + c] *
               (double)cb[(((int64_t)r * G + j) * n_codes + c) * g + k];
      o[(int64_t)j * g + k] = s;
    }
  if (hist) memcpy(hist, H, sizeof(double) * (size_t)R * G * n_codes);
  free(H);
  return ORACLE_OK;
}

/* One soft-assignment EM step with temperature tau (review, "Assumptions & free
 * parameters": the paper stabilises its EM with soft assignment and annealing; the caller
 * lowers tau from step to step). For each (row n, group j), with the encoder's fp32
 * distances d_c and d_min = min_c d_c:
 *   w_c = exp(-(d_c - d_min) / tau) / sum_c' exp(-(d_c' - d_min) / tau)      (fp64),
 * and each entry becomes (float)(sum_n w x / sum_n w); an entry whose weight sum is 0 keeps
 * its value. sse_out = sum over (row, group) of d_min (fp64, the hard distortion against the
 * input codebook). tau must be > 0 (tau -> 0 gives the hard step when there are no ties). */
int oracle_em_soft_step(const float* rows, int64_t N, int d, int g, int n_codes, float* cb, double tau,
                        double* sse_out) {
  if (!valid_shape(d, g, 1, n_codes) || N < 0 || !rows || !cb || !(tau > 0.0)) return ORACLE_BAD_ARG;
  const int G = d / g;
  double* sum = (double*)calloc((size_t)G * n_codes * g, sizeof(double));
  double* wsum = (double*)calloc((size_t)G * n_codes, sizeof(double));
  double* w = (double*)malloc(sizeof(double) * (size_t)n_codes);
  float* dist = (float*)malloc(sizeof(float) * (size_t)n_codes);
  if (!sum || !wsum || !w || !dist) { free(sum); free(wsum); free(w); free(dist); return ORACLE_NO_MEM; }
  double sse = 0.0;
  for (int64_t n = 0; n < N; ++n)
    for (int j = 0; j < G; ++j) {
      const float* x = rows + n * d + (int64_t)j * g;
      const float* sub = cb + (int64_t)j * n_codes * g;
      float dmin = INFINITY;
      for (int c = 0; c < n_codes; ++c) {
        float acc = 0.0f;
        for (int k = 0; k < g; ++k) {
          float e = x[k] - sub[(int64_t)c * g + k];
          acc = fmaf(e, e, acc);
        }
        dist[c] = acc;
        if (acc < dmin) dmin = acc;
      }
      sse += (double)dmin;
      double Z = 0.0;
      for (int c = 0; c < n_codes; ++c) {
        w[c] = exp(-((double)dist[c] - (double)dmin) / tau);
        Z += w[c];
      }
      for (int c = 0; c < n_codes; ++c) {
        const double wc = w[c] / Z;
        if (wc == 0.0) continue;
        wsum[(int64_t)j * n_codes + c] += wc;
        for (int k = 0; k < g; ++k) sum[((int64_t)j * n_codes + c) * g + k] += wc * (double)x[k];
      }
    }
  for (int j = 0; j < G; ++j)
    for (int c = 0; c < n_codes; ++c) {
      const double m = wsum[(int64_t)j * n_codes + c];
      if (!(m > 0.0)) continue;
      for (int k = 0; k < g; ++k) {
        const int64_t at = ((int64_t)j * n_codes + c) * g + k;
        cb[at] = (float)(sum[at] / m);
      }
    }
  free(sum); free(wsum); free(w); free(dist);
  if (sse_out) *sse_out = sse;
  return ORACLE_OK;
}
