/* Memory Sparse Attention -- plain fp64 CPU oracle (test infrastructure only).
 *
 * Only the test suite, the smoke check and the CPU-baseline leg of the
 * benchmark may load this code; the product path never does.
 *
 * Sources:
 *   [A] "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts",
 *       section "How MSA compresses and routes documents".
 *   [B] "EverMind Releases Memory-Sparse Attention Code for Long-Context AI
 *       Models", section "Architectural Design and Inference".
 *
 * Readings where the pages are silent (each is repeated at its use):
 *   - RoPE pairs dimension i with i + d/2 and turns it by pos * theta^(-2i/d);
 *     only keys (K) are rotated, never V or the router keys Kr.
 *   - cos(x, y) = x.y / (max(|x|, 1e-12) * max(|y|, 1e-12)), clamped to [-1, 1].
 *   - query head h is scored against router-key head h / (H_q / H_kv).
 *   - "retrieved blocks" in the global RoPE offset = top_k documents.
 *
 * Arithmetic is IEEE fp64 with every sum taken in index order and no fused
 * multiply-add (the build passes -ffp-contract=off), so each result is one
 * well-defined double.
 */
#include "msa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int g_threads = 0;

int orc_set_threads(int n) {
  g_threads = n > 0 ? n : 0;
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#endif
  return 0;
}

int orc_get_threads(void) {
#ifdef _OPENMP
  return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
  return 1;
#endif
}

/* One stored element as an exact double. */
static double ld(const void* p, int dtype, int64_t i) {
  if (dtype == ORC_F32) return (double)((const float*)p)[i];
  uint32_t u = (uint32_t)((const uint16_t*)p)[i] << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* theta^(-2i/d) for i < d/2. */
static void inv_freq(int d, double theta, double* w) {
  for (int i = 0; i < d / 2; ++i) w[i] = pow(theta, -2.0 * (double)i / (double)d);
}

static void rope_w(const double* x, int d, double pos, const double* w, double* y) {
  int h = d / 2;
  for (int i = 0; i < h; ++i) {
    double a = pos * w[i];
    double c = cos(a), s = sin(a);
    double x0 = x[i], x1 = x[i + h];
    y[i] = x0 * c - x1 * s;
    y[i + h] = x1 * c + x0 * s;
  }
}

int orc_rope(const double* x, int d, double pos, double theta, double* y) {
  if (d <= 0 || (d & 1)) return -1;
  double* w = (double*)malloc(sizeof(double) * (size_t)(d / 2));
  if (!w) return -2;
  inv_freq(d, theta, w);
  rope_w(x, d, pos, w, y);
  free(w);
  return 0;
}

int64_t orc_chunk_offsets(int64_t n_docs, const int64_t* doc_tok_off, int chunk,
                          int64_t* doc_chunk_off) {
  if (n_docs < 0 || chunk <= 0) return -1;
  doc_chunk_off[0] = 0;
  for (int64_t s = 0; s < n_docs; ++s) {
    int64_t L = doc_tok_off[s + 1] - doc_tok_off[s];
    if (L <= 0) return -1;                      /* every document holds >= 1 token */
    doc_chunk_off[s + 1] = doc_chunk_off[s] + (L + chunk - 1) / chunk;
  }
  return doc_chunk_off[n_docs];
}

/* Offline encoding [A][B]: positions restart at 0 in every document; each
 * pooled vector is the plain mean of the (rotated, for K) token vectors of its
 * chunk, the sum taken in token order and divided by the tokens present. */
int orc_encode(int64_t n_docs, const int64_t* doc_tok_off, int H, int d, int dr,
               int chunk, double theta, int dtype, const void* k_tok,
               const void* v_tok, const void* kr_tok, double* k_pool,
               double* v_pool, double* kr_pool) {
  if (n_docs < 0 || H <= 0 || d <= 0 || (d & 1) || dr <= 0 || chunk <= 0) return -1;
  int64_t* coff = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_docs + 1));
  double* w = (double*)malloc(sizeof(double) * (size_t)(d / 2));
  if (!coff || !w) { free(coff); free(w); return -2; }
  if (orc_chunk_offsets(n_docs, doc_tok_off, chunk, coff) < 0) { free(coff); free(w); return -1; }
  inv_freq(d, theta, w);
  int err = 0;
#pragma omp parallel
  {
    double* x = (double*)malloc(sizeof(double) * (size_t)d);
    double* y = (double*)malloc(sizeof(double) * (size_t)d);
    double* acc = (double*)malloc(sizeof(double) * (size_t)(d > dr ? d : dr));
    if (!x || !y || !acc) {
#pragma omp atomic write
      err = -2;
    } else {
#pragma omp for schedule(dynamic, 16)
      for (int64_t s = 0; s < n_docs; ++s) {
        int64_t t0 = doc_tok_off[s], L = doc_tok_off[s + 1] - doc_tok_off[s];
        for (int64_t c = coff[s]; c < coff[s + 1]; ++c) {
          int64_t p0 = (c - coff[s]) * chunk;            /* doc-local position */
          int64_t n = L - p0 < chunk ? L - p0 : chunk;    /* tokens in chunk */
          for (int g = 0; g < H; ++g) {
            /* K: rotate at the document-local position, then average. */
            for (int i = 0; i < d; ++i) acc[i] = 0.0;
            for (int64_t p = p0; p < p0 + n; ++p) {
              int64_t base = ((t0 + p) * H + g) * (int64_t)d;
              for (int i = 0; i < d; ++i) x[i] = ld(k_tok, dtype, base + i);
              rope_w(x, d, (double)p, w, y);
              for (int i = 0; i < d; ++i) acc[i] += y[i];
            }
            for (int i = 0; i < d; ++i) k_pool[(c * H + g) * (int64_t)d + i] = acc[i] / (double)n;
            /* V: plain average. */
            for (int i = 0; i < d; ++i) acc[i] = 0.0;
            for (int64_t p = p0; p < p0 + n; ++p) {
              int64_t base = ((t0 + p) * H + g) * (int64_t)d;
              for (int i = 0; i < d; ++i) acc[i] += ld(v_tok, dtype, base + i);
            }
            for (int i = 0; i < d; ++i) v_pool[(c * H + g) * (int64_t)d + i] = acc[i] / (double)n;
            /* Kr: plain average. */
            for (int i = 0; i < dr; ++i) acc[i] = 0.0;
            for (int64_t p = p0; p < p0 + n; ++p) {
              int64_t base = ((t0 + p) * H + g) * (int64_t)dr;
              for (int i = 0; i < dr; ++i) acc[i] += ld(kr_tok, dtype, base + i);
            }
            for (int i = 0; i < dr; ++i) kr_pool[(c * H + g) * (int64_t)dr + i] = acc[i] / (double)n;
          }
        }
      }
    }
    free(x); free(y); free(acc);
  }
  free(coff);
  free(w);
  return err;
}

/* Routing [A][B]: cosine per head, mean over all query heads, max over the
 * query tokens and the document's pooled chunks; Top-k by (score desc,
 * index asc). */
int orc_route(int B, int T, int Hq, int Hkv, int dr, const double* qr,
              int64_t n_docs, const int64_t* doc_chunk_off, int dtype,
              const void* kr, int top_k, int32_t* out_idx, double* out_score,
              double* doc_score) {
  if (B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || dr <= 0) return -1;
  if (n_docs <= 0 || top_k <= 0 || top_k > n_docs) return -1;
  int G = Hq / Hkv;
  double* score = (double*)malloc(sizeof(double) * (size_t)n_docs);
  double* qn = (double*)malloc(sizeof(double) * (size_t)(T * Hq));
  char* taken = (char*)malloc((size_t)n_docs);
  if (!score || !qn || !taken) { free(score); free(qn); free(taken); return -2; }
  int err = 0;
  for (int b = 0; b < B && !err; ++b) {
    const double* Q = qr + (int64_t)b * T * Hq * dr;
    for (int th = 0; th < T * Hq; ++th) {       /* |Qr[t,h]| */
      double s = 0.0;
      for (int i = 0; i < dr; ++i) s += Q[(int64_t)th * dr + i] * Q[(int64_t)th * dr + i];
      qn[th] = sqrt(s);
    }
#pragma omp parallel
    {
      double* kv = (double*)malloc(sizeof(double) * (size_t)Hkv * dr);
      double* kn = (double*)malloc(sizeof(double) * (size_t)Hkv);
      if (!kv || !kn) {
#pragma omp atomic write
        err = -2;
      } else {
#pragma omp for schedule(dynamic, 64)
        for (int64_t s = 0; s < n_docs; ++s) {
          double best = -INFINITY;
          for (int64_t c = doc_chunk_off[s]; c < doc_chunk_off[s + 1]; ++c) {
            for (int g = 0; g < Hkv; ++g) {   /* the pooled router key and |Kr[c,g]| */
              double nn = 0.0;
              for (int i = 0; i < dr; ++i) {
                double x = ld(kr, dtype, (c * Hkv + g) * (int64_t)dr + i);
                kv[g * dr + i] = x;
                nn += x * x;
              }
              kn[g] = sqrt(nn);
            }
            for (int t = 0; t < T; ++t) {
              double sum = 0.0;
              for (int h = 0; h < Hq; ++h) {
                int g = h / G;
                const double* q = Q + ((int64_t)t * Hq + h) * dr;
                double dot = 0.0;
                for (int i = 0; i < dr; ++i) dot += q[i] * kv[g * dr + i];
                double den = fmax(qn[t * Hq + h], 1e-12) * fmax(kn[g], 1e-12);
                double cs = dot / den;
                cs = fmin(fmax(cs, -1.0), 1.0);
                sum += cs;
              }
              double S = sum / (double)Hq;
              if (S > best) best = S;
            }
          }
          score[s] = best;
        }
      }
      free(kv); free(kn);
    }
    if (err) break;
    if (doc_score) memcpy(doc_score + (int64_t)b * n_docs, score, sizeof(double) * (size_t)n_docs);
    /* Top-k: repeatedly take the best remaining document. */
    memset(taken, 0, (size_t)n_docs);
    for (int r = 0; r < top_k; ++r) {
      int64_t arg = -1;
      for (int64_t s = 0; s < n_docs; ++s) {
        if (taken[s]) continue;
        if (arg < 0 || score[s] > score[arg]) arg = s;  /* strict: lower index wins ties */
      }
      taken[arg] = 1;
      out_idx[(int64_t)b * top_k + r] = (int32_t)arg;
      if (out_score) out_score[(int64_t)b * top_k + r] = score[arg];
    }
  }
  free(score); free(qn); free(taken);
  return err;
}

/* Sparse decode [A][B]: the selected documents' pooled K/V (keys kept with
 * their document-local rotation from encoding) are placed ahead of the local
 * context; the query and local keys take global positions offset by top_k. */
int orc_decode(int B, int T, int Hq, int Hkv, int d, double theta, int top_k,
               const int32_t* sel, int64_t n_docs, const int64_t* doc_chunk_off,
               int dtype, int kv_layout, const void* k_pool, const void* v_pool,
               const double* q, const int64_t* local_off, const void* local_k,
               const void* local_v, double* out) {
  if (B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || d <= 0 || (d & 1)) return -1;
  if (top_k <= 0 || top_k > n_docs) return -1;
  for (int b = 0; b < B; ++b) {
    if (local_off[b + 1] - local_off[b] < T) return -1;
    for (int r = 0; r < top_k; ++r) {
      int32_t s = sel[(int64_t)b * top_k + r];
      if (s < 0 || s >= n_docs) return -1;
    }
  }
  int G = Hq / Hkv;
  double* w = (double*)malloc(sizeof(double) * (size_t)(d / 2));
  if (!w) return -2;
  inv_freq(d, theta, w);
  const double scale_div = sqrt((double)d);
  int err = 0;
#pragma omp parallel
  {
    int64_t cap = 0;
    double *keys = NULL, *vals = NULL, *logit = NULL;
    double* x = (double*)malloc(sizeof(double) * (size_t)d);
    double* qrot = (double*)malloc(sizeof(double) * (size_t)d);
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    if (!x || !qrot || !acc) {
#pragma omp atomic write
      err = -2;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t bg = 0; bg < (int64_t)B * Hkv; ++bg) {
      if (err) continue;
      int b = (int)(bg / Hkv), g = (int)(bg % Hkv);
      int64_t Ltot = local_off[b + 1] - local_off[b], Lb = Ltot - T;
      int64_t nmem = 0;
      for (int r = 0; r < top_k; ++r) {
        int32_t s = sel[(int64_t)b * top_k + r];
        nmem += doc_chunk_off[s + 1] - doc_chunk_off[s];
      }
      int64_t nk = nmem + Ltot;
      if (nk > cap) {
        free(keys); free(vals); free(logit);
        cap = nk;
        keys = (double*)malloc(sizeof(double) * (size_t)(cap * d));
        vals = (double*)malloc(sizeof(double) * (size_t)(cap * d));
        logit = (double*)malloc(sizeof(double) * (size_t)cap);
        if (!keys || !vals || !logit) {
#pragma omp atomic write
          err = -2;
          cap = 0;
          continue;
        }
      }
      /* Context assembly: selected documents in rank order, chunks in order. */
      int64_t n = 0;
      for (int r = 0; r < top_k; ++r) {
        int32_t s = sel[(int64_t)b * top_k + r];
        int64_t c0 = doc_chunk_off[s], nc = doc_chunk_off[s + 1] - c0;
        for (int64_t c = c0; c < c0 + nc; ++c, ++n) {
          int64_t krow, vrow;
          const void* vsrc;
          if (kv_layout == ORC_KV_DOC_INTERLEAVED) {
            krow = c0 + c;            /* doc block starts at row 2*c0 */
            vrow = c0 + c + nc;
            vsrc = k_pool;
          } else {
            krow = c;
            vrow = c;
            vsrc = v_pool;
          }
          for (int i = 0; i < d; ++i) {
            keys[n * d + i] = ld(k_pool, dtype, (krow * Hkv + g) * (int64_t)d + i);
            vals[n * d + i] = ld(vsrc, dtype, (vrow * Hkv + g) * (int64_t)d + i);
          }
        }
      }
      /* Local context and the query tokens' own keys at global positions top_k + j. */
      int64_t lbase = (local_off[b] * Hkv + (int64_t)g * Ltot) * d;
      for (int64_t j = 0; j < Ltot; ++j, ++n) {
        for (int i = 0; i < d; ++i) x[i] = ld(local_k, dtype, lbase + j * d + i);
        rope_w(x, d, (double)(top_k + j), w, keys + n * d);
        for (int i = 0; i < d; ++i) vals[n * d + i] = ld(local_v, dtype, lbase + j * d + i);
      }
      for (int t = 0; t < T; ++t) {
        int64_t visible = nmem + Lb + t + 1;   /* memory + local j <= L_b + t */
        for (int hh = 0; hh < G; ++hh) {
          int h = g * G + hh;
          const double* qv = q + (((int64_t)b * T + t) * Hq + h) * d;
          rope_w(qv, d, (double)(top_k + Lb + t), w, qrot);
          double m = -INFINITY;
          for (int64_t j = 0; j < visible; ++j) {
            double dot = 0.0;
            for (int i = 0; i < d; ++i) dot += qrot[i] * keys[j * d + i];
            logit[j] = dot / scale_div;
            if (logit[j] > m) m = logit[j];
          }
          double den = 0.0;
          for (int i = 0; i < d; ++i) acc[i] = 0.0;
          for (int64_t j = 0; j < visible; ++j) {
            double p = exp(logit[j] - m);
            den += p;
            for (int i = 0; i < d; ++i) acc[i] += p * vals[j * d + i];
          }
          double* o = out + (((int64_t)b * T + t) * Hq + h) * d;
          for (int i = 0; i < d; ++i) o[i] = acc[i] / den;
        }
      }
    }
    free(keys); free(vals); free(logit); free(x); free(qrot); free(acc);
  }
  free(w);
  return err;
}

/* Memory Interleave expansion round [A][B]: the per_round best documents of
 * each query outside its selected set, appended in (score desc, index asc)
 * order. */
int orc_interleave_expand(int B, int64_t n_docs, const double* doc_score, int n_sel,
                          const int32_t* sel_old, int per_round, int32_t* sel_new) {
  if (B <= 0 || n_docs <= 0 || n_sel < 0 || per_round <= 0) return -1;
  if ((int64_t)n_sel + per_round > n_docs || (n_sel > 0 && !sel_old)) return -1;
  char* taken = (char*)malloc((size_t)n_docs);
  if (!taken) return -2;
  int n_new = n_sel + per_round;
  for (int b = 0; b < B; ++b) {
    const double* score = doc_score + (int64_t)b * n_docs;
    memset(taken, 0, (size_t)n_docs);
    for (int i = 0; i < n_sel; ++i) {
      int32_t s = sel_old[(int64_t)b * n_sel + i];
      if (s < 0 || s >= n_docs || taken[s]) { free(taken); return -1; }
      taken[s] = 1;
      sel_new[(int64_t)b * n_new + i] = s;
    }
    for (int r = 0; r < per_round; ++r) {
      int64_t arg = -1;
      for (int64_t s = 0; s < n_docs; ++s) {
        if (taken[s]) continue;
        if (arg < 0 || score[s] > score[arg]) arg = s;
      }
      taken[arg] = 1;
      sel_new[(int64_t)b * n_new + n_sel + r] = (int32_t)arg;
    }
  }
  free(taken);
  return 0;
}
