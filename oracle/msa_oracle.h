/* Memory Sparse Attention -- plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA library and must never be used as a
 * fallback for it.
 *
 * Sources (the method is described in words only):
 *   [A] "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts",
 *       section "How MSA compresses and routes documents".
 *   [B] "EverMind Releases Memory-Sparse Attention Code for Long-Context AI
 *       Models", section "Architectural Design and Inference".
 *
 * Every function returns 0 on success and a negative value on a bad argument.
 * Element storage types: ORC_F32 (float) or ORC_BF16 (bfloat16 bit patterns).
 */
#ifndef MSA_ORACLE_H
#define MSA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1 };
enum { ORC_KV_CHUNK_MAJOR = 0, ORC_KV_DOC_INTERLEAVED = 1 };

int orc_set_threads(int n);
int orc_get_threads(void);

/* Rotary embedding, rotate-half pairing (i, i + d/2), frequency theta^(-2i/d),
 * applied to one vector x[d] at position pos.  [A][B] name RoPE only. */
int orc_rope(const double* x, int d, double pos, double theta, double* y);

/* Pooled-chunk CSR: doc_chunk_off[D+1], ceil(L_d / chunk) chunks per doc.
 * Returns the total chunk count C (>= 0) or a negative error. */
int64_t orc_chunk_offsets(int64_t n_docs, const int64_t* doc_tok_off, int chunk,
                          int64_t* doc_chunk_off);

/* Offline memory encoding [A][B]: per document, RoPE each key at its
 * document-local position (0-based), then mean-pool K, V and Kr over runs of
 * `chunk` tokens (last run may be shorter).  Inputs [N_tok][H][dim] in dtype;
 * outputs fp64 [C][H][dim]. */
int orc_encode(int64_t n_docs, const int64_t* doc_tok_off, int H, int d, int dr,
               int chunk, double theta, int dtype, const void* k_tok,
               const void* v_tok, const void* kr_tok, double* k_pool,
               double* v_pool, double* kr_pool);

/* Online routing [A][B]: for each of B queries, the score of document d is
 * max over its pooled chunks c and query tokens t of
 *   (1/H_q) sum_h clamp(cos(Qr[t,h], Kr[c, h / (H_q/H_kv)]), -1, 1)
 * and the top_k documents are returned ordered by (score desc, index asc).
 * qr: [B][T][H_q][dr] fp64; kr: [C][H_kv][dr] in dtype.
 * out_idx/out_score: [B][top_k]; doc_score: [B][D] or NULL. */
int orc_route(int B, int T, int Hq, int Hkv, int dr, const double* qr,
              int64_t n_docs, const int64_t* doc_chunk_off, int dtype,
              const void* kr, int top_k, int32_t* out_idx, double* out_score,
              double* doc_score);

/* Sparse decode [A][B]: for query b, token t, head h (kv head g = h / G):
 * keys = [pooled K of the selected docs' chunks, rank order] ++
 *        [RoPE(localK[j], top_k + j) for j = 0 .. L_b + t];
 * the query is RoPE(Q[t,h], top_k + L_b + t); softmax(q.k / sqrt(d)) over the
 * keys weights [pooled V ++ local V].
 * q: [B][T][H_q][d] fp64; local_k/local_v: per query b at token offset
 * local_off[b] (element offset local_off[b]*H_kv*d), laid out [H_kv][Ltot_b][d]
 * with Ltot_b = local_off[b+1]-local_off[b] = L_b + T.  kv_layout selects
 * chunk-major k_pool/v_pool [C][H_kv][d] or one per-document interleaved
 * array in k_pool (doc s: its K chunks then its V chunks).  out: fp64 like q. */
int orc_decode(int B, int T, int Hq, int Hkv, int d, double theta, int top_k,
               const int32_t* sel, int64_t n_docs, const int64_t* doc_chunk_off,
               int dtype, int kv_layout, const void* k_pool, const void* v_pool,
               const double* q, const int64_t* local_off, const void* local_k,
               const void* local_v, double* out);

/* Memory Interleave, one context-expansion round ([A] "How MSA compresses
 * and routes documents"; [B], section "Core Contributions": retrieval,
 * context expansion and generation alternate).  The pages give no formula; the
 * reading: the selected set S_b of query b (n_sel documents, joining order)
 * grows by the per_round documents of highest score that are not in S_b,
 * ordered by (score desc, index asc), appended after S_b.
 * doc_score: [B][D] fp64 (orc_route's doc_score); sel_old: [B][n_sel] or NULL
 * when n_sel = 0; sel_new: [B][n_sel + per_round]. */
int orc_interleave_expand(int B, int64_t n_docs, const double* doc_score, int n_sel,
                          const int32_t* sel_old, int per_round, int32_t* sel_new);

#ifdef __cplusplus
}
#endif
#endif
