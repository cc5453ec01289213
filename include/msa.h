/* msa.h -- C ABI of the B200 (sm_100a) Memory Sparse Attention hot path.
 *
 * Memory Sparse Attention keeps a compressed memory of a corpus and, while
 * decoding, attends only over the few documents a router selects.  The three
 * stages below follow the pages' description of the inference pipeline:
 *   [A] "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts",
 *       section "How MSA compresses and routes documents";
 *   [B] "EverMind Releases Memory-Sparse Attention Code for Long-Context AI
 *       Models", section "Architectural Design and Inference" (the three
 *       numbered stages: global memory encoding, online routing and context
 *       assembly, sparse generation).
 *
 * Conventions for every entry point
 *   - Pointers marked (device) are CUDA device pointers, (host) are host
 *     pointers, (pinned) are page-locked host memory (cudaHostAlloc or
 *     cudaHostRegister).  The caller allocates and owns every buffer; the
 *     library allocates nothing and keeps no state except a thread-local error
 *     message and one device status word per GPU.
 *   - Work is enqueued on the given stream and runs asynchronously, with the
 *     usual CUDA stream semantics; no call synchronises unless stated.
 *   - Element storage is layout->dtype: MSA_F32 (float) or MSA_BF16
 *     (bfloat16).  Every device pointer must be 16-byte aligned.
 *   - Bad arguments return MSA_ERR_INVALID_ARG before anything is launched;
 *     shapes the kernels do not implement return MSA_ERR_UNSUPPORTED; launch
 *     or copy failures return MSA_ERR_CUDA; msa_last_error() then describes
 *     the failure.  Kernels never trap: an out-of-range value they meet (a
 *     position beyond the RoPE table, a selected document index out of range)
 *     sets a bit in the device status word, read with msa_device_status().
 *     Nothing aborts or exits the process.
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1,
  MSA_ERR_UNSUPPORTED = 2,
  MSA_ERR_CUDA = 3,
  MSA_ERR_WORKSPACE_TOO_SMALL = 4,
  MSA_ERR_TIMEOUT = 5,
  MSA_ERR_INTERNAL = 6
} msa_status;

typedef enum { MSA_F32 = 0, MSA_BF16 = 1 } msa_dtype;

/* Bits of the device status word. */
#define MSA_DEV_ROPE_RANGE   0x1u  /* a position beyond the RoPE table */
#define MSA_DEV_BAD_DOC      0x2u  /* a selected document index out of range */
#define MSA_DEV_PIPE_TIMEOUT 0x4u  /* a bounded in-kernel wait gave up */
#define MSA_DEV_BAD_SHAPE    0x8u  /* a shape the launch was not planned for */
#define MSA_DEV_BAD_SET      0x10u /* an interleave set holds a document twice or out of range */

/* Attention-head layout of one routing layer.  H_q query heads share H_kv
 * key/value heads (grouped-query attention, group G = H_q / H_kv).  Router
 * keys Kr have H_kv heads of router_dim (their pooled size, 2 bytes x 8 x 128
 * per chunk at 100M tokens, matches H_kv heads).  Rotary embedding: dims
 * (i, i + head_dim/2) turn by pos * rope_theta^(-2i/head_dim). */
typedef struct {
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t head_dim;     /* 64 or 128 */
  int32_t router_dim;   /* router_dim * element size must be 256 bytes */
  int32_t chunk_size;   /* tokens per pooled chunk, e.g. 64 */
  int32_t dtype;        /* msa_dtype */
  double rope_theta;
} msa_layout;

/* A pooled memory bank (output of stage 1, input of stages 2 and 3).
 * Chunk c of document s is row c, doc_chunk_off[s] <= c < doc_chunk_off[s+1];
 * rows are [H_kv][dim] (chunk-major, one row = H_kv * dim elements). */
typedef struct {
  int64_t n_docs;
  int64_t n_chunks;
  const int64_t* doc_chunk_off;       /* (device) [n_docs + 1] */
  const int64_t* doc_chunk_off_host;  /* (host) [n_docs + 1]; required when kv_on_host */
  int32_t max_doc_chunks;             /* max over documents of their chunk count */
  int32_t kv_on_host;                 /* 0: k, v in device memory; 1: host_kv */
  const void* kr;                     /* (device) [n_chunks][H_kv][router_dim] */
  const void* k;                      /* (device) [n_chunks][H_kv][head_dim], kv_on_host = 0 */
  const void* v;                      /* (device) [n_chunks][H_kv][head_dim], kv_on_host = 0 */
  const void* host_kv;                /* (pinned) kv_on_host = 1: document s occupies rows
                                         [2*doc_chunk_off[s], 2*doc_chunk_off[s+1]): its K
                                         chunks, then its V chunks, rows of [H_kv][head_dim] */
  const float* kr_inv_norm;           /* (device) optional, NULL allowed: the router keys'
                                         inverse norms as msa_kr_inv_norms writes them; the
                                         tensor-core routing scan reads them instead of
                                         recomputing them on every call */
} msa_index;

/* Instrumentation and test hooks (a scan timer, an injected copy failure, an
 * expiring in-kernel wait) are declared apart, in msa_debug.h. */

/* ---------------------------------------------------------------- helpers */

int msa_version(void);
const char* msa_last_error(void);            /* thread-local; "" when none */
const char* msa_status_string(msa_status s);

/* Reads and clears this GPU's device status word (MSA_DEV_* bits).
 * Synchronises `stream`. */
msa_status msa_device_status(uint32_t* bits, cudaStream_t stream);

/* Pooled-chunk CSR from token offsets (host computation): document s holds
 * doc_tok_off[s+1] - doc_tok_off[s] >= 1 tokens and ceil(L_s / chunk_size)
 * pooled chunks ([A] "chunk-mean pooled").  Writes doc_chunk_off_host[n+1]
 * and, when non-NULL, the largest chunk count and the largest length. */
msa_status msa_chunk_offsets(int64_t n_docs, const int64_t* doc_tok_off_host,
                             int32_t chunk_size, int64_t* doc_chunk_off_host,
                             int32_t* max_doc_chunks, int64_t* max_doc_len);

/* Rotary table (device) [n_pos][head_dim/2] of (cos, sin) float pairs for
 * positions 0 .. n_pos-1, computed in fp64 on the GPU and rounded once to
 * fp32.  Build it once per layout; encode and decode read it. */
msa_status msa_rope_table(const msa_layout* layout, int32_t n_pos, float* table,
                          cudaStream_t stream);

/* --------------------------------------------- stage 1: memory encoding */

/* [A][B] "Global Memory Encoding (offline)": per document, rotate each key
 * at its document-local position (positions restart at 0 in every document,
 * "parallel document-wise RoPE"), then mean-pool K, V and Kr over runs of
 * chunk_size tokens (the last run of a document may be shorter; it is
 * averaged over the tokens it holds).  Accumulation in fp32, one rounding to
 * dtype at the end.
 *   doc_tok_off, doc_chunk_off: (device) [n_docs + 1] token / chunk CSR
 *   k_tok, v_tok: (device) [N_tok][H_kv][head_dim]; kr_tok: [N_tok][H_kv][router_dim]
 *   rope_table: (device) from msa_rope_table, rope_rows >= the longest document
 *   k_pool, v_pool, kr_pool: (device) [n_chunks][H_kv][dim] outputs. */
msa_status msa_encode_memory(const msa_layout* layout, int64_t n_docs, int64_t n_chunks,
                             const int64_t* doc_tok_off, const int64_t* doc_chunk_off,
                             int64_t max_doc_len, const void* k_tok, const void* v_tok,
                             const void* kr_tok, const float* rope_table, int32_t rope_rows,
                             void* k_pool, void* v_pool, void* kr_pool, cudaStream_t stream);

/* msa_encode_memory with K and V written to one buffer in the host tier's
 * row layout (msa_index.host_kv): document s with chunks [c0, c1) gets its K
 * chunks in rows [2*c0, c0 + c1) and its V chunks in rows [c0 + c1, 2*c1),
 * so the buffer can be copied to pinned host memory as it is.
 *   kv_pool: (device) [2 * n_chunks][H_kv][head_dim]; kr_pool as above. */
msa_status msa_encode_memory_kv_interleaved(const msa_layout* layout, int64_t n_docs, int64_t n_chunks,
                                            const int64_t* doc_tok_off, const int64_t* doc_chunk_off,
                                            int64_t max_doc_len, const void* k_tok, const void* v_tok,
                                            const void* kr_tok, const float* rope_table, int32_t rope_rows,
                                            void* kv_pool, void* kr_pool, cudaStream_t stream);

/* ------------------------------- stage 1b: streaming offline encoding */

/* [A] "How MSA compresses and routes documents": the pooled triples are
 * cached offline by one pass over the corpus, and the content K/V of a
 * 100M-token memory stays in host memory.  A streaming encoder builds such a
 * bank from per-token batches that need not fit on the GPU together: each
 * push copies one batch of whole documents to the device, encodes it there
 * (msa_encode_memory arithmetic) and appends its pooled rows to the outputs --
 * Kr in device memory; K/V either in device memory, chunk-major, or in the
 * host tier's row layout in host memory.  Copies in, the encode and copies
 * out of consecutive batches overlap on three streams the encoder owns, with
 * two device slots of staging.
 *
 * Not thread-safe: one host thread drives an encoder. */
typedef struct msa_encoder msa_encoder;

/* max_batch_tokens / max_batch_docs: the largest push; max_doc_len: the
 * longest document of the whole bank; capacity_chunks: pooled rows the
 * outputs hold.  Outputs (all written in push order, chunk rows appended):
 *   kr_out: (device) [capacity_chunks][H_kv][router_dim]
 *   host tier: host_kv_out (pinned) [2 * capacity_chunks][H_kv][head_dim],
 *     k_out = v_out = NULL;
 *   device tier: k_out, v_out (device) [capacity_chunks][H_kv][head_dim],
 *     host_kv_out = NULL.
 * Device memory held: two slots of max_batch_tokens per-token rows of K, V
 * and Kr, plus for the host tier two slots of
 * 2 * (max_batch_tokens / chunk_size + max_batch_docs) pooled K/V rows.
 * Arguments are checked before anything is allocated. */
msa_status msa_encoder_create(const msa_layout* layout, int64_t max_batch_tokens, int32_t max_batch_docs,
                              int64_t max_doc_len, int64_t capacity_chunks, void* kr_out, void* k_out,
                              void* v_out, void* host_kv_out, msa_encoder** out);

/* Appends n_docs whole documents.  doc_tok_off_host: (host) [n_docs + 1],
 * starting at 0, every document at least 1 and at most max_doc_len tokens.
 * k_tok, v_tok: [N][H_kv][head_dim], kr_tok: [N][H_kv][router_dim],
 * N = doc_tok_off_host[n_docs] <= max_batch_tokens, in host memory (pinned
 * for the copies to overlap) or device memory, 16-byte aligned.
 * Returns once the batch is queued.  The inputs of one push may be reused
 * once the next push has returned, or after msa_encoder_finish.  An error
 * of an earlier batch's copies or launch is returned by the next call. */
msa_status msa_encoder_push(msa_encoder* enc, int32_t n_docs, const int64_t* doc_tok_off_host,
                            const void* k_tok, const void* v_tok, const void* kr_tok);

/* Waits for every pushed batch (all outputs written) and reports the bank so
 * far: documents, pooled chunks and the largest chunk count of a document
 * (any pointer may be NULL). */
msa_status msa_encoder_finish(msa_encoder* enc, int64_t* n_docs, int64_t* n_chunks, int32_t* max_doc_chunks);

/* The bank's chunk CSR so far, (host) [n_docs + 1] (msa_chunk_offsets of all
 * pushed documents, in push order). */
msa_status msa_encoder_chunk_offsets(const msa_encoder* enc, int64_t* doc_chunk_off_host);

/* Waits for outstanding work and frees the encoder's buffers and streams. */
void msa_encoder_destroy(msa_encoder* enc);

/* ------------------------------------------- persistent pooled index file */

/* A pooled bank on disk, so that the offline encoding runs once.  Format
 * (little-endian):
 *   bytes [0, 512): header
 *     0   char[8]  magic "MSAIDX01"
 *     8   u32      format version (1);  12 u32 header bytes (512)
 *     16  i32 x 6  n_q_heads, n_kv_heads, head_dim, router_dim, chunk_size, dtype
 *     40  f64      rope_theta
 *     48  i64      n_docs;  56 i64 n_chunks
 *     64  i32      max_doc_chunks;  68 i32 kv_on_host
 *     72  4 x {u64 offset, u64 bytes, u64 hash}: the sections
 *           0: doc_chunk_off, i64 [n_docs + 1]
 *           1: Kr [n_chunks][H_kv][router_dim]
 *           2: kv_on_host = 0: K [n_chunks][H_kv][head_dim];
 *              kv_on_host = 1: host_kv [2 * n_chunks][H_kv][head_dim]
 *           3: kv_on_host = 0: V [n_chunks][H_kv][head_dim]; else empty
 *     168..503 zero;  504 u64 hash of bytes [0, 504)
 *   sections at 4096-byte aligned offsets, in order, zero padding between.
 * Hash (msa64, of n bytes): the bytes as little-endian u64 words w_i, the
 * last one zero-padded; M1 = 0x9E3779B97F4A7C15, M2 = 0xD6E8FEB86659FD93;
 * four lanes h_j = M2 * (j + 1); word i updates lane i mod 4:
 * h = rotl64(h ^ (w_i * M1), 29) * M2.  Then r = n; for j = 0..3:
 * r = rotl64(r ^ (h_j * M1), 31) * M2; finally r ^= r >> 33, r *= M1,
 * r ^= r >> 29 (all mod 2^64). */
#define MSA_INDEX_HEADER_BYTES 512

/* Writes the bank `index` (device tier, or host tier with host_kv) to
 * `path` (written to a temporary name first, then renamed).  The CSR is read
 * from index->doc_chunk_off_host when given, else from the device.  Blocks
 * until the file is complete; `stream` carries the device-to-host copies. */
msa_status msa_index_save(const char* path, const msa_layout* layout, const msa_index* index,
                          cudaStream_t stream);

/* Reads and checks the header of an index file (no CUDA call): its layout
 * and sizes, for the caller to allocate the buffers of msa_index_load. */
msa_status msa_index_file_info(const char* path, msa_layout* layout, int64_t* n_docs, int64_t* n_chunks,
                               int32_t* max_doc_chunks, int32_t* kv_on_host);

/* Loads an index file into caller buffers, sized from msa_index_file_info:
 *   doc_chunk_off_host: (host) [n_docs + 1], required
 *   doc_chunk_off: (device) [n_docs + 1] or NULL
 *   kr: (device or host) [n_chunks][H_kv][router_dim], required
 *   k, v: (device or host) [n_chunks][H_kv][head_dim] -- files with
 *     kv_on_host = 0; host_kv: (host, pinned for the fetch) [2 * n_chunks]
 *     [H_kv][head_dim] -- files with kv_on_host = 1.
 * verify != 0 checks every section's hash (MSA_ERR_INVALID_ARG on a
 * mismatch; the buffers then hold whatever was read).  The header hash is
 * always checked.  Blocks until the buffers are filled. */
msa_status msa_index_load(const char* path, int32_t verify, int64_t* doc_chunk_off_host, int64_t* doc_chunk_off,
                          void* kr, void* k, void* v, void* host_kv, cudaStream_t stream);

/* ----------------------------------------------------- stage 2: routing */

/* Number of floats msa_kr_inv_norms writes: H_kv * ceil(n_chunks / 128) * 128. */
size_t msa_kr_inv_norm_count(const msa_layout* layout, int64_t n_chunks);

/* Static per-bank data for routing: out[g * P + c] = rsqrt(max(|Kr[c][g]|^2,
 * 1e-24)) for chunk c < n_chunks and kv head g, P = ceil(n_chunks/128) * 128
 * (entries c >= n_chunks are written as 0), with the fp32 sum of squares the
 * fast router score uses.  Computed once per bank (it reads the whole Kr) and
 * passed back as index->kr_inv_norm.  out: (device), 16-byte aligned. */
msa_status msa_kr_inv_norms(const msa_layout* layout, const msa_index* index, float* out,
                            cudaStream_t stream);

/* Workspace bytes msa_route / msa_route_scores need for a bank of n_docs
 * documents in n_chunks pooled chunks (index->n_docs, index->n_chunks): the
 * tensor-core scan keeps one entry per 128-chunk tile, so the size depends on
 * both.  0 for arguments no call accepts. */
size_t msa_route_workspace_size(const msa_layout* layout, int64_t n_docs, int64_t n_chunks,
                                int32_t batch, int32_t T, int32_t top_k);

/* [A][B] "Online Routing": for each of `batch` independent queries with T
 * query tokens, the router score of document s is
 *     S_s = max over query tokens t and pooled chunks c of s of
 *           (1/H_q) * sum_h clamp(cos(Qr[t,h], Kr[c, h/G]), -1, 1)
 * (cosine per head, mean over heads, max over tokens and chunks), with
 * cos(x,y) = x.y / (max(|x|,1e-12) * max(|y|,1e-12)).  The top_k documents by
 * (S desc, index asc) are returned in that order.
 * The whole Kr bank is streamed once per group of query rows on the GPU (up
 * to 4 rows per pass on the CUDA cores; on bf16 banks, more than 4 rows go to
 * the tensor cores, 32 to 128 rows per pass); candidates within a proven
 * error band of the k-th fast (fp32) score are re-scored in IEEE fp64 in a
 * fixed operation order, so the returned indices and scores are the exact
 * fp64 result of the formula above.
 *   batch: 1 .. 512 queries (MSA_ERR_UNSUPPORTED beyond)
 *   qr: (device) [batch][T][H_q][router_dim] in dtype
 *   out_doc_idx: (device) [batch][top_k] int32; out_score: (device) [batch][top_k]
 *     double, or NULL; out_doc_idx_host: (pinned) [batch][top_k] or NULL -- when
 *     given, the indices are also copied there on `stream` (for msa_fetch_selected).
 *   1 <= top_k <= min(n_docs, 64). */
msa_status msa_route(const msa_layout* layout, const msa_index* index, int32_t batch,
                     int32_t T, const void* qr, int32_t top_k, int32_t* out_doc_idx,
                     double* out_score, int32_t* out_doc_idx_host, void* ws, size_t ws_bytes,
                     cudaStream_t stream);

/* Largest workspace msa_route_noalloc can serve from its built-in scratch. */
#define MSA_ROUTE_NOALLOC_MAX_BYTES ((size_t)16 << 20)

/* Routing for callers that cannot allocate device memory.  The paper has no
 * counterpart: this is an operational variant of msa_route.  Some callers may
 * not call cudaMalloc at all -- a plug-in inside a host application that owns
 * every device allocation, or a latency-critical serving loop that cannot
 * afford cudaMalloc's device-wide synchronisation -- and so cannot supply the
 * msa_route workspace.  This entry point computes exactly what msa_route
 * computes (same arguments minus ws / ws_bytes) using a scratch array compiled
 * into the library: 16 MiB (MSA_ROUTE_NOALLOC_MAX_BYTES) of device memory that
 * every GPU which loads the library holds until the process exits.
 *   - Sizes whose msa_route_workspace_size exceeds that maximum are rejected
 *     with MSA_ERR_WORKSPACE_TOO_SMALL before anything is launched (e.g. one
 *     query over up to about 500,000 documents fits).
 *   - The first call on a device looks up the scratch's device address with the
 *     device current; make that first call before any stream capture.  The
 *     address is kept for the life of the process: after cudaDeviceReset (or
 *     any other end of the device's primary context) it is stale, so a process
 *     that resets a device must not call this entry point on it again.
 *   - All calls share the one array, which keeps the previous call's contents
 *     (every value the routing reads is written by the same call first).  Calls
 *     whose work overlaps on the GPU -- different streams, or different host
 *     threads -- race on it: serialise them.
 *   - It allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
msa_status msa_route_noalloc(const msa_layout* layout, const msa_index* index, int32_t batch,
                             int32_t T, const void* qr, int32_t top_k, int32_t* out_doc_idx,
                             double* out_score, int32_t* out_doc_idx_host, cudaStream_t stream);

/* The fast (fp32) router score of every document, [batch][n_docs] float
 * (device), i.e. the first pass of msa_route without the selection. */
msa_status msa_route_scores(const msa_layout* layout, const msa_index* index, int32_t batch,
                            int32_t T, const void* qr, float* out_doc_score, void* ws,
                            size_t ws_bytes, cudaStream_t stream);

/* [A] "How MSA compresses and routes documents" and [B] "Core
 * Contributions": Memory Interleave alternates retrieval, context expansion
 * and generation for multi-hop questions.  One context-expansion round:
 * query b's selected set S_b (n_sel documents, in the order they joined)
 * grows by the per_round documents of highest router score outside S_b, in
 * (score desc, index asc) order, appended after S_b.  The caller routes the
 * round's query with top_k = n_sel + per_round (msa_route) and passes that
 * ranking here; at least per_round of its documents lie outside S_b and the
 * first per_round of them are the ones to add.  The decode of the round then
 * takes sel_new with top_k = n_sel + per_round (the global RoPE offset), and
 * the local keys are rotated again at that offset (msa_rope_local).
 *   n_docs: the bank's document count; batch: 1 .. 512
 *   n_sel: 0 .. 63; per_round >= 1; n_sel + per_round <= min(n_docs, 64)
 *   ranked: (device) [batch][n_sel + per_round] int32, msa_route's output
 *   sel_old: (device) [batch][n_sel] int32; NULL allowed when n_sel = 0
 *   sel_new: (device) [batch][n_sel + per_round] int32; it must not overlap
 *     ranked or sel_old
 *   sel_new_host: (pinned) [batch][n_sel + per_round] or NULL -- when given,
 *     sel_new is also copied there on `stream` (for msa_fetch_selected).
 * A set that holds a document twice or out of range raises MSA_DEV_BAD_SET
 * in the device status word and leaves -1 in the slots it could not fill.
 * Asynchronous on `stream`; one launch. */
msa_status msa_interleave_expand(int64_t n_docs, int32_t batch, int32_t n_sel, int32_t per_round,
                                 const int32_t* ranked, const int32_t* sel_old, int32_t* sel_new,
                                 int32_t* sel_new_host, cudaStream_t stream);

/* ----------------------------- stage 2b: fetching host-resident content */

/* Bytes of the device staging buffer msa_fetch_selected fills: one slot per
 * (query, rank) of 2 * max_doc_chunks rows of [H_kv][head_dim]. */
size_t msa_fetch_staging_size(const msa_layout* layout, const msa_index* index, int32_t batch,
                              int32_t top_k);

/* [A][B]: content K/V stay in host memory and are "fetched asynchronously
 * when selected".  Waits on the host for `sel_ready` (an event recorded after
 * msa_route wrote out_doc_idx_host) for at most timeout_ms milliseconds
 * (MSA_ERR_TIMEOUT past that; nothing is enqueued then), then enqueues on
 * fetch_stream one host-to-device copy per selected document into its
 * staging slot (b, r) = rows [(b*top_k + r) * 2 * max_doc_chunks, ...) and
 * records fetch_done (if not NULL) on fetch_stream.  Requires
 * index->kv_on_host. */
msa_status msa_fetch_selected(const msa_layout* layout, const msa_index* index, int32_t batch,
                              int32_t top_k, const int32_t* sel_idx_host, cudaEvent_t sel_ready,
                              int32_t timeout_ms, void* staging, size_t staging_bytes,
                              cudaStream_t fetch_stream, cudaEvent_t fetch_done);

/* The same fetch without the host in the loop: one kernel on `stream` reads
 * the selection from device memory (sel_idx, e.g. msa_route's out_doc_idx,
 * in stream order after the routing) and copies each selected document's K/V
 * rows from the host tier straight into its staging slot (the layout above),
 * reading the pinned host memory through its device mapping over the host
 * link.  Nothing waits on the host, so a layer that decodes right after its
 * own routing does not pay a device -> host -> device round trip; the
 * per-document cudaMemcpyAsync path above stays the default for fetches that
 * overlap the next layer's routing on a side stream.
 *   index->host_kv: page-locked host memory mapped for the device (memory
 *     from cudaHostAlloc, or cudaHostRegister with cudaHostRegisterMapped);
 *     checked at both ends before anything is launched (MSA_ERR_INVALID_ARG)
 *   sel_idx: (device) [batch][top_k]; a document out of range, or with more
 *     than max_doc_chunks chunks, raises MSA_DEV_BAD_DOC and its slot is not
 *     written
 *   staging: (device) msa_fetch_staging_size bytes, 16-byte aligned.
 * One launch, B * top_k CTAs; allocates nothing. */
msa_status msa_fetch_selected_device(const msa_layout* layout, const msa_index* index, int32_t batch,
                                     int32_t top_k, const int32_t* sel_idx, void* staging,
                                     size_t staging_bytes, cudaStream_t stream);

/* --------------------------------------------- stage 3: sparse decode */

/* Local key/value cache layout (msa_rope_local, msa_sparse_decode): query b
 * owns token rows [local_off_host[b], local_off_host[b+1]), laid out
 * [H_kv][cap_b][head_dim] with cap_b = local_off_host[b+1] - local_off_host[b];
 * its live tokens are the first len_b = local_len_host[b] of them (local_len_host
 * NULL: len_b = cap_b), so a cache can grow by appending tokens in place up to
 * its capacity.  Live tokens are the L_b context tokens, then the T query
 * tokens of the current call (L_b = len_b - T). */

/* Workspace bytes msa_sparse_decode needs for these local lengths.  The
 * workspace must be zero-filled before its first use with msa_sparse_decode
 * (it holds per-(query, kv head) completion counters that every call leaves at
 * zero again); calls that share one workspace must not overlap on the GPU. */
size_t msa_decode_workspace_size(const msa_layout* layout, int32_t batch, int32_t T,
                                 const int64_t* local_off_host, const int64_t* local_len_host);

/* [A][B] Global RoPE of the local context: writes the local keys in the
 * rotated form msa_sparse_decode reads.  For query b, kv head g and live
 * local token j in [first_host[b], len_b):
 *     dst[b][g][j] = RoPE(src[b][g][j], top_k + j)
 * (the local context starts after the k retrieved documents), fp32
 * arithmetic, rounded once to dtype.  A key cache calls it once per token as
 * the token is appended, e.g. first_host[b] = len_b - T for the T new tokens
 * of a decode step; rows before first_host[b] or past len_b are untouched.
 *   src, dst: (device) the local cache layout above; dst == src rotates in
 *     place, otherwise the two must not overlap
 *   local_off_host: (host) [batch + 1] row offsets (capacities)
 *   local_len_host: (host) [batch] live lengths <= capacity, or NULL (full)
 *   first_host: (host) [batch] first token to rotate per query; NULL = 0
 *   rope_table: (device) rope_rows >= top_k + max_b len_b */
msa_status msa_rope_local(const msa_layout* layout, int32_t batch, const int64_t* local_off_host,
                          const int64_t* local_len_host, const int64_t* first_host, int32_t top_k,
                          const void* src, void* dst, const float* rope_table, int32_t rope_rows,
                          cudaStream_t stream);

/* Appends one generated token per query to a local cache in one launch: the
 * token of query b goes to row len_b (local_len_host[b], the live length
 * before the append; it must be below the capacity) of each kv head --
 * its value into v, its key into k_raw (when not NULL) as given and into
 * k_rot as RoPE(key, top_k + len_b), the form msa_sparse_decode reads.
 *   k_new, v_new: (device) [batch][H_kv][head_dim] in dtype
 *   k_raw (or NULL), k_rot, v: (device) the local cache layout above
 *   rope_table: (device) rope_rows > top_k + max_b len_b
 * The caller then passes len_b + 1 as the live length. */
msa_status msa_append_local(const msa_layout* layout, int32_t batch, const int64_t* local_off_host,
                            const int64_t* local_len_host, const void* k_new, const void* v_new, int32_t top_k,
                            const float* rope_table, int32_t rope_rows, void* k_raw, void* k_rot, void* v,
                            cudaStream_t stream);

/* ---- live lengths in device memory (CUDA-graph replay of a decode loop)
 *
 * The calls below read the live lengths from device memory instead of the
 * host, so that their launch parameters stay the same from one generated
 * token to the next and a token's work (append, decode, for every layer) can
 * be captured once into a CUDA graph and replayed.
 *   local_len_dev: (device) [batch] int64 live lengths; msa_append_local_devlen
 *     writes row local_len_dev[b] (it must be below the capacity, else
 *     MSA_DEV_BAD_SHAPE and nothing is written), msa_sparse_decode_devlen
 *     attends over local_len_dev[b] tokens (clamped to [T, capacity] with
 *     MSA_DEV_BAD_SHAPE), msa_advance_local_len adds `by` to every entry.
 * The decode is planned for the capacities (msa_decode_workspace_size with
 * local_len_host = NULL gives its workspace); splits past a query's live
 * tokens do no work.  Other arguments as in msa_append_local and
 * msa_sparse_decode (no wait event: order the host-tier fetch before). */
msa_status msa_append_local_devlen(const msa_layout* layout, int32_t batch, const int64_t* local_off_host,
                                   const int64_t* local_len_dev, const void* k_new, const void* v_new,
                                   int32_t top_k, const float* rope_table, int32_t rope_rows, void* k_raw,
                                   void* k_rot, void* v, cudaStream_t stream);
msa_status msa_sparse_decode_devlen(const msa_layout* layout, const msa_index* index, int32_t batch, int32_t T,
                                    const void* q, const void* local_k, const void* local_v,
                                    const int64_t* local_off_host, const int64_t* local_len_dev,
                                    const int32_t* sel_idx, int32_t top_k, const void* mem_staging,
                                    const float* rope_table, int32_t rope_rows, void* out, void* ws,
                                    size_t ws_bytes, cudaStream_t stream);
msa_status msa_advance_local_len(int32_t batch, int64_t* local_len_dev, int64_t by, cudaStream_t stream);

/* In short: msa_sparse_decode reads local keys ALREADY ROTATED at top_k + j
 * (a key cache written by msa_rope_local or msa_append_local); for keys as
 * they come from the projection, use msa_sparse_decode_raw below.
 *
 * [A][B] "Sparse Generation": for query b, query token t, query head h
 * (kv head g = h / G) the keys are
 *   [ pooled K of the selected documents' chunks, rank order, chunk order ]
 *   ++ [ RoPE(local token j's key, top_k + j) for j = 0 .. L_b + t ]
 * and the query is RoPE(q[b][t][h], top_k + L_b + t): the global RoPE start
 * is offset by k, the number of retrieved documents, keeping the order
 * memory -> local context -> generated tokens.  Pooled keys keep the
 * document-local rotation they received in stage 1; local keys arrive
 * rotated, as msa_rope_local writes them.  out = softmax(q.k / sqrt(head_dim))
 * weighted sum of [pooled V ++ local V], fp32 accumulation, rounded once to
 * dtype (bf16 banks: the rotated query and the softmax weights enter the
 * tensor-core products as bf16).
 *   q: (device) [batch][T][H_q][head_dim], unrotated
 *   local_k, local_v: (device) the local cache layout above, live length
 *     len_b = L_b + T (its L_b context tokens, then its T query tokens' own
 *     K/V); local_k rotated by msa_rope_local
 *   local_off_host: (host) [batch + 1] row offsets (capacities)
 *   local_len_host: (host) [batch] live lengths, T <= len_b <= cap_b, or NULL
 *   sel_idx: (device) [batch][top_k] selected documents (msa_route output)
 *   mem_staging: (device) staging buffer filled by msa_fetch_selected when
 *     index->kv_on_host, else NULL
 *   rope_table: (device) rope_rows >= top_k + max_b len_b
 *   wait_event: if not NULL, `stream` waits for it first (e.g. fetch_done)
 *   out: (device) [batch][T][H_q][head_dim]
 *   batch <= 256. */
msa_status msa_sparse_decode(const msa_layout* layout, const msa_index* index, int32_t batch,
                             int32_t T, const void* q, const void* local_k, const void* local_v,
                             const int64_t* local_off_host, const int64_t* local_len_host,
                             const int32_t* sel_idx,
                             int32_t top_k, const void* mem_staging, const float* rope_table,
                             int32_t rope_rows, void* out, void* ws, size_t ws_bytes,
                             cudaEvent_t wait_event, cudaStream_t stream);

/* Workspace bytes of msa_sparse_decode_raw: the decode's own workspace, a
 * rotated copy of the local keys ([capacity rows][H_kv][head_dim] in dtype)
 * and, for a host-tier bank, the staging of the selected documents.  0 when
 * the arguments are rejected. */
size_t msa_sparse_decode_raw_workspace_size(const msa_layout* layout, const msa_index* index, int32_t batch,
                                            int32_t T, int32_t top_k, const int64_t* local_off_host,
                                            const int64_t* local_len_host);

/* [A][B] stage 3 in one call, in the form the pages state it: the local keys
 * are the raw (unrotated) keys of the L_b context tokens and the T query
 * tokens, and for a host-tier bank the selected documents' K/V are fetched
 * inside the call.  On `stream`, with no host wait: the host-tier fetch by
 * one kernel reading the selection on the device (msa_fetch_selected_device),
 * the rotation of every live local key at top_k + j into the workspace
 * (msa_rope_local), then msa_sparse_decode on that copy -- the same
 * arithmetic and output as msa_rope_local + msa_sparse_decode.  It writes and
 * reads the local keys once more per call than a decode loop that keeps a
 * rotated key cache and rotates only each step's new tokens.
 *   local_k_raw, local_v: (device) the local cache layout above, keys unrotated
 *   ws: msa_sparse_decode_raw_workspace_size bytes, zero-filled before its
 *     first use (it starts with the decode's completion counters); calls that
 *     share it must not overlap on the GPU.
 *   host-tier banks: index->host_kv page-locked and mapped for the device.
 * Other arguments as in msa_sparse_decode. */
msa_status msa_sparse_decode_raw(const msa_layout* layout, const msa_index* index, int32_t batch, int32_t T,
                                 const void* q, const void* local_k_raw, const void* local_v,
                                 const int64_t* local_off_host, const int64_t* local_len_host,
                                 const int32_t* sel_idx, int32_t top_k, const float* rope_table, int32_t rope_rows,
                                 void* out, void* ws, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------ training-time routing layer */

/* [A] "How MSA compresses and routes documents" and "MSA against a
 * conventional RAG stack": routing and generation are trained end to end;
 * [B] "Implementation Details": continued pre-training adds an auxiliary
 * routing loss.  Neither gives a formula; the readings implemented here:
 * the layer's forward is the inference forward (route, top_k selection with
 * no gradient, sparse attention over [selected pooled K/V ++ local K/V] with
 * the global RoPE offset top_k); the router score is differentiable (through
 * the query token and chunk that maximise it) and trained by
 *     loss_b = logsumexp_d(S_d / tau) - logsumexp_{d in P_b}(S_d / tau),
 * the cross-entropy of a softmax over all documents against the query's set
 * P_b of relevant documents.  Training banks are device-tier. */

/* msa_sparse_decode plus the per-row log-sum-exp the backward needs:
 * lse (device) [batch][T][H_q] float, natural log of sum_j exp(q~ . k_j /
 * sqrt(head_dim)) over the keys the row sees.  Host-tier banks:
 * MSA_ERR_UNSUPPORTED. */
msa_status msa_sparse_attention_forward(const msa_layout* layout, const msa_index* index, int32_t batch,
                                        int32_t T, const void* q, const void* local_k, const void* local_v,
                                        const int64_t* local_off_host, const int64_t* local_len_host,
                                        const int32_t* sel_idx, int32_t top_k, const float* rope_table,
                                        int32_t rope_rows, void* out, float* lse, void* ws, size_t ws_bytes,
                                        cudaStream_t stream);

/* Workspace bytes of msa_sparse_attention_backward. */
size_t msa_attention_backward_workspace_size(const msa_layout* layout, int32_t batch, int32_t T);

/* Gradients of the sparse attention given dout = dL/dout, from the forward's
 * inputs, its output `out` and `lse`:
 *   d_q: (device) [batch][T][H_q][head_dim] float, overwritten: w.r.t. the
 *     unrotated query q;
 *   d_mem_k, d_mem_v: (device) [n_chunks][H_kv][head_dim] float, ADDED to:
 *     w.r.t. the bank's pooled K (as stored, with its document-local
 *     rotation) and V, on the chunks of the selected documents (a chunk two
 *     queries selected gets both contributions);
 *   d_local_k, d_local_v: (device) float, the local cache layout
 *     ([H_kv][capacity][head_dim] per query), live rows overwritten: w.r.t.
 *     the unrotated local keys (the rotation at top_k + j is undone) and the
 *     local values.
 * local_k is the rotated key cache the forward read (msa_rope_local).
 * Arithmetic: fp32 on fp32 copies of the tiles; batch 1..256; head_dim 64
 * or 128; the index needs max_doc_chunks.  The selected documents' chunk
 * total above top_k * max_doc_chunks raises MSA_DEV_BAD_SHAPE. */
msa_status msa_sparse_attention_backward(const msa_layout* layout, const msa_index* index, int32_t batch,
                                         int32_t T, const void* q, const void* local_k, const void* local_v,
                                         const int64_t* local_off_host, const int64_t* local_len_host,
                                         const int32_t* sel_idx, int32_t top_k, const float* rope_table,
                                         int32_t rope_rows, const void* out, const float* lse, const void* dout,
                                         float* d_q, float* d_mem_k, float* d_mem_v, float* d_local_k,
                                         float* d_local_v, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes of the routing loss; the forward's workspace must reach
 * the backward unchanged (it keeps the scores and their maximisers). */
size_t msa_route_loss_workspace_size(const msa_layout* layout, const msa_index* index, int32_t batch, int32_t T);

/* The auxiliary routing loss of `batch` queries of T tokens (qr as in
 * msa_route).  Scores in fp32: S_d = max over t and the document's chunks c
 * of (1/H_q) sum_h cos(Qr[t,h], Kr[c, h/G]) (norms clamped at 1e-12; the
 * clamp of each cosine to [-1, 1] acts only on rounding excess and is left
 * out).
 *   pos_off: (device) [batch + 1] int32, pos_doc: (device) the relevant
 *     documents of query b at [pos_off[b], pos_off[b+1]); at least one each
 *     (MSA_DEV_BAD_SHAPE otherwise);
 *   tau > 0; loss: (device) [batch] float; doc_score: (device) [batch][n_docs]
 *     float or NULL.  router_dim <= 128. */
msa_status msa_route_loss_forward(const msa_layout* layout, const msa_index* index, int32_t batch, int32_t T,
                                  const void* qr, const int32_t* pos_off, const int32_t* pos_doc, float tau,
                                  float* loss, float* doc_score, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Gradients of sum_b d_loss[b] * loss_b:
 *   d_qr: (device) [batch][T][H_q][router_dim] float, overwritten;
 *   d_kr: (device) [n_chunks][H_kv][router_dim] float, ADDED to (only the
 *     maximising chunk of each document receives a gradient). */
msa_status msa_route_loss_backward(const msa_layout* layout, const msa_index* index, int32_t batch, int32_t T,
                                   const void* qr, const int32_t* pos_off, const int32_t* pos_doc, float tau,
                                   const float* d_loss, float* d_qr, float* d_kr, void* ws, size_t ws_bytes,
                                   cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MSA_H */
