// Streaming offline encoding: a bank built batch by batch from per-token
// K/V/Kr that need not fit on the GPU together.
//
// "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts", section
// "How MSA compresses and routes documents": the pooled triples are cached
// offline by one pass over the corpus; the content K/V of a 100M-token memory
// lives in host memory and only the router keys stay on the GPU.
//
// Pipeline: three streams and two device slots.  Batch i's inputs are copied
// in on `in` while batch i-1 is encoded on `run` and batch i-2's pooled K/V
// go back to host memory on `out`.  Cross-stream order is kept with events:
//   copy-in of slot s    waits for the last encode that read slot s;
//   encode of slot s     waits for its copy-in and (host tier) the copy-out
//                        that last read slot s's pooled rows;
//   copy-out of slot s   waits for its encode.
// The host waits only when it reuses a slot's pinned CSR staging (whose
// previous copy-in finished long before) and, per the push contract, for the
// previous batch's copy-in, so the caller can double-buffer its inputs.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <string>
#include <vector>

#include "api_internal.h"
#include "msa.h"

using namespace msa_host;

struct msa_encoder {
  msa_layout L{};
  int64_t max_tok = 0, max_docs = 0, max_doc_len = 0, cap = 0, slot_chunks = 0;
  void* kr_out = nullptr;
  void* k_out = nullptr;
  void* v_out = nullptr;
  void* host_kv = nullptr;
  bool host_tier = false;
  float* rope = nullptr;
  int dev = 0;
  cudaStream_t in = nullptr, run = nullptr, out = nullptr;
  struct Slot {
    char* tok = nullptr;           // device: K rows, V rows, Kr rows of one batch
    int64_t* csr_dev = nullptr;    // device: token CSR [max_docs + 1], chunk CSR [max_docs + 1]
    int64_t* csr_host = nullptr;   // pinned staging of the two CSRs
    char* kv = nullptr;            // device: pooled K/V in host-tier rows (host tier only)
    cudaEvent_t in_done = nullptr, run_done = nullptr, out_done = nullptr;
    bool used = false;
  } slot[2];
  int next = 0;
  cudaEvent_t prev_in = nullptr;   // copy-in of the previous push
  std::vector<int64_t> chunk_off{0};
  int64_t n_chunks = 0;
  int32_t max_doc_chunks = 0;
  msa_status sticky = MSA_OK;      // first failure; every later call returns it
  std::string sticky_msg;
};

namespace {

int64_t row_k(const msa_layout& L) { return (int64_t)L.n_kv_heads * L.head_dim * esize(&L); }
int64_t row_r(const msa_layout& L) { return (int64_t)L.n_kv_heads * L.router_dim * esize(&L); }

msa_status stick(msa_encoder* e, msa_status s) {
  if (s != MSA_OK && e->sticky == MSA_OK) {
    e->sticky = s;
    e->sticky_msg = msa_last_error();
  }
  return s;
}

msa_status sticky_error(const msa_encoder* e) {
  return fail(e->sticky, "encoder stopped by an earlier error: %s", e->sticky_msg.c_str());
}

#define ENC_CUDA(call, what)                                   \
  do {                                                         \
    cudaError_t e_ = (call);                                   \
    if (e_ != cudaSuccess) return stick(enc, cuda_fail(e_, what)); \
  } while (0)

void release(msa_encoder* e) {
  cudaSetDevice(e->dev);
  for (cudaStream_t s : {e->in, e->run, e->out})
    if (s) cudaStreamSynchronize(s);
  for (auto& sl : e->slot) {
    cudaFree(sl.tok);
    cudaFree(sl.csr_dev);
    cudaFree(sl.kv);
    cudaFreeHost(sl.csr_host);
    for (cudaEvent_t ev : {sl.in_done, sl.run_done, sl.out_done})
      if (ev) cudaEventDestroy(ev);
  }
  cudaFree(e->rope);
  for (cudaStream_t s : {e->in, e->run, e->out})
    if (s) cudaStreamDestroy(s);
}

}  // namespace

extern "C" {

msa_status msa_encoder_create(const msa_layout* L, int64_t max_tok, int32_t max_docs, int64_t max_doc_len,
                              int64_t cap, void* kr_out, void* k_out, void* v_out, void* host_kv,
                              msa_encoder** out) {
  msa_status s = check_layout(L);
  if (s) return s;
  if (!out) return fail(MSA_ERR_INVALID_ARG, "encoder: out is NULL");
  *out = nullptr;
  if (max_tok <= 0 || max_docs <= 0 || max_doc_len <= 0 || cap <= 0)
    return fail(MSA_ERR_INVALID_ARG, "encoder: max_batch_tokens %lld, max_batch_docs %d, max_doc_len %lld, "
                "capacity %lld must be positive", (long long)max_tok, max_docs, (long long)max_doc_len,
                (long long)cap);
  if (max_doc_len > INT32_MAX) return fail(MSA_ERR_UNSUPPORTED, "max_doc_len %lld", (long long)max_doc_len);
  if (!kr_out || !aligned16(kr_out)) return fail(MSA_ERR_INVALID_ARG, "encoder: kr_out NULL or not 16-byte aligned");
  const bool host_tier = host_kv != nullptr;
  if (host_tier && (k_out || v_out))
    return fail(MSA_ERR_INVALID_ARG, "encoder: give host_kv_out or k_out and v_out, not both");
  if (!host_tier && (!k_out || !v_out || !aligned16(k_out) || !aligned16(v_out)))
    return fail(MSA_ERR_INVALID_ARG, "encoder: k_out and v_out (device, 16-byte aligned) are required");
  auto* e = new msa_encoder;
  e->L = *L;
  e->max_tok = max_tok; e->max_docs = max_docs; e->max_doc_len = max_doc_len; e->cap = cap;
  e->slot_chunks = max_tok / L->chunk_size + max_docs;   // sum of ceil(len / chunk) over the batch
  e->kr_out = kr_out; e->k_out = k_out; e->v_out = v_out; e->host_kv = host_kv; e->host_tier = host_tier;
  cudaGetDevice(&e->dev);
  auto bail = [&](msa_status st) { release(e); delete e; return st; };
  const int64_t tok_bytes = max_tok * (2 * row_k(*L) + row_r(*L));
  cudaError_t ce = cudaSuccess;
  for (cudaStream_t* st : {&e->in, &e->run, &e->out})
    if (ce == cudaSuccess) ce = cudaStreamCreateWithFlags(st, cudaStreamNonBlocking);
  for (auto& sl : e->slot) {
    if (ce == cudaSuccess) ce = cudaMalloc(&sl.tok, (size_t)tok_bytes);
    if (ce == cudaSuccess) ce = cudaMalloc(&sl.csr_dev, sizeof(int64_t) * 2 * (size_t)(max_docs + 1));
    if (ce == cudaSuccess) ce = cudaHostAlloc(&sl.csr_host, sizeof(int64_t) * 2 * (size_t)(max_docs + 1), 0);
    if (ce == cudaSuccess && host_tier) ce = cudaMalloc(&sl.kv, (size_t)(2 * e->slot_chunks * row_k(*L)));
    for (cudaEvent_t* ev : {&sl.in_done, &sl.run_done, &sl.out_done})
      if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  }
  if (ce == cudaSuccess) ce = cudaMalloc(&e->rope, sizeof(float) * (size_t)max_doc_len * L->head_dim);
  if (ce != cudaSuccess) return bail(cuda_fail(ce, "encoder: allocate staging"));
  if ((s = msa_rope_table(L, (int32_t)max_doc_len, e->rope, e->run))) return bail(s);
  *out = e;
  return MSA_OK;
}

msa_status msa_encoder_push(msa_encoder* enc, int32_t n, const int64_t* tok, const void* k_tok, const void* v_tok,
                            const void* kr_tok) {
  NvtxRange nvtx_("msa_encoder_push");
  if (!enc) return fail(MSA_ERR_INVALID_ARG, "encoder is NULL");
  if (enc->sticky) return sticky_error(enc);
  const msa_layout& L = enc->L;
  if (n <= 0 || n > enc->max_docs) return fail(MSA_ERR_INVALID_ARG, "push: %d documents (1..%lld)", n,
                                               (long long)enc->max_docs);
  if (!tok || !k_tok || !v_tok || !kr_tok) return fail(MSA_ERR_INVALID_ARG, "push: missing pointer");
  if (!aligned16(k_tok) || !aligned16(v_tok) || !aligned16(kr_tok))
    return fail(MSA_ERR_INVALID_ARG, "push: inputs must be 16-byte aligned");
  if (tok[0] != 0) return fail(MSA_ERR_INVALID_ARG, "push: doc_tok_off_host[0] must be 0");
  int64_t C = 0;
  int32_t max_ch = 0;
  for (int i = 0; i < n; ++i) {
    const int64_t len = tok[i + 1] - tok[i];
    if (len < 1 || len > enc->max_doc_len)
      return fail(MSA_ERR_INVALID_ARG, "push: document %d has %lld tokens (1..%lld)", i, (long long)len,
                  (long long)enc->max_doc_len);
    const int64_t ch = (len + L.chunk_size - 1) / L.chunk_size;
    C += ch;
    max_ch = std::max<int32_t>(max_ch, (int32_t)ch);
  }
  const int64_t N = tok[n];
  if (N > enc->max_tok) return fail(MSA_ERR_INVALID_ARG, "push: %lld tokens > max_batch_tokens %lld", (long long)N,
                                    (long long)enc->max_tok);
  if (enc->n_chunks + C > enc->cap)
    return fail(MSA_ERR_INVALID_ARG, "push: %lld pooled chunks would exceed the capacity %lld",
                (long long)(enc->n_chunks + C), (long long)enc->cap);
  ENC_CUDA(cudaSetDevice(enc->dev), "push: set device");
  // the caller may now reuse the previous push's inputs
  if (enc->prev_in) ENC_CUDA(cudaEventSynchronize(enc->prev_in), "push: previous copy-in");
  auto& sl = enc->slot[enc->next];
  if (sl.used) ENC_CUDA(cudaEventSynchronize(sl.in_done), "push: slot copy-in");
  int64_t* ht = sl.csr_host;
  int64_t* hc = sl.csr_host + (enc->max_docs + 1);
  hc[0] = 0;
  for (int i = 0; i < n; ++i) {
    ht[i] = tok[i];
    hc[i + 1] = hc[i] + (tok[i + 1] - tok[i] + L.chunk_size - 1) / L.chunk_size;
  }
  ht[n] = tok[n];
  const int64_t rk = row_k(L), rr = row_r(L);
  char* dk = sl.tok;
  char* dv = dk + enc->max_tok * rk;
  char* dr = dv + enc->max_tok * rk;
  int64_t* dt = sl.csr_dev;
  int64_t* dc = sl.csr_dev + (enc->max_docs + 1);
  // copy in (after the last encode that read this slot)
  if (sl.used) ENC_CUDA(cudaStreamWaitEvent(enc->in, sl.run_done, 0), "push: order copy-in");
  ENC_CUDA(cudaMemcpyAsync(dt, ht, sizeof(int64_t) * (size_t)(n + 1), cudaMemcpyHostToDevice, enc->in), "copy CSR");
  ENC_CUDA(cudaMemcpyAsync(dc, hc, sizeof(int64_t) * (size_t)(n + 1), cudaMemcpyHostToDevice, enc->in), "copy CSR");
  ENC_CUDA(cudaMemcpyAsync(dk, k_tok, (size_t)(N * rk), cudaMemcpyDefault, enc->in), "copy K");
  ENC_CUDA(cudaMemcpyAsync(dv, v_tok, (size_t)(N * rk), cudaMemcpyDefault, enc->in), "copy V");
  ENC_CUDA(cudaMemcpyAsync(dr, kr_tok, (size_t)(N * rr), cudaMemcpyDefault, enc->in), "copy Kr");
  ENC_CUDA(cudaEventRecord(sl.in_done, enc->in), "record copy-in");
  // encode
  ENC_CUDA(cudaStreamWaitEvent(enc->run, sl.in_done, 0), "order encode");
  if (enc->host_tier && sl.used) ENC_CUDA(cudaStreamWaitEvent(enc->run, sl.out_done, 0), "order encode");
  char* kr_dst = static_cast<char*>(enc->kr_out) + enc->n_chunks * rr;
  msa_status s;
  if (enc->host_tier) {
    s = msa_encode_memory_kv_interleaved(&L, n, C, dt, dc, enc->max_doc_len, dk, dv, dr, enc->rope,
                                         (int32_t)enc->max_doc_len, sl.kv, kr_dst, enc->run);
  } else {
    s = msa_encode_memory(&L, n, C, dt, dc, enc->max_doc_len, dk, dv, dr, enc->rope, (int32_t)enc->max_doc_len,
                          static_cast<char*>(enc->k_out) + enc->n_chunks * rk,
                          static_cast<char*>(enc->v_out) + enc->n_chunks * rk, kr_dst, enc->run);
  }
  if (s) return stick(enc, s);
  ENC_CUDA(cudaEventRecord(sl.run_done, enc->run), "record encode");
  // copy out (host tier): the batch's rows are contiguous in host_kv
  if (enc->host_tier) {
    ENC_CUDA(cudaStreamWaitEvent(enc->out, sl.run_done, 0), "order copy-out");
    ENC_CUDA(cudaMemcpyAsync(static_cast<char*>(enc->host_kv) + 2 * enc->n_chunks * rk, sl.kv, (size_t)(2 * C * rk),
                             cudaMemcpyDeviceToHost, enc->out), "copy K/V out");
    ENC_CUDA(cudaEventRecord(sl.out_done, enc->out), "record copy-out");
  }
  sl.used = true;
  enc->prev_in = sl.in_done;
  enc->next ^= 1;
  for (int i = 0; i < n; ++i) enc->chunk_off.push_back(enc->n_chunks + hc[i + 1]);
  enc->n_chunks += C;
  enc->max_doc_chunks = std::max(enc->max_doc_chunks, max_ch);
  return MSA_OK;
}

msa_status msa_encoder_finish(msa_encoder* enc, int64_t* n_docs, int64_t* n_chunks, int32_t* max_doc_chunks) {
  NvtxRange nvtx_("msa_encoder_finish");
  if (!enc) return fail(MSA_ERR_INVALID_ARG, "encoder is NULL");
  if (enc->sticky) return sticky_error(enc);
  ENC_CUDA(cudaSetDevice(enc->dev), "finish: set device");
  for (cudaStream_t st : {enc->in, enc->run, enc->out}) ENC_CUDA(cudaStreamSynchronize(st), "finish: wait");
  if (n_docs) *n_docs = (int64_t)enc->chunk_off.size() - 1;
  if (n_chunks) *n_chunks = enc->n_chunks;
  if (max_doc_chunks) *max_doc_chunks = enc->max_doc_chunks;
  return MSA_OK;
}

msa_status msa_encoder_chunk_offsets(const msa_encoder* enc, int64_t* out) {
  if (!enc || !out) return fail(MSA_ERR_INVALID_ARG, "chunk_offsets: NULL argument");
  std::memcpy(out, enc->chunk_off.data(), sizeof(int64_t) * enc->chunk_off.size());
  return MSA_OK;
}

void msa_encoder_destroy(msa_encoder* enc) {
  if (!enc) return;
  release(enc);
  delete enc;
}

}  // extern "C"
