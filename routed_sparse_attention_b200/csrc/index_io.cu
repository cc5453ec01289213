// Persistent pooled index: a bank written to one file and read back, so the
// offline encoding ("EverMind-AI/MSA: Memory Sparse Attention for 100M-Token
// Contexts", section "How MSA compresses and routes documents": the pooled
// triples are cached offline) runs once per corpus.  The file format and the
// msa64 hash are specified in include/msa.h.
//
// Device sections move through two pinned bounce buffers: the copy of one
// piece overlaps the hashing and file I/O of the other.  Host sections (the
// CSR, a host-tier K/V array, host destinations) are read or written in place.
#include <cuda_runtime.h>
#include <unistd.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "api_internal.h"
#include "msa.h"

using namespace msa_host;

namespace {

constexpr uint64_t kM1 = 0x9E3779B97F4A7C15ull, kM2 = 0xD6E8FEB86659FD93ull;
constexpr int64_t kSectionAlign = 4096;
constexpr size_t kPiece = (size_t)64 << 20;   // bounce buffer size (a multiple of 32 bytes)
constexpr char kMagic[8] = {'M', 'S', 'A', 'I', 'D', 'X', '0', '1'};
constexpr uint32_t kVersion = 1;
constexpr int kSections = 4;

inline uint64_t rotl(uint64_t x, int r) { return (x << r) | (x >> (64 - r)); }

// Incremental msa64: four multiply-rotate lanes over little-endian u64 words.
struct Msa64 {
  uint64_t h[4] = {kM2, 2 * kM2, 3 * kM2, 4 * kM2};
  uint64_t bytes = 0, words = 0;
  unsigned char tail[8];
  int nt = 0;

  void word(uint64_t w) {
    uint64_t& x = h[words & 3];
    x = rotl(x ^ (w * kM1), 29) * kM2;
    ++words;
  }
  void update(const void* p, size_t n) {
    const unsigned char* c = static_cast<const unsigned char*>(p);
    bytes += n;
    while (nt && n) {                       // finish a pending partial word
      tail[nt++] = *c++;
      --n;
      if (nt == 8) { uint64_t w; std::memcpy(&w, tail, 8); word(w); nt = 0; }
    }
    while (n >= 8 && (words & 3)) { uint64_t w; std::memcpy(&w, c, 8); word(w); c += 8; n -= 8; }
    uint64_t a = h[0], b = h[1], d = h[2], e = h[3];
    while (n >= 32) {                       // four lanes, one word each
      uint64_t w[4];
      std::memcpy(w, c, 32);
      a = rotl(a ^ (w[0] * kM1), 29) * kM2;
      b = rotl(b ^ (w[1] * kM1), 29) * kM2;
      d = rotl(d ^ (w[2] * kM1), 29) * kM2;
      e = rotl(e ^ (w[3] * kM1), 29) * kM2;
      c += 32; n -= 32; words += 4;
    }
    h[0] = a; h[1] = b; h[2] = d; h[3] = e;
    while (n >= 8) { uint64_t w; std::memcpy(&w, c, 8); word(w); c += 8; n -= 8; }
    while (n) { tail[nt++] = *c++; --n; }
  }
  uint64_t final() const {
    Msa64 t = *this;
    if (t.nt) {
      std::memset(t.tail + t.nt, 0, 8 - t.nt);
      uint64_t w;
      std::memcpy(&w, t.tail, 8);
      t.word(w);
    }
    uint64_t r = bytes;
    for (int j = 0; j < 4; ++j) r = rotl(r ^ (t.h[j] * kM1), 31) * kM2;
    r ^= r >> 33;
    r *= kM1;
    r ^= r >> 29;
    return r;
  }
};

uint64_t msa64(const void* p, size_t n) {
  Msa64 m;
  m.update(p, n);
  return m.final();
}

struct Header {
  msa_layout L{};
  int64_t n_docs = 0, n_chunks = 0;
  int32_t max_doc_chunks = 0, kv_on_host = 0;
  uint64_t off[kSections] = {}, bytes[kSections] = {}, hash[kSections] = {};
};

template <typename T>
void put(unsigned char* b, int at, T v) { std::memcpy(b + at, &v, sizeof v); }
template <typename T>
T get(const unsigned char* b, int at) { T v; std::memcpy(&v, b + at, sizeof v); return v; }

void encode_header(const Header& h, unsigned char* b) {
  std::memset(b, 0, MSA_INDEX_HEADER_BYTES);
  std::memcpy(b, kMagic, 8);
  put<uint32_t>(b, 8, kVersion);
  put<uint32_t>(b, 12, MSA_INDEX_HEADER_BYTES);
  const int32_t f[6] = {h.L.n_q_heads, h.L.n_kv_heads, h.L.head_dim, h.L.router_dim, h.L.chunk_size, h.L.dtype};
  for (int i = 0; i < 6; ++i) put<int32_t>(b, 16 + 4 * i, f[i]);
  put<double>(b, 40, h.L.rope_theta);
  put<int64_t>(b, 48, h.n_docs);
  put<int64_t>(b, 56, h.n_chunks);
  put<int32_t>(b, 64, h.max_doc_chunks);
  put<int32_t>(b, 68, h.kv_on_host);
  for (int s = 0; s < kSections; ++s) {
    put<uint64_t>(b, 72 + 24 * s, h.off[s]);
    put<uint64_t>(b, 80 + 24 * s, h.bytes[s]);
    put<uint64_t>(b, 88 + 24 * s, h.hash[s]);
  }
  put<uint64_t>(b, 504, msa64(b, 504));
}

int64_t row_bytes(const msa_layout& L, int dim) { return (int64_t)L.n_kv_heads * dim * esize(&L); }

// Section sizes implied by the layout and counts.
void section_sizes(Header& h) {
  h.bytes[0] = sizeof(int64_t) * (uint64_t)(h.n_docs + 1);
  h.bytes[1] = (uint64_t)(h.n_chunks * row_bytes(h.L, h.L.router_dim));
  const uint64_t kv = (uint64_t)(h.n_chunks * row_bytes(h.L, h.L.head_dim));
  h.bytes[2] = h.kv_on_host ? 2 * kv : kv;
  h.bytes[3] = h.kv_on_host ? 0 : kv;
  uint64_t at = kSectionAlign;
  for (int s = 0; s < kSections; ++s) {
    h.off[s] = at;
    at = (at + h.bytes[s] + kSectionAlign - 1) / kSectionAlign * kSectionAlign;
  }
}

msa_status decode_header(const unsigned char* b, Header* h) {
  if (std::memcmp(b, kMagic, 8) != 0) return fail(MSA_ERR_INVALID_ARG, "index file: bad magic");
  if (get<uint32_t>(b, 8) != kVersion) return fail(MSA_ERR_UNSUPPORTED, "index file: version %u", get<uint32_t>(b, 8));
  if (get<uint32_t>(b, 12) != MSA_INDEX_HEADER_BYTES) return fail(MSA_ERR_INVALID_ARG, "index file: header size");
  if (get<uint64_t>(b, 504) != msa64(b, 504)) return fail(MSA_ERR_INVALID_ARG, "index file: header checksum mismatch");
  h->L.n_q_heads = get<int32_t>(b, 16);
  h->L.n_kv_heads = get<int32_t>(b, 20);
  h->L.head_dim = get<int32_t>(b, 24);
  h->L.router_dim = get<int32_t>(b, 28);
  h->L.chunk_size = get<int32_t>(b, 32);
  h->L.dtype = get<int32_t>(b, 36);
  h->L.rope_theta = get<double>(b, 40);
  h->n_docs = get<int64_t>(b, 48);
  h->n_chunks = get<int64_t>(b, 56);
  h->max_doc_chunks = get<int32_t>(b, 64);
  h->kv_on_host = get<int32_t>(b, 68);
  msa_status s = check_layout(&h->L);
  if (s) return s;
  if (h->n_docs <= 0 || h->n_chunks < h->n_docs || h->max_doc_chunks <= 0 || (h->kv_on_host & ~1))
    return fail(MSA_ERR_INVALID_ARG, "index file: bad counts");
  Header want = *h;
  section_sizes(want);
  for (int i = 0; i < kSections; ++i) {
    h->off[i] = get<uint64_t>(b, 72 + 24 * i);
    h->bytes[i] = get<uint64_t>(b, 80 + 24 * i);
    h->hash[i] = get<uint64_t>(b, 88 + 24 * i);
    if (h->off[i] != want.off[i] || h->bytes[i] != want.bytes[i])
      return fail(MSA_ERR_INVALID_ARG, "index file: section %d placement does not match the counts", i);
  }
  return MSA_OK;
}

bool is_device(const void* p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) { cudaGetLastError(); return false; }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

struct Bounce {
  void* buf[2] = {nullptr, nullptr};
  cudaEvent_t ev[2] = {nullptr, nullptr};
  ~Bounce() {
    for (int i = 0; i < 2; ++i) {
      if (ev[i]) { cudaEventSynchronize(ev[i]); cudaEventDestroy(ev[i]); }
      if (buf[i]) cudaFreeHost(buf[i]);
    }
  }
  cudaError_t init() {
    for (int i = 0; i < 2; ++i) {
      cudaError_t e = cudaHostAlloc(&buf[i], kPiece, 0);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
};

struct File {
  FILE* f = nullptr;
  ~File() { if (f) fclose(f); }
};

// Writes `bytes` from src (device or host) at the file's current position.
msa_status write_section(FILE* f, const void* src, uint64_t bytes, Bounce& bo, cudaStream_t st, uint64_t* hash) {
  Msa64 m;
  if (!is_device(src)) {
    const char* p = static_cast<const char*>(src);
    for (uint64_t at = 0; at < bytes; at += kPiece) {
      const size_t n = (size_t)std::min<uint64_t>(kPiece, bytes - at);
      m.update(p + at, n);
      if (fwrite(p + at, 1, n, f) != n) return fail(MSA_ERR_INTERNAL, "index file: write failed");
    }
  } else {
    const char* p = static_cast<const char*>(src);
    const uint64_t pieces = (bytes + kPiece - 1) / kPiece;
    auto piece_n = [&](uint64_t i) { return (size_t)std::min<uint64_t>(kPiece, bytes - i * kPiece); };
    for (uint64_t i = 0; i <= pieces; ++i) {
      if (i < pieces) {     // start piece i while piece i-1 is hashed and written
        cudaError_t e = cudaMemcpyAsync(bo.buf[i & 1], p + i * kPiece, piece_n(i), cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaEventRecord(bo.ev[i & 1], st);
        if (e != cudaSuccess) return cuda_fail(e, "index file: copy to host");
      }
      if (i > 0) {
        const uint64_t j = i - 1;
        cudaError_t e = cudaEventSynchronize(bo.ev[j & 1]);
        if (e != cudaSuccess) return cuda_fail(e, "index file: copy to host");
        m.update(bo.buf[j & 1], piece_n(j));
        if (fwrite(bo.buf[j & 1], 1, piece_n(j), f) != piece_n(j))
          return fail(MSA_ERR_INTERNAL, "index file: write failed");
      }
    }
  }
  *hash = m.final();
  return MSA_OK;
}

// Reads `bytes` at the file's current position into dst (device or host).
msa_status read_section(FILE* f, void* dst, uint64_t bytes, Bounce& bo, cudaStream_t st, uint64_t* hash) {
  Msa64 m;
  if (!is_device(dst)) {
    char* p = static_cast<char*>(dst);
    for (uint64_t at = 0; at < bytes; at += kPiece) {
      const size_t n = (size_t)std::min<uint64_t>(kPiece, bytes - at);
      if (fread(p + at, 1, n, f) != n) return fail(MSA_ERR_INVALID_ARG, "index file: truncated");
      m.update(p + at, n);
    }
  } else {
    char* p = static_cast<char*>(dst);
    bool used[2] = {false, false};
    for (uint64_t at = 0, i = 0; at < bytes; at += kPiece, ++i) {
      const size_t n = (size_t)std::min<uint64_t>(kPiece, bytes - at);
      if (used[i & 1]) {    // the copy that last read this buffer must be done
        cudaError_t e = cudaEventSynchronize(bo.ev[i & 1]);
        if (e != cudaSuccess) return cuda_fail(e, "index file: copy to device");
      }
      if (fread(bo.buf[i & 1], 1, n, f) != n) return fail(MSA_ERR_INVALID_ARG, "index file: truncated");
      m.update(bo.buf[i & 1], n);
      cudaError_t e = cudaMemcpyAsync(p + at, bo.buf[i & 1], n, cudaMemcpyHostToDevice, st);
      if (e == cudaSuccess) e = cudaEventRecord(bo.ev[i & 1], st);
      if (e != cudaSuccess) return cuda_fail(e, "index file: copy to device");
      used[i & 1] = true;
    }
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "index file: copy to device");
  }
  *hash = m.final();
  return MSA_OK;
}

msa_status pad_to(FILE* f, uint64_t off) {
  const long at = ftell(f);
  if (at < 0 || (uint64_t)at > off) return fail(MSA_ERR_INTERNAL, "index file: bad position");
  static const unsigned char zero[kSectionAlign] = {};
  uint64_t need = off - (uint64_t)at;
  while (need) {
    const size_t n = (size_t)std::min<uint64_t>(need, sizeof zero);
    if (fwrite(zero, 1, n, f) != n) return fail(MSA_ERR_INTERNAL, "index file: write failed");
    need -= n;
  }
  return MSA_OK;
}

msa_status read_header(const char* path, Header* h) {
  if (!path) return fail(MSA_ERR_INVALID_ARG, "index file: path is NULL");
  File fl;
  fl.f = fopen(path, "rb");
  if (!fl.f) return fail(MSA_ERR_INVALID_ARG, "index file: cannot open %s", path);
  unsigned char b[MSA_INDEX_HEADER_BYTES];
  if (fread(b, 1, sizeof b, fl.f) != sizeof b) return fail(MSA_ERR_INVALID_ARG, "index file: truncated header");
  return decode_header(b, h);
}

}  // namespace

extern "C" {

msa_status msa_index_save(const char* path, const msa_layout* L, const msa_index* I, cudaStream_t st) {
  NvtxRange nvtx_("msa_index_save");
  msa_status s = check_layout(L);
  if (s) return s;
  if (!path || !I) return fail(MSA_ERR_INVALID_ARG, "index_save: NULL argument");
  if (I->n_docs <= 0 || I->n_chunks < I->n_docs || !I->kr || (!I->doc_chunk_off && !I->doc_chunk_off_host))
    return fail(MSA_ERR_INVALID_ARG, "index_save: empty bank, or Kr or the CSR missing");
  if (I->kv_on_host ? !I->host_kv : (!I->k || !I->v))
    return fail(MSA_ERR_INVALID_ARG, "index_save: K/V missing");
  Header h;
  h.L = *L;
  h.n_docs = I->n_docs;
  h.n_chunks = I->n_chunks;
  h.kv_on_host = I->kv_on_host ? 1 : 0;
  std::vector<int64_t> csr((size_t)I->n_docs + 1);
  if (I->doc_chunk_off_host) {
    std::memcpy(csr.data(), I->doc_chunk_off_host, sizeof(int64_t) * csr.size());
  } else {
    cudaError_t e = cudaMemcpyAsync(csr.data(), I->doc_chunk_off, sizeof(int64_t) * csr.size(),
                                    cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "index_save: read the CSR");
  }
  if (csr[0] != 0 || csr.back() != I->n_chunks) return fail(MSA_ERR_INVALID_ARG, "index_save: CSR does not span the chunks");
  int64_t mx = 0;
  for (int64_t d = 0; d < I->n_docs; ++d) {
    const int64_t n = csr[d + 1] - csr[d];
    if (n < 1) return fail(MSA_ERR_INVALID_ARG, "index_save: document %lld has no chunk", (long long)d);
    mx = std::max(mx, n);
  }
  h.max_doc_chunks = (int32_t)mx;
  section_sizes(h);
  Bounce bo;
  cudaError_t ce = bo.init();
  if (ce != cudaSuccess) return cuda_fail(ce, "index_save: pinned buffers");
  const std::string tmp = std::string(path) + ".tmp" + std::to_string((long long)getpid());
  {
    File fl;
    fl.f = fopen(tmp.c_str(), "wb");
    if (!fl.f) return fail(MSA_ERR_INVALID_ARG, "index_save: cannot create %s", tmp.c_str());
    const void* src[kSections] = {csr.data(), I->kr, I->kv_on_host ? I->host_kv : I->k, I->kv_on_host ? nullptr : I->v};
    for (int i = 0; i < kSections; ++i) {
      if ((s = pad_to(fl.f, h.off[i]))) break;
      if (h.bytes[i] && (s = write_section(fl.f, src[i], h.bytes[i], bo, st, &h.hash[i]))) break;
      if (!h.bytes[i]) h.hash[i] = msa64(nullptr, 0);
    }
    unsigned char hb[MSA_INDEX_HEADER_BYTES];
    encode_header(h, hb);
    if (!s && (fseek(fl.f, 0, SEEK_SET) != 0 || fwrite(hb, 1, sizeof hb, fl.f) != sizeof hb))
      s = fail(MSA_ERR_INTERNAL, "index_save: header write failed");
    if (!s && (fflush(fl.f) != 0 || fsync(fileno(fl.f)) != 0)) s = fail(MSA_ERR_INTERNAL, "index_save: flush failed");
  }
  if (!s && rename(tmp.c_str(), path) != 0) s = fail(MSA_ERR_INTERNAL, "index_save: rename to %s failed", path);
  if (s) std::remove(tmp.c_str());
  return s;
}

msa_status msa_index_file_info(const char* path, msa_layout* L, int64_t* n_docs, int64_t* n_chunks,
                               int32_t* max_doc_chunks, int32_t* kv_on_host) {
  Header h;
  msa_status s = read_header(path, &h);
  if (s) return s;
  if (L) *L = h.L;
  if (n_docs) *n_docs = h.n_docs;
  if (n_chunks) *n_chunks = h.n_chunks;
  if (max_doc_chunks) *max_doc_chunks = h.max_doc_chunks;
  if (kv_on_host) *kv_on_host = h.kv_on_host;
  return MSA_OK;
}

msa_status msa_index_load(const char* path, int32_t verify, int64_t* csr_host, int64_t* csr_dev, void* kr, void* k,
                          void* v, void* host_kv, cudaStream_t st) {
  NvtxRange nvtx_("msa_index_load");
  Header h;
  msa_status s = read_header(path, &h);
  if (s) return s;
  if (!csr_host || !kr) return fail(MSA_ERR_INVALID_ARG, "index_load: doc_chunk_off_host and kr are required");
  if (h.kv_on_host ? !host_kv : (!k || !v))
    return fail(MSA_ERR_INVALID_ARG, h.kv_on_host ? "index_load: the file holds a host-tier bank: host_kv is required"
                                                  : "index_load: the file holds a device bank: k and v are required");
  File fl;
  fl.f = fopen(path, "rb");
  if (!fl.f) return fail(MSA_ERR_INVALID_ARG, "index_load: cannot open %s", path);
  Bounce bo;
  cudaError_t ce = bo.init();
  if (ce != cudaSuccess) return cuda_fail(ce, "index_load: pinned buffers");
  void* dst[kSections] = {csr_host, kr, h.kv_on_host ? host_kv : k, h.kv_on_host ? nullptr : v};
  for (int i = 0; i < kSections; ++i) {
    if (!h.bytes[i]) continue;
    if (fseek(fl.f, (long)h.off[i], SEEK_SET) != 0) return fail(MSA_ERR_INVALID_ARG, "index_load: truncated");
    uint64_t got = 0;
    if ((s = read_section(fl.f, dst[i], h.bytes[i], bo, st, &got))) return s;
    if (verify && got != h.hash[i]) return fail(MSA_ERR_INVALID_ARG, "index_load: section %d checksum mismatch", i);
  }
  if (csr_host[0] != 0 || csr_host[h.n_docs] != h.n_chunks)
    return fail(MSA_ERR_INVALID_ARG, "index_load: CSR does not span the chunks");
  if (csr_dev) {
    cudaError_t e = cudaMemcpyAsync(csr_dev, csr_host, sizeof(int64_t) * (size_t)(h.n_docs + 1), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "index_load: copy the CSR");
  }
  return MSA_OK;
}

}  // extern "C"
