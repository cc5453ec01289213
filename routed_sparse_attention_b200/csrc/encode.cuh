// Stage 1 kernels: rotary table and document-wise RoPE + chunk-mean pooling.
//
// Method: "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts",
// section "How MSA compresses and routes documents" (K/V/Kr chunk-mean pooled;
// every document restarts its RoPE positions at zero) and "EverMind Releases
// Memory-Sparse Attention Code for Long-Context AI Models", section
// "Architectural Design and Inference" (stage 1, global memory encoding).
#pragma once
#include "msa_common.cuh"

namespace msa {

// table[p][i] = (cos, sin)(p * theta^(-2i/d)) for p < n_pos, i < d/2, computed
// in fp64 and rounded once to fp32.
__global__ void rope_table_kernel(int n_pos, int d, double theta, float2* table) {
  const int half = d / 2;
  const long long n = (long long)n_pos * half;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(idx % half);
    const long long p = idx / half;
    const double inv = pow(theta, -2.0 * (double)i / (double)d);
    double s, c;
    sincos((double)p * inv, &s, &c);
    table[idx] = make_float2((float)c, (float)s);
  }
}

// Persistent CTAs (three per SM, two 4-token stages each: 93 % of the copy
// peak on the 1M bank, against 89 % for two CTAs of two 8-token stages and
// 54 % for one CTA of four) take documents round-robin.  A producer warp
// streams each document's token rows -- contiguous per tensor -- into a
// shared-memory ring by bulk TMA, kEncStageTok tokens of K, V and Kr per
// stage, so that the loads in flight are bounded by the ring and not by the
// registers; three consumer roles accumulate from shared memory:
//   [0, TK)        K : a thread owns head h, pair block a: dims [a*V, a*V+V) and
//                      the rotate-half partners [d/2 + a*V, ...), so each
//                      thread rotates whole pairs with no shuffles;
//   [TK, 2TK)      V : same mapping, no rotation;
//   [2TK, 2TK+TR)  Kr: same mapping over router_dim, no rotation.
// One chunk's sum stays in fp32 registers, token by token in order, and is
// divided by the number of tokens the chunk holds (the last chunk of a
// document may be short).  The producer passes each stage's document, first
// token and token count through shared memory and ends with an empty stage.
constexpr int kEncStageTok = 4;
constexpr int kEncMaxStages = 4;
constexpr int kEncThreads = 256;               // up to 7 consumer warps + the producer warp

struct EncodeArgs {
  const int64_t* doc_tok_off;
  const int64_t* doc_chunk_off;
  const void* k_tok;
  const void* v_tok;
  const void* kr_tok;
  const float2* rope;
  void* k_pool;
  void* v_pool;
  void* kr_pool;
  int64_t n_docs;
  int rope_rows, H, d, dr, chunk, kv_interleaved, n_stages, stage_bytes;
};

template <typename T>
__global__ void __launch_bounds__(kEncThreads, 3) encode_pool_kernel(const __grid_constant__ EncodeArgs a) {
  constexpr int V = Elem<T>::kPerVec;
  extern __shared__ __align__(128) unsigned char smem[];
  const int NS = a.n_stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)NS * a.stage_bytes);
  uint64_t* empty = full + kEncMaxStages;
  int64_t* slot_len = reinterpret_cast<int64_t*>(empty + kEncMaxStages);   // document length
  int64_t* slot_c0 = slot_len + kEncMaxStages;                             // its first chunk
  int64_t* slot_nch = slot_c0 + kEncMaxStages;                             // its chunk count
  int* slot_p = reinterpret_cast<int*>(slot_nch + kEncMaxStages);          // first token of the stage
  int* slot_n = slot_p + kEncMaxStages;                                    // tokens in the stage
  const int TK = a.H * (a.d / 2) / V;
  const int TR = a.H * (a.dr / 2) / V;
  const int n_cons = 2 * TK + TR;
  const int cons_warps = (n_cons + 31) / 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int esz = (int)sizeof(T);
  const int rowK = a.H * a.d * esz, rowR = a.H * a.dr * esz;   // bytes per token row
  if (tid == 0) {
    for (int st = 0; st < NS; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], cons_warps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kEncThreads / 32 - 1) {          // ---- producer
    if (lane == 0) {
      int64_t st = 0;
      bool ok = true;
      const int ropeb = (a.d / 2) * (int)sizeof(float2);   // bytes per rotary row
      for (int64_t s = blockIdx.x; s < a.n_docs && ok; s += gridDim.x) {
        const int64_t t0 = a.doc_tok_off[s];
        const int64_t L = a.doc_tok_off[s + 1] - t0;
        const int64_t c0 = a.doc_chunk_off[s], nch = a.doc_chunk_off[s + 1] - c0;
        if (L > a.rope_rows) dev_flag(MSA_DEV_ROPE_RANGE);
        for (int64_t p = 0; p < L; p += kEncStageTok, ++st) {
          const int slot = (int)(st % NS);
          if (st >= NS && !mbar_wait(&empty[slot], (uint32_t)((st / NS - 1) & 1))) { ok = false; break; }
          const int n = (int)min64(kEncStageTok, L - p);
          const int64_t rem = (int64_t)a.rope_rows - p;              // rotary rows inside the table
          const int nr = rem <= 0 ? 0 : (int)min64(n, rem);
          slot_len[slot] = L;
          slot_c0[slot] = c0;
          slot_nch[slot] = nch;
          slot_p[slot] = (int)p;
          slot_n[slot] = n;
          unsigned char* dst = smem + (size_t)slot * a.stage_bytes;
          mbar_arrive_expect_tx(&full[slot], (uint32_t)(n * (2 * rowK + rowR) + nr * ropeb));
          if (nr > 0)
            tma_load_1d(dst + kEncStageTok * (2 * rowK + rowR), reinterpret_cast<const unsigned char*>(a.rope) +
                        p * ropeb, (uint32_t)(nr * ropeb), &full[slot]);
          const int64_t row = t0 + p;
          tma_load_1d(dst, static_cast<const unsigned char*>(a.k_tok) + row * rowK, (uint32_t)(n * rowK), &full[slot]);
          tma_load_1d(dst + kEncStageTok * rowK, static_cast<const unsigned char*>(a.v_tok) + row * rowK,
                      (uint32_t)(n * rowK), &full[slot]);
          tma_load_1d(dst + 2 * kEncStageTok * rowK, static_cast<const unsigned char*>(a.kr_tok) + row * rowR,
                      (uint32_t)(n * rowR), &full[slot]);
        }
      }
      if (ok) {                                // the end marker
        const int slot = (int)(st % NS);
        if (st < NS || mbar_wait(&empty[slot], (uint32_t)((st / NS - 1) & 1))) {
          slot_n[slot] = 0;
          mbar_arrive(&full[slot]);
        }
      }
    }
    return;
  }
  if (warp >= cons_warps) return;

  // ---- consumers
  const bool active = tid < n_cons;
  int role = 0, lt = 0, dim = a.d, region = 0, rowb = rowK;
  T* dst = reinterpret_cast<T*>(a.k_pool);
  if (tid < TK) { role = 0; lt = tid; }
  else if (tid < 2 * TK) { role = 1; lt = tid - TK; region = kEncStageTok * rowK; dst = reinterpret_cast<T*>(a.v_pool); }
  else { role = 2; lt = tid - 2 * TK; dim = a.dr; region = 2 * kEncStageTok * rowK; rowb = rowR;
         dst = reinterpret_cast<T*>(a.kr_pool); }
  const int bpp = (dim / 2) / V;               // pair blocks per head
  const int h = lt / bpp, ab = lt % bpp;
  const int half = dim / 2;
  const int64_t row = (int64_t)a.H * dim;     // elements per token / chunk row
  const int off_lo = h * dim + ab * V, off_hi = off_lo + half;
  float acc[2 * V];
#pragma unroll
  for (int i = 0; i < 2 * V; ++i) acc[i] = 0.f;
  int cnt = 0;                                 // tokens in the current chunk
  for (int64_t st = 0;; ++st) {
    const int slot = (int)(st % NS);
    if (!mbar_wait(&full[slot], (uint32_t)((st / NS) & 1))) return;
    const int n = slot_n[slot];
    if (n == 0) break;
    const int p0 = slot_p[slot];
    if (active) {
      const int64_t L = slot_len[slot], c0 = slot_c0[slot], nch = slot_nch[slot];
      const T* base = reinterpret_cast<const T*>(smem + (size_t)slot * a.stage_bytes + region);
      const float2* rs = reinterpret_cast<const float2*>(smem + (size_t)slot * a.stage_bytes +
                                                         kEncStageTok * (2 * rowK + rowR));
      for (int j = 0; j < n; ++j) {
        const int pos = p0 + j;
        const T* tr = reinterpret_cast<const T*>(reinterpret_cast<const unsigned char*>(base) + (int64_t)j * rowb);
        float x0[V], x1[V];
        Elem<T>::unpack(*reinterpret_cast<const uint4*>(tr + off_lo), x0);
        Elem<T>::unpack(*reinterpret_cast<const uint4*>(tr + off_hi), x1);
        if (role == 0) {                       // the stage's rotary rows (past the table: its last row)
          const float2* cs = pos < a.rope_rows ? rs + (int64_t)j * half + ab * V
                                               : a.rope + (int64_t)(a.rope_rows - 1) * half + ab * V;
#pragma unroll
          for (int i = 0; i < V; ++i) {
            const float2 w = cs[i];
            acc[i] += x0[i] * w.x - x1[i] * w.y;
            acc[V + i] += x1[i] * w.x + x0[i] * w.y;
          }
        } else {
#pragma unroll
          for (int i = 0; i < V; ++i) {
            acc[i] += x0[i];
            acc[V + i] += x1[i];
          }
        }
        ++cnt;
        if (cnt == a.chunk || pos == L - 1) {  // the chunk is complete
          const int64_t cc = pos / a.chunk;
          const float fn = (float)cnt;
#pragma unroll
          for (int i = 0; i < 2 * V; ++i) acc[i] = acc[i] / fn;
          // chunk-major rows; or, with kv_interleaved, the host tier's rows: a
          // document's K chunks at [2*c0, 2*c0 + nch), then its V chunks
          int64_t orow = c0 + cc;
          if (a.kv_interleaved && role < 2) orow += role == 0 ? c0 : c0 + nch;
          T* o = dst + orow * row;
          *reinterpret_cast<uint4*>(o + off_lo) = Elem<T>::pack(acc);
          *reinterpret_cast<uint4*>(o + off_hi) = Elem<T>::pack(acc + V);
#pragma unroll
          for (int i = 0; i < 2 * V; ++i) acc[i] = 0.f;
          cnt = 0;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
}

// ---------------------------------------------------- global RoPE of local keys
// "Global RoPE" of the MSA pages ("EverMind-AI/MSA: Memory Sparse Attention for
// 100M-Token Contexts", section "How MSA compresses and routes documents"): the
// local context starts at position k, after the k retrieved documents, so local
// token j is rotated at k + j.  A key cache applies it once per appended token.

constexpr int kRopeLocalMaxB = 256;

struct RopeLocalArgs {
  const void* src;
  void* dst;
  const float2* rope;
  int d, Hkv, top_k, rope_rows;
  int64_t local_off[kRopeLocalMaxB + 1];   // row offsets of each query's cache (capacity = difference)
  int64_t len[kRopeLocalMaxB];             // live tokens, per query
  int64_t first[kRopeLocalMaxB];           // first token to rotate, per query
};

// grid.y = query b.  A thread takes one row and one 16-byte group of the low
// half plus its rotate-half partner group; rows are [H_kv][cap_b][d].
template <typename T>
__global__ void __launch_bounds__(256) rope_local_kernel(const __grid_constant__ RopeLocalArgs a) {
  constexpr int V = Elem<T>::kPerVec;
  const int b = blockIdx.y;
  const int half = a.d / 2, groups = half / V;
  const int64_t cap = a.local_off[b + 1] - a.local_off[b];
  const int64_t j0 = a.first[b];
  const int64_t n_rot = a.len[b] - j0;
  if (n_rot <= 0) return;
  const int64_t n_items = (int64_t)a.Hkv * n_rot * groups;
  const int64_t base = a.local_off[b] * a.Hkv;              // first row of query b
  const T* src = reinterpret_cast<const T*>(a.src);
  T* dst = reinterpret_cast<T*>(a.dst);
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < n_items;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int grp = (int)(it % groups);
    const int64_t rr = it / groups;                           // (head, token) within the rotated span
    const int g = (int)(rr / n_rot);
    const int64_t j = j0 + rr % n_rot;
    const int64_t row = base + (int64_t)g * cap + j;
    int64_t pos = (int64_t)a.top_k + j;
    if (pos >= a.rope_rows) { dev_flag(MSA_DEV_ROPE_RANGE); pos = a.rope_rows - 1; }
    const T* sp = src + row * a.d + grp * V;
    float x0[V], x1[V], y0[V], y1[V];
    Elem<T>::unpack(*reinterpret_cast<const uint4*>(sp), x0);   // plain loads: dst may be src
    Elem<T>::unpack(*reinterpret_cast<const uint4*>(sp + half), x1);
    const float2* cs = a.rope + pos * half + grp * V;
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const float2 w = __ldg(cs + i);
      y0[i] = x0[i] * w.x - x1[i] * w.y;
      y1[i] = x1[i] * w.x + x0[i] * w.y;
    }
    T* dp = dst + row * a.d + grp * V;
    *reinterpret_cast<uint4*>(dp) = Elem<T>::pack(y0);
    *reinterpret_cast<uint4*>(dp + half) = Elem<T>::pack(y1);
  }
}

// Appends one token per query to a local key/value cache: the token of query
// b lands at row len_b of every kv head (rows [H_kv][cap_b][d] per query), its
// key both as given (raw cache, optional) and rotated at top_k + len_b.
struct AppendLocalArgs {
  const void* k_new;                       // [B][H_kv][d]
  const void* v_new;
  void* k_raw;                             // may be null
  void* k_rot;
  void* v;
  const float2* rope;
  int d, Hkv, top_k, rope_rows;
  const int64_t* len_dev;                  // live tokens before the append on the device, or null: len
  int64_t local_off[kRopeLocalMaxB + 1];
  int64_t len[kRopeLocalMaxB];             // live tokens before the append
};

// grid (H_kv, B); a thread takes one 16-byte group of the low half plus its
// rotate-half partner.
template <typename T>
__global__ void __launch_bounds__(64) append_local_kernel(const __grid_constant__ AppendLocalArgs a) {
  constexpr int V = Elem<T>::kPerVec;
  const int g = blockIdx.x, b = blockIdx.y;
  const int half = a.d / 2, groups = half / V;
  const int grp = threadIdx.x;
  if (grp >= groups) return;
  const int64_t cap = a.local_off[b + 1] - a.local_off[b];
  const int64_t j = a.len_dev ? a.len_dev[b] : a.len[b];
  if (j < 0 || j >= cap) {                          // no room (device lengths only)
    if (grp == 0) dev_flag(MSA_DEV_BAD_SHAPE);
    return;
  }
  const int64_t row = a.local_off[b] * a.Hkv + (int64_t)g * cap + j;
  int64_t pos = (int64_t)a.top_k + j;
  if (pos >= a.rope_rows) { dev_flag(MSA_DEV_ROPE_RANGE); pos = a.rope_rows - 1; }
  const int64_t in = ((int64_t)b * a.Hkv + g) * a.d + grp * V;
  const T* kp = reinterpret_cast<const T*>(a.k_new) + in;
  const T* vp = reinterpret_cast<const T*>(a.v_new) + in;
  const uint4 k0 = *reinterpret_cast<const uint4*>(kp), k1 = *reinterpret_cast<const uint4*>(kp + half);
  const int64_t out = row * a.d + grp * V;
  T* vd = reinterpret_cast<T*>(a.v) + out;
  *reinterpret_cast<uint4*>(vd) = *reinterpret_cast<const uint4*>(vp);
  *reinterpret_cast<uint4*>(vd + half) = *reinterpret_cast<const uint4*>(vp + half);
  if (a.k_raw) {
    T* kr = reinterpret_cast<T*>(a.k_raw) + out;
    *reinterpret_cast<uint4*>(kr) = k0;
    *reinterpret_cast<uint4*>(kr + half) = k1;
  }
  float x0[V], x1[V], y0[V], y1[V];
  Elem<T>::unpack(k0, x0);
  Elem<T>::unpack(k1, x1);
  const float2* cs = a.rope + pos * half + grp * V;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const float2 w = __ldg(cs + i);
    y0[i] = x0[i] * w.x - x1[i] * w.y;
    y1[i] = x1[i] * w.x + x0[i] * w.y;
  }
  T* kd = reinterpret_cast<T*>(a.k_rot) + out;
  *reinterpret_cast<uint4*>(kd) = Elem<T>::pack(y0);
  *reinterpret_cast<uint4*>(kd + half) = Elem<T>::pack(y1);
}

// Live lengths on the device advance by `by` tokens (after a step's appends).
__global__ void advance_len_kernel(int64_t* len, int B, int64_t by) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) len[b] += by;
}

}  // namespace msa
