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

// One CTA per document; three thread roles stream the document's tokens once:
//   [0, TK)        K : a thread owns head h, pair block a: dims [a*V, a*V+V) and
//                      the rotate-half partners [d/2 + a*V, ...), so each
//                      thread rotates whole pairs with no shuffles;
//   [TK, 2TK)      V : same mapping, no rotation;
//   [2TK, 2TK+TR)  Kr: same mapping over router_dim, no rotation.
// Each token row of a tensor is H_kv*dim contiguous elements, read as 16-byte
// vectors; one chunk's sum stays in fp32 registers and is divided by the
// number of tokens the chunk holds (the last chunk of a document may be short).
template <typename T>
__global__ void __launch_bounds__(256) encode_pool_kernel(
    const int64_t* __restrict__ doc_tok_off, const int64_t* __restrict__ doc_chunk_off,
    const T* __restrict__ k_tok, const T* __restrict__ v_tok, const T* __restrict__ kr_tok,
    const float2* __restrict__ rope, int rope_rows, int H, int d, int dr, int chunk,
    T* __restrict__ k_pool, T* __restrict__ v_pool, T* __restrict__ kr_pool, int kv_interleaved) {
  constexpr int V = Elem<T>::kPerVec;
  const int s = blockIdx.x;
  const int TK = H * (d / 2) / V;
  const int TR = H * (dr / 2) / V;
  const int tid = threadIdx.x;
  int role, lt, dim;
  const T* src;
  T* dst;
  if (tid < TK) { role = 0; lt = tid; dim = d; src = k_tok; dst = k_pool; }
  else if (tid < 2 * TK) { role = 1; lt = tid - TK; dim = d; src = v_tok; dst = v_pool; }
  else if (tid < 2 * TK + TR) { role = 2; lt = tid - 2 * TK; dim = dr; src = kr_tok; dst = kr_pool; }
  else return;
  const int bpp = (dim / 2) / V;          // pair blocks per head
  const int h = lt / bpp, a = lt % bpp;
  const int half = dim / 2;
  const int64_t row = (int64_t)H * dim;   // elements per token row
  const int64_t t0 = doc_tok_off[s];
  const int64_t L = doc_tok_off[s + 1] - t0;
  const int64_t c0 = doc_chunk_off[s];
  const int64_t nch = doc_chunk_off[s + 1] - c0;
  const int off_lo = h * dim + a * V, off_hi = off_lo + half;
  if (role == 0 && L > rope_rows) dev_flag(MSA_DEV_ROPE_RANGE);

  for (int64_t cc = 0; cc < nch; ++cc) {
    const int64_t p0 = cc * chunk;
    const int n = (int)min64(chunk, L - p0);
    float acc[2 * V];
#pragma unroll
    for (int i = 0; i < 2 * V; ++i) acc[i] = 0.f;
    const T* base = src + (t0 + p0) * row;
    int p = 0;
    for (; p < n; p += 4) {
      uint4 lo[4], hi[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (p + u < n) {
          lo[u] = ldg_nc_v4(base + (int64_t)(p + u) * row + off_lo);
          hi[u] = ldg_nc_v4(base + (int64_t)(p + u) * row + off_hi);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (p + u >= n) break;
        float x0[V], x1[V];
        Elem<T>::unpack(lo[u], x0);
        Elem<T>::unpack(hi[u], x1);
        if (role == 0) {
          const int pos = (int)(p0 + p + u);
          const int prow = pos < rope_rows ? pos : rope_rows - 1;
          const float2* cs = rope + (int64_t)prow * half + a * V;
#pragma unroll
          for (int i = 0; i < V; ++i) {
            const float2 w = __ldg(cs + i);
            const float r0 = x0[i] * w.x - x1[i] * w.y;
            const float r1 = x1[i] * w.x + x0[i] * w.y;
            acc[i] += r0;
            acc[V + i] += r1;
          }
        } else {
#pragma unroll
          for (int i = 0; i < V; ++i) {
            acc[i] += x0[i];
            acc[V + i] += x1[i];
          }
        }
      }
    }
    const float fn = (float)n;
#pragma unroll
    for (int i = 0; i < 2 * V; ++i) acc[i] = acc[i] / fn;
    // chunk-major rows; or, with kv_interleaved, the host tier's rows: a
    // document's K chunks at [2*c0, 2*c0 + nch), then its V chunks
    int64_t orow = c0 + cc;
    if (kv_interleaved && role < 2) orow += role == 0 ? c0 : c0 + nch;
    T* o = dst + orow * row;
    *reinterpret_cast<uint4*>(o + off_lo) = Elem<T>::pack(acc);
    *reinterpret_cast<uint4*>(o + off_hi) = Elem<T>::pack(acc + V);
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
