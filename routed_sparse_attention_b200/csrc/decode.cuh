// Stage 3 kernels: split-K GQA decode over [selected pooled K/V ++ local K/V].
//
// Method: "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts",
// section "How MSA compresses and routes documents" (compressed K/V of the
// Top-k documents concatenated with the query's local K/V; global RoPE offsets
// the query's start by k, order background -> query -> generation) and
// "EverMind Releases Memory-Sparse Attention Code for Long-Context AI Models",
// section "Architectural Design and Inference" (stage 3, sparse generation).
//
// Work split: for query b and kv head g, split 0 holds every memory key (the
// selected documents' pooled chunks, rank order) and splits 1.. hold runs of
// S local keys.  A CTA takes one (split, kv head, group of 4 query rows),
// where the rows of kv head g are (t, h) for the G query heads of the group and
// the T query tokens.  It writes the split's softmax partial (max, sum,
// unnormalised output); decode_combine_kernel merges the splits.
//
// Rotary positions: the query token t sits at top_k + L_b + t, local key j at
// top_k + j.  For local keys the CTA turns the query once by
// (L_b + t - j_lo), j_lo the split's first key, and each key by (j - j_lo), so
// only table rows 0 .. S-1 are read per key; <R(a)q, R(b)k> depends on a - b
// only.  Pooled memory keys keep their document-local rotation from encoding
// and meet the query turned by its absolute position.
#pragma once
#include "msa_common.cuh"

namespace msa {

constexpr int kDecMaxB = 256;
constexpr int kDecRows = 4;          // query rows per CTA
constexpr int kDecWarps = 4;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecNB = 2;            // key batches per softmax rescale

struct DecodeArgs {
  int B, T, Hq, Hkv, G, R, n_rg, S, top_k, rope_rows, kv_on_host;
  int max_doc_chunks;
  float scale_log2;                  // log2(e) / sqrt(d)
  const void* q;
  const void* lk;
  const void* lv;
  const int32_t* sel;
  const int64_t* doc_chunk_off;
  int64_t n_docs;
  const void* mem_k;                 // device chunk-major K / V, or staging (host tier)
  const void* mem_v;
  const float2* rope;
  float* part_o;                     // [S_tot][Hkv][R][d]
  float* part_ml;                    // [S_tot][Hkv][R][2] (max, sum) in log2 units
  void* out;
  int32_t split_off[kDecMaxB + 1];   // first split id of query b
  int64_t local_off[kDecMaxB + 1];   // token offset of query b's local rows
};

// 8 consecutive elements as floats.
template <typename T> __device__ __forceinline__ void load8(const T* p, float* f);
template <> __device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float* f) {
  Elem<__nv_bfloat16>::unpack(ldg_nc_v4(p), f);
}
template <> __device__ __forceinline__ void load8<float>(const float* p, float* f) {
  Elem<float>::unpack(ldg_nc_v4(p), f);
  Elem<float>::unpack(ldg_nc_v4(p + 4), f + 4);
}

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads)
decode_split_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int LPK = D / 16;             // lanes per key (16 dims each)
  constexpr int KPW = 32 / LPK;           // keys per warp step
  constexpr int HALF = D / 2;
  __shared__ int64_t s_mem_pref[65];
  __shared__ float s_ml[kDecWarps][kDecRows][2];
  __shared__ float s_o[kDecWarps][kDecRows][D];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kg = lane / LPK, sl = lane % LPK;
  // query b and split s of this CTA
  int b = 0;
  while (b + 1 < a.B && a.split_off[b + 1] <= (int)blockIdx.x) ++b;
  const int s = blockIdx.x - a.split_off[b];
  const int g = blockIdx.y / a.n_rg, rg = blockIdx.y % a.n_rg;
  const int64_t Ltot = a.local_off[b + 1] - a.local_off[b];
  const int64_t Lb = Ltot - a.T;
  const int k = a.top_k;

  // key range
  int64_t nkeys, j_lo = 0;
  if (s == 0) {
    if (threadIdx.x == 0) {
      int64_t acc = 0;
      s_mem_pref[0] = 0;
      for (int r = 0; r < k; ++r) {
        int doc = a.sel[(int64_t)b * k + r];
        if (doc < 0 || doc >= a.n_docs) { dev_flag(MSA_DEV_BAD_DOC); doc = 0; }
        const int64_t nc = a.doc_chunk_off[doc + 1] - a.doc_chunk_off[doc];
        acc += (nc <= a.max_doc_chunks) ? nc : 0;
        s_mem_pref[r + 1] = acc;
      }
    }
    __syncthreads();
    nkeys = s_mem_pref[k];
  } else {
    j_lo = (int64_t)(s - 1) * a.S;
    nkeys = min64(a.S, Ltot - j_lo);
  }

  // rows, query slices (dims [8 sl, 8 sl + 8) and their rotate-half partners)
  const T* Q = reinterpret_cast<const T*>(a.q);
  float qv[kDecRows][16];
  int row_t[kDecRows];
  bool row_on[kDecRows];
#pragma unroll
  for (int i = 0; i < kDecRows; ++i) {
    const int r = rg * kDecRows + i;
    row_on[i] = r < a.R;
    const int t = row_on[i] ? r / a.G : 0, hh = row_on[i] ? r % a.G : 0;
    row_t[i] = t;
    const int h = g * a.G + hh;
    // position of the turn applied to the query
    int64_t pos = (s == 0) ? (int64_t)k + Lb + t : Lb + t - j_lo;
    if (pos < 0) { row_on[i] = false; pos = 0; }      // every key of the split is in its future
    if (pos >= a.rope_rows) { dev_flag(MSA_DEV_ROPE_RANGE); pos = a.rope_rows - 1; }
    float x0[8], x1[8];
    const T* qp = Q + (((int64_t)b * a.T + t) * a.Hq + h) * D;
    load8<T>(qp + 8 * sl, x0);
    load8<T>(qp + HALF + 8 * sl, x1);
    const float2* cs = a.rope + pos * HALF + 8 * sl;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float2 w = __ldg(cs + e);
      qv[i][e] = row_on[i] ? (x0[e] * w.x - x1[e] * w.y) * a.scale_log2 : 0.f;
      qv[i][8 + e] = row_on[i] ? (x1[e] * w.x + x0[e] * w.y) * a.scale_log2 : 0.f;
    }
  }

  float m[kDecRows], l[kDecRows], o[kDecRows][16];
#pragma unroll
  for (int i = 0; i < kDecRows; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) o[i][e] = 0.f;
  }

  const T* LK = reinterpret_cast<const T*>(a.lk) + (a.local_off[b] * a.Hkv + (int64_t)g * Ltot) * D;
  const T* LV = reinterpret_cast<const T*>(a.lv) + (a.local_off[b] * a.Hkv + (int64_t)g * Ltot) * D;
  const T* MK = reinterpret_cast<const T*>(a.mem_k);
  const T* MV = reinterpret_cast<const T*>(a.mem_v);

  for (int64_t base = (int64_t)warp * kDecNB * KPW; base < nkeys;
       base += (int64_t)kDecWarps * kDecNB * KPW) {
    float kx[kDecNB][16], vx[kDecNB][16];
    float x[kDecNB][kDecRows];
    bool kv[kDecNB];
#pragma unroll
    for (int u = 0; u < kDecNB; ++u) {
      const int64_t kk = base + u * KPW + kg;
      kv[u] = kk < nkeys;
      if (!kv[u]) {
#pragma unroll
        for (int e = 0; e < 16; ++e) { kx[u][e] = 0.f; vx[u][e] = 0.f; }
        continue;
      }
      const T *kp, *vp;
      if (s == 0) {
        int r = 0;
        while (s_mem_pref[r + 1] <= kk) ++r;
        int doc = a.sel[(int64_t)b * k + r];
        if (doc < 0 || doc >= a.n_docs) doc = 0;
        const int64_t ci = kk - s_mem_pref[r];
        const int64_t c0 = a.doc_chunk_off[doc];
        if (a.kv_on_host) {
          const int64_t nc = a.doc_chunk_off[doc + 1] - c0;
          const int64_t slot = ((int64_t)b * k + r) * 2 * a.max_doc_chunks;
          kp = MK + ((slot + ci) * a.Hkv + g) * D;
          vp = MK + ((slot + nc + ci) * a.Hkv + g) * D;
        } else {
          kp = MK + ((c0 + ci) * a.Hkv + g) * D;
          vp = MV + ((c0 + ci) * a.Hkv + g) * D;
        }
      } else {
        kp = LK + (j_lo + kk) * D;
        vp = LV + (j_lo + kk) * D;
      }
      load8<T>(kp + 8 * sl, kx[u]);
      load8<T>(kp + HALF + 8 * sl, kx[u] + 8);
      load8<T>(vp + 8 * sl, vx[u]);
      load8<T>(vp + HALF + 8 * sl, vx[u] + 8);
      if (s != 0) {                                 // turn the local key by (j - j_lo)
        const int64_t rr = kk < a.rope_rows ? kk : a.rope_rows - 1;
        const float2* cs = a.rope + rr * HALF + 8 * sl;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 w = __ldg(cs + e);
          const float k0 = kx[u][e], k1 = kx[u][8 + e];
          kx[u][e] = k0 * w.x - k1 * w.y;
          kx[u][8 + e] = k1 * w.x + k0 * w.y;
        }
      }
    }
    // logits (log2 units): partial dots over this lane's 16 dims, reduced
    // over the LPK lanes that hold one key
#pragma unroll
    for (int u = 0; u < kDecNB; ++u)
#pragma unroll
      for (int i = 0; i < kDecRows; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) acc = fmaf(qv[i][e], kx[u][e], acc);
#pragma unroll
        for (int o2 = 1; o2 < LPK; o2 <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o2);
        x[u][i] = acc;
      }
    // mask: keys past the split end, rows off, local keys after the row's token
#pragma unroll
    for (int u = 0; u < kDecNB; ++u) {
      const int64_t kk = base + u * KPW + kg;
#pragma unroll
      for (int i = 0; i < kDecRows; ++i) {
        bool vis = kv[u] && row_on[i];
        if (s != 0) vis = vis && (j_lo + kk <= Lb + row_t[i]);
        if (!vis) x[u][i] = -INFINITY;
      }
    }
#pragma unroll
    for (int i = 0; i < kDecRows; ++i) {
      float mb = m[i];
#pragma unroll
      for (int u = 0; u < kDecNB; ++u) mb = fmaxf(mb, x[u][i]);
      if (mb == -INFINITY) continue;
      const float sc = exp2f(m[i] - mb);
      l[i] *= sc;
#pragma unroll
      for (int e = 0; e < 16; ++e) o[i][e] *= sc;
      m[i] = mb;
#pragma unroll
      for (int u = 0; u < kDecNB; ++u) {
        const float p = exp2f(x[u][i] - mb);
        l[i] += p;
#pragma unroll
        for (int e = 0; e < 16; ++e) o[i][e] = fmaf(p, vx[u][e], o[i][e]);
      }
    }
  }

  // merge the KPW key slots of the warp (lanes with equal sl)
#pragma unroll
  for (int i = 0; i < kDecRows; ++i) {
#pragma unroll
    for (int o2 = LPK; o2 < 32; o2 <<= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[i], o2);
      const float lo = __shfl_xor_sync(0xffffffffu, l[i], o2);
      const float mn = fmaxf(m[i], mo);
      const float s1 = (m[i] == -INFINITY) ? 0.f : exp2f(m[i] - mn);
      const float s2 = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
      l[i] = l[i] * s1 + lo * s2;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float oo = __shfl_xor_sync(0xffffffffu, o[i][e], o2);
        o[i][e] = o[i][e] * s1 + oo * s2;
      }
      m[i] = mn;
    }
  }
  if (kg == 0) {
#pragma unroll
    for (int i = 0; i < kDecRows; ++i) {
      if (sl == 0) { s_ml[warp][i][0] = m[i]; s_ml[warp][i][1] = l[i]; }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        s_o[warp][i][8 * sl + e] = o[i][e];
        s_o[warp][i][HALF + 8 * sl + e] = o[i][8 + e];
      }
    }
  }
  __syncthreads();
  // merge the warps and write this split's partial
  const int sid = a.split_off[b] + s;
  for (int idx = threadIdx.x; idx < kDecRows * D; idx += kDecThreads) {
    const int i = idx / D, dd = idx % D;
    const int r = rg * kDecRows + i;
    if (r >= a.R) continue;
    float mt = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) mt = fmaxf(mt, s_ml[w][i][0]);
    float lt = 0.f, ot = 0.f;
    if (mt != -INFINITY) {
      for (int w = 0; w < kDecWarps; ++w) {
        const float mw = s_ml[w][i][0];
        if (mw == -INFINITY) continue;
        const float sc = exp2f(mw - mt);
        lt += s_ml[w][i][1] * sc;
        ot += s_o[w][i][dd] * sc;
      }
    }
    const int64_t prow = ((int64_t)sid * a.Hkv + g) * a.R + r;
    a.part_o[prow * D + dd] = ot;
    if (dd == 0) {
      a.part_ml[prow * 2] = mt;
      a.part_ml[prow * 2 + 1] = lt;
    }
  }
}

// One CTA per (query, token, head): merge the splits' partials.
template <typename T, int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(const __grid_constant__ DecodeArgs a) {
  const int bid = blockIdx.x;
  const int h = bid % a.Hq;
  const int t = (bid / a.Hq) % a.T;
  const int b = bid / (a.Hq * a.T);
  const int g = h / a.G, r = t * a.G + (h % a.G);
  const int s0 = a.split_off[b], s1 = a.split_off[b + 1];
  const int dd = threadIdx.x;
  float mt = -INFINITY;
  for (int sid = s0; sid < s1; ++sid) {
    const int64_t prow = ((int64_t)sid * a.Hkv + g) * a.R + r;
    mt = fmaxf(mt, a.part_ml[prow * 2]);
  }
  float lt = 0.f, ot = 0.f;
  for (int sid = s0; sid < s1; ++sid) {
    const int64_t prow = ((int64_t)sid * a.Hkv + g) * a.R + r;
    const float ms = a.part_ml[prow * 2];
    if (ms == -INFINITY) continue;
    const float sc = exp2f(ms - mt);
    lt += a.part_ml[prow * 2 + 1] * sc;
    ot += a.part_o[prow * D + dd] * sc;
  }
  T* out = reinterpret_cast<T*>(a.out);
  Elem<T>::store1(out + (((int64_t)b * a.T + t) * a.Hq + h) * D + dd, ot / lt);
}

}  // namespace msa
