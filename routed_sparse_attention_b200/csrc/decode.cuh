// Stage 3 kernel: split-K GQA decode over [selected pooled K/V ++ local K/V].
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
// the T query tokens.  Keys arrive in shared-memory tiles of 64: a local tile
// is two contiguous rows ranges (K and V of one head) fetched by bulk TMA, two
// stages deep; a memory tile is gathered row by row by all threads.  The CTA
// writes its softmax partial (max, sum, unnormalised output); the last CTA of
// each (query, kv head, row group) to finish -- counted with an atomic in the
// workspace, which it resets to zero -- merges every split and writes the output.
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
constexpr int kDecNB = 2;            // key steps per softmax rescale
constexpr int kDecTile = 64;         // keys per shared-memory tile
constexpr int kDecStages = 2;
constexpr int kDecMaxSplits = 512;   // splits per (query, kv head)
constexpr int kMaxTopKDecode = 64;   // selected documents per query

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
  int* counters;                     // [B][Hkv][n_rg], zero between calls
  void* out;
  int32_t split_off[kDecMaxB + 1];   // first split id of query b
  int64_t local_off[kDecMaxB + 1];   // token offset of query b's local rows
};

template <typename T, int D>
struct DecSmem {
  T k[kDecStages][kDecTile][D];
  T v[kDecStages][kDecTile][D];
  uint64_t full[kDecStages];
  int64_t mem_pref[kMaxTopKDecode + 1];
  int64_t mem_krow[kMaxTopKDecode];    // first K row of rank r's document (element rows of [H_kv][d])
  int64_t mem_vrow[kMaxTopKDecode];    // first V row
  int64_t key_krow[kDecTile];          // K / V source rows of the current memory tile's keys
  int64_t key_vrow[kDecTile];
  float ml[kDecWarps][kDecRows][2];
  float o[kDecWarps][kDecRows][D];
  float w[kDecMaxSplits][kDecRows];
  float red[kDecWarps][kDecRows];
  float rowl[kDecRows];
  int last;
};

// 8 consecutive elements as floats (global, streaming).
template <typename T> __device__ __forceinline__ void load8(const T* p, float* f);
template <> __device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float* f) {
  Elem<__nv_bfloat16>::unpack(ldg_nc_v4(p), f);
}
template <> __device__ __forceinline__ void load8<float>(const float* p, float* f) {
  Elem<float>::unpack(ldg_nc_v4(p), f);
  Elem<float>::unpack(ldg_nc_v4(p + 4), f + 4);
}
// 8 consecutive elements as floats (shared memory).
template <typename T> __device__ __forceinline__ void lds8(const T* p, float* f);
template <> __device__ __forceinline__ void lds8<__nv_bfloat16>(const __nv_bfloat16* p, float* f) {
  Elem<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(p), f);
}
template <> __device__ __forceinline__ void lds8<float>(const float* p, float* f) {
  Elem<float>::unpack(*reinterpret_cast<const uint4*>(p), f);
  Elem<float>::unpack(*reinterpret_cast<const uint4*>(p + 4), f + 4);
}

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads)
decode_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int LPK = D / 16;             // lanes per key (16 dims each)
  constexpr int KPW = 32 / LPK;           // keys per warp step
  constexpr int HALF = D / 2;
  constexpr int ROWB = D * (int)sizeof(T);
  extern __shared__ __align__(128) unsigned char smem_raw[];
  DecSmem<T, D>& sm = *reinterpret_cast<DecSmem<T, D>*>(smem_raw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kg = lane / LPK, sl = lane % LPK;
  int b = 0;
  while (b + 1 < a.B && a.split_off[b + 1] <= (int)blockIdx.x) ++b;
  const int s = blockIdx.x - a.split_off[b];
  const int nsplit = a.split_off[b + 1] - a.split_off[b];
  const int g = blockIdx.y / a.n_rg, rg = blockIdx.y % a.n_rg;
  const int64_t Ltot = a.local_off[b + 1] - a.local_off[b];
  const int64_t Lb = Ltot - a.T;
  const int k = a.top_k;
  const bool mem = (s == 0);

  const T* LK = reinterpret_cast<const T*>(a.lk) + (a.local_off[b] * a.Hkv + (int64_t)g * Ltot) * D;
  const T* LV = reinterpret_cast<const T*>(a.lv) + (a.local_off[b] * a.Hkv + (int64_t)g * Ltot) * D;
  const T* MK = reinterpret_cast<const T*>(a.mem_k);
  const T* MV = reinterpret_cast<const T*>(a.mem_v);

  // ---- key range; issue the first local tiles at once
  int64_t nkeys, j_lo = 0;
  if (mem) {
    // rank r's chunk count and first K / V rows, in parallel over the ranks
    if (threadIdx.x < k) {
      const int r = threadIdx.x;
      int doc = a.sel[(int64_t)b * k + r];
      if (doc < 0 || doc >= a.n_docs) { dev_flag(MSA_DEV_BAD_DOC); doc = 0; }
      const int64_t c0 = a.doc_chunk_off[doc];
      int64_t nc = a.doc_chunk_off[doc + 1] - c0;
      if (nc > a.max_doc_chunks) nc = 0;
      if (a.kv_on_host) {
        const int64_t slot = ((int64_t)b * k + r) * 2 * a.max_doc_chunks;
        sm.mem_krow[r] = slot;
        sm.mem_vrow[r] = slot + nc;
      } else {
        sm.mem_krow[r] = c0;
        sm.mem_vrow[r] = c0;
      }
      sm.mem_pref[r + 1] = nc;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      sm.mem_pref[0] = 0;
      for (int r = 0; r < k; ++r) sm.mem_pref[r + 1] += sm.mem_pref[r];
    }
    __syncthreads();
    nkeys = sm.mem_pref[k];
  } else {
    j_lo = (int64_t)(s - 1) * a.S;
    nkeys = min64(a.S, Ltot - j_lo);
  }
  const int ntiles = (int)((nkeys + kDecTile - 1) / kDecTile);
  auto issue_local = [&](int t) {                      // thread 0 only
    const int st = t % kDecStages;
    const int64_t n_t = min64(kDecTile, nkeys - (int64_t)t * kDecTile);
    const uint32_t bytes = (uint32_t)(n_t * ROWB);
    mbar_arrive_expect_tx(&sm.full[st], 2 * bytes);
    tma_load_1d(&sm.k[st][0][0], LK + (j_lo + (int64_t)t * kDecTile) * D, bytes, &sm.full[st]);
    tma_load_1d(&sm.v[st][0][0], LV + (j_lo + (int64_t)t * kDecTile) * D, bytes, &sm.full[st]);
  };
  if (!mem) {
    if (threadIdx.x == 0) {
      for (int st = 0; st < kDecStages; ++st) mbar_init(&sm.full[st], 1);
      fence_mbar_init();
      for (int t = 0; t < ntiles && t < kDecStages; ++t) issue_local(t);
    }
    __syncthreads();
  }

  // ---- rows and rotated query slices (dims [8 sl, 8 sl + 8) and partners)
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
    int64_t pos = mem ? (int64_t)k + Lb + t : Lb + t - j_lo;
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

  for (int t = 0; t < ntiles; ++t) {
    const int st = t % kDecStages;
    const int64_t kb = (int64_t)t * kDecTile;            // first key of the tile (split-relative)
    const int n_t = (int)min64(kDecTile, nkeys - kb);
    if (mem) {                                           // gather memory rows into the stage
      __syncthreads();
      if (threadIdx.x < n_t) {                           // source rows of each key, once
        const int64_t kk = kb + threadIdx.x;
        int r = 0;
        while (sm.mem_pref[r + 1] <= kk) ++r;
        const int64_t ci = kk - sm.mem_pref[r];
        sm.key_krow[threadIdx.x] = sm.mem_krow[r] + ci;
        sm.key_vrow[threadIdx.x] = sm.mem_vrow[r] + ci;
      }
      __syncthreads();
      for (int idx = threadIdx.x; idx < n_t * 2 * (ROWB / 16); idx += kDecThreads) {
        const int vec = idx % (ROWB / 16), kv = (idx / (ROWB / 16)) & 1, i = idx / (2 * (ROWB / 16));
        const int64_t row = kv ? sm.key_vrow[i] : sm.key_krow[i];
        const T* src = ((kv && !a.kv_on_host) ? MV : MK) + (row * a.Hkv + g) * D;
        T* dst = kv ? &sm.v[st][i][0] : &sm.k[st][i][0];
        cp_async_16(reinterpret_cast<unsigned char*>(dst) + 16 * vec,
                    reinterpret_cast<const unsigned char*>(src) + 16 * vec);
      }
      cp_async_wait_all();
      __syncthreads();
    } else {
      if (!mbar_wait(&sm.full[st], (uint32_t)((t / kDecStages) & 1))) break;
    }
    const T* Ks = &sm.k[st][0][0];
    const T* Vs = &sm.v[st][0][0];
    for (int i0 = warp * kDecNB * KPW; i0 < n_t; i0 += kDecWarps * kDecNB * KPW) {
      float x[kDecNB][kDecRows];
      bool kv[kDecNB];
#pragma unroll
      for (int u = 0; u < kDecNB; ++u) {
        const int i = i0 + u * KPW + kg;
        kv[u] = i < n_t;
        float kx[16];
        const int ii = kv[u] ? i : 0;
        lds8<T>(Ks + ii * D + 8 * sl, kx);
        lds8<T>(Ks + ii * D + HALF + 8 * sl, kx + 8);
        if (!mem) {                                      // turn the local key by (j - j_lo)
          int64_t rr = kb + ii;
          rr = rr < a.rope_rows ? rr : a.rope_rows - 1;
          const float4* cs = reinterpret_cast<const float4*>(a.rope + rr * HALF + 8 * sl);
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const float4 w = __ldg(cs + e2);
            const float k0 = kx[2 * e2], k1 = kx[8 + 2 * e2];
            kx[2 * e2] = k0 * w.x - k1 * w.y;
            kx[8 + 2 * e2] = k1 * w.x + k0 * w.y;
            const float k2 = kx[2 * e2 + 1], k3 = kx[8 + 2 * e2 + 1];
            kx[2 * e2 + 1] = k2 * w.z - k3 * w.w;
            kx[8 + 2 * e2 + 1] = k3 * w.z + k2 * w.w;
          }
        }
#pragma unroll
        for (int r = 0; r < kDecRows; ++r) {
          float acc = 0.f;
#pragma unroll
          for (int e = 0; e < 16; ++e) acc = fmaf(qv[r][e], kx[e], acc);
#pragma unroll
          for (int o2 = 1; o2 < LPK; o2 <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o2);
          bool vis = kv[u] && row_on[r];
          if (!mem) vis = vis && (j_lo + kb + i <= Lb + row_t[r]);
          x[u][r] = vis ? acc : -INFINITY;
        }
      }
#pragma unroll
      for (int r = 0; r < kDecRows; ++r) {
        float mb = m[r];
#pragma unroll
        for (int u = 0; u < kDecNB; ++u) mb = fmaxf(mb, x[u][r]);
        if (mb == -INFINITY) continue;
        const float sc = exp2f(m[r] - mb);
        l[r] *= sc;
#pragma unroll
        for (int e = 0; e < 16; ++e) o[r][e] *= sc;
        m[r] = mb;
      }
#pragma unroll
      for (int u = 0; u < kDecNB; ++u) {
        if (!kv[u]) continue;
        const int i = i0 + u * KPW + kg;
        float vx[16];
        lds8<T>(Vs + i * D + 8 * sl, vx);
        lds8<T>(Vs + i * D + HALF + 8 * sl, vx + 8);
#pragma unroll
        for (int r = 0; r < kDecRows; ++r) {
          if (x[u][r] == -INFINITY) continue;
          const float p = exp2f(x[u][r] - m[r]);
          l[r] += p;
#pragma unroll
          for (int e = 0; e < 16; ++e) o[r][e] = fmaf(p, vx[e], o[r][e]);
        }
      }
    }
    if (!mem) {
      __syncthreads();                                   // stage free again
      if (threadIdx.x == 0 && t + kDecStages < ntiles) issue_local(t + kDecStages);
    }
  }

  // ---- merge the KPW key slots of the warp (lanes with equal sl)
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
      if (sl == 0) { sm.ml[warp][i][0] = m[i]; sm.ml[warp][i][1] = l[i]; }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        sm.o[warp][i][8 * sl + e] = o[i][e];
        sm.o[warp][i][HALF + 8 * sl + e] = o[i][8 + e];
      }
    }
  }
  __syncthreads();
  // ---- merge the warps and write this split's partial
  const int sid = a.split_off[b] + s;
  for (int idx = threadIdx.x; idx < kDecRows * D; idx += kDecThreads) {
    const int i = idx / D, dd = idx % D;
    const int r = rg * kDecRows + i;
    if (r >= a.R) continue;
    float mt = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) mt = fmaxf(mt, sm.ml[w][i][0]);
    float lt = 0.f, ot = 0.f;
    if (mt != -INFINITY) {
      for (int w = 0; w < kDecWarps; ++w) {
        const float mw = sm.ml[w][i][0];
        if (mw == -INFINITY) continue;
        const float sc = exp2f(mw - mt);
        lt += sm.ml[w][i][1] * sc;
        ot += sm.o[w][i][dd] * sc;
      }
    }
    const int64_t prow = ((int64_t)sid * a.Hkv + g) * a.R + r;
    a.part_o[prow * D + dd] = ot;
    if (dd == 0) {
      a.part_ml[prow * 2] = mt;
      a.part_ml[prow * 2 + 1] = lt;
    }
  }

  // ---- the last split of this (query, kv head, row group) merges them all
  __syncthreads();
  int* counter = a.counters + ((int64_t)b * a.Hkv + g) * a.n_rg + rg;
  if (threadIdx.x == 0) {
    __threadfence();
    const int done = atomicAdd(counter, 1);
    sm.last = (done == nsplit - 1);
  }
  __syncthreads();
  if (!sm.last) return;
  __threadfence();
  const int nrow = min(kDecRows, a.R - rg * kDecRows);
  // row maxima over the splits
  float mx[kDecRows];
#pragma unroll
  for (int i = 0; i < kDecRows; ++i) mx[i] = -INFINITY;
  for (int ss = threadIdx.x; ss < nsplit; ss += kDecThreads) {
    const int64_t base = ((int64_t)(a.split_off[b] + ss) * a.Hkv + g) * a.R + rg * kDecRows;
#pragma unroll
    for (int i = 0; i < kDecRows; ++i)
      if (i < nrow) mx[i] = fmaxf(mx[i], __ldcg(&a.part_ml[(base + i) * 2]));
  }
#pragma unroll
  for (int i = 0; i < kDecRows; ++i) {
    float v = mx[i];
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o2));
    if (lane == 0) sm.red[warp][i] = v;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < kDecRows; ++i) {
    float v = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) v = fmaxf(v, sm.red[w][i]);
    mx[i] = v;
  }
  __syncthreads();
  // split weights and the row sums
  float ls[kDecRows];
#pragma unroll
  for (int i = 0; i < kDecRows; ++i) ls[i] = 0.f;
  for (int ss = threadIdx.x; ss < nsplit; ss += kDecThreads) {
    const int64_t base = ((int64_t)(a.split_off[b] + ss) * a.Hkv + g) * a.R + rg * kDecRows;
#pragma unroll
    for (int i = 0; i < kDecRows; ++i) {
      float w = 0.f;
      if (i < nrow) {
        const float ms = __ldcg(&a.part_ml[(base + i) * 2]);
        if (ms != -INFINITY) w = exp2f(ms - mx[i]);
        ls[i] += w * __ldcg(&a.part_ml[(base + i) * 2 + 1]);
      }
      sm.w[ss][i] = w;
    }
  }
#pragma unroll
  for (int i = 0; i < kDecRows; ++i) {
    float v = ls[i];
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o2);
    if (lane == 0) sm.red[warp][i] = v;
  }
  __syncthreads();
  if (threadIdx.x < kDecRows) {
    float v = 0.f;
    for (int w = 0; w < kDecWarps; ++w) v += sm.red[w][threadIdx.x];
    sm.rowl[threadIdx.x] = v;
  }
  __syncthreads();
  T* out = reinterpret_cast<T*>(a.out);
  if (threadIdx.x < D) {                               // thread = one output dim, all rows
    const int dd = threadIdx.x;
    float acc[kDecRows];
#pragma unroll
    for (int i = 0; i < kDecRows; ++i) acc[i] = 0.f;
    constexpr int kBatch = 8;                          // splits whose partials load together
    for (int s0 = 0; s0 < nsplit; s0 += kBatch) {
      float v[kBatch][kDecRows];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
#pragma unroll
        for (int i = 0; i < kDecRows; ++i) {
          const int ss = s0 + u;
          const int64_t prow = ((int64_t)(a.split_off[b] + ss) * a.Hkv + g) * a.R + rg * kDecRows + i;
          v[u][i] = (ss < nsplit && i < nrow) ? __ldcg(&a.part_o[prow * D + dd]) : 0.f;
        }
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
#pragma unroll
        for (int i = 0; i < kDecRows; ++i)
          if (s0 + u < nsplit) acc[i] = fmaf(sm.w[s0 + u][i], v[u][i], acc[i]);
    }
#pragma unroll
    for (int i = 0; i < kDecRows; ++i) {
      if (i >= nrow) break;
      const int r = rg * kDecRows + i;
      const int t = r / a.G, h = g * a.G + r % a.G;
      Elem<T>::store1(out + (((int64_t)b * a.T + t) * a.Hq + h) * D + dd, acc[i] / sm.rowl[i]);
    }
  }
  if (threadIdx.x == 0) *counter = 0;                   // ready for the next call
}

}  // namespace msa
