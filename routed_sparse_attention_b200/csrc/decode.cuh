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
// is two contiguous row ranges (K and V of one head) fetched by bulk TMA, two
// stages deep; a memory tile is gathered row by row with cp.async.  The CTA
// writes its softmax partial (reference max, sum, unnormalised output); the
// last CTA of each (query, kv head, row group) to finish -- counted with an
// atomic in the workspace, which it resets to zero -- merges every split and
// writes the output.
//
// Rotary positions: the query token t sits at top_k + L_b + t and is rotated
// there once per CTA; local key j was rotated at top_k + j when it entered the
// key cache (msa_rope_local), and pooled memory keys keep their
// document-local rotation from encoding.  Within a tile a warp takes 16
// consecutive keys and each lane group every KPW-th of them.
//
// This CUDA-core kernel serves fp32 banks, where the tensor-core path's bf16
// operands would not meet fp32 accuracy; bf16 banks use decode_mma.cuh.  The
// key loop is kept rolled (one key per lane group per trip) and the softmax
// rescales lazily.
#pragma once
#include <climits>
#include <cstddef>

#include "msa_common.cuh"

namespace msa {

constexpr int kDecMaxB = 256;
constexpr int kDecRows = 4;          // query rows per CTA
constexpr int kDecWarps = 4;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecTile = 64;         // keys per shared-memory tile
constexpr int kDecWarpKeys = kDecTile / kDecWarps;
constexpr int kDecStages = 2;
constexpr int kDecMaxSplits = 512;   // splits per (query, kv head)
constexpr int kMaxTopKDecode = 64;   // selected documents per query
// A lane keeps its reference max until a score exceeds it by this much (log2
// units); the terms it sums then stay below 2^8 each.
constexpr float kLazyRescale = 8.0f;

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
  float* part_ml;                    // [S_tot][Hkv][R][2] (reference max, sum) in log2 units
  int* counters;                     // [B][Hkv][n_rg], zero between calls
  void* out;
  float* lse;                        // [B][T][Hq] natural-log log-sum-exp of the scaled logits, or null
  const int64_t* local_len_dev;      // live lengths read on the device ([B]), or null: local_len below
  int32_t split_off[kDecMaxB + 1];   // first split id of query b
  int64_t local_off[kDecMaxB + 1];   // row offset of query b's local cache (capacity = difference)
  int64_t local_len[kDecMaxB];       // live local tokens of query b
};

template <typename T, int D>
struct DecSmem {
  static constexpr int kSrc = kDecWarps * 32 / (D / 16);   // lane groups per CTA
  union {
    struct {                           // key tiles while the keys stream
      T k[kDecStages][kDecTile][D];
      T v[kDecStages][kDecTile][D];
    } tile;
    struct {                           // merge scratch afterwards
      float2 o[kSrc][kDecRows][D / 2]; // lane group partials, dims (p, p + d/2) paired
      float2 ml[kSrc][kDecRows];       // (reference max, sum)
      float w[kSrc][kDecRows];
      float cw[kDecMaxSplits][kDecRows];   // split weights (last CTA)
      float cl[kDecMaxSplits][kDecRows];   // split sums (last CTA)
    } post;
  } u;
  uint64_t full[kDecStages];
  int64_t mem_pref[kMaxTopKDecode + 1];
  int64_t mem_krow[kMaxTopKDecode];    // first K row of rank r's document (rows of [H_kv][d])
  int64_t mem_vrow[kMaxTopKDecode];    // first V row
  int64_t key_krow[kDecTile];          // K / V source rows of the current memory tile's keys
  int64_t key_vrow[kDecTile];
  float rowm[kDecRows], rowl[kDecRows];
  int last;
};

// Live local tokens of query b: from the kernel parameters, or from device
// memory when the caller keeps them there (clamped to [T, capacity]; a value
// outside that range raises MSA_DEV_BAD_SHAPE).
__device__ __forceinline__ int64_t live_len(const DecodeArgs& a, int b) {
  if (!a.local_len_dev) return a.local_len[b];
  const int64_t cap = a.local_off[b + 1] - a.local_off[b];
  int64_t n = a.local_len_dev[b];
  if (n < a.T || n > cap) {
    if (threadIdx.x == 0) dev_flag(MSA_DEV_BAD_SHAPE);
    n = n < a.T ? a.T : cap;
  }
  return n;
}

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
// A row's 16 dims of this lane as pairs (dim 8 sl + e, dim d/2 + 8 sl + e).
template <typename T, int HALF>
__device__ __forceinline__ void lds_pairs(const T* row, int sl, float2 (&x)[8]) {
  float f[16];
  lds8<T>(row + 8 * sl, f);
  lds8<T>(row + HALF + 8 * sl, f + 8);
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = make_float2(f[e], f[8 + e]);
}
// (cos, sin) of this lane's 8 rotary pairs at table row `row`.
__device__ __forceinline__ void rope8(const float2* rope, int64_t row, int half, int sl, float2 (&z)[8]) {
  const float4* cs = reinterpret_cast<const float4*>(rope + row * half + 8 * sl);
#pragma unroll
  for (int e2 = 0; e2 < 4; ++e2) {
    const float4 w = __ldg(cs + e2);
    z[2 * e2] = make_float2(w.x, w.y);
    z[2 * e2 + 1] = make_float2(w.z, w.w);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads)
decode_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int LPK = D / 16;             // lanes per key (16 dims each)
  constexpr int KPW = 32 / LPK;           // keys per warp step
  constexpr int HALF = D / 2;
  constexpr int ROWB = D * (int)sizeof(T);
  constexpr int NPL = kDecWarpKeys / KPW; // keys of a lane group per tile
  using Smem = DecSmem<T, D>;
  constexpr int NSRC = Smem::kSrc;
  static_assert(NPL * KPW == kDecWarpKeys, "a warp's keys split into whole steps");
  static_assert(HALF <= 64 && NSRC <= 32, "head_dim 64 or 128");
  static_assert(kDecWarps >= kDecRows, "one warp per row in the merges");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kg = lane / LPK, sl = lane % LPK;
  int b = 0;
  while (b + 1 < a.B && a.split_off[b + 1] <= (int)blockIdx.x) ++b;
  const int s = blockIdx.x - a.split_off[b];
  const int nsplit = a.split_off[b + 1] - a.split_off[b];
  const int g = blockIdx.y / a.n_rg, rg = blockIdx.y % a.n_rg;
  const int64_t cap = a.local_off[b + 1] - a.local_off[b];   // row stride of a head
  const int64_t Ltot = live_len(a, b);                       // live local tokens
  const int64_t Lb = Ltot - a.T;
  const int k = a.top_k;
  const bool mem = (s == 0);
  // the memory split's first dependent load goes out before anything else
  int doc = 0;
  if (mem && threadIdx.x < k) doc = __ldg(a.sel + (int64_t)b * k + threadIdx.x);

  const T* LK = reinterpret_cast<const T*>(a.lk) + (a.local_off[b] * a.Hkv + (int64_t)g * cap) * D;
  const T* LV = reinterpret_cast<const T*>(a.lv) + (a.local_off[b] * a.Hkv + (int64_t)g * cap) * D;
  const T* MK = reinterpret_cast<const T*>(a.mem_k);
  const T* MV = reinterpret_cast<const T*>(a.mem_v);

  // ---- local splits: key range known at once; issue the first tiles
  const int64_t j_lo = mem ? 0 : (int64_t)(s - 1) * a.S;
  int64_t nkeys = mem ? 0 : min64(a.S, Ltot - j_lo);
  if (nkeys < 0) nkeys = 0;                                   // a split past the live tokens
  auto issue_local = [&](int t) {                      // thread 0 only
    const int st = t % kDecStages;
    const int64_t n_t = min64(kDecTile, nkeys - (int64_t)t * kDecTile);
    const uint32_t bytes = (uint32_t)(n_t * ROWB);
    mbar_arrive_expect_tx(&sm.full[st], 2 * bytes);
    tma_load_1d(&sm.u.tile.k[st][0][0], LK + (j_lo + (int64_t)t * kDecTile) * D, bytes, &sm.full[st]);
    tma_load_1d(&sm.u.tile.v[st][0][0], LV + (j_lo + (int64_t)t * kDecTile) * D, bytes, &sm.full[st]);
  };
  if (!mem && threadIdx.x == 0) {
    const int nt0 = (int)((nkeys + kDecTile - 1) / kDecTile);
    for (int st = 0; st < kDecStages; ++st) mbar_init(&sm.full[st], 1);
    fence_mbar_init();
    for (int t = 0; t < nt0 && t < kDecStages; ++t) issue_local(t);
  }

  // ---- rows and rotated query pairs (dims 8 sl + e and d/2 + 8 sl + e)
  const T* Q = reinterpret_cast<const T*>(a.q);
  float2 qp[kDecRows][8];
  int lim[kDecRows];                 // last split-relative key a row sees (-1: none)
#pragma unroll
  for (int i = 0; i < kDecRows; ++i) {
    const int r = rg * kDecRows + i;
    bool on = r < a.R;
    const int t = on ? r / a.G : 0, hh = on ? r % a.G : 0;
    const int h = g * a.G + hh;
    int64_t pos = (int64_t)k + Lb + t;
    const int64_t last = Lb + t - j_lo;                // last split-relative local key the row sees
    if (!mem && last < 0) on = false;                  // every key of the split is in its future
    lim[i] = !on ? -1 : (mem ? INT_MAX : (int)min64(last, INT_MAX));
    if (pos >= a.rope_rows) { dev_flag(MSA_DEV_ROPE_RANGE); pos = a.rope_rows - 1; }
    float x0[8], x1[8];
    const T* qr = Q + (((int64_t)b * a.T + t) * a.Hq + h) * D;
    load8<T>(qr + 8 * sl, x0);
    load8<T>(qr + HALF + 8 * sl, x1);
    float2 w[8];
    rope8(a.rope, pos, HALF, sl, w);
    const float sc = on ? a.scale_log2 : 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      qp[i][e] = make_float2((x0[e] * w[e].x - x1[e] * w[e].y) * sc, (x1[e] * w[e].x + x0[e] * w[e].y) * sc);
  }
  const int wb = warp * kDecWarpKeys;                  // this warp's first key of a tile

  // ---- memory split: rank r's chunk count and first K / V rows
  if (mem) {
    if (threadIdx.x < k) {
      const int r = threadIdx.x;
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
    __syncthreads();                                   // barriers initialised
  }
  const int ntiles = (int)((nkeys + kDecTile - 1) / kDecTile);

  float mref[kDecRows], l[kDecRows];
  float2 o[kDecRows][8];
#pragma unroll
  for (int i = 0; i < kDecRows; ++i) {
    mref[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[i][e] = make_float2(0.f, 0.f);
  }

#pragma unroll 1
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
        T* dst = kv ? &sm.u.tile.v[st][i][0] : &sm.u.tile.k[st][i][0];
        cp_async_16(reinterpret_cast<unsigned char*>(dst) + 16 * vec,
                    reinterpret_cast<const unsigned char*>(src) + 16 * vec);
      }
      cp_async_wait_all();
      __syncthreads();
    } else {
      // every thread leaves together if the wait ran out (the loop has CTA barriers)
      if (!__syncthreads_and(mbar_wait(&sm.full[st], (uint32_t)((t / kDecStages) & 1)))) break;
    }
    const T* Ks = &sm.u.tile.k[st][0][0];
    const T* Vs = &sm.u.tile.v[st][0][0];
#pragma unroll 1
    for (int mm = 0; mm < NPL; ++mm) {
      const int i = wb + kg + KPW * mm;
      const bool kval = i < n_t;
      const int ii = kval ? i : 0;
      float2 kp[8];
      lds_pairs<T, HALF>(Ks + ii * D, sl, kp);
      float xs[kDecRows];
#pragma unroll
      for (int r = 0; r < kDecRows; ++r) {
        float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc2 = __ffma2_rn(qp[r][e], kp[e], acc2);
        float acc = acc2.x + acc2.y;
#pragma unroll
        for (int o2 = 1; o2 < LPK; o2 <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o2);
        xs[r] = (kval && kb + i <= lim[r]) ? acc : -INFINITY;
      }
      float2 vp[8];
      lds_pairs<T, HALF>(Vs + ii * D, sl, vp);
#pragma unroll
      for (int r = 0; r < kDecRows; ++r) {
        if (xs[r] == -INFINITY) continue;
        if (xs[r] > mref[r] + kLazyRescale) {            // new reference max
          const float sc = exp2f(mref[r] - xs[r]);
          const float2 sc2 = make_float2(sc, sc);
          l[r] *= sc;
#pragma unroll
          for (int e = 0; e < 8; ++e) o[r][e] = __fmul2_rn(o[r][e], sc2);
          mref[r] = xs[r];
        }
        const float p = exp2f(xs[r] - mref[r]);
        const float2 p2 = make_float2(p, p);
        l[r] += p;
#pragma unroll
        for (int e = 0; e < 8; ++e) o[r][e] = __ffma2_rn(p2, vp[e], o[r][e]);
      }
    }
    if (!mem) {
      __syncthreads();                                   // stage free again
      if (threadIdx.x == 0 && t + kDecStages < ntiles) issue_local(t + kDecStages);
    }
  }
  __syncthreads();                                       // tiles done: shared memory becomes merge scratch

  // ---- merge the CTA's lane groups and write this split's partial
  const int src = warp * KPW + kg;
#pragma unroll
  for (int i = 0; i < kDecRows; ++i) {
    float4* dst = reinterpret_cast<float4*>(&sm.u.post.o[src][i][8 * sl]);
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2)
      dst[e2] = make_float4(o[i][2 * e2].x, o[i][2 * e2].y, o[i][2 * e2 + 1].x, o[i][2 * e2 + 1].y);
    if (sl == 0) sm.u.post.ml[src][i] = make_float2(mref[i], l[i]);
  }
  __syncthreads();
  if (warp < kDecRows) {                                 // warp i: row i's reference max and weights
    const int i = warp;
    const float2 ml = lane < NSRC ? sm.u.post.ml[lane][i] : make_float2(-INFINITY, 0.f);
    float mt = ml.x;
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o2));
    const float wgt = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - mt);
    const float lt = warp_sum(wgt * ml.y);
    if (lane < NSRC) sm.u.post.w[lane][i] = wgt;
    if (lane == 0) { sm.rowm[i] = mt; sm.rowl[i] = lt; }
  }
  __syncthreads();
  const int sid = a.split_off[b] + s;
  for (int idx = threadIdx.x; idx < kDecRows * HALF; idx += kDecThreads) {
    const int i = idx / HALF, p = idx % HALF;
    const int r = rg * kDecRows + i;
    if (r >= a.R) continue;
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll 4
    for (int q = 0; q < NSRC; ++q) {
      const float wq = sm.u.post.w[q][i];
      acc = __ffma2_rn(make_float2(wq, wq), sm.u.post.o[q][i][p], acc);
    }
    const int64_t prow = ((int64_t)sid * a.Hkv + g) * a.R + r;
    a.part_o[prow * D + p] = acc.x;
    a.part_o[prow * D + HALF + p] = acc.y;
    if (p == 0) reinterpret_cast<float2*>(a.part_ml)[prow] = make_float2(sm.rowm[i], sm.rowl[i]);
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
  for (int ss = threadIdx.x; ss < nsplit; ss += kDecThreads) {   // every split's (max, sum)
    const int64_t base = ((int64_t)(a.split_off[b] + ss) * a.Hkv + g) * a.R + rg * kDecRows;
#pragma unroll
    for (int i = 0; i < kDecRows; ++i) {
      const float2 v = i < nrow ? __ldcg(reinterpret_cast<const float2*>(a.part_ml) + base + i)
                                : make_float2(-INFINITY, 0.f);
      sm.u.post.cw[ss][i] = v.x;
      sm.u.post.cl[ss][i] = v.y;
    }
  }
  __syncthreads();
  if (warp < kDecRows) {                                 // warp i: row i's max and weighted sum
    const int i = warp;
    float mx = -INFINITY;
    for (int ss = lane; ss < nsplit; ss += 32) mx = fmaxf(mx, sm.u.post.cw[ss][i]);
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
    float lsum = 0.f;
    for (int ss = lane; ss < nsplit; ss += 32) {
      const float ms = sm.u.post.cw[ss][i];
      const float wgt = (ms == -INFINITY) ? 0.f : exp2f(ms - mx);
      sm.u.post.cw[ss][i] = wgt;
      lsum += wgt * sm.u.post.cl[ss][i];
    }
    lsum = warp_sum(lsum);
    if (lane == 0) {
      sm.rowl[i] = lsum;
      const int r = rg * kDecRows + i;
      if (a.lse && i < nrow)                           // (max + log2 sum) in log2 units, to natural log
        a.lse[((int64_t)b * a.T + r / a.G) * a.Hq + g * a.G + r % a.G] = (mx + log2f(lsum)) * 0.6931471805599453f;
    }
  }
  __syncthreads();
  T* out = reinterpret_cast<T*>(a.out);
  constexpr int QD = D / 4;                            // float4 quads per row
  constexpr int kBatch = 8;                            // split partials loaded together
  for (int idx = threadIdx.x; idx < nrow * QD; idx += kDecThreads) {
    const int i = idx / QD, qd = idx % QD;
    const int r = rg * kDecRows + i;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
    for (int s0 = 0; s0 < nsplit; s0 += kBatch) {
      float4 v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int ss = min(s0 + u, nsplit - 1);
        const int64_t prow = ((int64_t)(a.split_off[b] + ss) * a.Hkv + g) * a.R + r;
        v[u] = __ldcg(reinterpret_cast<const float4*>(a.part_o + prow * D) + qd);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const float wgt = (s0 + u < nsplit) ? sm.u.post.cw[s0 + u][i] : 0.f;
        acc.x = fmaf(wgt, v[u].x, acc.x);
        acc.y = fmaf(wgt, v[u].y, acc.y);
        acc.z = fmaf(wgt, v[u].z, acc.z);
        acc.w = fmaf(wgt, v[u].w, acc.w);
      }
    }
    const float inv = 1.0f / sm.rowl[i];
    const int t = r / a.G, h = g * a.G + r % a.G;
    T* op = out + (((int64_t)b * a.T + t) * a.Hq + h) * D + 4 * qd;
    Elem<T>::store1(op + 0, acc.x * inv);
    Elem<T>::store1(op + 1, acc.y * inv);
    Elem<T>::store1(op + 2, acc.z * inv);
    Elem<T>::store1(op + 3, acc.w * inv);
  }
  if (threadIdx.x == 0) *counter = 0;                   // ready for the next call
}

}  // namespace msa
