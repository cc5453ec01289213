// Stage 2 kernels: router-key scan, Top-k, certified exact re-scoring.
//
// Method: "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts",
// section "How MSA compresses and routes documents" (router projector scores
// relevance by cosine similarity, mean over heads, max over tokens, Top-k) and
// "EverMind Releases Memory-Sparse Attention Code for Long-Context AI Models",
// section "Architectural Design and Inference" (stage 2, online routing).
//
// Pipeline of one msa_route call (all on one stream, no host round trip):
//   route_prep_kernel   : per query token, u[t][g] = (1/H_q) sum_{h in g}
//                         Qr[t,h] / max(|Qr[t,h]|, 1e-12); zero the per-document
//                         score array; first document of each scan CTA.
//   kr_scan_kernel      : stream the whole Kr bank once (bulk TMA into a
//                         shared-memory ring); per chunk and kv head the dot
//                         with u and the norm of Kr; the head-mean cosine of
//                         the chunk is sum_g dot_g / max(|Kr_g|, 1e-12), whose
//                         max over chunks and tokens goes to the document
//                         (atomicMax on an order-preserving encoding).
//   topk_local_kernel   : per slice of documents, its top-k keys and every
//                         document within 2*eps of its k-th score.
//   merge_band_kernel   : per query, the global k-th fast score tau and the
//                         band {s : fast_s >= tau - 2*eps}.
//   rescore_kernel      : exact fp64 score of every band document, in the
//                         fixed operation order of the formula.
//   final_select_kernel : top-k of the band by (exact desc, index asc).
// Certification: every fast score is within eps of the exact one (fp32 error
// analysis gives ~1.2e-5 for 128-dim keys; eps = 2^-12), so the exact top-k
// lies inside the band, and the re-scored result equals the fp64 formula.
#pragma once
#include <climits>

#include "msa_common.cuh"

namespace msa {

constexpr float kRouteEps = 1.0f / 4096.0f;           // eps: bound on |fast - exact|
constexpr float kBandMargin = 2.0f * kRouteEps + 1.0f / 1048576.0f;  // 2 eps + rounding slack
constexpr int kTopkSlice = 2048;                      // documents per top-k slice
constexpr int kMaxTopK = 64;

// ----------------------------------------------------------------- prep
template <typename T>
__global__ void route_prep_kernel(const T* __restrict__ qr, int NQ, int Hq, int Hkv, int dr,
                                  float* __restrict__ u, uint32_t* __restrict__ score,
                                  int64_t n_score, const int64_t* __restrict__ doc_chunk_off,
                                  int64_t D, int64_t C, int n_cta, int* __restrict__ cta_first_doc) {
  extern __shared__ float s_inv[];     // [Hq]
  const int G = Hq / Hkv;
  if ((int)blockIdx.x < NQ) {
    const int q = blockIdx.x;
    const T* Q = qr + (int64_t)q * Hq * dr;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int h = warp; h < Hq; h += nw) {
      float ss = 0.f;
      for (int i = lane; i < dr; i += 32) {
        const float x = Elem<T>::load1(Q + (int64_t)h * dr + i);
        ss += x * x;
      }
      ss = warp_sum(ss);
      if (lane == 0) s_inv[h] = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
    }
    __syncthreads();
    for (int gi = threadIdx.x; gi < Hkv * dr; gi += blockDim.x) {
      const int g = gi / dr, i = gi % dr;
      float acc = 0.f;
      for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        acc += Elem<T>::load1(Q + (int64_t)h * dr + i) * s_inv[h];
      }
      u[(int64_t)q * Hkv * dr + gi] = acc / (float)Hq;
    }
  }
  const int64_t gt = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t gs = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = gt; i < n_score; i += gs) score[i] = 0u;
  // CTA i of the scan starts at chunk floor(i*C/n_cta); record the document
  // holding that chunk.
  for (int64_t s = gt; s < D; s += gs) {
    const int64_t a = doc_chunk_off[s], b = doc_chunk_off[s + 1];
    const int64_t ilo = (a * n_cta + C - 1) / C, ihi = (b * n_cta + C - 1) / C;
    for (int64_t i = ilo; i < ihi && i < n_cta; ++i) cta_first_doc[i] = (int)s;
  }
}

// ----------------------------------------------------------------- scan
// Chunk row = H_kv heads x 256 bytes (router_dim * element size = 256), read
// as 16-byte units: lane l reads units l + 32j (j < SEG = H_kv / 2), which is
// conflict-free in shared memory.  Unit l + 32j covers head 2j + (l >> 4),
// dims [(l & 15) * E, +E) with E elements per unit, so each head is spread over
// 16 lanes of one half-warp and reduced with four xor-shuffles.
template <typename T, int NQG, int SEG>
struct ScanCfg {
  static constexpr int E = Elem<T>::kPerVec;
  static constexpr int ROW = SEG * 512;                 // bytes per chunk row
  static constexpr int STAGE_BYTES = 16384;
  static constexpr int SCH = STAGE_BYTES / ROW;         // chunks per stage
  static constexpr int NSTAGE = 6;
  static constexpr int NCW = 8;                         // consumer warps
  static constexpr int THREADS = (NCW + 1) * 32;        // + 1 producer warp
  static constexpr int SMEM = NSTAGE * STAGE_BYTES + 2 * NSTAGE * 8;
};

template <typename T, int NQG, int SEG>
__global__ void __launch_bounds__(ScanCfg<T, NQG, SEG>::THREADS)
kr_scan_kernel(const T* __restrict__ kr, const float* __restrict__ u, int NQ, int Ttok,
               const int64_t* __restrict__ doc_chunk_off, int64_t C, const int* __restrict__ cta_first_doc,
               uint32_t* __restrict__ score, int64_t D) {
  using Cfg = ScanCfg<T, NQG, SEG>;
  constexpr int E = Cfg::E, ROW = Cfg::ROW, SCH = Cfg::SCH, NSTAGE = Cfg::NSTAGE, NCW = Cfg::NCW;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NSTAGE * Cfg::STAGE_BYTES);
  uint64_t* empty = full + NSTAGE;

  const int n_cta = gridDim.x;
  const int64_t cs = (int64_t)blockIdx.x * C / n_cta;
  const int64_t ce = (int64_t)(blockIdx.x + 1) * C / n_cta;
  if (cs >= ce) return;
  const int64_t nst = (ce - cs + SCH - 1) / SCH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = blockIdx.y * NQG;
  const int nq = min(NQG, NQ - q0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NCW) {                               // producer warp
    if (lane == 0) {
      const unsigned char* src = reinterpret_cast<const unsigned char*>(kr) + cs * ROW;
      for (int64_t st = 0; st < nst; ++st) {
        const int slot = (int)(st % NSTAGE);
        if (st >= NSTAGE && !mbar_wait(&empty[slot], (uint32_t)((st / NSTAGE - 1) & 1))) break;
        const int64_t nch = min64(SCH, ce - cs - st * SCH);
        const uint32_t bytes = (uint32_t)(nch * ROW);
        mbar_arrive_expect_tx(&full[slot], bytes);
        tma_load_1d(smem + slot * Cfg::STAGE_BYTES, src + st * SCH * ROW, bytes, &full[slot]);
      }
    }
    return;
  }

  // consumer warps: query slices in registers
  float uq[NQG][SEG][E];
  const int hsel = lane >> 4, dsel = (lane & 15) * E;
#pragma unroll
  for (int q = 0; q < NQG; ++q)
#pragma unroll
    for (int j = 0; j < SEG; ++j) {
      const int head = 2 * j + hsel;
#pragma unroll
      for (int e = 0; e < E; ++e)
        uq[q][j][e] = (q < nq) ? u[((int64_t)(q0 + q) * (2 * SEG) + head) * (16 * E) + dsel + e] : 0.f;
    }

  int64_t cur = cta_first_doc[blockIdx.x];
  for (int64_t st = 0; st < nst; ++st) {
    const int slot = (int)(st % NSTAGE);
    if (!mbar_wait(&full[slot], (uint32_t)((st / NSTAGE) & 1))) return;
    const int64_t cbase = cs + st * SCH;
    const int nch = (int)min64(SCH, ce - cbase);
    const unsigned char* stage = smem + slot * Cfg::STAGE_BYTES;
    for (int ci = warp; ci < nch; ci += NCW) {
      const uint4* rowp = reinterpret_cast<const uint4*>(stage + ci * ROW);
      float dot[SEG][NQG], nrm[SEG];
#pragma unroll
      for (int j = 0; j < SEG; ++j) {
        float x[E];
        Elem<T>::unpack(rowp[lane + 32 * j], x);
        float n2 = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) n2 = fmaf(x[e], x[e], n2);
        nrm[j] = n2;
#pragma unroll
        for (int q = 0; q < NQG; ++q) {
          float a = 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) a = fmaf(x[e], uq[q][j][e], a);
          dot[j][q] = a;
        }
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
#pragma unroll
        for (int j = 0; j < SEG; ++j) {
          nrm[j] += __shfl_xor_sync(0xffffffffu, nrm[j], o);
#pragma unroll
          for (int q = 0; q < NQG; ++q) dot[j][q] += __shfl_xor_sync(0xffffffffu, dot[j][q], o);
        }
      }
      float sq[NQG];
#pragma unroll
      for (int q = 0; q < NQG; ++q) {
        float a = 0.f;
#pragma unroll
        for (int j = 0; j < SEG; ++j) a += dot[j][q] / fmaxf(sqrtf(nrm[j]), 1e-12f);
        sq[q] = a + __shfl_xor_sync(0xffffffffu, a, 16);
      }
      const int64_t c = cbase + ci;
      while (doc_chunk_off[cur + 1] <= c) ++cur;
      if (lane == 0) {
#pragma unroll
        for (int q = 0; q < NQG; ++q)
          if (q < nq) atomicMax(&score[(int64_t)((q0 + q) / Ttok) * D + cur], enc_f32(sq[q]));
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
}

// ------------------------------------------------------------ block argmax
__device__ __forceinline__ unsigned long long block_max_u64(unsigned long long v, unsigned long long* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w > v ? w : v;
  }
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  unsigned long long r = 0;
  for (int i = 0; i < nw; ++i) r = red[i] > r ? red[i] : r;
  return r;
}

// key = enc(score) << 32 | (0xffffffff - doc): larger key = better (score
// desc, index asc); 0 = none.
__device__ __forceinline__ unsigned long long doc_key(uint32_t enc, int64_t doc) {
  return ((unsigned long long)enc << 32) | (0xffffffffull - (unsigned long long)doc);
}

// ------------------------------------------------------------ local top-k
constexpr int kTopkThreads = 256;
constexpr int kTopkPer = kTopkSlice / kTopkThreads;

__global__ void __launch_bounds__(kTopkThreads)
topk_local_kernel(const uint32_t* __restrict__ score, int64_t D, int k,
                  unsigned long long* __restrict__ loc_keys, int* __restrict__ cand,
                  int* __restrict__ cand_cnt) {
  __shared__ unsigned long long red[kTopkThreads / 32];
  __shared__ int s_cnt;
  const int p = blockIdx.x, b = blockIdx.y, P = gridDim.x;
  const int64_t d0 = (int64_t)p * kTopkSlice;
  const uint32_t* sc = score + (int64_t)b * D;
  unsigned long long key[kTopkPer];
#pragma unroll
  for (int i = 0; i < kTopkPer; ++i) {
    const int64_t doc = d0 + threadIdx.x + i * kTopkThreads;
    key[i] = doc < D ? doc_key(sc[doc], doc) : 0ull;
  }
  unsigned long long last = ~0ull;
  unsigned long long* out = loc_keys + ((int64_t)b * P + p) * k;
  for (int r = 0; r < k; ++r) {
    unsigned long long best = 0;
#pragma unroll
    for (int i = 0; i < kTopkPer; ++i)
      if (key[i] < last && key[i] > best) best = key[i];
    best = block_max_u64(best, red);
    if (threadIdx.x == 0) out[r] = best;
    last = best;
  }
  // candidates: every document within the band of this slice's k-th score
  uint32_t thr = 0;
  if (last != 0) thr = enc_f32(dec_f32((uint32_t)(last >> 32)) - kBandMargin);
  if (threadIdx.x == 0) s_cnt = 0;
  __syncthreads();
  int* cl = cand + ((int64_t)b * P + p) * kTopkSlice;
#pragma unroll
  for (int i = 0; i < kTopkPer; ++i) {
    const int64_t doc = d0 + threadIdx.x + i * kTopkThreads;
    if (key[i] != 0 && (uint32_t)(key[i] >> 32) >= thr) cl[atomicAdd(&s_cnt, 1)] = (int)(doc - d0);
  }
  __syncthreads();
  if (threadIdx.x == 0) cand_cnt[(int64_t)b * P + p] = s_cnt;
}

// ------------------------------------------------------------ merge + band
constexpr int kMergeThreads = 1024;

__global__ void __launch_bounds__(kMergeThreads)
merge_band_kernel(const uint32_t* __restrict__ score, int64_t D, int k, int P, int Ttok,
                  const unsigned long long* __restrict__ loc_keys, const int* __restrict__ cand,
                  const int* __restrict__ cand_cnt, const int64_t* __restrict__ doc_chunk_off,
                  int* __restrict__ band, int* __restrict__ band_cnt,
                  unsigned long long* __restrict__ band_exact, int64_t* __restrict__ item_off) {
  __shared__ unsigned long long red[kMergeThreads / 32];
  __shared__ int s_cnt;
  __shared__ int64_t s_scan[kMergeThreads / 32];
  const int b = blockIdx.x;
  const int64_t nkeys = (int64_t)P * k;
  const unsigned long long* keys = loc_keys + (int64_t)b * nkeys;
  unsigned long long last = ~0ull;
  for (int r = 0; r < k; ++r) {
    unsigned long long best = 0;
    for (int64_t i = threadIdx.x; i < nkeys; i += blockDim.x) {
      const unsigned long long x = keys[i];
      if (x < last && x > best) best = x;
    }
    last = block_max_u64(best, red);
  }
  const uint32_t thr = enc_f32(dec_f32((uint32_t)(last >> 32)) - kBandMargin);
  if (threadIdx.x == 0) s_cnt = 0;
  __syncthreads();
  const uint32_t* sc = score + (int64_t)b * D;
  int* bl = band + (int64_t)b * D;
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    const int n = cand_cnt[(int64_t)b * P + p];
    const int* cl = cand + ((int64_t)b * P + p) * kTopkSlice;
    for (int i = 0; i < n; ++i) {
      const int64_t doc = (int64_t)p * kTopkSlice + cl[i];
      if (sc[doc] >= thr) bl[atomicAdd(&s_cnt, 1)] = (int)doc;
    }
  }
  __syncthreads();
  const int nb = s_cnt;
  // exclusive prefix of work items (chunks x query tokens) over band entries
  int64_t* io = item_off + (int64_t)b * (D + 1);
  unsigned long long* ex = band_exact + (int64_t)b * D;
  int64_t carry = 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int base = 0; base < nb; base += blockDim.x) {
    const int e = base + threadIdx.x;
    int64_t v = 0;
    if (e < nb) {
      const int doc = bl[e];
      v = (doc_chunk_off[doc + 1] - doc_chunk_off[doc]) * (int64_t)Ttok;
      ex[e] = 0ull;
    }
    int64_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_scan[warp] = incl;
    __syncthreads();
    int64_t wofs = 0;
    for (int w = 0; w < warp; ++w) wofs += s_scan[w];
    int64_t tot = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += s_scan[w];
    if (e < nb) io[e] = carry + wofs + incl - v;
    carry += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    io[nb] = carry;
    band_cnt[b] = nb;
  }
}

// ------------------------------------------------------------ exact rescoring
// One warp per (band document, query token, chunk) item.  Lane h computes the
// cosine of query head h against the chunk's router key of head h / G:
// dot, |q|^2 and |k|^2 are each summed over i = 0 .. dr-1 in order with
// separately rounded IEEE products and sums (no fused multiply-add), then
//   cos = dot / (max(sqrt(|q|^2), 1e-12) * max(sqrt(|k|^2), 1e-12)), clamped;
// the head sum runs h = 0 .. H_q-1 in order and is divided by H_q.
template <typename T>
__device__ __forceinline__ double ld_elem_f64(const T* p) { return (double)Elem<T>::load1(p); }

constexpr int kRescoreThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kRescoreThreads)
rescore_kernel(const T* __restrict__ qr, const T* __restrict__ kr, int B, int Ttok, int Hq, int Hkv,
               int dr, int64_t D, const int64_t* __restrict__ doc_chunk_off,
               const int* __restrict__ band, const int* __restrict__ band_cnt,
               const int64_t* __restrict__ item_off, unsigned long long* __restrict__ band_exact) {
  extern __shared__ double s_cos[];     // [warps][Hq]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw_blk = blockDim.x >> 5;
  double* cb = s_cos + warp * Hq;
  const int64_t gw = (int64_t)blockIdx.x * nw_blk + warp;
  const int64_t nwarps = (int64_t)gridDim.x * nw_blk;
  const int G = Hq / Hkv;
  for (int b = 0; b < B; ++b) {
    const int nb = band_cnt[b];
    const int64_t* io = item_off + (int64_t)b * (D + 1);
    const int64_t total = io[nb];
    const int* bl = band + (int64_t)b * D;
    for (int64_t it = gw; it < total; it += nwarps) {
      int lo = 0, hi = nb;                       // last e with io[e] <= it
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (io[mid] <= it) lo = mid; else hi = mid;
      }
      const int e = lo;
      const int doc = bl[e];
      const int64_t c0 = doc_chunk_off[doc];
      const int64_t nc = doc_chunk_off[doc + 1] - c0;
      const int64_t rem = it - io[e];
      const int t = (int)(rem / nc);
      const int64_t c = c0 + rem % nc;
      for (int h = lane; h < Hq; h += 32) {
        const T* qp = qr + (((int64_t)b * Ttok + t) * Hq + h) * dr;
        const T* kp = kr + (c * Hkv + h / G) * dr;
        double dot = 0.0, nq = 0.0, nk = 0.0;
        for (int i = 0; i < dr; ++i) {
          const double x = ld_elem_f64(qp + i), y = ld_elem_f64(kp + i);
          dot = __dadd_rn(dot, __dmul_rn(x, y));
          nq = __dadd_rn(nq, __dmul_rn(x, x));
          nk = __dadd_rn(nk, __dmul_rn(y, y));
        }
        const double den = __dmul_rn(fmax(__dsqrt_rn(nq), 1e-12), fmax(__dsqrt_rn(nk), 1e-12));
        double cs = __ddiv_rn(dot, den);
        cs = fmin(fmax(cs, -1.0), 1.0);
        cb[h] = cs;
      }
      __syncwarp();
      if (lane == 0) {
        double sum = 0.0;
        for (int h = 0; h < Hq; ++h) sum = __dadd_rn(sum, cb[h]);
        const double S = __ddiv_rn(sum, (double)Hq);
        atomicMax(&band_exact[(int64_t)b * D + e], enc_f64(S));
      }
      __syncwarp();
    }
  }
}

// ------------------------------------------------------------ final selection
constexpr int kFinalThreads = 256;

__device__ __forceinline__ bool better(unsigned long long ea, int da, unsigned long long eb, int db) {
  return ea > eb || (ea == eb && da < db);
}

__global__ void __launch_bounds__(kFinalThreads)
final_select_kernel(int64_t D, int k, const int* __restrict__ band, const int* __restrict__ band_cnt,
                    const unsigned long long* __restrict__ band_exact, int* __restrict__ out_idx,
                    double* __restrict__ out_score) {
  __shared__ unsigned long long r_e[kFinalThreads / 32];
  __shared__ int r_d[kFinalThreads / 32];
  const int b = blockIdx.x;
  const int nb = band_cnt[b];
  const int* bl = band + (int64_t)b * D;
  const unsigned long long* ex = band_exact + (int64_t)b * D;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  unsigned long long le = ~0ull;                 // last pick (start: above everything)
  int ld = -1;
  for (int r = 0; r < k; ++r) {
    unsigned long long be = 0;
    int bd = INT_MAX;   // no document yet
    for (int e = threadIdx.x; e < nb; e += blockDim.x) {
      const unsigned long long x = ex[e];
      const int d = bl[e];
      // candidates strictly after the last pick in (exact desc, doc asc) order
      const bool after = (x < le) || (x == le && d > ld);
      if (after && better(x, d, be, bd)) { be = x; bd = d; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long xe = __shfl_xor_sync(0xffffffffu, be, o);
      const int xd = __shfl_xor_sync(0xffffffffu, bd, o);
      if (better(xe, xd, be, bd)) { be = xe; bd = xd; }
    }
    __syncthreads();
    if (lane == 0) { r_e[warp] = be; r_d[warp] = bd; }
    __syncthreads();
    be = r_e[0]; bd = r_d[0];
    for (int w = 1; w < nw; ++w)
      if (better(r_e[w], r_d[w], be, bd)) { be = r_e[w]; bd = r_d[w]; }
    if (threadIdx.x == 0) {
      out_idx[(int64_t)b * k + r] = bd;
      if (out_score) out_score[(int64_t)b * k + r] = dec_f64(be);
    }
    le = be;
    ld = bd;
  }
}

__global__ void scores_to_float_kernel(const uint32_t* __restrict__ score, int64_t n, float* __restrict__ out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = dec_f32(score[i]);
}

}  // namespace msa
