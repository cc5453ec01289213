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
//   topk_local_kernel   : per slice of documents, a lower bound on its k-th
//                         fast score (one histogram pass) and every document
//                         within 2*eps of it, appended to a candidate list.
//   merge_band_kernel   : per query, a lower bound tau' on the global k-th
//                         fast score (same method over the candidates) and
//                         the band {s : fast_s >= tau' - 2*eps}.
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
constexpr int kRouteMaxB = 512;                       // queries per routing call

// ----------------------------------------------------------------- prep
constexpr int kPrepThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kPrepThreads)
route_prep_kernel(const T* __restrict__ qr, int NQ, int Hq, int Hkv, int dr,
                  float* __restrict__ u, uint32_t* __restrict__ score, int64_t n_score,
                  const int64_t* __restrict__ doc_chunk_off, int64_t D, int64_t C, int n_units,
                  int* __restrict__ unit_first_doc, int* __restrict__ cand_cnt, int B, int unit_chunks,
                  double* __restrict__ qn2, int* __restrict__ unit_counter, int n_counters) {
  extern __shared__ float s_qn[];      // [G][dr] query heads of one group, then [G] inverse norms
  const int G = Hq / Hkv;
  pdl_trigger();                       // the scan may set up its ring meanwhile
  if ((int)blockIdx.x < NQ * Hkv) {    // block (q, g): u[q][g], and |Qr[q][h]|^2 in fp64 for the re-scoring
    const int q = blockIdx.x / Hkv, g = blockIdx.x % Hkv;
    const T* Q = qr + ((int64_t)q * Hq + (int64_t)g * G) * dr;
    float* s_inv = s_qn + G * dr;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int hh = warp; hh < G; hh += nw) {
      float ss = 0.f;
      for (int i = lane; i < dr; i += 32) {
        const float x = Elem<T>::load1(Q + (int64_t)hh * dr + i);
        s_qn[hh * dr + i] = x;
        ss += x * x;
      }
      ss = warp_sum(ss);
      if (lane == 0) s_inv[hh] = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
    }
    __syncthreads();
    if ((int)threadIdx.x < G) {        // sequential fp64 sum of squares, the exact score's order
      double n2 = 0.0;
      for (int i = 0; i < dr; ++i) {
        const double x = (double)s_qn[threadIdx.x * dr + i];
        n2 = __dadd_rn(n2, __dmul_rn(x, x));
      }
      qn2[(int64_t)q * Hq + g * G + threadIdx.x] = n2;
    }
    for (int i = threadIdx.x; i < dr; i += blockDim.x) {
      float acc = 0.f;
      for (int hh = 0; hh < G; ++hh) acc += s_qn[hh * dr + i] * s_inv[hh];
      u[((int64_t)q * Hkv + g) * dr + i] = acc / (float)Hq;
    }
  }
  const int64_t gt = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t gs = (int64_t)gridDim.x * blockDim.x;
  uint4* s4 = reinterpret_cast<uint4*>(score);
  for (int64_t i = gt; i < n_score / 4; i += gs) s4[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int64_t i = (n_score / 4) * 4 + gt; i < n_score; i += gs) score[i] = 0u;
  if (gt < B) cand_cnt[gt] = 0;
  if (gt < n_counters) unit_counter[gt] = 0;
  // Scan unit i (a unit of work the CUDA-core scan claims, or a tile of the
  // tensor-core scan) starts at chunk i*unit_chunks; record the document
  // holding that chunk.
  constexpr int kDocsPerThread = 8;    // CSR loads of one thread issued together
  for (int64_t s0 = gt * kDocsPerThread; s0 < D; s0 += gs * kDocsPerThread) {
    int64_t off[kDocsPerThread + 1];
#pragma unroll
    for (int j = 0; j <= kDocsPerThread; ++j) off[j] = (s0 + j <= D) ? doc_chunk_off[s0 + j] : C;
#pragma unroll
    for (int j = 0; j < kDocsPerThread; ++j) {
      if (s0 + j >= D) break;
      const int64_t ilo = (off[j] + unit_chunks - 1) / unit_chunks;
      const int64_t ihi = (off[j + 1] + unit_chunks - 1) / unit_chunks;
      for (int64_t i = ilo; i < ihi && i < n_units; ++i) unit_first_doc[i] = (int)(s0 + j);
    }
  }
}

// ----------------------------------------------------------------- scan
// A chunk row is H_kv heads x 256 bytes (router_dim * element size = 256 B),
// i.e. H_kv*16 vectors of 16 bytes.  Lane l owns UPL = H_kv/2 consecutive
// vectors, all of one head (head = l / (32/H_kv)); it reads them in an order
// rotated by f(l) so that the 8 lanes of each shared-memory wavefront touch 8
// different 16-byte bank groups.  Per lane: squared norm and one dot per query
// row with packed fp32 FMA; the head's partial sums are combined over its
// 32/H_kv lanes, scaled by rsqrt(max(|Kr_g|^2, 1e-24)), and summed over the
// heads with xor-shuffles, leaving the chunk's fast score in every lane.
template <typename T, int NQG, int HKV>
struct ScanCfg {
  static constexpr int E = Elem<T>::kPerVec;            // elements per 16-byte vector
  static constexpr int ROW = HKV * 256;                 // bytes per chunk row
  static constexpr int UPL = HKV / 2;                   // vectors per lane
  static constexpr int LPH = 32 / HKV;                  // lanes per head
  static constexpr int STAGE_BYTES = 32768;
  static constexpr int SCH = STAGE_BYTES / ROW;         // chunks per stage
  static constexpr int NSTAGE = 2;                      // 2 x 2 CTAs leave ~100 KB per SM for co-running kernels
  static constexpr int NCW = 8;                         // consumer warps
  static constexpr int CPW = SCH / NCW;                 // chunks per warp per stage
  static constexpr int THREADS = (NCW + 1) * 32;        // + 1 producer warp
  static constexpr int SMEM = NSTAGE * STAGE_BYTES + 2 * NSTAGE * 8 + NSTAGE * 16;
  static_assert(CPW >= 1 && SCH % NCW == 0, "stage must split evenly over warps");
};

template <typename T, int NQG, int HKV>
__device__ __forceinline__ void chunk_scores(const unsigned char* row, int lane,
                                             const float2 (&up)[NQG][HKV / 2][Elem<T>::kPerVec / 2],
                                             float (&s)[NQG]) {
  using Cfg = ScanCfg<T, NQG, HKV>;
  constexpr int UPL = Cfg::UPL, E = Cfg::E, LPH = Cfg::LPH;
  const int f = (lane / (8 / UPL)) % UPL;
  const uint4* rp = reinterpret_cast<const uint4*>(row);
  float2 nn = make_float2(0.f, 0.f);
  float2 dd[NQG];
#pragma unroll
  for (int q = 0; q < NQG; ++q) dd[q] = make_float2(0.f, 0.f);
#pragma unroll
  for (int k = 0; k < UPL; ++k) {
    const uint4 v = rp[UPL * lane + ((k + f) % UPL)];
    float x[E];
    Elem<T>::unpack(v, x);
#pragma unroll
    for (int i = 0; i < E / 2; ++i) {
      const float2 p = make_float2(x[2 * i], x[2 * i + 1]);
      nn = __ffma2_rn(p, p, nn);
#pragma unroll
      for (int q = 0; q < NQG; ++q) dd[q] = __ffma2_rn(p, up[q][k][i], dd[q]);
    }
  }
  float n2 = nn.x + nn.y;
  float d[NQG];
#pragma unroll
  for (int q = 0; q < NQG; ++q) d[q] = dd[q].x + dd[q].y;
#pragma unroll
  for (int o = 1; o < LPH; o <<= 1) {
    n2 += __shfl_xor_sync(0xffffffffu, n2, o);
#pragma unroll
    for (int q = 0; q < NQG; ++q) d[q] += __shfl_xor_sync(0xffffffffu, d[q], o);
  }
  const float r = rsqrtf(fmaxf(n2, 1e-24f));
#pragma unroll
  for (int q = 0; q < NQG; ++q) {
    float t = d[q] * r;
#pragma unroll
    for (int o = LPH; o < 32; o <<= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    s[q] = t;
  }
}

template <typename T, int NQG, int HKV>
__global__ void __launch_bounds__(ScanCfg<T, NQG, HKV>::THREADS)
kr_scan_kernel(const T* __restrict__ kr, const float* __restrict__ u, int NQ, int Ttok,
               const int64_t* __restrict__ doc_chunk_off, int64_t C, const int* __restrict__ unit_first_doc,
               int64_t n_units, int unit_chunks, int* __restrict__ unit_counter, uint32_t* __restrict__ score,
               int64_t D) {
  using Cfg = ScanCfg<T, NQG, HKV>;
  constexpr int E = Cfg::E, ROW = Cfg::ROW, SCH = Cfg::SCH, NSTAGE = Cfg::NSTAGE, NCW = Cfg::NCW,
                UPL = Cfg::UPL, CPW = Cfg::CPW;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NSTAGE * Cfg::STAGE_BYTES);
  uint64_t* empty = full + NSTAGE;
  // per ring slot: first chunk of the stage, its chunk count (0: no more
  // work), and the document holding its first chunk when the stage opens a
  // unit (-1 when it continues the previous stage)
  int64_t* slot_base = reinterpret_cast<int64_t*>(empty + NSTAGE);
  int* slot_n = reinterpret_cast<int*>(slot_base + NSTAGE);
  int* slot_doc = slot_n + NSTAGE;

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
  pdl_wait();                          // u, the zeroed scores and the unit counter

  // The bank is cut into units of unit_chunks chunks (a multiple of SCH);
  // each CTA's producer claims the next unclaimed unit from a counter until
  // none is left, so CTAs that stream faster take more units and all finish
  // within about one unit.
  if (warp == NCW) {                               // producer warp
    if (lane == 0) {
      const unsigned char* src = reinterpret_cast<const unsigned char*>(kr);
      int64_t st = 0;
      bool ok = true;
      for (;;) {
        const int64_t un = atomicAdd(&unit_counter[blockIdx.y], 1);
        if (un >= n_units) break;
        const int64_t c0 = un * unit_chunks, c1 = min64(C, c0 + unit_chunks);
        for (int64_t cb = c0; cb < c1 && ok; cb += SCH, ++st) {
          const int slot = (int)(st % NSTAGE);
          if (st >= NSTAGE && !mbar_wait(&empty[slot], (uint32_t)((st / NSTAGE - 1) & 1))) { ok = false; break; }
          const int nch = (int)min64(SCH, c1 - cb);
          slot_base[slot] = cb;
          slot_n[slot] = nch;
          slot_doc[slot] = cb == c0 ? unit_first_doc[un] : -1;
          mbar_arrive_expect_tx(&full[slot], (uint32_t)(nch * ROW));
          tma_load_1d(smem + slot * Cfg::STAGE_BYTES, src + cb * ROW, (uint32_t)(nch * ROW), &full[slot]);
        }
        if (!ok) break;
      }
      if (ok) {                                    // the end marker: a stage with no chunks
        const int slot = (int)(st % NSTAGE);
        if (st < NSTAGE || mbar_wait(&empty[slot], (uint32_t)((st / NSTAGE - 1) & 1))) {
          slot_n[slot] = 0;
          mbar_arrive(&full[slot]);
        }
      }
    }
    return;
  }

  // consumer warps: this lane's slices of the query rows, as float pairs in the
  // (rotated) order the lane reads its vectors
  float2 up[NQG][UPL][E / 2];
  {
    const int f = (lane / (8 / UPL)) % UPL;
#pragma unroll
    for (int q = 0; q < NQG; ++q)
#pragma unroll
      for (int k = 0; k < UPL; ++k) {
        const int e0 = (UPL * lane + ((k + f) % UPL)) * E;   // element index within the row
        const float* uq = u + (int64_t)(q0 + q) * (HKV * 16 * E) + e0;
#pragma unroll
        for (int i = 0; i < E / 2; ++i)
          up[q][k][i] = (q < nq) ? make_float2(uq[2 * i], uq[2 * i + 1]) : make_float2(0.f, 0.f);
      }
  }

  int64_t cur = 0;
  int64_t run_doc = -1;
  float run_max[NQG];
#pragma unroll
  for (int q = 0; q < NQG; ++q) run_max[q] = -INFINITY;
  auto flush = [&]() {
    float val = run_max[0];
#pragma unroll
    for (int q = 1; q < NQG; ++q)
      if (lane == q) val = run_max[q];
    if (lane < nq) atomicMax(&score[(int64_t)((q0 + lane) / Ttok) * D + run_doc], enc_f32(val));
  };

  for (int64_t st = 0;; ++st) {
    const int slot = (int)(st % NSTAGE);
    if (!mbar_wait(&full[slot], (uint32_t)((st / NSTAGE) & 1))) return;
    const int nch = slot_n[slot];
    if (nch == 0) break;                           // no more work
    const int64_t cbase = slot_base[slot];
    const int first_doc = slot_doc[slot];
    if (first_doc >= 0) cur = first_doc;           // a new unit: the run restarts (atomicMax merges)
    const unsigned char* stage = smem + slot * Cfg::STAGE_BYTES;
    float s[CPW][NQG];
#pragma unroll
    for (int k2 = 0; k2 < CPW; ++k2)
      chunk_scores<T, NQG, HKV>(stage + (warp * CPW + k2) * ROW, lane, up, s[k2]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
#pragma unroll
    for (int k2 = 0; k2 < CPW; ++k2) {
      const int ci = warp * CPW + k2;
      if (ci >= nch) break;
      const int64_t c = cbase + ci;
      while (doc_chunk_off[cur + 1] <= c) ++cur;
      if (cur != run_doc) {
        if (run_doc >= 0) flush();
        run_doc = cur;
#pragma unroll
        for (int q = 0; q < NQG; ++q) run_max[q] = s[k2][q];
      } else {
#pragma unroll
        for (int q = 0; q < NQG; ++q) run_max[q] = fmaxf(run_max[q], s[k2][q]);
      }
    }
  }
  if (run_doc >= 0) flush();
}

// ------------------------------------------------------------ k-th score bound
// A lower bound on the k-th largest of n nonzero 32-bit score encodings spread
// over a CTA (k <= number of nonzero keys; zero keys are absent): one pass for
// the score range, one shared-memory histogram of 1024 equal-width score bins,
// one warp that finds the bin where the count from the top reaches k, and the
// smallest key inside that bin.  Binning is a monotone fp32 map, so the k-th
// largest key lies in that bin and is at least its smallest key.  Any lower
// bound keeps the band a superset of the exact one.
constexpr int kHistBins = 1024;
struct HistSmem {
  unsigned int hist[kHistBins];
  unsigned int wmin[32], wmax[32];
  unsigned int lo, hi, bin, minv;
};

__device__ __forceinline__ int score_bin(uint32_t v, float flo, float scale) {
  return min(kHistBins - 1, (int)((dec_f32(v) - flo) * scale));
}

template <typename KeyFn>
__device__ uint32_t block_kth_lower_bound(int n, int k, KeyFn key, HistSmem& hs) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t mn = 0xffffffffu, mx = 0u;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const uint32_t v = key(i);
    if (v) { mn = min(mn, v); mx = max(mx, v); }
  }
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (lane == 0) { hs.wmin[warp] = mn; hs.wmax[warp] = mx; }
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hs.hist[i] = 0u;
  __syncthreads();
  if (warp == 0) {
    uint32_t a = lane < nw ? hs.wmin[lane] : 0xffffffffu, c = lane < nw ? hs.wmax[lane] : 0u;
    a = __reduce_min_sync(0xffffffffu, a);
    c = __reduce_max_sync(0xffffffffu, c);
    if (lane == 0) { hs.lo = a; hs.hi = c; hs.bin = 0u; hs.minv = 0xffffffffu; }
  }
  __syncthreads();
  const float flo = dec_f32(hs.lo), fhi = dec_f32(hs.hi);
  const float scale = fhi > flo ? (float)kHistBins / (fhi - flo) : 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const uint32_t v = key(i);
    if (v) atomicAdd(&hs.hist[score_bin(v, flo, scale)], 1u);
  }
  __syncthreads();
  if (warp == 0) {                       // lane l holds bins 1023-32l .. 992-32l, descending
    constexpr int PER = kHistBins / 32;
    uint32_t sum = 0u;
#pragma unroll 8
    for (int j = 0; j < PER; ++j) sum += hs.hist[kHistBins - 1 - PER * lane - j];
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t excl = incl - sum, kk = (uint32_t)k;
    if (excl < kk && kk <= incl) {
      uint32_t acc = excl;
      for (int j = 0; j < PER; ++j) {
        const int bin = kHistBins - 1 - PER * lane - j;
        acc += hs.hist[bin];
        if (acc >= kk) { hs.bin = (unsigned)bin; break; }
      }
    }
  }
  __syncthreads();
  const int bstar = (int)hs.bin;
  uint32_t bm = 0xffffffffu;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const uint32_t v = key(i);
    if (v && score_bin(v, flo, scale) == bstar) bm = min(bm, v);
  }
  bm = __reduce_min_sync(0xffffffffu, bm);
  if (lane == 0 && bm != 0xffffffffu) atomicMin(&hs.minv, bm);
  __syncthreads();
  return hs.minv == 0xffffffffu ? hs.lo : hs.minv;
}

// Band threshold below a k-th score bound: bound - 2 eps - rounding slack, as
// an encoding; 0 keeps everything.
__device__ __forceinline__ uint32_t band_threshold(uint32_t tau_enc) {
  return tau_enc ? enc_f32(dec_f32(tau_enc) - kBandMargin) : 0u;
}

// ------------------------------------------------------------ local top-k
constexpr int kTopkThreads = 256;
constexpr int kTopkPer = kTopkSlice / kTopkThreads;

// One CTA per (slice of 2048 documents, query): a lower bound tau_s on the
// slice's k-th fast score, then every document with fast score >= tau_s -
// 2 eps is appended, packed as (score encoding << 32 | document), to the
// query's candidate list (one reservation per CTA).  Any document of the
// global band is a candidate, since tau_s <= the global k-th score.
__global__ void __launch_bounds__(kTopkThreads)
topk_local_kernel(const uint32_t* __restrict__ score, int64_t D, int k,
                  unsigned long long* __restrict__ cand, int* __restrict__ cand_cnt) {
  __shared__ uint32_t s_key[kTopkSlice];
  __shared__ HistSmem hs;
  __shared__ int s_cnt, s_base;
  const int p = blockIdx.x, b = blockIdx.y;
  const int64_t d0 = (int64_t)p * kTopkSlice;
  const uint32_t* sc = score + (int64_t)b * D;
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  uint32_t key[kTopkPer];
#pragma unroll
  for (int i = 0; i < kTopkPer; ++i) {
    const int64_t doc = d0 + threadIdx.x + i * kTopkThreads;
    key[i] = doc < D ? sc[doc] : 0u;
    s_key[threadIdx.x + i * kTopkThreads] = key[i];
  }
  if (threadIdx.x == 0) s_cnt = 0;
  __syncthreads();
  const int64_t n_real = min64(kTopkSlice, D - d0);
  const uint32_t thr = n_real <= k ? 0u
                       : band_threshold(block_kth_lower_bound(kTopkSlice, k, [&](int i) { return s_key[i]; }, hs));
  int mine = 0;
#pragma unroll
  for (int i = 0; i < kTopkPer; ++i) mine += (key[i] != 0u && key[i] >= thr) ? 1 : 0;
  int off = 0;
  {
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int wbase = 0;
    if (lane == 31 && incl) wbase = atomicAdd(&s_cnt, incl);
    wbase = __shfl_sync(0xffffffffu, wbase, 31);
    off = wbase + incl - mine;
  }
  __syncthreads();
  if (threadIdx.x == 0) s_base = s_cnt ? atomicAdd(&cand_cnt[b], s_cnt) : 0;
  __syncthreads();
  unsigned long long* cl = cand + (int64_t)b * D + s_base + off;
#pragma unroll
  for (int i = 0; i < kTopkPer; ++i) {
    if (key[i] != 0u && key[i] >= thr) {
      const int64_t doc = d0 + threadIdx.x + i * kTopkThreads;
      *cl++ = ((unsigned long long)key[i] << 32) | (unsigned long long)doc;
    }
  }
}

// ------------------------------------------------------------ merge + band
constexpr int kMergeThreads = 1024;

// One CTA per query.  tau' = a lower bound on the k-th score of the
// candidates, which is the global k-th fast score (the global top-k are
// candidates); band = candidates with fast score >= tau' - 2 eps; then the work
// items of the exact re-scoring (chunks x query tokens) as an exclusive prefix
// over the band.
__global__ void __launch_bounds__(kMergeThreads)
merge_band_kernel(int64_t D, int k, int Ttok, const unsigned long long* __restrict__ cand,
                  const int* __restrict__ cand_cnt, const int64_t* __restrict__ doc_chunk_off,
                  int* __restrict__ band, int* __restrict__ band_cnt,
                  unsigned long long* __restrict__ band_exact, int64_t* __restrict__ item_off) {
  __shared__ HistSmem hs;
  __shared__ int s_cnt;
  __shared__ int64_t s_scan[kMergeThreads / 32];
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  pdl_wait();
  pdl_trigger();
  const int ncand = cand_cnt[b];
  const unsigned long long* cl = cand + (int64_t)b * D;
  if (threadIdx.x == 0) s_cnt = 0;
  const uint32_t thr =
      band_threshold(block_kth_lower_bound(ncand, k, [&](int i) { return (uint32_t)(cl[i] >> 32); }, hs));
  int* bl = band + (int64_t)b * D;
  for (int i0 = 0; i0 < ncand; i0 += blockDim.x) {
    const int i = i0 + threadIdx.x;
    unsigned long long x = 0ull;
    bool in = false;
    if (i < ncand) {
      x = cl[i];
      in = (uint32_t)(x >> 32) >= thr;
    }
    const unsigned m = __ballot_sync(0xffffffffu, in);
    int base = 0;
    if (lane == 0 && m) base = atomicAdd(&s_cnt, __popc(m));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (in) bl[base + __popc(m & ((1u << lane) - 1))] = (int)(x & 0xffffffffull);
  }
  __syncthreads();
  const int nb = s_cnt;
  int64_t* io = item_off + (int64_t)b * (D + 1);
  unsigned long long* ex = band_exact + (int64_t)b * D;
  int64_t carry = 0;
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
    int64_t wofs = 0, tot = 0;
    for (int w = 0; w < nw; ++w) {
      const int64_t sw = s_scan[w];
      if (w < warp) wofs += sw;
      tot += sw;
    }
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
constexpr int kRescoreThreads = 256;
constexpr int kRescoreSmemItems = 4096;      // band item offsets (all queries) cached in shared memory

// The rows (256 bytes each) are loaded into registers before the ordered sum
// starts, so no load waits inside the sequential chain: the empty asm
// statements take every loaded word as an input, which pins all loads ahead
// of the first add.
#define MSA_USE4(v) "r"((v).x), "r"((v).y), "r"((v).z), "r"((v).w)
#define MSA_USE8x4(a, i) MSA_USE4(a[i]), MSA_USE4(a[i + 1]), MSA_USE4(a[i + 2]), MSA_USE4(a[i + 3]), \
                         MSA_USE4(a[i + 4]), MSA_USE4(a[i + 5]), MSA_USE4(a[i + 6]), MSA_USE4(a[i + 7])
__device__ __forceinline__ void pin16(const uint4 (&a)[16]) {
  asm volatile("" ::MSA_USE8x4(a, 0));
  asm volatile("" ::MSA_USE8x4(a, 8));
}
// q.k, and (when want_nk) |k|^2, each summed sequentially in element order;
// the two chains run interleaved from the same loaded registers.
template <typename T>
__device__ __forceinline__ void seq_dot_nk(const T* qp, const T* kp, bool want_nk, double& dot, double& nk) {
  constexpr int E = Elem<T>::kPerVec;
  constexpr int NV = 256 / 16;                 // router_dim * element size = 256 bytes
  uint4 qv[NV], kv[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {                 // volatile loads: all 32 issue before the chain starts
    qv[j] = ldg_nc_v4(reinterpret_cast<const uint4*>(qp) + j);
    kv[j] = ldg_nc_v4(reinterpret_cast<const uint4*>(kp) + j);
  }
  pin16(qv);
  pin16(kv);
  double d = 0.0, n = 0.0;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    float x[E], y[E];
    Elem<T>::unpack(qv[j], x);
    Elem<T>::unpack(kv[j], y);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const double yd = (double)y[e];
      d = __dadd_rn(d, __dmul_rn((double)x[e], yd));
      if (want_nk) n = __dadd_rn(n, __dmul_rn(yd, yd));
    }
  }
  dot = d;
  nk = n;
}

// Work items are (query b, band entry e, token t, chunk c), numbered over all
// queries at once: every CTA caches the per-query item offsets of all bands
// in shared memory (when they fit) and locates an item by two binary searches.
template <typename T>
__global__ void __launch_bounds__(kRescoreThreads)
rescore_kernel(const T* __restrict__ qr, const T* __restrict__ kr, int B, int Ttok, int Hq, int Hkv,
               int dr, int64_t D, const int64_t* __restrict__ doc_chunk_off,
               const int* __restrict__ band, const int* __restrict__ band_cnt,
               const int64_t* __restrict__ item_off, const double* __restrict__ qn2,
               unsigned long long* __restrict__ band_exact) {
  extern __shared__ double s_dyn[];
  double* s_cos = s_dyn;                                  // [warps][Hq]
  double* s_nk = s_cos + (kRescoreThreads / 32) * Hq;     // [warps][Hkv] key norms of the item's chunk
  int64_t* s_tot = reinterpret_cast<int64_t*>(s_nk + (kRescoreThreads / 32) * Hkv);   // [B+1] item prefix
  int* s_cnt = reinterpret_cast<int*>(s_tot + (B + 1));                                // [B]
  int* s_eb = s_cnt + B;                                                               // [B+1] entry prefix
  int64_t* s_io = reinterpret_cast<int64_t*>(s_cnt + 2 * B + 2);                       // [kRescoreSmemItems], 8-aligned
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw_blk = blockDim.x >> 5;
  double* cb = s_cos + warp * Hq;
  double* nkb = s_nk + warp * Hkv;
  const int G = Hq / Hkv;
  pdl_wait();
  pdl_trigger();
  for (int b = threadIdx.x; b < B; b += blockDim.x) s_cnt[b] = band_cnt[b];
  __syncthreads();
  if (threadIdx.x == 0) {
    s_eb[0] = 0;
    for (int b = 0; b < B; ++b) s_eb[b + 1] = s_eb[b] + s_cnt[b] + 1;
  }
  __syncthreads();
  const bool cached = s_eb[B] <= kRescoreSmemItems;
  if (cached) {                         // every query's offsets, loads in flight together
    constexpr int kBatch = 8;
    const int n_e = s_eb[B];
    for (int i0 = threadIdx.x; i0 < n_e; i0 += kBatch * blockDim.x) {
      int64_t v[kBatch];
      int at[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * blockDim.x;
        at[u] = -1;
        if (i < n_e) {
          int lo = 0, hi = B - 1;       // last b with s_eb[b] <= i
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_eb[mid] <= i) lo = mid; else hi = mid - 1;
          }
          v[u] = item_off[(int64_t)lo * (D + 1) + (i - s_eb[lo])];
          at[u] = i;
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (at[u] >= 0) s_io[at[u]] = v[u];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    s_tot[0] = 0;
    for (int b = 0; b < B; ++b)
      s_tot[b + 1] = s_tot[b] + (cached ? s_io[s_eb[b] + s_cnt[b]] : item_off[(int64_t)b * (D + 1) + s_cnt[b]]);
  }
  __syncthreads();
  const int64_t total = s_tot[B];
  for (int64_t git = (int64_t)blockIdx.x * nw_blk + warp; git < total; git += (int64_t)gridDim.x * nw_blk) {
    int b = 0;
    {
      int lo = 0, hi = B - 1;                             // last b with s_tot[b] <= git
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_tot[mid] <= git) lo = mid; else hi = mid - 1;
      }
      b = lo;
    }
    const int64_t it = git - s_tot[b];
    const int nb = s_cnt[b];
    const int64_t* io = cached ? s_io + s_eb[b] : item_off + (int64_t)b * (D + 1);
    int lo = 0, hi = nb;                                  // last e with io[e] <= it
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (io[mid] <= it) lo = mid; else hi = mid;
    }
    const int e = lo;
    const int doc = band[(int64_t)b * D + e];
    const int64_t c0 = doc_chunk_off[doc];
    const int64_t nc = doc_chunk_off[doc + 1] - c0;
    const int64_t rem = it - io[e];
    const int t = (int)(rem / nc);
    const int64_t c = c0 + rem % nc;
    // lane h: q_h . k_{h/G}; the first head of each group also takes |k|^2,
    // which the group's G heads share
    for (int h = lane; h < Hq; h += 32) {
      const T* qp = qr + (((int64_t)b * Ttok + t) * Hq + h) * dr;
      const T* kp = kr + (c * Hkv + h / G) * dr;
      double dot, nk;
      seq_dot_nk<T>(qp, kp, h % G == 0, dot, nk);
      if (h % G == 0) nkb[h / G] = nk;
      cb[h] = dot;
    }
    __syncwarp();
    for (int h = lane; h < Hq; h += 32) {
      const double nq = qn2[((int64_t)b * Ttok + t) * Hq + h];
      const double den = __dmul_rn(fmax(__dsqrt_rn(nq), 1e-12), fmax(__dsqrt_rn(nkb[h / G]), 1e-12));
      double cs = __ddiv_rn(cb[h], den);
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

// ------------------------------------------------------------ final selection
constexpr int kFinalThreads = 1024;

__device__ __forceinline__ bool better(unsigned long long ea, int da, unsigned long long eb, int db) {
  return ea > eb || (ea == eb && da < db);
}

// One CTA per query: rank every band entry by (exact desc, index asc); entries
// of rank < k are the output.  Bands of up to 1024 entries are ranked directly
// from shared memory; larger ones (degenerate, e.g. many equal scores) fall
// back to k rounds of block argmax.
__global__ void __launch_bounds__(kFinalThreads)
final_select_kernel(int64_t D, int k, const int* __restrict__ band, const int* __restrict__ band_cnt,
                    const unsigned long long* __restrict__ band_exact, int* __restrict__ out_idx,
                    double* __restrict__ out_score) {
  __shared__ unsigned long long s_e[kFinalThreads];
  __shared__ int s_d[kFinalThreads];
  __shared__ unsigned long long r_e[kFinalThreads / 32];
  __shared__ int r_d[kFinalThreads / 32];
  const int b = blockIdx.x;
  pdl_wait();
  const int nb = band_cnt[b];
  const int* bl = band + (int64_t)b * D;
  const unsigned long long* ex = band_exact + (int64_t)b * D;
  if (nb <= kFinalThreads) {
    const int e = threadIdx.x;
    if (e < nb) { s_e[e] = ex[e]; s_d[e] = bl[e]; }
    __syncthreads();
    if (e < nb) {
      const unsigned long long me = s_e[e];
      const int md = s_d[e];
      int rank = 0;
      for (int j = 0; j < nb; ++j) rank += better(s_e[j], s_d[j], me, md) ? 1 : 0;
      if (rank < k) {
        out_idx[(int64_t)b * k + rank] = md;
        if (out_score) out_score[(int64_t)b * k + rank] = dec_f64(me);
      }
    }
    return;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  unsigned long long le = ~0ull;                 // last pick (start: above everything)
  int ld = -1;
  for (int r = 0; r < k; ++r) {
    unsigned long long be = 0;
    int bd = INT_MAX;                            // no document yet
    for (int e = threadIdx.x; e < nb; e += blockDim.x) {
      const unsigned long long x = ex[e];
      const int d = bl[e];
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
