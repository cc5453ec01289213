// Stage 2 router-key scan on the 5th-generation tensor cores, for many query
// rows at once (batched queries, or many query tokens).
//
// Method: "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts",
// section "How MSA compresses and routes documents" (cosine of the query's
// router projection with each document's pooled router keys, mean over heads,
// max over query tokens and over the document's chunks) -- the same fast
// score as kr_scan_kernel in route.cuh, which serves up to 4 query rows per
// pass and stays HBM-bound there.  With 32 or 64 rows the CUDA-core scan needs
// 8-16 passes over the bank; here one pass serves up to 128 rows.
//
// Per 128-chunk tile and kv head g the MMA computes D_g = Kr_g u_g^T:
//   A = Kr[c0 .. c0+127][g][0..127] (M = 128 chunks, K = 128 dims, bf16),
//       a 3D TMA box, 128-byte swizzle, K-major;
//   B = [u_hi ; u_lo][g] (N = 2 x rows of the pass), the fp32 head-group
//       mean query split into two bf16 terms so that u_hi + u_lo carries
//       16 significant bits: |u - u_hi - u_lo| <= 2^-16 |u|;
//   D = fp32 accumulator columns in tensor memory (TMEM), one buffer per
//       in-flight (tile, head).
// The four epilogue warps own the 128 TMEM lanes, i.e. one chunk each: they
// read D_g's hi and lo columns and add (hi + lo) * rsqrt(max(|Kr_g|^2, 1e-24))
// into the chunk's per-row score, the norm coming from the same
// shared-memory tile.  After the last head each row's score goes to its
// query and document as a max, on the order-preserving encoding
// kr_scan_kernel uses.
//
// Error: the bf16 split adds at most 2^-16 * sum_g |u_g| <= 2^-16 to the score
// and the fp32 accumulation of 128 exact products a few 2^-17, both far
// inside the certified eps = 2^-12 of the selection that follows.
//
// Roles (one CTA per SM, persistent over a contiguous run of tiles):
//   warps 0-3     : epilogue (TMEM lanes 32w .. 32w + 31)
//   warps 4-7     : norms -- rsqrt(max(|Kr_g|^2, 1e-24)) of each chunk row of
//                   a stage, handed to the epilogue through shared memory
//   warp 8 lane 0 : TMA producer of the (tile, head) stage ring
//   warp 9        : TMEM allocation; lane 0 issues tcgen05.mma and commits
// The per-document maxima leave each warp as one global atomicMax per
// (query, run of chunks of one document) after a shared-memory transpose.
// Every wait is bounded (mbar_wait); a timeout flags MSA_DEV_PIPE_TIMEOUT.
#pragma once
#include <cuda.h>

#include "route.cuh"

namespace msa {

constexpr int kScanTile = 128;                 // chunks per tile (MMA M)
constexpr int kScanEpiWarps = 4;
constexpr int kScanNormWarps = 4;
constexpr int kScanProducerWarp = kScanEpiWarps + kScanNormWarps;
constexpr int kScanMmaWarp = kScanProducerWarp + 1;
constexpr int kScanMmaThreads = (kScanMmaWarp + 1) * 32;
constexpr int kScanMaxRows = 128;              // query rows per pass
constexpr int kScanDocCols = kScanTile + 1;    // documents a tile may touch

struct ScanMmaArgs {
  CUtensorMap tm_kr;                           // {d_r, H_kv, C} bf16, box {64, 1, 128}
  CUtensorMap tm_u;                            // {d_r, passes * H_kv * 2 * NQP} bf16, box {64, 2 * NQP}
  const int64_t* doc_chunk_off;
  const int* tile_first_doc;                   // document holding each tile's first chunk
  uint32_t* score;                             // [B][D] encoded maxima
  const float* rnorm;                          // [H_kv][P] inverse router-key norms, or NULL
  int64_t C, D, P;
  int Hkv, NQ, Ttok, pass, n_tiles;
};

template <int NQP>
struct ScanMmaCfg {
  static constexpr int NP2 = 2 * NQP;                          // hi rows, then lo rows
  static constexpr int A_BYTES = kScanTile * 256;              // two 64-dim halves of 16 KiB
  static constexpr int B_BYTES = NP2 * 256;
  static constexpr int NORM_BYTES = kScanTile * 4;             // the stage's 128 inverse norms
  static constexpr int STAGE = (A_BYTES + B_BYTES + NORM_BYTES + 1023) / 1024 * 1024;
  static constexpr int DOC_BYTES = kScanEpiWarps * 32 * 33 * 4;                // epilogue transpose buffers
  static constexpr int EXTRA = 27 * 1024;                      // transposes, norms, windows, barriers
  static constexpr int NSTAGE = (227 * 1024 - EXTRA - 1024) / STAGE;
  static constexpr int NTB = (512 / NP2) >= 4 ? 4 : 512 / NP2; // TMEM accumulator buffers
  static constexpr int TCOLS_RAW = NTB * NP2;
  static constexpr int TCOLS = TCOLS_RAW <= 32 ? 32 : TCOLS_RAW <= 64 ? 64 : TCOLS_RAW <= 128 ? 128
                               : TCOLS_RAW <= 256 ? 256 : 512;
  static constexpr int SMEM = NSTAGE * STAGE + EXTRA + 1024;   // + room for 1 KiB alignment
  static_assert(NSTAGE >= 2, "at least two stages");
  static_assert(NQP % 32 == 0 && NQP <= kScanMaxRows, "rows per pass: whole 32-column TMEM loads");
  static_assert(DOC_BYTES + NSTAGE * kScanTile * 4 + 2 * kScanDocCols * 8 + kScanNormWarps * kScanDocCols * 8 +
                    512 <= EXTRA, "extra space");
  static_assert(DOC_BYTES % 16 == 0 && (NSTAGE * kScanTile * 4) % 16 == 0 && (2 * kScanDocCols * 8) % 16 == 0,
                "16-byte aligned regions (the windows are int64, the barriers 8-byte mbarriers)");
};

// ------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tm, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_s(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t umma_sdesc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D, M = 128, N = n.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}
// tcgen05.ld of 32 (or 16) consecutive fp32 columns of this warp's 32 TMEM
// lanes, without waiting; tmem_wait_tie / reg_tie then make every use of the
// registers come after tcgen05.wait::ld (the registers pass through the asm).
#define MSA_R8(i) "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), \
                  "+r"(r[i + 4]), "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7])
__device__ __forceinline__ void tmem_ld32_issue(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16_issue(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
template <int N>
__device__ __forceinline__ void tmem_wait_tie(uint32_t (&r)[N]) {
  static_assert(N == 16 || N == 32, "16 or 32 registers");
  if constexpr (N == 32)
    asm volatile("tcgen05.wait::ld.sync.aligned;" : MSA_R8(0), MSA_R8(8), MSA_R8(16), MSA_R8(24) :: "memory");
  else
    asm volatile("tcgen05.wait::ld.sync.aligned;" : MSA_R8(0), MSA_R8(8) :: "memory");
}
template <int N>
__device__ __forceinline__ void reg_tie(uint32_t (&r)[N]) {
  static_assert(N == 16 || N == 32, "16 or 32 registers");
  if constexpr (N == 32)
    asm volatile("" : MSA_R8(0), MSA_R8(8), MSA_R8(16), MSA_R8(24));
  else
    asm volatile("" : MSA_R8(0), MSA_R8(8));
}
#undef MSA_R8
// Bounded wait whose outcome every lane of the warp shares (the TMEM loads
// that follow are warp-collective).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}
// Barrier of the 128 epilogue threads that also ANDs `ok` over them, so that
// they leave their loop together.
__device__ __forceinline__ bool epi_bar_and(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
      " bar.red.and.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r) : "r"((uint32_t)ok), "n"(kScanEpiWarps * 32) : "memory");
  return r != 0;
}

// -------------------------------------------------------------- u split
// ub[pass][g][i] = bf16(u[q][g]) and ub[pass][g][NQP + i] = bf16(u - that),
// q = pass * NQP + i (rows past NQ are zero).
__global__ void u_split_kernel(const float* __restrict__ u, int NQ, int Hkv, int dr, int NQP, int n_pass,
                               __nv_bfloat16* __restrict__ ub) {
  const int64_t n = (int64_t)n_pass * Hkv * NQP * dr;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < n;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int e = (int)(idx % dr);
    const int i = (int)((idx / dr) % NQP);
    const int g = (int)((idx / ((int64_t)dr * NQP)) % Hkv);
    const int pass = (int)(idx / ((int64_t)dr * NQP * Hkv));
    const int q = pass * NQP + i;
    const float x = q < NQ ? u[((int64_t)q * Hkv + g) * dr + e] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
    const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
    __nv_bfloat16* row = ub + (((int64_t)pass * Hkv + g) * 2 * NQP) * dr;
    row[(int64_t)i * dr + e] = hi;
    row[(int64_t)(NQP + i) * dr + e] = lo;
  }
}

// ------------------------------------------------------ inverse key norms
// out[g][c] = rsqrt(max(|Kr[c][g]|^2, 1e-24)) with the fp32 sum of squares of
// the fast score; rows c >= C of the padded layout are 0.  One thread per
// (g, c), four partial sums.
template <typename T>
__global__ void kr_inv_norms_kernel(const T* __restrict__ kr, int64_t C, int Hkv, int dr, int64_t P,
                                    float* __restrict__ out) {
  constexpr int E = Elem<T>::kPerVec;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < (int64_t)Hkv * P;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int g = (int)(idx / P);
    const int64_t c = idx % P;
    float r = 0.f;
    if (c < C) {
      const uint4* row = reinterpret_cast<const uint4*>(kr + (c * Hkv + g) * dr);
      float2 nn[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      for (int j = 0; j < dr / E; ++j) {
        float x[E];
        Elem<T>::unpack(ldg_nc_v4(row + j), x);
#pragma unroll
        for (int i = 0; i < E / 2; ++i) nn[i & 1] = __ffma2_rn(make_float2(x[2 * i], x[2 * i + 1]),
                                                              make_float2(x[2 * i], x[2 * i + 1]), nn[i & 1]);
      }
      r = rsqrtf(fmaxf((nn[0].x + nn[0].y) + (nn[1].x + nn[1].y), 1e-24f));
    }
    out[idx] = r;
  }
}

// One warp's 32 chunk rows, staged in sw = [row][33] (row = chunk of the
// warp, column = query row of this 32-wide block); doc_l = this lane's row's
// document relative to fdoc (-1 past the bank).  Lane q walks the rows in
// chunk order and posts one atomicMax per (query, run of one document's
// chunks); when all 32 query rows belong to one query the warp reduces first.
__device__ __forceinline__ void post_runs(const float* sw, int doc_l, int lane, int qb, int q1, int Ttok, int64_t D,
                                          int fdoc, uint32_t* score) {
  const int q = qb + lane;
  const bool qv = q < q1;
  const int64_t brow = qv ? (int64_t)(q / Ttok) * D + fdoc : 0;
  const bool one_b = qb / Ttok == (qb + 31) / Ttok && qb + 31 < q1;
  float m = -INFINITY;
  int cur = -1;
  auto post = [&]() {
    if (cur < 0) return;
    if (one_b) {
      const uint32_t e = __reduce_max_sync(0xffffffffu, enc_f32(m));
      if (lane == 0) atomicMax(&score[brow + cur], e);
    } else if (qv) {
      atomicMax(&score[brow + cur], enc_f32(m));
    }
  };
  for (int r = 0; r < 32; ++r) {
    const int d = __shfl_sync(0xffffffffu, doc_l, r);           // the same for every lane
    const float v = sw[r * 33 + lane];
    if (d != cur) {
      post();
      cur = d;
      m = v;
    } else {
      m = fmaxf(m, v);
    }
  }
  post();
}
// The largest j in [0, 128] with wn[j] <= c.
__device__ __forceinline__ int window_find(const int64_t* wn, int64_t c) {
  int lo = 0, hi = kScanTile;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (wn[mid] <= c) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ----------------------------------------------------------------- scan
template <int NQP>
__global__ void __launch_bounds__(kScanMmaThreads, 1)
kr_scan_mma_kernel(const __grid_constant__ ScanMmaArgs a) {
  using Cfg = ScanMmaCfg<NQP>;
  constexpr int NP2 = Cfg::NP2, NSTAGE = Cfg::NSTAGE, NTB = Cfg::NTB;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~uintptr_t(1023));
  unsigned char* extra = smem + NSTAGE * Cfg::STAGE;
  float* s_acc = reinterpret_cast<float*>(extra);                               // [4 warps][32][33]
  float* s_rn = reinterpret_cast<float*>(extra + Cfg::DOC_BYTES);               // [NSTAGE][128]
  int64_t* win = reinterpret_cast<int64_t*>(extra + Cfg::DOC_BYTES + NSTAGE * kScanTile * 4);   // [2][129]
  int64_t* wpost = win + 2 * kScanDocCols;                                       // [4][129] post-warp windows
  uint64_t* pfull = reinterpret_cast<uint64_t*>(wpost + kScanNormWarps * kScanDocCols);   // [4] rows handed over
  uint64_t* pempty = pfull + kScanEpiWarps;                                      // [4] transpose buffer free
  uint64_t* full = pempty + kScanEpiWarps;
  uint64_t* empty = full + NSTAGE;
  uint64_t* nready = empty + NSTAGE;
  uint64_t* tfull = nready + NSTAGE;
  uint64_t* tempty = tfull + NTB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + NTB);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = (int)((int64_t)blockIdx.x * a.n_tiles / gridDim.x);
  const int t1 = (int)((int64_t)(blockIdx.x + 1) * a.n_tiles / gridDim.x);
  const int ntile = t1 - t0;
  const int H = a.Hkv;
  const int nwork = ntile * H;                                  // (tile, head) items
  const bool pre = a.rnorm != nullptr;                          // inverse norms come with the stage

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kScanEpiWarps + (pre ? 0 : kScanNormWarps));   // MMA, epilogue (, norm) warps
      mbar_init(&nready[s], kScanNormWarps);
    }
    for (int s = 0; s < NTB; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], kScanEpiWarps);
    }
    for (int s = 0; s < kScanEpiWarps; ++s) {
      mbar_init(&pfull[s], 1);
      mbar_init(&pempty[s], 1);
    }
    fence_mbar_init();
  }
  if (warp == kScanMmaWarp) {                                   // TMEM columns for NTB accumulators
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(tmem_slot)), "n"(Cfg::TCOLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kScanProducerWarp) {                              // ---- TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int w = 0; w < nwork; ++w) {
        const int slot = w % NSTAGE;
        if (w >= NSTAGE && !mbar_wait(&empty[slot], (uint32_t)(((w / NSTAGE) - 1) & 1))) break;
        const int tile = t0 + w / H, g = w % H;
        unsigned char* sa = smem + slot * Cfg::STAGE;
        unsigned char* sb = sa + Cfg::A_BYTES;
        mbar_arrive_expect_tx(&full[slot], Cfg::A_BYTES + Cfg::B_BYTES + (pre ? Cfg::NORM_BYTES : 0));
        if (pre)
          tma_load_1d(sb + Cfg::B_BYTES, a.rnorm + (int64_t)g * a.P + (int64_t)tile * kScanTile, Cfg::NORM_BYTES,
                      &full[slot]);
        tma_load_3d(sa, &a.tm_kr, 0, g, tile * kScanTile, &full[slot]);
        tma_load_3d(sa + Cfg::A_BYTES / 2, &a.tm_kr, 64, g, tile * kScanTile, &full[slot]);
        const int brow = (a.pass * H + g) * NP2;
        tma_load_2d_s(sb, &a.tm_u, 0, brow, &full[slot]);
        tma_load_2d_s(sb + Cfg::B_BYTES / 2, &a.tm_u, 64, brow, &full[slot]);
        issued = w + 1;
      }
      // the copies of the last stages land before the CTA may leave
      for (int w = issued > NSTAGE ? issued - NSTAGE : 0; w < issued; ++w)
        mbar_wait(&full[w % NSTAGE], (uint32_t)((w / NSTAGE) & 1));
    }
  } else if (warp == kScanMmaWarp) {                            // ---- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(NP2);
      int done = 0;
      for (int w = 0; w < nwork; ++w) {
        const int slot = w % NSTAGE, tb = w % NTB;
        if (!mbar_wait(&full[slot], (uint32_t)((w / NSTAGE) & 1))) break;
        if (w >= NTB && !mbar_wait(&tempty[tb], (uint32_t)(((w / NTB) - 1) & 1))) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + slot * Cfg::STAGE), sb = sa + Cfg::A_BYTES;
        const uint32_t d = tmem + (uint32_t)(tb * NP2);
#pragma unroll
        for (int k = 0; k < 8; ++k) {                           // K = 128 dims in steps of 16
          const uint32_t ao = (uint32_t)((k >> 2) * (Cfg::A_BYTES / 2) + (k & 3) * 32);
          const uint32_t bo = (uint32_t)((k >> 2) * (Cfg::B_BYTES / 2) + (k & 3) * 32);
          umma_bf16(d, umma_sdesc(sa + ao), umma_sdesc(sb + bo), idesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&tfull[tb]);
        umma_commit(&empty[slot]);
        done = w + 1;
      }
      if (done > 0) {                                           // the last products are complete
        const int w = done - 1;
        mbar_wait(&tfull[w % NTB], (uint32_t)((w / NTB) & 1));
      }
    }
  } else if (warp >= kScanEpiWarps && pre) {                    // ---- post: runs of epilogue warp p's rows
    const int p = warp - kScanEpiWarps;
    const float* sw = s_acc + p * 32 * 33;
    int64_t* wp = wpost + p * kScanDocCols;
    const int q0 = a.pass * NQP;
    const int q1 = min(q0 + NQP, a.NQ);
    int h = 0;                                                  // hand-overs received
    bool ok = true;
    for (int it = 0; it < ntile && ok; ++it) {
      const int tile = t0 + it;
      const int fdoc = a.tile_first_doc[tile];
      for (int j = lane; j <= kScanTile; j += 32) wp[j] = (int64_t)fdoc + j <= a.D ? a.doc_chunk_off[fdoc + j] : a.C;
      __syncwarp();
      const int64_t c = (int64_t)tile * kScanTile + p * 32 + lane;
      const int doc_l = c < a.C ? window_find(wp, c) : -1;
      for (int kq = 0; kq < NQP / 32; ++kq, ++h) {
        if (!mbar_wait_warp(&pfull[p], (uint32_t)(h & 1))) { ok = false; break; }
        post_runs(sw, doc_l, lane, q0 + 32 * kq, q1, a.Ttok, a.D, fdoc, a.score);
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty[p]);
      }
    }
  } else if (warp >= kScanEpiWarps) {                           // ---- norms: chunk row = thread
    const int row = threadIdx.x - kScanEpiWarps * 32;
    for (int w = 0; w < nwork; ++w) {
      const int slot = w % NSTAGE;
      if (!mbar_wait_warp(&full[slot], (uint32_t)((w / NSTAGE) & 1))) break;
      const unsigned char* sa = smem + slot * Cfg::STAGE;
      float2 nn[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int j = 0; j < 8; ++j) {                           // logical chunk j sits at j ^ (row mod 8)
          const uint4 v = *reinterpret_cast<const uint4*>(sa + h * (Cfg::A_BYTES / 2) + row * 128 +
                                                          ((j ^ (row & 7)) << 4));
          float x[8];
          Elem<__nv_bfloat16>::unpack(v, x);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 p = make_float2(x[2 * i], x[2 * i + 1]);
            nn[i] = __ffma2_rn(p, p, nn[i]);
          }
        }
      const float n2 = ((nn[0].x + nn[0].y) + (nn[1].x + nn[1].y)) + ((nn[2].x + nn[2].y) + (nn[3].x + nn[3].y));
      s_rn[slot * kScanTile + row] = rsqrtf(fmaxf(n2, 1e-24f));
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&nready[slot]);
        mbar_arrive(&empty[slot]);
      }
    }
  } else {                                                      // ---- epilogue: chunk row = thread
    const int row = threadIdx.x;
    const uint32_t tlane = (uint32_t)(warp * 32) << 16;
    const int q0 = a.pass * NQP;
    const int q1 = min(q0 + NQP, a.NQ);                         // rows of this pass: [q0, q1)
    // document window of tile t0 + i: doc_chunk_off[fdoc .. fdoc + 128] (past D: C);
    // the next tile's window is fetched during this tile's heads
    auto win_val = [&](int fd, int j) -> int64_t {
      return (int64_t)fd + j <= a.D ? a.doc_chunk_off[fd + j] : a.C;
    };
    int fdoc_next = (ntile > 0 && !pre) ? a.tile_first_doc[t0] : 0;
    if (ntile > 0 && !pre) {
      win[row] = win_val(fdoc_next, row);
      if (row == 0) win[kScanTile] = win_val(fdoc_next, kScanTile);
    }
    bool ok = true;
    for (int it = 0; it < ntile && ok; ++it) {
      const int tile = t0 + it;
      const int64_t c = (int64_t)tile * kScanTile + row;
      const int fdoc = fdoc_next;
      int64_t* wn = win + (it & 1) * kScanDocCols;
      const bool more = !pre && it + 1 < ntile;               // the window is only needed here without the table
      fdoc_next = more ? a.tile_first_doc[tile + 1] : 0;
      int64_t wnext = 0, wnext_last = 0;
      float acc[NQP];
#pragma unroll
      for (int q = 0; q < NQP; ++q) acc[q] = 0.f;
      for (int g = 0; g < H; ++g) {
        const int w = it * H + g, slot = w % NSTAGE, tb = w % NTB;
        if (g == H / 2 && more) {                               // next window, loads in flight
          wnext = win_val(fdoc_next, row);
          if (row == 0) wnext_last = win_val(fdoc_next, kScanTile);
        }
        if (!mbar_wait_warp(pre ? &full[slot] : &nready[slot], (uint32_t)((w / NSTAGE) & 1))) { ok = false; break; }
        const float rn = pre ? reinterpret_cast<const float*>(smem + slot * Cfg::STAGE + Cfg::A_BYTES +
                                                              Cfg::B_BYTES)[row]
                             : s_rn[slot * kScanTile + row];
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (!mbar_wait_warp(&tfull[tb], (uint32_t)((w / NTB) & 1))) { ok = false; break; }
        tc_fence_after();
        if constexpr (NQP <= 64) {                            // hi and lo columns in flight together
#pragma unroll
          for (int cb = 0; cb < NQP / 32; ++cb) {
            uint32_t hi[32], lo[32];
            tmem_ld32_issue(tmem + tlane + (uint32_t)(tb * NP2 + 32 * cb), hi);
            tmem_ld32_issue(tmem + tlane + (uint32_t)(tb * NP2 + NQP + 32 * cb), lo);
            tmem_wait_tie(hi);
            reg_tie(lo);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              acc[32 * cb + i] = fmaf(__uint_as_float(hi[i]) + __uint_as_float(lo[i]), rn, acc[32 * cb + i]);
          }
        } else {                                                // 128 rows: narrower loads keep acc in registers
#pragma unroll
          for (int cb = 0; cb < NQP / 16; ++cb) {
            uint32_t hi[16], lo[16];
            tmem_ld16_issue(tmem + tlane + (uint32_t)(tb * NP2 + 16 * cb), hi);
            tmem_ld16_issue(tmem + tlane + (uint32_t)(tb * NP2 + NQP + 16 * cb), lo);
            tmem_wait_tie(hi);
            reg_tie(lo);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              acc[16 * cb + i] = fmaf(__uint_as_float(hi[i]) + __uint_as_float(lo[i]), rn, acc[16 * cb + i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[tb]);
      }
      float* sw = s_acc + warp * 32 * 33;                      // [row][33], padded: no bank conflicts
      if (pre) {                                                // rows go to the post warp; next tile at once
        if (!ok) break;
#pragma unroll
        for (int kq = 0; kq < NQP / 32; ++kq) {
          const int h = it * (NQP / 32) + kq;
          if (h > 0 && !mbar_wait_warp(&pempty[warp], (uint32_t)((h - 1) & 1))) { ok = false; break; }
#pragma unroll
          for (int i = 0; i < 32; ++i) sw[lane * 33 + i] = acc[32 * kq + i];
          __syncwarp();
          if (lane == 0) mbar_arrive(&pfull[warp]);
        }
        continue;
      }
      if (more) {                                               // the buffer tile it - 1 used
        int64_t* wx = win + ((it + 1) & 1) * kScanDocCols;
        wx[row] = wnext;
        if (row == 0) wx[kScanTile] = wnext_last;
      }
      ok = epi_bar_and(ok);                                     // document windows written
      if (!ok) break;
      const int doc_l = c < a.C ? window_find(wn, c) : -1;
#pragma unroll
      for (int kq = 0; kq < NQP / 32; ++kq) {
#pragma unroll
        for (int i = 0; i < 32; ++i) sw[lane * 33 + i] = acc[32 * kq + i];
        __syncwarp();
        post_runs(sw, doc_l, lane, q0 + 32 * kq, q1, a.Ttok, a.D, fdoc, a.score);
        __syncwarp();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kScanMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(Cfg::TCOLS) : "memory");
  }
}

}  // namespace msa
