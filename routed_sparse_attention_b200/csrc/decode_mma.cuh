// Stage 3 kernel for bf16 banks: split-K GQA decode on the tensor cores.
//
// Method: "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts",
// section "How MSA compresses and routes documents", and "EverMind Releases
// Memory-Sparse Attention Code for Long-Context AI Models", section
// "Architectural Design and Inference" (stage 3): attention of the query over
// [pooled K/V of the Top-k documents ++ local K/V], global RoPE offset k.
//
// Same work split and partials as decode_kernel (decode.cuh); what changes is
// the inner product and the merge.  A CTA owns 16 * WR query rows (WR = 1 or
// 2) of one kv head (rows r = t * G + h_in_group, padded to whole m16 blocks)
// and one split of keys.  The last CTA of a (query, kv head, row group),
// found by an acquire-release counter, merges the splits (merge_splits).  Its 4 warps form WR row blocks x (4 / WR) key groups: warp (rb, kw)
// computes, per 64-key tile, S = Q_rb K^T over its 64 / (4/WR) keys and
// O_rb += P V with mma.sync m16n8k16 (bf16 operands, fp32 accumulators), the
// softmax running on the accumulator fragments with a lazily moved reference
// max.  Per tile and warp that is a few dozen tensor instructions instead of
// the ~1000 scalar ones a CUDA-core dot product needs for bf16 keys, which is
// what lets a T = 1 decode stream at HBM rate.
//
// Tiles sit in shared memory as rows of 128 bytes (64 dims; d = 128 uses two
// such halves) with the 16-byte chunk index XOR-ed with the row index mod 8:
// the layout TMA's 128-byte swizzle writes for local tiles, and the one the
// memory-key gather reproduces with cp.async.  ldmatrix then reads 8 rows of
// one logical chunk from 8 distinct bank groups.
//
// Numerics: the rotated query and the probabilities P enter the products as
// bf16 (relative rounding 2^-9), keys and values are the stored bf16 values,
// every sum is fp32.
#pragma once
#include <cuda.h>

#include "decode.cuh"

namespace msa {

constexpr int kMmaWarps = 4;
constexpr int kMmaThreads = kMmaWarps * 32;
constexpr int kMmaStages = 2;

struct DecodeMmaArgs {
  CUtensorMap tm_k;                        // local K / V: [rows][d] bf16, box 64 x 64, 128-byte swizzle
  CUtensorMap tm_v;
  CUtensorMap tm_q;                        // tensor-core kernel only: Q [B*T][Hq][128], box 128 x G x 128/G
  DecodeArgs d;
};

// Scratch of the merge of a CTA's warps (their key groups) into one partial.
template <int D>
struct DecWarpMerge {
  float o[kMmaWarps][16][D];                                // warp partials, [warp][row in block][dim]
  float ml[kMmaWarps][16][2];
  float w[kMmaWarps][64];                                   // per-warp weight of each CTA row
  float rowm[64], rowl[64];                                 // per CTA row: reference max, sum
};

template <int D>
struct DecMmaSmem {
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kHalves * 64 * 128;     // one tensor of one 64-key tile
  union {
    unsigned char kv[kMmaStages][2][kTileBytes];            // [stage][K, V] swizzled tiles
    DecWarpMerge<D> merge;
  } u;
  uint64_t full[kMmaStages];
  int64_t mem_pref[kMaxTopKDecode + 1];
  int64_t mem_krow[kMaxTopKDecode];
  int64_t mem_vrow[kMaxTopKDecode];
  int64_t key_krow[kMmaStages][kDecTile];                   // source rows of a memory tile's keys
  int64_t key_vrow[kMmaStages][kDecTile];
  int last;
};

// ------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// D += A (16x16 bf16, row) * B (16x8 bf16, col), fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
// Add to a split counter with acquire-release semantics at GPU scope: after a
// CTA barrier, one thread's call publishes the CTA's earlier global writes,
// and the thread that reads the final count (followed by a CTA barrier) sees
// every other CTA's writes.
__device__ __forceinline__ int atom_add_acq_rel(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
// Byte offset of (row, logical 16-byte chunk) in a swizzled tile.
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)((chunk >> 3) * (64 * 128) + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

// The merge of a (query, kv head, row group)'s splits sfirst .. sfirst +
// nsplit - 1: for every item (row r0 + rr, 4 dims) the splits' partial outputs
// are added with weights
// 2^(m_s - m), m the running maximum, one rescale per batch of NBT splits with
// all the batch's loads in flight; NI items per thread at a time.
template <int D, int NI, int NBT>
__device__ __forceinline__ void merge_splits(const DecodeArgs& a, int b, int g, int r0, int nrow, int sfirst,
                                             int nsplit) {
  constexpr int QD = D / 4;
  const int n_items = nrow * QD;
  const int64_t sstride = (int64_t)a.Hkv * a.R;             // rows between consecutive splits
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
  for (int i0 = threadIdx.x; i0 < n_items; i0 += NI * kMmaThreads) {
    float4 acc[NI];
    float mrun[NI], lrun[NI];
    int64_t pbase[NI];
    int rr[NI], qd[NI];
#pragma unroll
    for (int j = 0; j < NI; ++j) {
      const int idx = min(i0 + j * kMmaThreads, n_items - 1);
      rr[j] = idx / QD;
      qd[j] = idx % QD;
      pbase[j] = ((int64_t)sfirst * a.Hkv + g) * a.R + r0 + rr[j];
      acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      mrun[j] = -INFINITY;
      lrun[j] = 0.f;
    }
#pragma unroll 1
    for (int s0 = 0; s0 < nsplit; s0 += NBT) {
      float4 v[NI][NBT];
      float2 ml[NI][NBT];
#pragma unroll
      for (int j = 0; j < NI; ++j)
#pragma unroll
        for (int u = 0; u < NBT; ++u) {
          const int64_t prow = pbase[j] + (int64_t)min(s0 + u, nsplit - 1) * sstride;
          ml[j][u] = __ldcg(reinterpret_cast<const float2*>(a.part_ml) + prow);
          v[j][u] = __ldcg(reinterpret_cast<const float4*>(a.part_o + prow * D) + qd[j]);
        }
#pragma unroll
      for (int j = 0; j < NI; ++j) {
        float mb = mrun[j];
#pragma unroll
        for (int u = 0; u < NBT; ++u)
          if (s0 + u < nsplit) mb = fmaxf(mb, ml[j][u].x);
        if (mb == -INFINITY) continue;                      // no key seen yet
        const float sa = exp2f(mrun[j] - mb);               // mrun = -inf gives 0
        acc[j].x *= sa; acc[j].y *= sa; acc[j].z *= sa; acc[j].w *= sa;
        lrun[j] *= sa;
#pragma unroll
        for (int u = 0; u < NBT; ++u) {
          const float wgt = (s0 + u >= nsplit || ml[j][u].x == -INFINITY) ? 0.f : exp2f(ml[j][u].x - mb);
          acc[j].x = fmaf(v[j][u].x, wgt, acc[j].x);
          acc[j].y = fmaf(v[j][u].y, wgt, acc[j].y);
          acc[j].z = fmaf(v[j][u].z, wgt, acc[j].z);
          acc[j].w = fmaf(v[j][u].w, wgt, acc[j].w);
          lrun[j] = fmaf(ml[j][u].y, wgt, lrun[j]);
        }
        mrun[j] = mb;
      }
    }
#pragma unroll
    for (int j = 0; j < NI; ++j) {
      if (i0 + j * kMmaThreads >= n_items) continue;
      const float inv = 1.0f / lrun[j];
      const int r = r0 + rr[j];
      const int t = r / a.G, h = g * a.G + r % a.G;
      if (a.lse && qd[j] == 0)
        a.lse[((int64_t)b * a.T + t) * a.Hq + h] = (mrun[j] + log2f(lrun[j])) * 0.6931471805599453f;
      __nv_bfloat16* op = out + (((int64_t)b * a.T + t) * a.Hq + h) * D + 4 * qd[j];
      *reinterpret_cast<uint2*>(op) =
          make_uint2(pack_bf16(acc[j].x * inv, acc[j].y * inv), pack_bf16(acc[j].z * inv, acc[j].w * inv));
    }
  }
}

// ------------------------------------------------- pieces shared by the kernels

// The memory split's set-up: rank r's first K / V source rows and its chunk
// count, then their prefix sums; mem_pref[k] is the split's key count.  `doc`
// is this thread's selected document (threads < k), already loaded.  Ends
// with a CTA barrier.
__device__ __forceinline__ void dec_mem_setup(const DecodeArgs& a, int b, int k, int doc, int64_t* mem_pref,
                                              int64_t* mem_krow, int64_t* mem_vrow) {
  if (threadIdx.x < k) {
    const int r = threadIdx.x;
    if (doc < 0 || doc >= a.n_docs) { dev_flag(MSA_DEV_BAD_DOC); doc = 0; }
    const int64_t c0 = a.doc_chunk_off[doc];
    int64_t nc = a.doc_chunk_off[doc + 1] - c0;
    if (nc > a.max_doc_chunks) nc = 0;
    if (a.kv_on_host) {
      const int64_t slot = ((int64_t)b * k + r) * 2 * a.max_doc_chunks;
      mem_krow[r] = slot;
      mem_vrow[r] = slot + nc;
    } else {
      mem_krow[r] = c0;
      mem_vrow[r] = c0;
    }
    mem_pref[r + 1] = nc;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mem_pref[0] = 0;
    for (int r = 0; r < k; ++r) mem_pref[r + 1] += mem_pref[r];
  }
  __syncthreads();
}

// Source rows of the memory keys of tile tt of the key range [kbeg, kend)
// (thread tid < 64: key kbeg + 64 tt + tid), found by a binary search of the
// rank in the chunk prefix.
__device__ __forceinline__ void dec_mem_rows(int tid, int tt, int64_t kbeg, int64_t kend, int k,
                                             const int64_t* mem_pref, const int64_t* mem_krow,
                                             const int64_t* mem_vrow, int64_t* key_krow, int64_t* key_vrow) {
  const int64_t kk = kbeg + (int64_t)tt * kDecTile + tid;
  if (tid < kDecTile && kk < kend) {
    int lo = 0, hi = k;                                     // mem_pref[lo] <= kk < mem_pref[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (mem_pref[mid] <= kk) lo = mid;
      else hi = mid;
    }
    const int64_t ci = kk - mem_pref[lo];
    key_krow[tid] = mem_krow[lo] + ci;
    key_vrow[tid] = mem_vrow[lo] + ci;
  }
}

// cp.async gather of memory tile tt of the key range [kbeg, kend) into the
// swizzled K / V tiles kt / vt by 128 threads (tid 0..127), one per key row
// of K or V (rows past the keys zero-filled, so no stale value reaches P V);
// one commit group.
template <int D>
__device__ __forceinline__ void dec_mem_gather(int tid, const DecodeArgs& a, int g, int tt, int64_t kbeg,
                                               int64_t kend, const int64_t* key_krow, const int64_t* key_vrow,
                                               unsigned char* kt, unsigned char* vt) {
  constexpr int CPR = D / 8;                                // 16-byte chunks per row
  static_assert(kMmaThreads == 2 * kDecTile, "one thread per key row of K or V");
  const int n2 = (int)min64(kDecTile, kend - kbeg - (int64_t)tt * kDecTile);
  const int i = tid >> 1, kv = tid & 1;
  unsigned char* dst = kv ? vt : kt;
  if (i < n2) {
    const int64_t row = kv ? key_vrow[i] : key_krow[i];
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>((kv && !a.kv_on_host) ? a.mem_v : a.mem_k)
                               + (row * a.Hkv + g) * D;
#pragma unroll
    for (int c = 0; c < CPR; ++c) cp_async_16(dst + swz(i, c), src + 8 * c);
  } else {
#pragma unroll
    for (int c = 0; c < CPR; ++c) *reinterpret_cast<uint4*>(dst + swz(i, c)) = make_uint4(0u, 0u, 0u, 0u);
  }
  cp_async_commit();
}

// The rotated query as bf16 A fragments for this lane's rows qr and qr + 8 of
// row block rb (CTA rows rg * RPC + rb * 16 + ...), and the last
// split-relative key each row sees (lim, -1: none; memory splits see every
// key).  The query token t sits at position top_k + L_b + t.
template <int D, int RPC>
__device__ __forceinline__ void dec_query_frags(const DecodeArgs& a, int b, int g, int rg, int rb, int qr, int qc,
                                                bool mem, int64_t Lb, int64_t j_lo, uint32_t (&qa)[D / 16][4],
                                                int (&lim)[2]) {
  constexpr int KB = D / 16, HALF = D / 2;
  const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.q);
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    if (rg * RPC + rb * 16 + 8 * hr >= a.R) {               // no real row in this half (warp-uniform)
      lim[hr] = -1;
#pragma unroll
      for (int kb = 0; kb < KB; ++kb) qa[kb][hr] = qa[kb][hr + 2] = 0u;
      continue;
    }
    const int r = rg * RPC + rb * 16 + qr + 8 * hr;
    bool on = r < a.R;
    const int t = on ? r / a.G : 0, h = g * a.G + (on ? r % a.G : 0);
    int64_t pos = (int64_t)a.top_k + Lb + t;
    const int64_t last = Lb + t - j_lo;
    if (!mem && last < 0) on = false;
    lim[hr] = !on ? -1 : (mem ? INT_MAX : (int)min64(last, INT_MAX));
    if (pos >= a.rope_rows) { dev_flag(MSA_DEV_ROPE_RANGE); pos = a.rope_rows - 1; }
    const __nv_bfloat16* qp = Q + (((int64_t)b * a.T + t) * a.Hq + h) * D;
    const float2* cs = a.rope + pos * HALF;
#pragma unroll
    for (int kb = 0; kb < KB / 2; ++kb) {
#pragma unroll
      for (int o8 = 0; o8 < 2; ++o8) {
        const int c = 16 * kb + 8 * o8 + 2 * qc;            // columns c, c + 1 and partners + d/2
        const float2 x0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(qp + c));
        const float2 x1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(qp + c + HALF));
        const float4 w = __ldg(reinterpret_cast<const float4*>(cs + c));   // (cos, sin) of c and c + 1
        const float lo0 = x0.x * w.x - x1.x * w.y, hi0 = x1.x * w.x + x0.x * w.y;
        const float lo1 = x0.y * w.z - x1.y * w.w, hi1 = x1.y * w.z + x0.y * w.w;
        const uint32_t plo = on ? pack_bf16(lo0, lo1) : 0u, phi = on ? pack_bf16(hi0, hi1) : 0u;
        qa[kb][hr + 2 * o8] = plo;
        qa[kb + KB / 2][hr + 2 * o8] = phi;
      }
    }
  }
}

// One 64-key tile (swizzled K at kt_s, V at vt_s; n_t real keys, first key kt
// split-relative) for this warp's NK keys from kbase: S = Q K^T, the online
// softmax on the fragments (reference max mref, sum lsum per fragment row),
// O += P V.
template <int D, int NK>
__device__ __forceinline__ void dec_attend_tile(const DecodeArgs& a, uint32_t kt_s, uint32_t vt_s, int n_t,
                                                int64_t kt, int kbase, int lane, int qc,
                                                const uint32_t (&qa)[D / 16][4], const int (&lim)[2],
                                                float (&oacc)[D / 8][4], float (&mref)[2], float (&lsum)[2]) {
  constexpr int NKB = NK / 8, KB = D / 16, NB = D / 8;
  float sacc[NKB][4];
#pragma unroll
  for (int nb = 0; nb < NKB; ++nb) sacc[nb][0] = sacc[nb][1] = sacc[nb][2] = sacc[nb][3] = 0.f;
#pragma unroll
  for (int nb = 0; nb < NKB; ++nb) {
    const int key = kbase + nb * 8 + (lane & 7);
#pragma unroll
    for (int kb2 = 0; kb2 < KB / 2; ++kb2) {
      uint32_t bf[4];
      ldsm_x4(kt_s + swz(key, 4 * kb2 + (lane >> 3)), bf);
      mma_bf16(sacc[nb], qa[2 * kb2], bf[0], bf[1]);
      mma_bf16(sacc[nb], qa[2 * kb2 + 1], bf[2], bf[3]);
    }
  }
  // softmax on the fragments: sacc[nb][0..1] row qr, [2..3] row qr + 8; keys kbase + 8 nb + 2 qc + {0, 1}
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nb = 0; nb < NKB; ++nb) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = kbase + nb * 8 + 2 * qc + (e & 1);
      const bool vis = key < n_t && kt + key <= lim[e >> 1];
      sacc[nb][e] = vis ? sacc[nb][e] * a.scale_log2 : -INFINITY;
      mx[e >> 1] = fmaxf(mx[e >> 1], sacc[nb][e]);
    }
  }
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 1));
    mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 2));
    if (mx[hr] > mref[hr] + kLazyRescale) {                 // new reference max for the row
      const float sc = exp2f(mref[hr] - mx[hr]);
      lsum[hr] *= sc;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        oacc[nb][2 * hr] *= sc;
        oacc[nb][2 * hr + 1] *= sc;
      }
      mref[hr] = mx[hr];
    }
  }
  uint32_t pa[NK / 16][4];
#pragma unroll
  for (int nb = 0; nb < NKB; ++nb) {
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      p[e] = sacc[nb][e] == -INFINITY ? 0.f : exp2f(sacc[nb][e] - mref[e >> 1]);
      lsum[e >> 1] += p[e];
    }
    pa[nb >> 1][2 * (nb & 1)] = pack_bf16(p[0], p[1]);
    pa[nb >> 1][2 * (nb & 1) + 1] = pack_bf16(p[2], p[3]);
  }
  // O += P V
#pragma unroll
  for (int j = 0; j < NK / 16; ++j) {
    const int key = kbase + 16 * j + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int np = 0; np < NB / 2; ++np) {
      uint32_t bf[4];
      ldsm_x4_t(vt_s + swz(key, 2 * np + (lane >> 4)), bf);
      mma_bf16(oacc[2 * np], pa[j], bf[0], bf[1]);
      mma_bf16(oacc[2 * np + 1], pa[j], bf[2], bf[3]);
    }
  }
}

// The second half of the warp merge, once every warp's partial (o, ml) is in
// mg: per CTA row the weights of the warps' reference maxima, then the
// weighted sum of their outputs.
template <int D, int WR, typename StoreML, typename StoreO>
__device__ __forceinline__ void dec_combine_warps(DecWarpMerge<D>& mg, int nrow, StoreML store_ml, StoreO store_o) {
  constexpr int KW = kMmaWarps / WR;
  if (threadIdx.x < nrow) {                                 // row rr: reference max, weights, sum
    const int rr = threadIdx.x, rbk = rr / 16, ri = rr % 16;
    float mt = -INFINITY;
#pragma unroll
    for (int w = 0; w < KW; ++w) mt = fmaxf(mt, mg.ml[w * WR + rbk][ri][0]);
    float lt = 0.f;
#pragma unroll
    for (int w = 0; w < KW; ++w) {
      const float mw = mg.ml[w * WR + rbk][ri][0];
      const float sc = mw == -INFINITY ? 0.f : exp2f(mw - mt);
      mg.w[w][rr] = sc;
      lt += mg.ml[w * WR + rbk][ri][1] * sc;
    }
    mg.rowm[rr] = mt;
    mg.rowl[rr] = lt;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < nrow * (D / 4); idx += kMmaThreads) {
    const int rr = idx / (D / 4), d4 = idx % (D / 4);       // row within the CTA, 4-dim group
    const int rbk = rr / 16, ri = rr % 16;
    float4 ot = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < KW; ++w) {
      const float wt = mg.w[w][rr];
      const float4 o = *reinterpret_cast<const float4*>(&mg.o[w * WR + rbk][ri][4 * d4]);
      ot.x = fmaf(wt, o.x, ot.x);
      ot.y = fmaf(wt, o.y, ot.y);
      ot.z = fmaf(wt, o.z, ot.z);
      ot.w = fmaf(wt, o.w, ot.w);
    }
    store_o(rr, d4, ot);
    if (d4 == 0) store_ml(rr, mg.rowm[rr], mg.rowl[rr]);
  }
}

// Merges the key groups (warps) of each row block into the CTA's partial for
// its nrow real rows: per row the reference max and sum go to store_ml(rr, m,
// l), the weighted output to store_o(rr, d4, float4) for 4 dims at a time.
// The caller has finished with the tiles (mg aliases them) and placed a CTA
// barrier after its last read of them.
template <int D, int WR, typename StoreML, typename StoreO>
__device__ __forceinline__ void dec_merge_warps(DecWarpMerge<D>& mg, int warp, int qr, int qc, int nrow,
                                                const float (&oacc)[D / 8][4], const float (&mref)[2],
                                                float (&lsum)[2], StoreML store_ml, StoreO store_o) {
  constexpr int NB = D / 8;
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    lsum[hr] += __shfl_xor_sync(0xffffffffu, lsum[hr], 1);
    lsum[hr] += __shfl_xor_sync(0xffffffffu, lsum[hr], 2);
  }
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    *reinterpret_cast<float2*>(&mg.o[warp][qr][8 * nb + 2 * qc]) = make_float2(oacc[nb][0], oacc[nb][1]);
    *reinterpret_cast<float2*>(&mg.o[warp][qr + 8][8 * nb + 2 * qc]) = make_float2(oacc[nb][2], oacc[nb][3]);
  }
  if (qc == 0) {
    mg.ml[warp][qr][0] = mref[0];
    mg.ml[warp][qr][1] = lsum[0];
    mg.ml[warp][qr + 8][0] = mref[1];
    mg.ml[warp][qr + 8][1] = lsum[1];
  }
  __syncthreads();
  dec_combine_warps<D, WR>(mg, nrow, store_ml, store_o);
}

// ------------------------------------------------------------- the kernel

template <int D, int WR>
__global__ void __launch_bounds__(kMmaThreads)
decode_mma_kernel(const __grid_constant__ DecodeMmaArgs A) {
  const DecodeArgs& a = A.d;
  constexpr int KW = kMmaWarps / WR;        // key groups
  constexpr int NK = kDecTile / KW;         // keys of a warp per tile
  constexpr int KB = D / 16;                // dim k-blocks of S
  constexpr int NB = D / 8;                 // dim n-blocks of O
  constexpr int RPC = 16 * WR;              // rows per CTA
  using Smem = DecMmaSmem<D>;
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(NK % 16 == 0, "whole 16-key blocks per warp");
  extern __shared__ unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = warp % WR, kw = warp / WR;
  const int qr = lane >> 2, qc = lane & 3;  // fragment row / column-pair of this lane
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
  int doc = 0;
  if (mem && threadIdx.x < k) doc = __ldg(a.sel + (int64_t)b * k + threadIdx.x);

  // ---- local splits: issue the first tiles
  const int64_t j_lo = mem ? 0 : (int64_t)(s - 1) * a.S;
  int64_t nkeys = mem ? 0 : min64(a.S, Ltot - j_lo);
  if (nkeys < 0) nkeys = 0;                                   // a split past the live tokens
  const int row0 = (int)(a.local_off[b] * a.Hkv + (int64_t)g * cap + j_lo);    // tensor-map row of key j_lo
  auto issue_local = [&](int t) {                         // thread 0 only
    const int st = t % kMmaStages;
    mbar_arrive_expect_tx(&sm.full[st], 2 * Smem::kTileBytes);
#pragma unroll
    for (int h = 0; h < Smem::kHalves; ++h) {
      tma_load_2d(&sm.u.kv[st][0][h * 64 * 128], &A.tm_k, 64 * h, row0 + t * kDecTile, &sm.full[st]);
      tma_load_2d(&sm.u.kv[st][1][h * 64 * 128], &A.tm_v, 64 * h, row0 + t * kDecTile, &sm.full[st]);
    }
  };
  if (!mem && threadIdx.x == 0) {
    const int nt0 = (int)((nkeys + kDecTile - 1) / kDecTile);
    for (int st = 0; st < kMmaStages; ++st) mbar_init(&sm.full[st], 1);
    fence_mbar_init();
    for (int t = 0; t < nt0 && t < kMmaStages; ++t) issue_local(t);
  }

  // ---- memory split: rank r's chunk count and first K / V rows; its first
  //      two tiles are gathered before the query is rotated, so the rotation
  //      overlaps their loads
  if (mem) {
    dec_mem_setup(a, b, k, doc, sm.mem_pref, sm.mem_krow, sm.mem_vrow);
    nkeys = sm.mem_pref[k];
  }
  auto mem_rows = [&](int tt) {
    dec_mem_rows(threadIdx.x, tt, 0, nkeys, k, sm.mem_pref, sm.mem_krow, sm.mem_vrow, sm.key_krow[tt % kMmaStages],
                 sm.key_vrow[tt % kMmaStages]);
  };
  auto mem_gather = [&](int tt) {
    const int sst = tt % kMmaStages;
    dec_mem_gather<D>(threadIdx.x, a, g, tt, 0, nkeys, sm.key_krow[sst], sm.key_vrow[sst], &sm.u.kv[sst][0][0],
                      &sm.u.kv[sst][1][0]);
  };
  const int ntiles = (int)((nkeys + kDecTile - 1) / kDecTile);
  if (mem && ntiles > 0) {
    mem_rows(0);
    if (ntiles > 1) mem_rows(1);
    __syncthreads();
    mem_gather(0);
    if (ntiles > 1) mem_gather(1);
  }

  // ---- rotated query as bf16 A fragments; rows qr and qr + 8 of block rb
  uint32_t qa[KB][4];
  int lim[2];                                // last split-relative key the row sees (-1: none)
  dec_query_frags<D, RPC>(a, b, g, rg, rb, qr, qc, mem, Lb, j_lo, qa, lim);

  if (!mem) __syncthreads();                                // barriers initialised

  float oacc[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) oacc[nb][0] = oacc[nb][1] = oacc[nb][2] = oacc[nb][3] = 0.f;
  float mref[2] = {-INFINITY, -INFINITY}, lsum[2] = {0.f, 0.f};
  const int kbase = kw * NK;                                // this warp's first key of a tile

#pragma unroll 1
  for (int t = 0; t < ntiles; ++t) {
    const int st = t % kMmaStages;
    const int64_t kt = (int64_t)t * kDecTile;               // first key of the tile (split-relative)
    const int n_t = (int)min64(kDecTile, nkeys - kt);
    if (mem) {
      if (t + 1 < ntiles) cp_async_wait_group<1>();         // tile t landed, t + 1 may still fly
      else cp_async_wait_group<0>();
      __syncthreads();
    } else {
      // every thread leaves together if the wait ran out (the loop has CTA barriers)
      if (!__syncthreads_and(mbar_wait(&sm.full[st], (uint32_t)((t / kMmaStages) & 1)))) break;
    }
    dec_attend_tile<D, NK>(a, smem_u32(&sm.u.kv[st][0][0]), smem_u32(&sm.u.kv[st][1][0]), n_t, kt, kbase, lane, qc,
                           qa, lim, oacc, mref, lsum);
    __syncthreads();                                        // stage free again
    if (t + kMmaStages < ntiles) {
      if (!mem) {
        if (threadIdx.x == 0) issue_local(t + kMmaStages);
      } else {
        mem_rows(t + kMmaStages);
        __syncthreads();
        mem_gather(t + kMmaStages);
      }
    }
  }
  cp_async_wait_group<0>();
  __syncthreads();                                          // tiles done: shared memory becomes merge scratch

  // ---- merge the key groups of each row block and write this split's partial
  const int nrow = min(RPC, a.R - rg * RPC);                // real rows of this CTA
  const int sid = a.split_off[b] + s;
  const int64_t prow0 = ((int64_t)sid * a.Hkv + g) * a.R + rg * RPC;
  dec_merge_warps<D, WR>(
      sm.u.merge, warp, qr, qc, nrow, oacc, mref, lsum,
      [&](int rr, float m, float l) { reinterpret_cast<float2*>(a.part_ml)[prow0 + rr] = make_float2(m, l); },
      [&](int rr, int d4, float4 ot) { reinterpret_cast<float4*>(a.part_o + (prow0 + rr) * D)[d4] = ot; });

  // ---- the last split of this (query, kv head, row group) merges them all
  __syncthreads();
  int* counter = a.counters + ((int64_t)b * a.Hkv + g) * a.n_rg + rg;
  if (threadIdx.x == 0) sm.last = (atom_add_acq_rel(counter, 1) == nsplit - 1);
  __syncthreads();
  if (!sm.last) return;
  // items (row, 4 dims): one per thread with batches of 16 splits when they
  // fit one pass of the CTA, else two per thread with batches of 8, so two
  // items' loads are in flight together
  const int sfirst = a.split_off[b];
  if (nrow * (D / 4) <= kMmaThreads) merge_splits<D, 1, 16>(a, b, g, rg * RPC, nrow, sfirst, nsplit);
  else merge_splits<D, 2, 8>(a, b, g, rg * RPC, nrow, sfirst, nsplit);
  if (threadIdx.x == 0) *counter = 0;                      // ready for the next call
}

}  // namespace msa
