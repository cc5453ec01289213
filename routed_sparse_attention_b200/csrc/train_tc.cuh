// Backward of the sparse attention on the 5th-generation tensor cores (bf16
// banks, head_dim 128).
//
// "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts", sections
// "How MSA compresses and routes documents" and "MSA against a conventional
// RAG stack" (routing and generation trained end to end).  The forward is the
// decode (attention over [selected pooled K/V ++ local K/V] with the query at
// position top_k + L_b + t); given dO, its log-sum-exp and D = sum dO * O per
// row, the gradients are, per (row r, key j) with P = 2^(s q~.k log2e - lse log2e),
//   dV_j += P dO_r,   dS = P (dO_r . v_j - D_r),
//   dK_j += s dS q~_r,   dq~_r += s dS k_j        (s = 1/sqrt(d)),
// with the rotated query q~ (dq~ is rotated back afterwards, and a local key's
// dK back to the unrotated key's frame in the epilogue).
//
// One CTA per (128-key tile, kv head, query): keys on the MMA's M side.  Per
// block of 128 query rows (r = t * G + h_in_group):
//   S^T  = K q~^T     M = 128 keys, N = 128 rows, K = 128 dims   -> TMEM 0..127
//   dP^T = V dO^T     M = 128 keys, N = 128 rows, K = 128 dims   -> TMEM 128..255
// eight softmax warps (lane = key = TMEM lane; two warps per lane quarter,
// each taking half of the rows) turn them into P^T and dS^T in bf16 in shared
// memory (key rows, 128-byte swizzle), then
//   dV  += P^T dO     M = 128 keys, N = 128 dims, K = 128 rows   -> TMEM 256..383
//   dK  += dS^T q~    M = 128 keys, N = 128 dims, K = 128 rows   -> TMEM 384..511
//   dq~  = dS K       M = 128 rows, N = 128 dims, K = 128 keys   -> TMEM 0..127
// and the same warps (lane = row) stage dq~ in shared memory, from where one
// tile reduce-add per 32 dims adds it to global memory.
// Every tile is one shared-memory layout ([dim or row half][128 rows][64],
// 128-byte swizzle) read either way: K-major where the contraction runs along
// its rows' contiguous elements (K, V in S^T and dP^T; q~, dO as B there;
// P^T, dS^T as A of dV, dK), MN-major otherwise (dO, q~ as B of dV, dK; dS^T as
// A and K as B of dq).  q~ and dO arrive by TMA (one box of 128 / G tokens x
// G heads per 64 dims), local K and V by TMA too, a memory tile's K and V by
// a cp.async gather (its keys are chunk rows of the selected documents).  At
// the end dV and dK are staged in shared memory and each warp stores (local
// keys; dK rotated back with the tile's RoPE rows, one bulk copy) or adds
// (memory keys) whole rows.  Every wait is bounded (mbar_wait).
#pragma once
#include "train.cuh"
#include "decode_tc.cuh"

namespace msa {

constexpr int kBwtKeys = 128;            // keys per CTA (MMA M)
constexpr int kBwtRows = 128;            // query rows per block
constexpr int kBwtSoftWarps = 8;         // softmax / epilogue: two warps per TMEM lane quarter
constexpr int kBwtSoft = kBwtSoftWarps * 32;
constexpr int kBwtProducerWarp = kBwtSoftWarps;
constexpr int kBwtMmaWarp = kBwtSoftWarps + 1;
constexpr int kBwtThreads = (kBwtSoftWarps + 2) * 32;
constexpr int kBwtTmemCols = 512;

struct BwdTcArgs {
  CUtensorMap tm_q;                      // rotated queries (bf16 workspace) [B*T][Hq][128], box 64 x G x 128/G
  CUtensorMap tm_do;                     // dO, same shape
  CUtensorMap tm_k;                      // local key / value caches [rows][128], box 64 x 128 rows
  CUtensorMap tm_v;
  CUtensorMap tm_dq;                     // fp32 dq~ [B*T][Hq][128], box 32 x G x 128/G (reduce-add)
  BwdArgs a;
};

struct BwdTcSmem {
  static constexpr int kTile = 128 * 256;              // [2 halves][128 rows][128 B]
  unsigned char k[kTile], v[kTile], q[kTile], dout[kTile], pt[kTile], dst[kTile];
  alignas(16) float lse2[2][kBwtRows];                 // per row block (double buffer)
  alignas(16) float drow[2][kBwtRows];
  int64_t krow[kBwtKeys];
  int64_t mem_pref[kMaxTopKDecode + 1];
  int64_t mem_c0[kMaxTopKDecode];
  uint64_t kvfull, qfull, sfull, pready, bdone, dqempty, ropefull;
  uint32_t tmem_slot;
};

// Byte offset of (row, 16-byte chunk) in a 128-row tile with the 128-byte swizzle.
__device__ __forceinline__ uint32_t swz128(int row, int chunk) {
  return (uint32_t)((chunk >> 3) * (128 * 128) + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}
// Tile reduce-add (TMA): global += the box at (x, y, z) from shared memory (bulk group).
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* tm, int x, int y, int z, const void* src) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4}], [%1];"
      ::"l"(reinterpret_cast<uint64_t>(tm)), "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The bulk group's reads of shared memory are done (its source may be rewritten).
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// The bulk group's writes are done.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Barrier of the softmax warps (named barrier 1) that also ANDs `pred` over
// them, so that they leave a loop together; and the plain barrier.
__device__ __forceinline__ bool soft_and(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred q, d;\n setp.ne.u32 q, %1, 0;\n bar.red.and.pred d, 1, %2, q;\n"
      " selp.u32 %0, 1, 0, d;\n}\n"
      : "=r"(r) : "r"((uint32_t)pred), "n"(kBwtSoft) : "memory");
  return r != 0;
}
__device__ __forceinline__ void soft_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kBwtSoft) : "memory"); }

// Instruction descriptor, kind::f16: bf16 A and B both MN-major, fp32 D, M = 128, N = n.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_amn_bmn(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

__global__ void __launch_bounds__(kBwtThreads, 1) attn_bwd_tc_kernel(const __grid_constant__ BwdTcArgs A) {
  constexpr int D = 128, H = D / 2, T16 = 16384;           // T16: bytes between a tile's halves
  const BwdArgs& a = A.a;
  extern __shared__ unsigned char smem_raw[];
  BwdTcSmem& sm = *reinterpret_cast<BwdTcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int g = blockIdx.y;
  const int slot = blockIdx.x;
  int b = 0;
  while (slot >= a.tile_off[b + 1]) ++b;
  const int tile = slot - a.tile_off[b];
  const int64_t cap = a.local_off[b + 1] - a.local_off[b];
  const int64_t Ltot = a.local_len[b], Lb = Ltot - a.T;
  const bool mem = tile < a.mem_tiles;
  if (mem) {                                                 // rank r's first chunk and chunk count, then their prefix
    if (tid < a.top_k) {
      int doc = a.sel[(int64_t)b * a.top_k + tid];
      if (doc < 0 || doc >= a.n_docs) { dev_flag(MSA_DEV_BAD_DOC); doc = 0; }
      const int64_t c0 = a.doc_chunk_off[doc];
      sm.mem_c0[tid] = c0;
      sm.mem_pref[tid + 1] = a.doc_chunk_off[doc + 1] - c0;
    }
    __syncthreads();
    if (tid == 0) {
      sm.mem_pref[0] = 0;
      for (int r = 0; r < a.top_k; ++r) sm.mem_pref[r + 1] += sm.mem_pref[r];
      if (tile == 0 && sm.mem_pref[a.top_k] > (int64_t)a.mem_tiles * kBwtKeys) dev_flag(MSA_DEV_BAD_SHAPE);
    }
    __syncthreads();
  }
  const int64_t k0 = (int64_t)(mem ? tile : tile - a.mem_tiles) * kBwtKeys;
  const int64_t nkey_all = mem ? sm.mem_pref[a.top_k] : Ltot;
  if (k0 >= nkey_all) return;                                // the whole CTA, before any barrier or TMEM
  const int nk = (int)min64(kBwtKeys, nkey_all - k0);
  // row blocks from the first one a row of which sees this tile (visibility grows with the token)
  const int nrb = (a.R + kBwtRows - 1) / kBwtRows;
  int rb0 = 0;
  if (!mem && k0 > Lb) rb0 = (int)min64((int64_t)nrb, (int64_t)a.G * (k0 - Lb) / kBwtRows);
  const int nb = nrb - rb0;                                  // >= 1: the tile's first key is seen by the last token

  // ---- set-up: barriers, TMEM, K/V gather (softmax warps), first q~ / dO box
  auto issue_rows = [&](int n) {                             // q~ and dO of row block rb0 + n (one lane)
    const int z = b * a.T + (rb0 + n) * (kBwtRows / a.G);
    mbar_arrive_expect_tx(&sm.qfull, 2u * BwdTcSmem::kTile);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      tma_load_3d(sm.q + h * T16, &A.tm_q, 64 * h, g * a.G, z, &sm.qfull);
      tma_load_3d(sm.dout + h * T16, &A.tm_do, 64 * h, g * a.G, z, &sm.qfull);
    }
  };
  const int row0 = mem ? 0 : (int)(a.local_off[b] * a.Hkv + (int64_t)g * cap + k0);   // cache row of key k0
  if (warp == kBwtProducerWarp && lane == 0) {               // barriers, then K / V and the first block's rows
    mbar_init(&sm.kvfull, mem ? 4 : 1);                      // memory tiles: one arrive per gathering warp
    mbar_init(&sm.qfull, 1);
    mbar_init(&sm.sfull, 1);
    mbar_init(&sm.pready, kBwtSoftWarps);
    mbar_init(&sm.bdone, 1);
    mbar_init(&sm.dqempty, kBwtSoftWarps);
    mbar_init(&sm.ropefull, 1);
    fence_mbar_init();
    prefetch_tensormap_desc(&A.tm_q);
    prefetch_tensormap_desc(&A.tm_do);
    if (!mem) {                                              // local keys are consecutive cache rows
      mbar_arrive_expect_tx(&sm.kvfull, 2u * BwdTcSmem::kTile);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        tma_load_2d(sm.k + h * T16, &A.tm_k, 64 * h, row0, &sm.kvfull);
        tma_load_2d(sm.v + h * T16, &A.tm_v, 64 * h, row0, &sm.kvfull);
      }
    }
    issue_rows(0);
  }
  if (warp == kBwtMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&sm.tmem_slot)), "n"(kBwtTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  float l_next = INFINITY, d_next = 0.f;                     // this thread's row of the next block
  auto row_stats = [&](int rb) {
    const int r = rb * kBwtRows + tid;
    l_next = INFINITY;
    d_next = 0.f;
    if (r < a.R) {
      const int64_t i = ((int64_t)b * a.T + r / a.G) * a.Hq + g * a.G + r % a.G;
      l_next = a.lse[i] * kLog2e;
      d_next = a.drow[i];
    }
  };
  if (warp < 4) {
    // key row tid's source row (-1 past the tile's keys); a memory tile's
    // keys are gathered here, one thread per key, zero past its keys
    int64_t row = -1;
    if (tid < nk) {
      if (mem) {
        const int64_t m = k0 + tid;
        int r = 0;
        while (sm.mem_pref[r + 1] <= m) ++r;
        row = (sm.mem_c0[r] + (m - sm.mem_pref[r])) * a.Hkv + g;
      } else {
        row = (int64_t)row0 + tid;
      }
    }
    sm.krow[tid] = row;
    row_stats(rb0);
  }
  tc_fence_before();
  __syncthreads();                                           // barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = sm.tmem_slot;
  if (warp < 4 && mem) {
    const int64_t row = sm.krow[tid];
    const __nv_bfloat16* Kb = reinterpret_cast<const __nv_bfloat16*>(a.mem_k);
    const __nv_bfloat16* Vb = reinterpret_cast<const __nv_bfloat16*>(a.mem_v);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      if (row >= 0) {
        cp_async_16(sm.k + swz128(tid, c), Kb + row * D + 8 * c);
        cp_async_16(sm.v + swz128(tid, c), Vb + row * D + 8 * c);
      } else {
        *reinterpret_cast<uint4*>(sm.k + swz128(tid, c)) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(sm.v + swz128(tid, c)) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    cp_async_commit();
    cp_async_wait_group<0>();
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.kvfull);
  }

  if (warp == kBwtProducerWarp) {                            // ---- TMA producer: q~ and dO of each row block
    for (int n = 1; n < nb; ++n) {
      if (!mbar_wait_warp(&sm.bdone, (uint32_t)((n - 1) & 1))) break;   // the block before is done with them
      if (elect_one()) issue_rows(n);
      __syncwarp();
    }
    // the last boxes have landed before the CTA may leave
    mbar_wait_warp(&sm.qfull, (uint32_t)((nb - 1) & 1));
    if (!mem) mbar_wait_warp(&sm.kvfull, 0u);
  } else if (warp == kBwtMmaWarp) {                          // ---- MMA issuer (all lanes; one elected issues)
    constexpr uint32_t id_kk = umma_idesc_bf16(128);           // A, B K-major
    constexpr uint32_t id_kmn = umma_idesc_bf16_bmn(128);      // A K-major, B MN-major
    constexpr uint32_t id_mnmn = umma_idesc_bf16_amn_bmn(128); // A, B MN-major
    const uint32_t sk = smem_u32(sm.k), sv = smem_u32(sm.v), sq = smem_u32(sm.q), so = smem_u32(sm.dout);
    const uint32_t sp = smem_u32(sm.pt), sd = smem_u32(sm.dst);
    const bool kv_in = mbar_wait_warp(&sm.kvfull, 0u);
    for (int n = 0; n < nb && kv_in; ++n) {
      if (!mbar_wait_warp(&sm.qfull, (uint32_t)(n & 1))) break;
      if (n > 0 && !mbar_wait_warp(&sm.dqempty, (uint32_t)((n - 1) & 1))) break;   // dq~ of the block before is read
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {                     // K = 128 dims in steps of 16
          const uint32_t off = (uint32_t)((kk >> 2) * T16 + (kk & 3) * 32);
          umma_bf16(tmem, umma_sdesc(sk + off), umma_sdesc(sq + off), id_kk, kk > 0 ? 1u : 0u);
          umma_bf16(tmem + 128, umma_sdesc(sv + off), umma_sdesc(so + off), id_kk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sm.sfull);
      }
      __syncwarp();
      if (!mbar_wait_warp(&sm.pready, (uint32_t)(n & 1))) break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {                     // K = 128 rows in steps of 16
          const uint32_t offa = (uint32_t)((kk >> 2) * T16 + (kk & 3) * 32);
          const uint32_t offb = (uint32_t)(kk * 16 * 128);
          const uint32_t acc = (n > 0 || kk > 0) ? 1u : 0u;
          umma_bf16(tmem + 256, umma_sdesc(sp + offa), umma_sdesc_mn(so + offb, T16), id_kmn, acc);
          umma_bf16(tmem + 384, umma_sdesc(sd + offa), umma_sdesc_mn(sq + offb, T16), id_kmn, acc);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {                     // K = 128 keys in steps of 16
          const uint32_t off = (uint32_t)(kk * 16 * 128);
          umma_bf16(tmem, umma_sdesc_mn(sd + off, T16), umma_sdesc_mn(sk + off, T16), id_mnmn, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sm.bdone);
      }
      __syncwarp();
    }
  } else {                                                   // ---- softmax and epilogue: 8 warps
    // Warps w and w + 4 share TMEM lane quarter w % 4 (lane = key for S^T, dP^T,
    // dV, dK; = row for dq~) and split the 128 columns: half 0 takes columns
    // 0..63, half 1 columns 64..127.
    const int q4 = warp & 3, half = warp >> 2;
    const uint32_t tlane = (uint32_t)(q4 * 32) << 16;
    const int j = q4 * 32 + lane;                            // this thread's TMEM lane
    // rows of a block that see key j: r >= rmin (causal for local keys), r < R, and j < nk
    const int64_t rmin_all = mem ? 0 : (int64_t)a.G * (k0 + j - Lb);
    // fp32 rows of 512 bytes staged in shared memory (dV and dK), 16-byte
    // chunk c of row i at chunk c ^ (i mod 32): a warp's writes of one chunk of
    // 32 rows and its reads of one row both spread over all banks
    auto stage_row = [&](unsigned char* base, int i, int cb, const uint32_t (&o)[32], float mul) {
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<float4*>(base + i * 512 + (((8 * cb + c) ^ (i & 31)) << 4)) =
            make_float4(__uint_as_float(o[4 * c]) * mul, __uint_as_float(o[4 * c + 1]) * mul,
                        __uint_as_float(o[4 * c + 2]) * mul, __uint_as_float(o[4 * c + 3]) * mul);
    };
    auto staged = [&](const unsigned char* base, int i, int c) -> float4 {
      return *reinterpret_cast<const float4*>(base + i * 512 + ((c ^ (i & 31)) << 4));
    };
    // dq~ rows staged as four [128 rows][32 floats] tiles with the 128-byte
    // swizzle, the layout of the reduce-add's boxes (dims 32 cb ..)
    auto stage_tile = [&](unsigned char* base, int i, int cb, const uint32_t (&o)[32], float mul) {
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<float4*>(base + cb * 16384 + i * 128 + ((c ^ (i & 7)) << 4)) =
            make_float4(__uint_as_float(o[4 * c]) * mul, __uint_as_float(o[4 * c + 1]) * mul,
                        __uint_as_float(o[4 * c + 2]) * mul, __uint_as_float(o[4 * c + 3]) * mul);
    };
    unsigned char* st_a = sm.pt;                             // 64 KB: pt and dst
    unsigned char* st_b = sm.q;                              // 64 KB: q and dout
    // The softmax warps meet at named barrier 1 every block (the row
    // statistics are shared), so each give-up decision is taken by all of them.
    bool ok = true;
    for (int n = 0; n < nb && ok; ++n) {
      const int rb = rb0 + n, buf = n & 1;
      if (tid < kBwtRows) {
        sm.lse2[buf][tid] = l_next;
        sm.drow[buf][tid] = d_next;
        if (n + 1 < nb) row_stats(rb + 1);
      }
      const int64_t rmin = rmin_all - (int64_t)rb * kBwtRows;   // first visible row of this block
      const int rlo = j >= nk ? kBwtRows : (int)(rmin < 0 ? 0 : (rmin > kBwtRows ? kBwtRows : rmin));
      if (tid == 0 && n > 0) bulk_wait_read();               // the block before's dq~ reduce has read its staging
      // (the barrier also publishes the row statistics, and orders these
      // writes of P^T and dS^T after that read)
      if (!soft_and(mbar_wait_warp(&sm.sfull, (uint32_t)(n & 1)))) { ok = false; break; }
      tc_fence_after();
      if (n == 0 && j >= nk)                                 // rows past the tile's keys: zero for dq~ = dS K
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(sm.k + swz128(j, 8 * half + c)) = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {                       // rows 32 cb .. 32 cb + 31
        const int cb = 2 * half + cc;
        uint32_t sr[32], dp[32];
        tmem_ld32_issue(tmem + tlane + (uint32_t)(32 * cb), sr);
        tmem_ld32_issue(tmem + tlane + 128u + (uint32_t)(32 * cb), dp);
        tmem_wait_tie(sr);
        reg_tie(dp);
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {                     // 8 rows = one 16-byte chunk of P^T and dS^T
          uint32_t pw[4], dw[4];
          float l8[8], d8[8];                                // the 8 rows' statistics, two 16-byte loads each
          *reinterpret_cast<float4*>(l8) = *reinterpret_cast<const float4*>(&sm.lse2[buf][32 * cb + 8 * c8]);
          *reinterpret_cast<float4*>(l8 + 4) = *reinterpret_cast<const float4*>(&sm.lse2[buf][32 * cb + 8 * c8 + 4]);
          *reinterpret_cast<float4*>(d8) = *reinterpret_cast<const float4*>(&sm.drow[buf][32 * cb + 8 * c8]);
          *reinterpret_cast<float4*>(d8 + 4) = *reinterpret_cast<const float4*>(&sm.drow[buf][32 * cb + 8 * c8 + 4]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float p2[2], d2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int c = 8 * c8 + 2 * e + u, rr = 32 * cb + c;
              const bool vis = rr >= rlo;
              const float p = vis ? ex2_approx(fmaf(__uint_as_float(sr[c]), a.scale_log2, -l8[2 * e + u])) : 0.f;
              p2[u] = p;
              d2[u] = vis ? p * (__uint_as_float(dp[c]) - d8[2 * e + u]) : 0.f;
            }
            pw[e] = pack_bf16(p2[0], p2[1]);
            dw[e] = pack_bf16(d2[0], d2[1]);
          }
          const uint32_t off = swz128(j, 4 * cb + c8);
          *reinterpret_cast<uint4*>(sm.pt + off) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
          *reinterpret_cast<uint4*>(sm.dst + off) = make_uint4(dw[0], dw[1], dw[2], dw[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.pready);
      // dq~ of the block (lane = row), staged over P^T / dS^T (free once the
      // block's products are done), then added to the rotated-frame gradient
      // by four tile reduce-adds (rows past R add zeros)
      if (!soft_and(mbar_wait_warp(&sm.bdone, (uint32_t)(n & 1)))) { ok = false; break; }
      tc_fence_after();
      if (tid == 0 && n == nb - 1 && !mem) {                 // K / V are read: the tile's rotary rows over them
        mbar_arrive_expect_tx(&sm.ropefull, (uint32_t)nk * 512u);
        tma_load_1d(sm.k, a.rope + (a.top_k + k0) * H, (uint32_t)nk * 512u, &sm.ropefull);
      }
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int cb = 2 * half + cc;
        uint32_t o[32];
        tmem_ld32_issue(tmem + tlane + (uint32_t)(32 * cb), o);
        tmem_wait_tie(o);
        stage_tile(st_a, j, cb, o, a.scale);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.dqempty);               // TMEM columns 0..127 are free
      soft_bar();
      if (tid == 0) {
        const int z = b * a.T + rb * (kBwtRows / a.G);
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) tma_reduce_add_3d(&A.tm_dq, 32 * cb, g * a.G, z, st_a + cb * 16384);
        bulk_commit();
      }
    }
    // ---- dV and dK (complete with the last block's products): lane j
    // stages key j's rows, then each warp stores or adds whole rows; a local
    // key's dK goes back to its unrotated frame, dims i and i + 64 held by
    // lanes l and l + 16.  The TMEM loads run in every lane (.sync.aligned).
    if (tid == 0) bulk_wait_read();                          // the last dq~ reduce has read st_a
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int cb = 2 * half + cc;
        uint32_t o[32];
        tmem_ld32_issue(tmem + tlane + 256u + (uint32_t)(32 * cb), o);
        tmem_wait_tie(o);
        stage_row(st_b, j, cb, o, 1.f);
      }
      soft_bar();                                            // st_a is free
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int cb = 2 * half + cc;
        uint32_t o[32];
        tmem_ld32_issue(tmem + tlane + 384u + (uint32_t)(32 * cb), o);
        tmem_wait_tie(o);
        stage_row(st_a, j, cb, o, a.scale);
      }
      const bool rope_in = mem || mbar_wait_warp(&sm.ropefull, 0u);   // the same in every lane (shuffles below)
      soft_bar();
      const int i4 = 4 * (lane & 15);                        // this lane's first dim within its half
      for (int kk = warp; kk < nk && rope_in; kk += kBwtSoftWarps) {
        const int64_t row = sm.krow[kk];
        const float4 dv = staged(st_b, kk, lane);
        const float4 dk = staged(st_a, kk, lane);
        if (mem) {                                           // memory keys are pooled, not rotated here
          atomicAdd(reinterpret_cast<float4*>(a.dmem_v + row * D) + lane, dv);
          atomicAdd(reinterpret_cast<float4*>(a.dmem_k + row * D) + lane, dk);
        } else {
          reinterpret_cast<float4*>(a.dlv + row * D)[lane] = dv;
          float4 pk;                                         // the partner dims (i + 64 or i - 64)
          pk.x = __shfl_xor_sync(0xffffffffu, dk.x, 16);
          pk.y = __shfl_xor_sync(0xffffffffu, dk.y, 16);
          pk.z = __shfl_xor_sync(0xffffffffu, dk.z, 16);
          pk.w = __shfl_xor_sync(0xffffffffu, dk.w, 16);
          // (cos, sin) of dims i4 .. i4 + 3 of key kk's position, from the staged rotary rows
          const float4* cs4 = reinterpret_cast<const float4*>(sm.k + kk * 512 + i4 * 8);
          const float4 c01 = cs4[0], c23 = cs4[1];
          const float cs[4] = {c01.x, c01.z, c23.x, c23.z}, sn[4] = {c01.y, c01.w, c23.y, c23.w};
          const float own[4] = {dk.x, dk.y, dk.z, dk.w}, par[4] = {pk.x, pk.y, pk.z, pk.w};
          float res[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)                        // y0 = dim i, y1 = dim i + 64
            res[e] = lane < 16 ? own[e] * cs[e] + par[e] * sn[e] : own[e] * cs[e] - par[e] * sn[e];
          reinterpret_cast<float4*>(a.dlk + row * D)[lane] = make_float4(res[0], res[1], res[2], res[3]);
        }
      }
    }
    if (tid == 0) bulk_wait_all();                           // the reduce-adds are complete before the CTA leaves
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kBwtMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(kBwtTmemCols) : "memory");
  }
}

}  // namespace msa
