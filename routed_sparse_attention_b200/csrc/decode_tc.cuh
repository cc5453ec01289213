// Stage 3 kernel for many query rows per kv head (bf16 banks, head_dim 128):
// split-K GQA decode on the 5th-generation tensor cores.
//
// Method: "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts",
// section "How MSA compresses and routes documents", and "EverMind Releases
// Memory-Sparse Attention Code for Long-Context AI Models", section
// "Architectural Design and Inference" (stage 3): attention of the query over
// [pooled K/V of the Top-k documents ++ local K/V], global RoPE offset k.
//
// With T query tokens a kv head has G * T query rows (256 at T = 64, G = 4):
// enough for the MMA's M = 128.  A CTA owns 128 rows of one kv head (row r =
// t * G + h_in_group) and one split of keys -- split 0 the selected
// documents' pooled keys, the others runs of local keys -- and per 64-key
// tile computes
//   S = Q K^T   (M = 128 rows, N = 64 keys, K = 128 dims) into TMEM,
//   the online softmax of each row in the thread that owns its TMEM lane,
//   O += P V    (M = 128 rows, N = 128 dims, K = 64 keys) into TMEM,
// with P written to shared memory in bf16.  Q (rotated at top_k + L_b + t)
// and the K tiles are K-major operands; V tiles, rows of keys as TMA or the
// memory gather leave them, are the MN-major B operand of P V (two 64-dim
// atoms 8 KB apart, 8-key groups 1 KB apart).  The split's partial (reference
// max, sum, unnormalised output) goes to the split plan's workspace;
// decode_tc_merge_kernel, launched right after (programmatic dependent
// launch), merges the splits of 4 rows per CTA.  The query rows (one TMA
// box of 128 / G tokens x G heads) and their rotary rows (a bulk copy) land
// in shared memory and are rotated there.
//
// Roles:
//   warps 0-7     : two softmax warpgroups; warpgroup w takes the tiles t with
//                   t % 2 == w and keeps its own (max, sum) per row and its
//                   own O in TMEM, so that one group's softmax overlaps the
//                   other's; thread i of a group = row i = TMEM lane i.  They
//                   also rotate Q into shared memory and, for the memory
//                   split, gather its tiles with cp.async; at the end group 0
//                   merges the two groups' partials of each row.
//   warp 8 lane 0 : TMA producer of the local K/V stage ring
//   warp 9        : TMEM allocation; lane 0 issues tcgen05.mma and commits
// Pipeline: S(t) goes to TMEM buffer t % 4 and is issued two tiles ahead,
// once its K/V stage has landed: S(0), S(1), then P V(u) after S(u + 2) for
// u = 0, 1, ...  P V(u) waits for the softmax of tile u to write P into its
// group's buffer.  The softmax moves each row's reference maximum lazily
// (when a score exceeds it by 2^8) and rescales that row's O in TMEM only
// then, after the group's previous P V has completed.  Every wait is bounded
// (mbar_wait); a timeout flags MSA_DEV_PIPE_TIMEOUT.
#pragma once
#include "decode_mma.cuh"
#include "route_mma.cuh"

namespace msa {

constexpr int kTcRows = 128;             // query rows per CTA (MMA M)
constexpr int kTcGroups = 2;             // softmax warpgroups
constexpr int kTcSoftWarps = 4 * kTcGroups;
constexpr int kTcProducerWarp = kTcSoftWarps;
constexpr int kTcMmaWarp = kTcSoftWarps + 1;
constexpr int kTcThreads = (kTcSoftWarps + 2) * 32;
constexpr int kTcStages = 4;             // K/V stages of 64 keys
constexpr int kTcSBufs = 4;              // S buffers of 64 columns
constexpr int kTcTmemCols = 512;         // S: 4 x 64 columns, then O of group 0 and of group 1: 128 each
constexpr int kTcOCol = kTcSBufs * 64;
constexpr int kTcMaxTok = 32;            // query tokens of a CTA's 128 rows (G >= 4)
constexpr int kTcMergeRows = 4;          // rows per CTA of the split merge: one item per thread,
                                         // few registers, so its CTAs fit beside a decode CTA

struct DecTcSmem {                       // head_dim 128
  unsigned char q[2][kTcRows * 128];            // rotated Q, K-major: [dim half][row][64 dims]
  unsigned char kv[kTcStages][2][2][64 * 128];  // [stage][K, V][dim half][64 keys x 64 dims]
  unsigned char p[kTcGroups][kTcRows * 128];    // P in bf16, K-major: [group][row][64 keys]; first the raw Q rows
  float2 rope_rows[kTcMaxTok][64];              // (cos, sin) of the CTA's query positions
  float2 ml1[kTcRows];                          // group 1's (reference max, sum) per row, for the merge
  uint64_t kvfull[kTcStages], kvempty[kTcStages];
  uint64_t qfull;
  uint64_t sfull[kTcSBufs], sempty[kTcSBufs];
  uint64_t pready[kTcGroups], pvdone[kTcGroups];
  uint64_t odone;
  int64_t mem_pref[kMaxTopKDecode + 1];
  int64_t mem_krow[kMaxTopKDecode];
  int64_t mem_vrow[kMaxTopKDecode];
  int64_t key_krow[kTcGroups][kDecTile];        // source rows of the memory tile a group gathers
  int64_t key_vrow[kTcGroups][kDecTile];
  uint32_t tmem_slot;
};

// Instruction descriptor, kind::f16: bf16 A (K-major) and B (MN-major), fp32
// D, M = 128, N = n.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_bmn(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
// Shared-memory descriptor of an MN-major operand, 128-byte swizzle: atoms of
// 64 elements (128 B) x 8 K-rows (1 KB); lbo bytes between atoms along MN,
// 1 KB between 8-row groups along K.
__device__ __forceinline__ uint64_t umma_sdesc_mn(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)((lbo >> 4) & 0x3fffu) << 16) |
         ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void prefetch_tensormap_desc(const CUtensorMap* tm) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm)) : "memory");
}
// Barrier of one softmax warpgroup's 128 threads (named barrier 1 + group)
// that also ANDs `pred` over them, so that they leave a loop together.
__device__ __forceinline__ bool group_sync_and(int grp, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred q, d;\n setp.ne.u32 q, %2, 0;\n bar.red.and.pred d, %1, 128, q;\n"
      " selp.u32 %0, 1, 0, d;\n}\n"
      : "=r"(r) : "r"(1 + grp), "r"((uint32_t)pred) : "memory");
  return r != 0;
}
__device__ __forceinline__ void group_sync(int grp) { asm volatile("bar.sync %0, 128;" ::"r"(1 + grp) : "memory"); }
// Generic-proxy writes to shared memory become visible to the tensor core's
// (async proxy) reads.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// True in one lane of the (converged) warp.
__device__ __forceinline__ bool elect_one() {
  uint32_t e;
  asm volatile("{\n .reg .pred p;\n elect.sync _|p, 0xffffffff;\n selp.u32 %0, 1, 0, p;\n}\n" : "=r"(e));
  return e != 0;
}
// 2^x by the SFU's ex2.approx (flush-to-zero): -inf gives +0; relative error
// about 2^-22, far below the bf16 rounding P takes next.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(kTcThreads, 1)
decode_tc_kernel(const __grid_constant__ DecodeMmaArgs A) {
  constexpr int D = 128, HALF = 64, NS = kTcStages, NB = kTcSBufs;
  const DecodeArgs& a = A.d;
  extern __shared__ unsigned char smem_raw[];
  DecTcSmem& sm = *reinterpret_cast<DecTcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int b = 0;
  while (b + 1 < a.B && a.split_off[b + 1] <= (int)blockIdx.x) ++b;
  const int s = blockIdx.x - a.split_off[b];
  const int g = blockIdx.y / a.n_rg, rg = blockIdx.y % a.n_rg;
  const int64_t cap = a.local_off[b + 1] - a.local_off[b];
  const int64_t Ltot = live_len(a, b);
  const int64_t Lb = Ltot - a.T;
  const int k = a.top_k;
  const bool mem = (s == 0);
  int doc = 0;
  if (mem && threadIdx.x < k) doc = __ldg(a.sel + (int64_t)b * k + threadIdx.x);
  const int64_t j_lo = mem ? 0 : (int64_t)(s - 1) * a.S;
  int64_t nkeys = mem ? 0 : min64(a.S, Ltot - j_lo);
  if (nkeys < 0) nkeys = 0;
  const int row0 = (int)(a.local_off[b] * a.Hkv + (int64_t)g * cap + j_lo);    // tensor-map row of key j_lo
  const int nrow = min(kTcRows, a.R - rg * kTcRows);
  pdl_trigger();                                             // the merge kernel may launch; it waits for this grid

  auto issue_local = [&](int t) {                            // producer lane only
    const int st = t % NS;
    mbar_arrive_expect_tx(&sm.kvfull[st], 4 * 64 * 128);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      tma_load_2d(&sm.kv[st][0][h][0], &A.tm_k, 64 * h, row0 + t * kDecTile, &sm.kvfull[st]);
      tma_load_2d(&sm.kv[st][1][h][0], &A.tm_v, 64 * h, row0 + t * kDecTile, &sm.kvfull[st]);
    }
  };
  // query tokens of this CTA's rows: [t0, t0 + ntok), G heads each, contiguous
  const int t0 = rg * kTcRows / a.G, ntok = (nrow + a.G - 1) / a.G;
  int ntiles = (int)((nkeys + kDecTile - 1) / kDecTile);    // the memory split's count follows its set-up

  // ---- set-up.  The producer lane initialises the barriers and at once
  // issues the raw query rows, their rotary rows and a local split's first
  // stages; meanwhile warp 9 allocates TMEM and a memory split finds its key count.
  if (warp == kTcProducerWarp && lane == 0) {
    for (int st = 0; st < NS; ++st) {
      mbar_init(&sm.kvfull[st], mem ? 4 : 1);              // memory tiles: one arrive per warp of the gathering group
      mbar_init(&sm.kvempty[st], 1);
    }
    for (int j = 0; j < NB; ++j) {
      mbar_init(&sm.sfull[j], 1);
      mbar_init(&sm.sempty[j], 4);
    }
    for (int j = 0; j < kTcGroups; ++j) {
      mbar_init(&sm.pready[j], 4);
      mbar_init(&sm.pvdone[j], 1);
    }
    mbar_init(&sm.odone, 1);
    mbar_init(&sm.qfull, 1);
    fence_mbar_init();
    // one box of 128 / G tokens x G heads x 128 dims = rows i = tt * G + h of
    // 256 bytes; tokens past the query's (rows i >= nrow) are never used
    mbar_arrive_expect_tx(&sm.qfull, (uint32_t)(kTcRows * D * 2 + ntok * HALF * 8));
    prefetch_tensormap_desc(&A.tm_q);
    tma_load_3d(&sm.p[0][0], &A.tm_q, 0, g * a.G, b * a.T + t0, &sm.qfull);
    tma_load_1d(&sm.rope_rows[0][0], a.rope + ((int64_t)k + Lb + t0) * HALF, (uint32_t)ntok * HALF * 8, &sm.qfull);
    if (!mem) {
      prefetch_tensormap_desc(&A.tm_k);
      prefetch_tensormap_desc(&A.tm_v);
      for (int t = 0; t < ntiles && t < NS; ++t) issue_local(t);
    }
  }
  if (warp == kTcMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&sm.tmem_slot)), "n"(kTcTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (mem) dec_mem_setup(a, b, k, doc, sm.mem_pref, sm.mem_krow, sm.mem_vrow);   // CTA barriers inside
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_slot;
  if (mem) {
    nkeys = sm.mem_pref[k];
    ntiles = (int)((nkeys + kDecTile - 1) / kDecTile);
  }

  // the memory split's tile t: cp.async by the 128 threads of group grp into stage t % NS
  auto mem_tile = [&](int grp, int tid, int t) {
    dec_mem_rows(tid, t, 0, nkeys, k, sm.mem_pref, sm.mem_krow, sm.mem_vrow, sm.key_krow[grp], sm.key_vrow[grp]);
    group_sync(grp);
    const int st = t % NS;
    dec_mem_gather<D>(tid, a, g, t, 0, nkeys, sm.key_krow[grp], sm.key_vrow[grp], &sm.kv[st][0][0][0],
                      &sm.kv[st][1][0][0]);
    cp_async_wait_group<0>();
    fence_proxy_async_smem();
    group_sync(grp);                                         // rows of the group's next tile may be rewritten
    if (lane == 0) mbar_arrive(&sm.kvfull[st]);
  };

  if (warp < kTcSoftWarps) {                                 // ---- softmax warps: Q, first memory tiles
    const int grp = warp >> 2, i = threadIdx.x & (kTcRows - 1);
    const int r = rg * kTcRows + i;
    const bool real = i < nrow;
    // rotated query row i (zero past the real rows), K-major with the 128-byte
    // swizzle, from the raw row and its rotary row in shared memory; group w
    // takes dims 32w .. 32w+31 and their partners + 64
    {
      const bool arrived = mbar_wait(&sm.qfull, 0u);
      const unsigned char* raw = &sm.p[0][0] + (size_t)i * D * 2;
      const float2* cs = sm.rope_rows[real ? r / a.G - t0 : 0];
#pragma unroll 2
      for (int j = 4 * grp; j < 4 * grp + 4; ++j) {         // dims 8j .. 8j+7
        uint32_t lo[4], hi[4];
        if (real && arrived) {
          float x0[8], x1[8];
          Elem<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(raw + 16 * j), x0);
          Elem<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(raw + 2 * HALF + 16 * j), x1);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float4 w = *reinterpret_cast<const float4*>(cs + 8 * j + 2 * e);   // (cos, sin) of 2 dims
            const float l0 = x0[2 * e] * w.x - x1[2 * e] * w.y, h0 = x1[2 * e] * w.x + x0[2 * e] * w.y;
            const float l1 = x0[2 * e + 1] * w.z - x1[2 * e + 1] * w.w, h1 = x1[2 * e + 1] * w.z + x0[2 * e + 1] * w.w;
            lo[e] = pack_bf16(l0, l1);
            hi[e] = pack_bf16(h0, h1);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) lo[e] = hi[e] = 0u;
        }
        const uint32_t off = (uint32_t)(i * 128 + (((j ^ (i & 7))) << 4));
        *reinterpret_cast<uint4*>(&sm.q[0][off]) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        *reinterpret_cast<uint4*>(&sm.q[1][off]) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      }
    }
    fence_proxy_async_smem();
    // every raw Q row is read before P overwrites it
    asm volatile("bar.sync 3, %0;" ::"n"(kTcSoftWarps * 32) : "memory");
    if (mem)                                                 // the group's first memory tiles
      for (int t = grp; t < ntiles && t < NS; t += kTcGroups) mem_tile(grp, i, t);
  }
  __syncthreads();                                           // Q and the first stages' copies in place

  // The producer and MMA warps run their loops with all 32 lanes, so that the
  // control flow and the operands (stage addresses, descriptors) stay
  // warp-uniform; one elected lane issues each copy or tensor-core instruction.
  if (warp == kTcProducerWarp) {                             // ---- TMA producer: the remaining stages
    if (!mem) {
      int issued = min(ntiles, NS);
      for (int t = NS; t < ntiles; ++t) {
        if (!mbar_wait_warp(&sm.kvempty[t % NS], (uint32_t)(((t / NS) - 1) & 1))) break;
        if (elect_one()) issue_local(t);
        __syncwarp();
        issued = t + 1;
      }
      // the last stages' copies land before the CTA may leave
      for (int t = issued > NS ? issued - NS : 0; t < issued; ++t)
        mbar_wait_warp(&sm.kvfull[t % NS], (uint32_t)((t / NS) & 1));
    }
  } else if (warp == kTcMmaWarp) {                           // ---- MMA issuer
    constexpr uint32_t idesc_s = umma_idesc_bf16(64);
    constexpr uint32_t idesc_o = umma_idesc_bf16_bmn(128);
    const uint32_t sq = smem_u32(&sm.q[0][0]);
    auto qk = [&](int t) -> bool {                           // S(t) = Q K(t)^T into buffer t % NB
      const int st = t % NS, sb = t % NB;
      if (!mbar_wait_warp(&sm.kvfull[st], (uint32_t)((t / NS) & 1))) return false;
      if (t >= NB && !mbar_wait_warp(&sm.sempty[sb], (uint32_t)(((t / NB) - 1) & 1))) return false;
      tc_fence_after();
      const uint32_t sk = smem_u32(&sm.kv[st][0][0][0]);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {                     // K = 128 dims in steps of 16
          const uint32_t off = (uint32_t)((kk >> 2) * (64 * 128) + (kk & 3) * 32);
          const uint32_t offq = (uint32_t)((kk >> 2) * (kTcRows * 128) + (kk & 3) * 32);
          umma_bf16(tmem + (uint32_t)(sb * 64), umma_sdesc(sq + offq), umma_sdesc(sk + off), idesc_s,
                    kk > 0 ? 1u : 0u);
        }
        umma_commit(&sm.sfull[sb]);
      }
      __syncwarp();
      return true;
    };
    auto pv = [&](int u) -> bool {                           // O(u % 2) += P(u) V(u)
      const int grp = u & 1, st = u % NS;
      if (!mbar_wait_warp(&sm.pready[grp], (uint32_t)((u >> 1) & 1))) return false;
      tc_fence_after();
      const uint32_t sp = smem_u32(&sm.p[grp][0]), sv = smem_u32(&sm.kv[st][1][0][0]);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)                       // K = 64 keys in steps of 16
          umma_bf16(tmem + kTcOCol + (uint32_t)(grp * 128), umma_sdesc(sp + kk * 32),
                    umma_sdesc_mn(sv + kk * 2048, 64 * 128), idesc_o, (u >= kTcGroups || kk > 0) ? 1u : 0u);
        umma_commit(&sm.pvdone[grp]);
        umma_commit(&sm.kvempty[st]);
      }
      __syncwarp();
      return true;
    };
    bool ok = true;
    for (int t = 0; t < ntiles && t < 2 && ok; ++t) ok = qk(t);
    for (int u = 0; u < ntiles && ok; ++u) {
      if (u + 2 < ntiles && !qk(u + 2)) { ok = false; break; }
      ok = pv(u);
    }
    if (ok && ntiles > 0 && elect_one()) umma_commit(&sm.odone);   // every product above is complete
    __syncwarp();
  } else {                                                   // ---- softmax and epilogue: group grp, row i
    const int grp = warp >> 2, i = threadIdx.x & (kTcRows - 1);
    const int r = rg * kTcRows + i;
    const bool real = i < nrow;
    const int t_q = real ? r / a.G : 0;
    const int64_t last = Lb + t_q - j_lo;
    const int lim = !real ? -1 : (mem ? INT_MAX : (last < 0 ? -1 : (int)min64(last, INT_MAX)));
    const uint32_t tlane = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t ocol = kTcOCol + (uint32_t)(grp * 128);
    unsigned char* prow = &sm.p[grp][0];
    float mref = -INFINITY, lsum = 0.f;
    bool ok = true;
    for (int t = grp, n = 0; t < ntiles && ok; t += kTcGroups, ++n) {   // n-th tile of the group
      const int sb = t % NB;
      const int n_t = (int)min64(kDecTile, nkeys - (int64_t)t * kDecTile);
      // a memory split's group meets at named barriers inside this loop, so
      // its warps take every give-up decision together (a warp that left alone
      // would leave the others at a barrier); local splits' warps decide alone
      bool got = mbar_wait_warp(&sm.sfull[sb], (uint32_t)((t / NB) & 1));
      if (mem) got = group_sync_and(grp, got);
      if (!got) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32_issue(tmem + tlane + (uint32_t)(sb * 64), sr[0]);
      tmem_ld32_issue(tmem + tlane + (uint32_t)(sb * 64 + 32), sr[1]);
      tmem_wait_tie(sr[0]);
      reg_tie(sr[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.sempty[sb]);            // S buffer sb may be overwritten
      // keys [0, nvis) of the tile are visible to row i (in the tile, and causal for local keys)
      const int64_t kt = (int64_t)t * kDecTile;
      const int64_t vis_rem = (int64_t)lim - kt + 1;
      const int nvis = vis_rem <= 0 ? 0 : (int)min64((int64_t)n_t, vis_rem);
      if (!__all_sync(0xffffffffu, nvis == kDecTile)) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= nvis) sr[c >> 5][c & 31] = __float_as_uint(-INFINITY);
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < 64; ++c) mx4[c & 3] = fmaxf(mx4[c & 3], __uint_as_float(sr[c >> 5][c & 31]));
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * a.scale_log2;   // the scale is positive
      // lazy reference maximum; O (in TMEM) is rescaled when it moves after the group's first tile
      const bool move = mx > mref + kLazyRescale;
      const float sc = move ? ex2_approx(mref - mx) : 1.f;   // mref = -inf gives 0
      // the group's previous P V is done before its O is rescaled or its P buffer rewritten
      if (n > 0) {
        got = mbar_wait_warp(&sm.pvdone[grp], (uint32_t)((n - 1) & 1));
        if (mem) got = group_sync_and(grp, got);
        if (!got) { ok = false; break; }
      }
      if (n > 0 && __any_sync(0xffffffffu, move)) {
        tc_fence_after();
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
          uint32_t o[32];
          tmem_ld32_issue(tmem + tlane + ocol + (uint32_t)(32 * cb), o);
          tmem_wait_tie(o);
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * sc);
          tmem_st32(tmem + tlane + ocol + (uint32_t)(32 * cb), o);
        }
        tmem_st_wait();
      }
      if (move) {
        lsum *= sc;
        mref = mx;
      }
      // P(t) in bf16; V rows past the tile's keys zeroed (their values may be
      // anything), so P V sees 0 x 0.  p = 2^(s * scale - mref): a hidden
      // key's -inf gives 0; a row with no visible key yet (mref = -inf)
      // subtracts 0 instead, all its p being 0.
      const float nm = mref == -INFINITY ? 0.f : -mref;
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 8 * j + 2 * e;
          const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c >> 5][c & 31]), a.scale_log2, nm));
          const float p1 = ex2_approx(fmaf(__uint_as_float(sr[(c + 1) >> 5][(c + 1) & 31]), a.scale_log2, nm));
          l4[e] += p0 + p1;
          w4[e] = pack_bf16(p0, p1);
        }
        *reinterpret_cast<uint4*>(prow + i * 128 + (((j ^ (i & 7))) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      lsum += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      if (n_t < kDecTile) {                                  // stage t % NS: V rows n_t .. 63 to zero
        unsigned char* vt = &sm.kv[t % NS][1][0][0];
        for (int idx = i; idx < (kDecTile - n_t) * 16; idx += kTcRows) {
          const int row = n_t + idx / 16, c = idx % 16;      // 16-byte chunk c of the row (two halves)
          *reinterpret_cast<uint4*>(vt + swz(row, c)) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.pready[grp]);
      if (mem && t + NS < ntiles) {                          // the memory split's tile t + NS into this stage
        if (!group_sync_and(grp, mbar_wait_warp(&sm.kvempty[t % NS], (uint32_t)((t / NS) & 1)))) { ok = false; break; }
        mem_tile(grp, i, t + NS);
      }
    }
    // ---- this split's partial: (reference max, sum) and the unnormalised O
    // rows.  Group 1 hands its (max, sum) to group 0, which merges the two
    // groups' O rows out of TMEM (group 1's only when it had a tile) and stages
    // them in the K/V ring (idle once the last P V is done), so that each warp
    // then stores whole 512-byte rows.  Row i's 16-byte chunk c sits at chunk
    // c ^ (i mod 32): a warp's writes of one chunk and its reads of one row
    // both spread over all banks.
    const bool have = ok && ntiles > 0 && mbar_wait_warp(&sm.odone, 0u);
    if (grp == 1) sm.ml1[i] = make_float2(have ? mref : -INFINITY, have ? lsum : 0.f);
    asm volatile("bar.sync 3, %0;" ::"n"(kTcSoftWarps * 32) : "memory");
    const int64_t prow0 = ((int64_t)(a.split_off[b] + s) * a.Hkv + g) * a.R + rg * kTcRows;
    unsigned char* ost = &sm.kv[0][0][0][0];
    if (grp == 0) {
      if (have) tc_fence_after();
      // `two` (group 1 had a tile) is the same for the whole warp, as the
      // .sync.aligned TMEM loads under it need; whether group 1 saw a key is
      // per row and only picks the weight (its O row is then not read at all)
      const float2 m1 = sm.ml1[i];
      const bool two = have && ntiles > 1;
      const bool use1 = two && m1.x != -INFINITY;
      const float m0 = have ? mref : -INFINITY;
      const float mt = fmaxf(m0, use1 ? m1.x : -INFINITY);
      const float w0 = m0 == -INFINITY ? 0.f : ex2_approx(m0 - mt);
      const float w1 = use1 ? ex2_approx(m1.x - mt) : 0.f;
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        uint32_t o[32], o1[32];
        if (have) {
          tmem_ld32_issue(tmem + tlane + kTcOCol + (uint32_t)(32 * cb), o);
          if (two) {
            tmem_ld32_issue(tmem + tlane + kTcOCol + 128u + (uint32_t)(32 * cb), o1);
            tmem_wait_tie(o1);
          }
          tmem_wait_tie(o);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            o[c] = __float_as_uint(use1 ? fmaf(__uint_as_float(o1[c]), w1, __uint_as_float(o[c]) * w0)
                                        : __uint_as_float(o[c]) * w0);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(ost + i * 512 + (((8 * cb + c) ^ (i & 31)) << 4)) =
              make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
      }
      const float lt = have ? lsum * w0 + (use1 ? m1.y * w1 : 0.f) : 0.f;
      if (real) reinterpret_cast<float2*>(a.part_ml)[prow0 + i] = make_float2(have ? mt : -INFINITY, lt);
    }
    asm volatile("bar.sync 3, %0;" ::"n"(kTcSoftWarps * 32) : "memory");
    for (int rr = warp; rr < nrow; rr += kTcSoftWarps)
      reinterpret_cast<uint4*>(a.part_o + (prow0 + rr) * D)[lane] =
          *reinterpret_cast<const uint4*>(ost + rr * 512 + ((lane ^ (rr & 31)) << 4));
  }

  // ---- teardown (decode_tc_merge_kernel merges the splits)
  tc_fence_before();
  __syncthreads();
  if (warp == kTcMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(kTcTmemCols) : "memory");
  }
}

// The splits of decode_tc_kernel merged into the output: one CTA per 4 rows
// of a (query, kv head, row group), one item (row, 4 dims) per thread with
// all its loads in flight at once.
__global__ void __launch_bounds__(kMmaThreads) decode_tc_merge_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int PER = kTcRows / kTcMergeRows;
  int idx = blockIdx.x;
  const int c = idx % PER;
  idx /= PER;
  const int rg = idx % a.n_rg;
  idx /= a.n_rg;
  const int g = idx % a.Hkv, b = idx / a.Hkv;
  const int r0 = rg * kTcRows + c * kTcMergeRows;
  const int nrow = min(kTcMergeRows, a.R - r0);
  // the split table is the host's, not the decode's: read it while the decode runs
  const int sfirst = a.split_off[b], nsplit = a.split_off[b + 1] - sfirst;
  pdl_wait();                                                // every split's partial is written
  if (nrow <= 0) return;
  merge_splits<128, kTcMergeRows * 32 / kMmaThreads, 8>(a, b, g, r0, nrow, sfirst, nsplit);
}

}  // namespace msa
