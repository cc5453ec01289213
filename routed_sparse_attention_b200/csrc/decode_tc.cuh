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
// launch), merges the splits of 16 rows per CTA.  The query rows (G per
// token, contiguous) and their rotary rows arrive by bulk copies into shared
// memory and are rotated there.
//
// Roles:
//   warps 0-3     : softmax and epilogue, thread i = row i = TMEM lane i; they
//                   also rotate Q into shared memory and, for the memory
//                   split, gather its tiles with cp.async
//   warp 4 lane 0 : TMA producer of the local K/V stage ring
//   warp 5        : TMEM allocation; lane 0 issues tcgen05.mma and commits
// Pipeline per tile t: S(t) is issued as soon as its K/V stage has landed and
// the S buffer t % 2 is free; P V of tile t - 1 follows once the softmax of
// t - 1 has written P.  The softmax moves each row's reference maximum
// lazily (when a score exceeds it by 2^8) and rescales that row's O in TMEM
// only then, after the previous P V has completed.  Every wait is bounded
// (mbar_wait); a timeout flags MSA_DEV_PIPE_TIMEOUT.
#pragma once
#include "decode_mma.cuh"
#include "route_mma.cuh"

namespace msa {

constexpr int kTcRows = 128;             // query rows per CTA (MMA M)
constexpr int kTcSoftWarps = 4;
constexpr int kTcProducerWarp = 4;
constexpr int kTcMmaWarp = 5;
constexpr int kTcThreads = 6 * 32;
constexpr int kTcStages = 4;             // K/V stages of 64 keys
constexpr int kTcTmemCols = 256;         // S: 2 x 64 columns, then O: 128 columns
constexpr int kTcOCol = 128;
constexpr int kTcMaxTok = 32;            // query tokens of a CTA's 128 rows (G >= 4)
constexpr int kTcMergeRows = 16;         // rows per CTA of the split merge

struct DecTcSmem {                       // head_dim 128
  unsigned char q[2][kTcRows * 128];            // rotated Q, K-major: [dim half][row][64 dims]
  unsigned char kv[kTcStages][2][2][64 * 128];  // [stage][K, V][dim half][64 keys x 64 dims]
  unsigned char p[2][kTcRows * 128];            // P in bf16, K-major: [buffer][row][64 keys]; first the raw Q rows
  float2 rope_rows[kTcMaxTok][64];              // (cos, sin) of the CTA's query positions
  uint64_t kvfull[kTcStages], kvempty[kTcStages];
  uint64_t qfull;
  uint64_t sfull[2], sempty[2], pready[2], pvdone[2];
  uint64_t odone;
  int64_t mem_pref[kMaxTopKDecode + 1];
  int64_t mem_krow[kMaxTopKDecode];
  int64_t mem_vrow[kMaxTopKDecode];
  int64_t key_krow[kDecTile];
  int64_t key_vrow[kDecTile];
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
// Barrier of the 128 softmax threads (named barrier 1) that also ANDs `pred`
// over them, so that they leave a loop together.
__device__ __forceinline__ bool soft_sync_and(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred q, d;\n setp.ne.u32 q, %1, 0;\n bar.red.and.pred d, 1, 128, q;\n"
      " selp.u32 %0, 1, 0, d;\n}\n"
      : "=r"(r) : "r"((uint32_t)pred) : "memory");
  return r != 0;
}
// Generic-proxy writes to shared memory become visible to the tensor core's
// (async proxy) reads.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__global__ void __launch_bounds__(kTcThreads, 1)
decode_tc_kernel(const __grid_constant__ DecodeMmaArgs A) {
  constexpr int D = 128, HALF = 64, NS = kTcStages;
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

  // ---- set-up: barriers, TMEM, the memory split's key count
  if (threadIdx.x == 0) {
    for (int st = 0; st < NS; ++st) {
      mbar_init(&sm.kvfull[st], mem ? kTcSoftWarps : 1);   // memory tiles: one arrive per gathering warp
      mbar_init(&sm.kvempty[st], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.sfull[i], 1);
      mbar_init(&sm.sempty[i], kTcSoftWarps);
      mbar_init(&sm.pready[i], kTcSoftWarps);
      mbar_init(&sm.pvdone[i], 1);
    }
    mbar_init(&sm.odone, 1);
    mbar_init(&sm.qfull, 1);
    fence_mbar_init();
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
  if (mem) nkeys = sm.mem_pref[k];
  const int ntiles = (int)((nkeys + kDecTile - 1) / kDecTile);

  // the memory split's tiles: cp.async by the softmax threads into stage t % NS
  auto mem_tile = [&](int t) {
    dec_mem_rows(threadIdx.x, t, 0, nkeys, k, sm.mem_pref, sm.mem_krow, sm.mem_vrow, sm.key_krow, sm.key_vrow);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const int st = t % NS;
    dec_mem_gather<D>(threadIdx.x, a, g, t, 0, nkeys, sm.key_krow, sm.key_vrow, &sm.kv[st][0][0][0],
                      &sm.kv[st][1][0][0]);
    cp_async_wait_group<0>();
    fence_proxy_async_smem();
    asm volatile("bar.sync 1, 128;" ::: "memory");          // rows of the next tile may be rewritten
    if (lane == 0) mbar_arrive(&sm.kvfull[st]);
  };

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
  if (warp == kTcProducerWarp) {                             // ---- the raw query rows, then the first stages
    if (lane == 0) {
      const uint32_t row_bytes = (uint32_t)a.G * D * 2;
      mbar_arrive_expect_tx(&sm.qfull, (uint32_t)ntok * (row_bytes + HALF * 8));
      const __nv_bfloat16* q0 = reinterpret_cast<const __nv_bfloat16*>(a.q) + (int64_t)g * a.G * D;
      for (int tt = 0; tt < ntok; ++tt)
        tma_load_1d(&sm.p[0][0] + (size_t)tt * row_bytes, q0 + (((int64_t)b * a.T + t0 + tt) * a.Hq) * D, row_bytes,
                    &sm.qfull);
      tma_load_1d(&sm.rope_rows[0][0], a.rope + ((int64_t)k + Lb + t0) * HALF, (uint32_t)ntok * HALF * 8, &sm.qfull);
      if (!mem) {
        prefetch_tensormap_desc(&A.tm_k);
        prefetch_tensormap_desc(&A.tm_v);
        for (int t = 0; t < ntiles && t < NS; ++t) issue_local(t);
      }
    }
  } else if (warp < kTcSoftWarps) {                          // ---- softmax warps: Q, first memory tiles
    const int i = threadIdx.x;
    const int r = rg * kTcRows + i;
    const bool real = i < nrow;
    // rotated query row i (zero past the real rows), K-major with the 128-byte swizzle,
    // from the raw row and its rotary row in shared memory
    {
      const bool arrived = mbar_wait(&sm.qfull, 0u);
      const unsigned char* raw = &sm.p[0][0] + (size_t)i * D * 2;
      const float2* cs = sm.rope_rows[real ? r / a.G - t0 : 0];
#pragma unroll 2
      for (int j = 0; j < 8; ++j) {                          // dims 8j .. 8j+7 and their partners + 64
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
    if (mem)                                                 // the first memory tiles
      for (int t = 0; t < ntiles && t < NS; ++t) mem_tile(t);
  }
  __syncthreads();                                           // Q and the first stages' copies in place

  if (warp == kTcProducerWarp) {                             // ---- TMA producer: the remaining stages
    if (lane == 0 && !mem) {
      int issued = min(ntiles, NS);
      for (int t = NS; t < ntiles; ++t) {
        if (!mbar_wait(&sm.kvempty[t % NS], (uint32_t)(((t / NS) - 1) & 1))) break;
        issue_local(t);
        issued = t + 1;
      }
      // the last stages' copies land before the CTA may leave
      for (int t = issued > NS ? issued - NS : 0; t < issued; ++t)
        mbar_wait(&sm.kvfull[t % NS], (uint32_t)((t / NS) & 1));
    }
  } else if (warp == kTcMmaWarp) {                           // ---- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(64);
      constexpr uint32_t idesc_o = umma_idesc_bf16_bmn(128);
      const uint32_t sq = smem_u32(&sm.q[0][0]);
      bool ok = true;
      auto pv = [&](int u) -> bool {                         // O += P(u) V(u)
        const int pb = u & 1, st = u % NS;
        if (!mbar_wait(&sm.pready[pb], (uint32_t)((u >> 1) & 1))) return false;
        tc_fence_after();
        const uint32_t sp = smem_u32(&sm.p[pb][0]), sv = smem_u32(&sm.kv[st][1][0][0]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)                       // K = 64 keys in steps of 16
          umma_bf16(tmem + kTcOCol, umma_sdesc(sp + kk * 32), umma_sdesc_mn(sv + kk * 2048, 64 * 128), idesc_o,
                    (u > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&sm.pvdone[pb]);
        umma_commit(&sm.kvempty[st]);
        return true;
      };
      for (int t = 0; t < ntiles && ok; ++t) {
        const int st = t % NS, sb = t & 1;
        if (!mbar_wait(&sm.kvfull[st], (uint32_t)((t / NS) & 1))) { ok = false; break; }
        if (t >= 2 && !mbar_wait(&sm.sempty[sb], (uint32_t)(((t >> 1) - 1) & 1))) { ok = false; break; }
        tc_fence_after();
        const uint32_t sk = smem_u32(&sm.kv[st][0][0][0]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {                     // K = 128 dims in steps of 16
          const uint32_t off = (uint32_t)((kk >> 2) * (64 * 128) + (kk & 3) * 32);
          const uint32_t offq = (uint32_t)((kk >> 2) * (kTcRows * 128) + (kk & 3) * 32);
          umma_bf16(tmem + (uint32_t)(sb * 64), umma_sdesc(sq + offq), umma_sdesc(sk + off), idesc_s,
                    kk > 0 ? 1u : 0u);
        }
        umma_commit(&sm.sfull[sb]);
        if (t >= 1 && !pv(t - 1)) { ok = false; break; }
      }
      if (ok && ntiles > 0 && pv(ntiles - 1)) umma_commit(&sm.odone);
    }
  } else {                                                   // ---- softmax and epilogue: row i
    const int i = threadIdx.x;
    const int r = rg * kTcRows + i;
    const bool real = i < nrow;
    const int t_q = real ? r / a.G : 0;
    const int64_t last = Lb + t_q - j_lo;
    const int lim = !real ? -1 : (mem ? INT_MAX : (last < 0 ? -1 : (int)min64(last, INT_MAX)));
    const uint32_t tlane = (uint32_t)(warp * 32) << 16;
    float mref = -INFINITY, lsum = 0.f;
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) {
      const int sb = t & 1;
      const int n_t = (int)min64(kDecTile, nkeys - (int64_t)t * kDecTile);
      if (!mbar_wait_warp(&sm.sfull[sb], (uint32_t)((t >> 1) & 1))) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32_issue(tmem + tlane + (uint32_t)(sb * 64), sr[0]);
      tmem_ld32_issue(tmem + tlane + (uint32_t)(sb * 64 + 32), sr[1]);
      tmem_wait_tie(sr[0]);
      reg_tie(sr[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.sempty[sb]);            // S buffer sb may be overwritten
      const int64_t kt = (int64_t)t * kDecTile;
      float sv[64];
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const bool vis = c < n_t && kt + c <= lim;
        sv[c] = vis ? __uint_as_float(sr[c >> 5][c & 31]) * a.scale_log2 : -INFINITY;
        mx = fmaxf(mx, sv[c]);
      }
      // lazy reference maximum; O (in TMEM) is rescaled when it moves after the first tile
      const bool move = mx > mref + kLazyRescale;
      const float sc = move ? exp2f(mref - mx) : 1.f;       // mref = -inf gives 0
      if (t > 0 && __any_sync(0xffffffffu, move)) {
        if (!mbar_wait_warp(&sm.pvdone[(t - 1) & 1], (uint32_t)(((t - 1) >> 1) & 1))) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
          uint32_t o[32];
          tmem_ld32_issue(tmem + tlane + (uint32_t)(kTcOCol + 32 * cb), o);
          tmem_wait_tie(o);
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * sc);
          tmem_st32(tmem + tlane + (uint32_t)(kTcOCol + 32 * cb), o);
        }
        tmem_st_wait();
      }
      if (move) {
        lsum *= sc;
        mref = mx;
      }
      // P(t) into buffer sb once P V(t - 2) is done with it; V rows past the
      // tile's keys zeroed (their values may be anything), so P V sees 0 x 0
      if (t >= 2 && !mbar_wait_warp(&sm.pvdone[sb], (uint32_t)(((t - 2) >> 1) & 1))) { ok = false; break; }
      unsigned char* prow = &sm.p[sb][0];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 8 * j + 2 * e;
          const float p0 = sv[c] == -INFINITY ? 0.f : exp2f(sv[c] - mref);
          const float p1 = sv[c + 1] == -INFINITY ? 0.f : exp2f(sv[c + 1] - mref);
          lsum += p0 + p1;
          w4[e] = pack_bf16(p0, p1);
        }
        *reinterpret_cast<uint4*>(prow + i * 128 + (((j ^ (i & 7))) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
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
      if (lane == 0) mbar_arrive(&sm.pready[sb]);
      if (mem && t + NS < ntiles) {                          // the memory split's next tile into this stage
        if (!soft_sync_and(mbar_wait_warp(&sm.kvempty[t % NS], (uint32_t)((t / NS) & 1)))) { ok = false; break; }
        mem_tile(t + NS);
      }
    }
    // ---- this split's partial: (reference max, sum) and the unnormalised O row
    const int sid = a.split_off[b] + s;
    const int64_t prow = ((int64_t)sid * a.Hkv + g) * a.R + rg * kTcRows + i;
    const bool have = ok && ntiles > 0 && mbar_wait_warp(&sm.odone, 0u);
    if (have) tc_fence_after();
#pragma unroll 1
    for (int cb = 0; cb < 4; ++cb) {
      uint32_t o[32];
      if (have) {
        tmem_ld32_issue(tmem + tlane + (uint32_t)(kTcOCol + 32 * cb), o);
        tmem_wait_tie(o);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = 0u;
      }
      if (real) {
        float4* dst = reinterpret_cast<float4*>(a.part_o + prow * D) + 8 * cb;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          dst[c] = make_float4(__uint_as_float(o[4 * c]), __uint_as_float(o[4 * c + 1]), __uint_as_float(o[4 * c + 2]),
                               __uint_as_float(o[4 * c + 3]));
      }
    }
    if (real) reinterpret_cast<float2*>(a.part_ml)[prow] = make_float2(have ? mref : -INFINITY, have ? lsum : 0.f);
  }

  // ---- teardown (decode_tc_merge_kernel merges the splits)
  tc_fence_before();
  __syncthreads();
  if (warp == kTcMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(kTcTmemCols) : "memory");
  }
}

// The splits of decode_tc_kernel merged into the output: one CTA per 16 rows
// of a (query, kv head, row group), all its loads in flight at once.
__global__ void __launch_bounds__(kMmaThreads) decode_tc_merge_kernel(const __grid_constant__ DecodeArgs a) {
  pdl_wait();                                                // every split's partial is written
  constexpr int PER = kTcRows / kTcMergeRows;
  int idx = blockIdx.x;
  const int c = idx % PER;
  idx /= PER;
  const int rg = idx % a.n_rg;
  idx /= a.n_rg;
  const int g = idx % a.Hkv, b = idx / a.Hkv;
  const int r0 = rg * kTcRows + c * kTcMergeRows;
  const int nrow = min(kTcMergeRows, a.R - r0);
  if (nrow <= 0) return;
  merge_splits<128, kTcMergeRows * 32 / kMmaThreads, 8>(a, b, g, r0, nrow, a.split_off[b + 1] - a.split_off[b]);
}

}  // namespace msa
