// Training-time MSA routing layer: backward of the sparse attention, and the
// auxiliary routing loss (forward and backward).
//
// "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts", sections
// "How MSA compresses and routes documents" and "MSA against a conventional
// RAG stack" (routing and generation trained end to end), and "EverMind
// Releases Memory-Sparse Attention Code for Long-Context AI Models", section
// "Implementation Details" (an auxiliary routing loss).  The forward of the
// layer is the inference path (the top-k selection carries no gradient); the
// router score is trained by the loss
//     loss_b = logsumexp_d(S_d / tau) - logsumexp_{d in P_b}(S_d / tau),
// its gradient following the query token and chunk that maximise S_d.
#pragma once
#include "msa_common.cuh"
#include "decode.cuh"
#include "decode_mma.cuh"

namespace msa {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ----------------------------------------------------- attention backward

constexpr int kBwdTile = 64;       // keys per CTA
constexpr int kBwdRows = 64;       // query rows per block
constexpr int kBwdThreads = 256;
constexpr int kBwdMmaThreads = 512;
constexpr int kBwdMaxB = 256;

struct BwdArgs {
  int B, T, Hq, Hkv, G, R, top_k, rope_rows, mem_tiles;
  float scale, scale_log2;           // 1/sqrt(d), log2(e)/sqrt(d)
  const void* q;                     // [B][T][Hq][d] unrotated
  const void* lk;                    // rotated local keys, [H_kv][cap_b][d] per query
  const void* lv;
  const int32_t* sel;
  const int64_t* doc_chunk_off;
  int64_t n_docs;
  const void* mem_k;                 // [C][H_kv][d]
  const void* mem_v;
  const float2* rope;
  const void* out;                   // forward output [B][T][Hq][d]
  const void* dout;                  // its gradient
  const float* lse;                  // [B][T][Hq] natural log
  float* qrot;                       // workspace: rotated queries [B][T][Hq][d] in the bank's type
  float* drow;                       // workspace: sum_d dO * O, [B][T][Hq]
  float* dq;                         // [B][T][Hq][d], accumulated in the rotated frame, then rotated back
  float* dmem_k;                     // [C][H_kv][d], += per selected chunk
  float* dmem_v;
  float* dlk;                        // local cache layout, w.r.t. the unrotated keys
  float* dlv;
  int32_t tile_off[kBwdMaxB + 1];    // first CTA slot of query b (its memory tiles, then local tiles)
  int64_t local_off[kBwdMaxB + 1];
  int64_t local_len[kBwdMaxB];
};

template <typename T>
__device__ __forceinline__ void load4f(const T* p, float* f);
template <> __device__ __forceinline__ void load4f<float>(const float* p, float* f) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
template <> __device__ __forceinline__ void load4f<__nv_bfloat16>(const __nv_bfloat16* p, float* f) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
}

// One warp per (b, t, h): the rotated query (position top_k + L_b + t), the
// row's D = sum dO * O, and a zeroed dq row.
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __grid_constant__ BwdArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + warp;
  if (row >= (int64_t)a.B * a.T * a.Hq) return;
  const int b = (int)(row / ((int64_t)a.T * a.Hq));
  const int t = (int)((row / a.Hq) % a.T);
  const int64_t pos = a.top_k + (a.local_len[b] - a.T) + t;
  const T* q = reinterpret_cast<const T*>(a.q) + row * D;
  const T* o = reinterpret_cast<const T*>(a.out) + row * D;
  const T* dO = reinterpret_cast<const T*>(a.dout) + row * D;
  constexpr int H = D / 2;
  T* qrot = reinterpret_cast<T*>(a.qrot) + row * D;     // in the bank's type: bf16 for the tensor cores
  float dsum = 0.f;
  for (int i = lane; i < H; i += 32) {
    const float2 cs = a.rope[pos * H + i];
    const float x0 = to_f32(q[i]), x1 = to_f32(q[i + H]);
    Elem<T>::store1(qrot + i, x0 * cs.x - x1 * cs.y);
    Elem<T>::store1(qrot + i + H, x1 * cs.x + x0 * cs.y);
    dsum += to_f32(dO[i]) * to_f32(o[i]) + to_f32(dO[i + H]) * to_f32(o[i + H]);
    a.dq[row * D + i] = 0.f;
    a.dq[row * D + i + H] = 0.f;
  }
  dsum = warp_sum(dsum);
  if (lane == 0) a.drow[row] = dsum;
}

// dq from the rotated frame back to the query's own: the transposed rotation.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_rotq_kernel(const __grid_constant__ BwdArgs a) {
  constexpr int H = D / 2;
  const int64_t n = (int64_t)a.B * a.T * a.Hq * H;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = idx / H;
    const int i = (int)(idx % H);
    const int b = (int)(row / ((int64_t)a.T * a.Hq));
    const int t = (int)((row / a.Hq) % a.T);
    const int64_t pos = a.top_k + (a.local_len[b] - a.T) + t;
    const float2 cs = a.rope[pos * H + i];
    float* p = a.dq + row * D;
    const float y0 = p[i], y1 = p[i + H];
    p[i] = y0 * cs.x + y1 * cs.y;
    p[i + H] = y1 * cs.x - y0 * cs.y;
  }
}

template <int D>
struct BwdSmem {
  static constexpr int KS = D + 4;    // row stride (floats): 16-byte rows spread over the banks
  float k[kBwdTile][KS];
  float v[kBwdTile][KS];
  float q[kBwdRows][KS];
  float dout[kBwdRows][KS];
  float p[kBwdRows][kBwdTile + 4];
  float ds[kBwdRows][kBwdTile + 1];
  float lse2[kBwdRows], drow[kBwdRows];
  int64_t krow[kBwdTile];             // source row (units of d elements) of each key, -1 past the tile's end
  int64_t mem_pref[kMaxTopKDecode + 1];
  int64_t mem_c0[kMaxTopKDecode];
};

// One CTA per (key tile, kv head): the tile's 64 keys (memory chunks of the
// selected documents, or local tokens) against every query row of that kv
// head, 64 rows at a time, flash-attention style:
//   S = q~ k^T, P = exp(S/sqrt(d) - lse), dP = dO v^T, dS = P (dP - D)
//   dV += P^T dO, dK += dS^T q~ / sqrt(d), dq~ += dS k / sqrt(d) (atomics)
// CUDA-core fp32 arithmetic on fp32 copies of the tiles.  Thread roles
// (DP = d/16 dims per thread): (A, B) rows ra + 16u x keys ka + 16v;
// (C) keys kc + 16v x dims DP*dc..; (D) rows rc + 16u x dims DP*dc.. --
// strides chosen so that the shared-memory reads of a warp hit distinct banks
// or broadcast.
template <typename T, int D>
__global__ void __launch_bounds__(kBwdThreads, 1) attn_bwd_kernel(const __grid_constant__ BwdArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  auto& sm = *reinterpret_cast<BwdSmem<D>*>(smem_raw);
  const int g = blockIdx.y;
  const int slot = blockIdx.x;
  int b = 0;
  while (slot >= a.tile_off[b + 1]) ++b;
  const int tile = slot - a.tile_off[b];
  const int tid = threadIdx.x;
  const int64_t cap = a.local_off[b + 1] - a.local_off[b];
  const int64_t Ltot = a.local_len[b], Lb = Ltot - a.T;
  if (tid == 0) {
    int64_t acc = 0;
    for (int r = 0; r < a.top_k; ++r) {
      int doc = a.sel[(int64_t)b * a.top_k + r];
      if (doc < 0 || doc >= a.n_docs) { dev_flag(MSA_DEV_BAD_DOC); doc = 0; }
      const int64_t c0 = a.doc_chunk_off[doc];
      sm.mem_c0[r] = c0;
      sm.mem_pref[r] = acc;
      acc += a.doc_chunk_off[doc + 1] - c0;
    }
    sm.mem_pref[a.top_k] = acc;
  }
  __syncthreads();
  if (tid == 0 && tile == 0 && sm.mem_pref[a.top_k] > (int64_t)a.mem_tiles * kBwdTile)
    dev_flag(MSA_DEV_BAD_SHAPE);                 // more memory keys than the launch planned for
  const bool mem = tile < a.mem_tiles;
  const int64_t k0 = (int64_t)(mem ? tile : tile - a.mem_tiles) * kBwdTile;
  const int64_t nkey_all = mem ? sm.mem_pref[a.top_k] : Ltot;
  if (k0 >= nkey_all) return;
  const int nk = (int)min64(kBwdTile, nkey_all - k0);
  if (tid < kBwdTile) {
    int64_t row = -1;
    if (tid < nk) {
      if (mem) {
        const int64_t m = k0 + tid;
        int r = 0;
        while (sm.mem_pref[r + 1] <= m) ++r;
        row = (sm.mem_c0[r] + (m - sm.mem_pref[r])) * a.Hkv + g;
      } else {
        row = a.local_off[b] * a.Hkv + (int64_t)g * cap + k0 + tid;
      }
    }
    sm.krow[tid] = row;
  }
  __syncthreads();
  {
    const T* Kb = reinterpret_cast<const T*>(mem ? a.mem_k : a.lk);
    const T* Vb = reinterpret_cast<const T*>(mem ? a.mem_v : a.lv);
    for (int idx = tid; idx < kBwdTile * (D / 8); idx += kBwdThreads) {
      const int kk = idx / (D / 8), c8 = idx % (D / 8);
      float fk[8], fv[8];
      const int64_t row = sm.krow[kk];
      if (row >= 0) {
        load8<T>(Kb + row * D + c8 * 8, fk);
        load8<T>(Vb + row * D + c8 * 8, fv);
      } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) fk[u] = fv[u] = 0.f;
      }
      *reinterpret_cast<float4*>(&sm.k[kk][c8 * 8]) = make_float4(fk[0], fk[1], fk[2], fk[3]);
      *reinterpret_cast<float4*>(&sm.k[kk][c8 * 8 + 4]) = make_float4(fk[4], fk[5], fk[6], fk[7]);
      *reinterpret_cast<float4*>(&sm.v[kk][c8 * 8]) = make_float4(fv[0], fv[1], fv[2], fv[3]);
      *reinterpret_cast<float4*>(&sm.v[kk][c8 * 8 + 4]) = make_float4(fv[4], fv[5], fv[6], fv[7]);
    }
  }
  constexpr int DP = D / 16;                  // dims per thread in phases C, D
  static_assert(DP % 4 == 0, "head_dim must be a multiple of 64");
  const int ra = tid >> 4, ka = tid & 15;     // phases A, B
  const int kc = tid & 15, dc = tid >> 4;     // phase C (keys), phase D (rows rc = kc); dims DP*dc..
  float dk[4][DP], dv[4][DP];
#pragma unroll
  for (int v = 0; v < 4; ++v)
#pragma unroll
    for (int e = 0; e < DP; ++e) dk[v][e] = dv[v][e] = 0.f;
  const T* dOg = reinterpret_cast<const T*>(a.dout);
  const int nrb = (a.R + kBwdRows - 1) / kBwdRows;
  for (int rb = 0; rb < nrb; ++rb) {
    const int r0 = rb * kBwdRows;
    if (!mem) {                                 // no row of the block sees a key of this tile
      const int t_last = min(a.R - 1, r0 + kBwdRows - 1) / a.G;
      if (Lb + t_last < k0) continue;
    }
    __syncthreads();                            // the previous block's readers are done
    for (int idx = tid; idx < kBwdRows * (D / 4); idx += kBwdThreads) {
      const int rr = idx / (D / 4), c4 = idx % (D / 4);
      const int r = r0 + rr;
      float4 qv = make_float4(0.f, 0.f, 0.f, 0.f), ov = qv;
      if (r < a.R) {
        const int t = r / a.G, h = g * a.G + r % a.G;
        const int64_t o = (((int64_t)b * a.T + t) * a.Hq + h) * D + c4 * 4;
        qv = *reinterpret_cast<const float4*>(a.qrot + o);
        float f[4];
        load4f<T>(dOg + o, f);
        ov = make_float4(f[0], f[1], f[2], f[3]);
      }
      *reinterpret_cast<float4*>(&sm.q[rr][c4 * 4]) = qv;
      *reinterpret_cast<float4*>(&sm.dout[rr][c4 * 4]) = ov;
    }
    if (tid < kBwdRows) {
      const int r = r0 + tid;
      float l2 = INFINITY, dr = 0.f;
      if (r < a.R) {
        const int64_t i = ((int64_t)b * a.T + r / a.G) * a.Hq + g * a.G + r % a.G;
        l2 = a.lse[i] * kLog2e;
        dr = a.drow[i];
      }
      sm.lse2[tid] = l2;
      sm.drow[tid] = dr;
    }
    __syncthreads();
    // A: S and dP
    float s[4][4], dp[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) s[u][v] = dp[u][v] = 0.f;
#pragma unroll 2
    for (int i = 0; i < D; i += 4) {
      float4 qv[4], ov[4], kv[4], vv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        qv[u] = *reinterpret_cast<const float4*>(&sm.q[ra + 16 * u][i]);
        ov[u] = *reinterpret_cast<const float4*>(&sm.dout[ra + 16 * u][i]);
        kv[u] = *reinterpret_cast<const float4*>(&sm.k[ka + 16 * u][i]);
        vv[u] = *reinterpret_cast<const float4*>(&sm.v[ka + 16 * u][i]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          s[u][v] = fmaf(qv[u].x, kv[v].x, fmaf(qv[u].y, kv[v].y, fmaf(qv[u].z, kv[v].z, fmaf(qv[u].w, kv[v].w, s[u][v]))));
          dp[u][v] = fmaf(ov[u].x, vv[v].x, fmaf(ov[u].y, vv[v].y, fmaf(ov[u].z, vv[v].z, fmaf(ov[u].w, vv[v].w, dp[u][v]))));
        }
    }
    // B: P and dS (zero where the key is not visible to the row)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int rr = ra + 16 * u, r = r0 + rr;
      const int t = r / a.G;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int kk = ka + 16 * v;
        const bool vis = r < a.R && kk < nk && (mem || k0 + kk <= Lb + t);
        const float pr = vis ? exp2f(fmaf(s[u][v], a.scale_log2, -sm.lse2[rr])) : 0.f;
        sm.p[rr][kk] = pr;
        sm.ds[rr][kk] = pr * (dp[u][v] - sm.drow[rr]);
      }
    }
    __syncthreads();
    // C: dV += P^T dO, dK += dS^T q~
#pragma unroll 4
    for (int rr = 0; rr < kBwdRows; ++rr) {
      float of[DP], qf[DP];
#pragma unroll
      for (int e = 0; e < DP; e += 4) {
        const float4 o4 = *reinterpret_cast<const float4*>(&sm.dout[rr][DP * dc + e]);
        const float4 q4 = *reinterpret_cast<const float4*>(&sm.q[rr][DP * dc + e]);
        of[e] = o4.x; of[e + 1] = o4.y; of[e + 2] = o4.z; of[e + 3] = o4.w;
        qf[e] = q4.x; qf[e + 1] = q4.y; qf[e + 2] = q4.z; qf[e + 3] = q4.w;
      }
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const float pv = sm.p[rr][kc + 16 * v], dsv = sm.ds[rr][kc + 16 * v];
#pragma unroll
        for (int e = 0; e < DP; ++e) {
          dv[v][e] = fmaf(pv, of[e], dv[v][e]);
          dk[v][e] = fmaf(dsv, qf[e], dk[v][e]);
        }
      }
    }
    // D: dq~ rows kc + 16u, dims DP*dc.. over the tile's keys
    float dq[4][DP];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int e = 0; e < DP; ++e) dq[u][e] = 0.f;
#pragma unroll 2
    for (int kk = 0; kk < nk; ++kk) {
      float kf[DP];
#pragma unroll
      for (int e = 0; e < DP; e += 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(&sm.k[kk][DP * dc + e]);
        kf[e] = k4.x; kf[e + 1] = k4.y; kf[e + 2] = k4.z; kf[e + 3] = k4.w;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float w = sm.ds[kc + 16 * u][kk];
#pragma unroll
        for (int e = 0; e < DP; ++e) dq[u][e] = fmaf(w, kf[e], dq[u][e]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = r0 + kc + 16 * u;
      if (r >= a.R) continue;
      const int t = r / a.G, h = g * a.G + r % a.G;
      float* dst = a.dq + (((int64_t)b * a.T + t) * a.Hq + h) * D + DP * dc;
#pragma unroll
      for (int e = 0; e < DP; ++e) atomicAdd(dst + e, dq[u][e] * a.scale);
    }
  }
  __syncthreads();
  if (mem) {                                    // chunks another query also selected add up
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int kk = kc + 16 * v;
      if (kk >= nk) continue;
      const int64_t row = sm.krow[kk];
#pragma unroll
      for (int e = 0; e < DP; ++e) {
        atomicAdd(a.dmem_k + row * D + DP * dc + e, dk[v][e] * a.scale);
        atomicAdd(a.dmem_v + row * D + DP * dc + e, dv[v][e]);
      }
    }
    return;
  }
  // local keys: dV as it is; dK through the transposed rotation at top_k + j
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const int kk = kc + 16 * v;
    if (kk >= nk) continue;
    float* dvp = a.dlv + sm.krow[kk] * D + DP * dc;
#pragma unroll
    for (int e = 0; e < DP; e += 4)
      *reinterpret_cast<float4*>(dvp + e) = make_float4(dv[v][e], dv[v][e + 1], dv[v][e + 2], dv[v][e + 3]);
#pragma unroll
    for (int e = 0; e < DP; ++e) sm.k[kk][DP * dc + e] = dk[v][e] * a.scale;
  }
  __syncthreads();
  constexpr int H = D / 2;
  for (int idx = tid; idx < nk * H; idx += kBwdThreads) {
    const int kk = idx / H, i = idx % H;
    const float2 cs = a.rope[(a.top_k + k0 + kk) * H + i];
    const float y0 = sm.k[kk][i], y1 = sm.k[kk][i + H];
    float* dkp = a.dlk + sm.krow[kk] * D;
    dkp[i] = y0 * cs.x + y1 * cs.y;
    dkp[i + H] = y1 * cs.x - y0 * cs.y;
  }
}

// ------------------------------------- attention backward on the tensor cores

template <int D>
struct BwdMmaSmem {
  static constexpr int kTile = D * 128;          // bytes of a [64][D] bf16 tile, 128-byte swizzled rows
  union {
    struct {
      unsigned char k[kTile];
      unsigned char v[kTile];
    } kv;
    float dk[kBwdTile][D + 4];                   // epilogue: the local keys' scaled dK
  } u;
  unsigned char q[2][kTile];                     // rotated queries of a row block, bf16 (double buffer)
  unsigned char o[2][kTile];                     // their dO
  unsigned char p[64 * 128];                     // P [row][key], bf16
  unsigned char ds[64 * 128];                    // dS [row][key], bf16
  float lse2[kBwdRows], drow[kBwdRows];
  int64_t krow[kBwdTile];
  int64_t mem_pref[kMaxTopKDecode + 1];
  int64_t mem_c0[kMaxTopKDecode];
};

// bf16 banks: the same CTA work as attn_bwd_kernel with the five products on
// the tensor cores (mma.sync m16n8k16, bf16 operands, fp32 accumulators).
// Tiles sit in shared memory as bf16 in the decode's 128-byte swizzle;
// ldmatrix (.trans where a product needs the transpose: P^T, dS^T as A
// operands, dO, q~, K as [k][n] B operands) feeds the fragments.  16 warps:
// wm = warp % 4 picks 16 rows (S, dP, dq) or 16 keys (dV, dK); wn = warp / 4
// picks 16 keys (S, dP) or a quarter of the dims (dV, dK, dq).  The rotated query, P
// and dS enter the products as bf16 (relative rounding 2^-9).
template <int D>
__global__ void __launch_bounds__(kBwdMmaThreads, 1) attn_bwd_mma_kernel(const __grid_constant__ BwdArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  auto& sm = *reinterpret_cast<BwdMmaSmem<D>*>(smem_raw);
  constexpr int CPR = D / 8;                     // 16-byte chunks per row
  constexpr int NB4 = D / 32;                    // n8 blocks of a warp's quarter of the dims
  const int g = blockIdx.y;
  const int slot = blockIdx.x;
  int b = 0;
  while (slot >= a.tile_off[b + 1]) ++b;
  const int tile = slot - a.tile_off[b];
  const int tid = threadIdx.x;
  const int64_t cap = a.local_off[b + 1] - a.local_off[b];
  const int64_t Ltot = a.local_len[b], Lb = Ltot - a.T;
  if (tid == 0) {
    int64_t acc = 0;
    for (int r = 0; r < a.top_k; ++r) {
      int doc = a.sel[(int64_t)b * a.top_k + r];
      if (doc < 0 || doc >= a.n_docs) { dev_flag(MSA_DEV_BAD_DOC); doc = 0; }
      const int64_t c0 = a.doc_chunk_off[doc];
      sm.mem_c0[r] = c0;
      sm.mem_pref[r] = acc;
      acc += a.doc_chunk_off[doc + 1] - c0;
    }
    sm.mem_pref[a.top_k] = acc;
  }
  __syncthreads();
  if (tid == 0 && tile == 0 && sm.mem_pref[a.top_k] > (int64_t)a.mem_tiles * kBwdTile)
    dev_flag(MSA_DEV_BAD_SHAPE);
  const bool mem = tile < a.mem_tiles;
  const int64_t k0 = (int64_t)(mem ? tile : tile - a.mem_tiles) * kBwdTile;
  const int64_t nkey_all = mem ? sm.mem_pref[a.top_k] : Ltot;
  if (k0 >= nkey_all) return;
  const int nk = (int)min64(kBwdTile, nkey_all - k0);
  if (tid < kBwdTile) {
    int64_t row = -1;
    if (tid < nk) {
      if (mem) {
        const int64_t m = k0 + tid;
        int r = 0;
        while (sm.mem_pref[r + 1] <= m) ++r;
        row = (sm.mem_c0[r] + (m - sm.mem_pref[r])) * a.Hkv + g;
      } else {
        row = a.local_off[b] * a.Hkv + (int64_t)g * cap + k0 + tid;
      }
    }
    sm.krow[tid] = row;
  }
  __syncthreads();
  {                                              // K and V tiles, zero past the tile's keys
    const __nv_bfloat16* Kb = reinterpret_cast<const __nv_bfloat16*>(mem ? a.mem_k : a.lk);
    const __nv_bfloat16* Vb = reinterpret_cast<const __nv_bfloat16*>(mem ? a.mem_v : a.lv);
    for (int idx = tid; idx < kBwdTile * 2 * CPR; idx += kBwdMmaThreads) {
      const int c = idx % CPR, kv = (idx / CPR) & 1, i = idx / (2 * CPR);
      unsigned char* dst = (kv ? sm.u.kv.v : sm.u.kv.k) + swz(i, c);
      const int64_t row = sm.krow[i];
      if (row >= 0) cp_async_16(dst, (kv ? Vb : Kb) + row * D + 8 * c);
      else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    cp_async_commit();
  }
  const int warp = tid >> 5, lane = tid & 31, wm = warp & 3, wn = warp >> 2;
  const int qr = lane >> 2, qc = lane & 3;
  const uint32_t k_s = smem_u32(sm.u.kv.k), v_s = smem_u32(sm.u.kv.v);
  const uint32_t p_s = smem_u32(sm.p), ds_s = smem_u32(sm.ds);
  float dkacc[NB4][4], dvacc[NB4][4];
#pragma unroll
  for (int nb = 0; nb < NB4; ++nb)
#pragma unroll
    for (int e = 0; e < 4; ++e) dkacc[nb][e] = dvacc[nb][e] = 0.f;
  const __nv_bfloat16* dOg = reinterpret_cast<const __nv_bfloat16*>(a.dout);
  const __nv_bfloat16* Qg = reinterpret_cast<const __nv_bfloat16*>(a.qrot);
  const int nrb = (a.R + kBwdRows - 1) / kBwdRows;
  // row blocks from the first one a row of which sees this tile (visibility
  // only grows with the token); q~ and dO of block rb go to buffer rb & 1
  int rb0 = 0;
  if (!mem)
    while (rb0 < nrb && Lb + min(a.R - 1, rb0 * kBwdRows + kBwdRows - 1) / a.G < k0) ++rb0;
  auto stage = [&](int rb) {
    const int r0s = rb * kBwdRows;
    unsigned char* qd = sm.q[rb & 1];
    unsigned char* od = sm.o[rb & 1];
    for (int idx = tid; idx < kBwdRows * CPR; idx += kBwdMmaThreads) {
      const int rr = idx / CPR, c = idx % CPR;
      const int r = r0s + rr;
      if (r < a.R) {
        const int t = r / a.G, h = g * a.G + r % a.G;
        const int64_t o = (((int64_t)b * a.T + t) * a.Hq + h) * D + 8 * c;
        cp_async_16(qd + swz(rr, c), Qg + o);
        cp_async_16(od + swz(rr, c), dOg + o);
      } else {
        *reinterpret_cast<uint4*>(qd + swz(rr, c)) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(od + swz(rr, c)) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    cp_async_commit();
  };
  if (rb0 < nrb) stage(rb0);
  for (int rb = rb0; rb < nrb; ++rb) {
    const int r0 = rb * kBwdRows;
    const uint32_t q_s = smem_u32(sm.q[rb & 1]), o_s = smem_u32(sm.o[rb & 1]);
    __syncthreads();                             // the previous block's readers are done
    if (rb + 1 < nrb) {
      stage(rb + 1);                             // in flight while this block computes
      cp_async_wait_group<1>();                  // K/V and this block's q~ / dO have landed
    } else {
      cp_async_wait_group<0>();
    }
    if (tid < kBwdRows) {
      const int r = r0 + tid;
      float l2 = INFINITY, dr = 0.f;
      if (r < a.R) {
        const int64_t i = ((int64_t)b * a.T + r / a.G) * a.Hq + g * a.G + r % a.G;
        l2 = a.lse[i] * kLog2e;
        dr = a.drow[i];
      }
      sm.lse2[tid] = l2;
      sm.drow[tid] = dr;
    }
    __syncthreads();
    // (1) S = q~ K^T and dP = dO V^T: rows 16 wm.., keys 16 wn..
    float sacc[2][4], pacc[2][4];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nb][e] = pacc[nb][e] = 0.f;
#pragma unroll
    for (int kb2 = 0; kb2 < D / 32; ++kb2) {
      uint32_t aq[2][4], ao[2][4];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int ks = 2 * kb2 + h2;
        ldsm_x4(q_s + swz(16 * wm + (lane & 15), 2 * ks + (lane >> 4)), aq[h2]);
        ldsm_x4(o_s + swz(16 * wm + (lane & 15), 2 * ks + (lane >> 4)), ao[h2]);
      }
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        const int key = 16 * wn + 8 * nb + (lane & 7);
        uint32_t bk[4], bv[4];
        ldsm_x4(k_s + swz(key, 4 * kb2 + (lane >> 3)), bk);
        ldsm_x4(v_s + swz(key, 4 * kb2 + (lane >> 3)), bv);
        mma_bf16(sacc[nb], aq[0], bk[0], bk[1]);
        mma_bf16(sacc[nb], aq[1], bk[2], bk[3]);
        mma_bf16(pacc[nb], ao[0], bv[0], bv[1]);
        mma_bf16(pacc[nb], ao[1], bv[2], bv[3]);
      }
    }
    // (2) P and dS on the fragments (rows 16 wm + qr (+8), keys 16 wn + 8 nb + 2 qc (+1)), stored bf16
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
      const int kk0 = 16 * wn + 8 * nb + 2 * qc;
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int rr = 16 * wm + qr + 8 * hr, r = r0 + rr;
        const int t = r / a.G;
        float pv[2], dv2[2];
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
          const int kk = kk0 + e2;
          const bool vis = r < a.R && kk < nk && (mem || k0 + kk <= Lb + t);
          pv[e2] = vis ? exp2f(fmaf(sacc[nb][2 * hr + e2], a.scale_log2, -sm.lse2[rr])) : 0.f;
          dv2[e2] = pv[e2] * (pacc[nb][2 * hr + e2] - sm.drow[rr]);
        }
        const uint32_t off = swz(rr, kk0 >> 3) + (kk0 & 7) * 2;
        *reinterpret_cast<uint32_t*>(sm.p + off) = pack_bf16(pv[0], pv[1]);
        *reinterpret_cast<uint32_t*>(sm.ds + off) = pack_bf16(dv2[0], dv2[1]);
      }
    }
    __syncthreads();
    // (3) dV += P^T dO and dK += dS^T q~: keys 16 wm.., dims (D/4) wn..
#pragma unroll
    for (int ks = 0; ks < kBwdRows / 16; ++ks) {
      uint32_t ap[4], ads[4];
      const int mi = lane >> 3;
      const int srow = 16 * ks + (lane & 7) + ((mi >> 1) << 3);
      ldsm_x4_t(p_s + swz(srow, 2 * wm + (mi & 1)), ap);
      ldsm_x4_t(ds_s + swz(srow, 2 * wm + (mi & 1)), ads);
      const int brow = 16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int np = 0; np < NB4 / 2; ++np) {
        const int chunk = (D / 32) * wn + 2 * np + (lane >> 4);
        uint32_t bo[4], bq[4];
        ldsm_x4_t(o_s + swz(brow, chunk), bo);
        ldsm_x4_t(q_s + swz(brow, chunk), bq);
        mma_bf16(dvacc[2 * np], ap, bo[0], bo[1]);
        mma_bf16(dvacc[2 * np + 1], ap, bo[2], bo[3]);
        mma_bf16(dkacc[2 * np], ads, bq[0], bq[1]);
        mma_bf16(dkacc[2 * np + 1], ads, bq[2], bq[3]);
      }
    }
    // (4) dq~ = dS K: rows 16 wm.., dims (D/4) wn..; then atomics
    float dqa[NB4][4];
#pragma unroll
    for (int nb = 0; nb < NB4; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) dqa[nb][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < kBwdTile / 16; ++ks) {
      uint32_t ads[4];
      ldsm_x4(ds_s + swz(16 * wm + (lane & 15), 2 * ks + (lane >> 4)), ads);
      const int key = 16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int np = 0; np < NB4 / 2; ++np) {
        const int chunk = (D / 32) * wn + 2 * np + (lane >> 4);
        uint32_t bk[4];
        ldsm_x4_t(k_s + swz(key, chunk), bk);
        mma_bf16(dqa[2 * np], ads, bk[0], bk[1]);
        mma_bf16(dqa[2 * np + 1], ads, bk[2], bk[3]);
      }
    }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int r = r0 + 16 * wm + qr + 8 * hr;
      if (r >= a.R) continue;
      const int t = r / a.G, h = g * a.G + r % a.G;
      float* dst = a.dq + (((int64_t)b * a.T + t) * a.Hq + h) * D + (D / 4) * wn + 2 * qc;
#pragma unroll
      for (int nb = 0; nb < NB4; ++nb)                      // two consecutive dims: one 8-byte atomic
        atomicAdd(reinterpret_cast<float2*>(dst + 8 * nb),
                  make_float2(dqa[nb][2 * hr] * a.scale, dqa[nb][2 * hr + 1] * a.scale));
    }
  }
  cp_async_wait_group<0>();
  __syncthreads();
  // dK, dV of keys 16 wm + qr (+8), dims (D/4) wn + 8 nb + 2 qc (+1)
  if (mem) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int kk = 16 * wm + qr + 8 * hr;
      if (kk >= nk) continue;
      const int64_t row = sm.krow[kk];
#pragma unroll
      for (int nb = 0; nb < NB4; ++nb) {
        const int d0 = (D / 4) * wn + 8 * nb + 2 * qc;
        atomicAdd(reinterpret_cast<float2*>(a.dmem_k + row * D + d0),
                  make_float2(dkacc[nb][2 * hr] * a.scale, dkacc[nb][2 * hr + 1] * a.scale));
        atomicAdd(reinterpret_cast<float2*>(a.dmem_v + row * D + d0),
                  make_float2(dvacc[nb][2 * hr], dvacc[nb][2 * hr + 1]));
      }
    }
    return;
  }
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int kk = 16 * wm + qr + 8 * hr;
    if (kk >= nk) continue;
    float* dvp = a.dlv + sm.krow[kk] * D;
#pragma unroll
    for (int nb = 0; nb < NB4; ++nb) {
      const int d0 = (D / 4) * wn + 8 * nb + 2 * qc;
      *reinterpret_cast<float2*>(dvp + d0) = make_float2(dvacc[nb][2 * hr], dvacc[nb][2 * hr + 1]);
      sm.u.dk[kk][d0] = dkacc[nb][2 * hr] * a.scale;
      sm.u.dk[kk][d0 + 1] = dkacc[nb][2 * hr + 1] * a.scale;
    }
  }
  __syncthreads();
  constexpr int H = D / 2;
  for (int idx = tid; idx < nk * H; idx += kBwdMmaThreads) {
    const int kk = idx / H, i = idx % H;
    const float2 cs = a.rope[(a.top_k + k0 + kk) * H + i];
    const float y0 = sm.u.dk[kk][i], y1 = sm.u.dk[kk][i + H];
    float* dkp = a.dlk + sm.krow[kk] * D;
    dkp[i] = y0 * cs.x + y1 * cs.y;
    dkp[i + H] = y1 * cs.x - y0 * cs.y;
  }
}

// ------------------------------------------------- auxiliary routing loss

struct LossArgs {
  int B, T, Hq, Hkv, G, dr;
  int64_t n_docs, n_chunks;
  float tau;
  const void* qr;                    // [B][T][Hq][dr]
  const void* kr;                    // [C][H_kv][dr]
  const int64_t* doc_chunk_off;
  const int32_t* pos_off;            // [B + 1]
  const int32_t* pos_doc;
  float* qinv;                       // [B][T][Hq] 1 / max(|q|, 1e-12)
  float* u;                          // [B][T][H_kv][dr] sum over the kv head's query heads of q / |q|
  float* chunk_best;                 // [B][C] max over t of the chunk's score
  int32_t* chunk_t;                  // [B][C] its token
  float* doc_score;                  // [B][D]
  int32_t* doc_t;                    // [B][D] maximising token
  int64_t* doc_c;                    // [B][D] maximising chunk
  float* lse;                        // [B][2]: logsumexp of S / tau over all documents, over the positives
  float* loss;                       // [B]
  const float* dloss;                // [B] (backward)
  float* dqr;                        // [B][T][Hq][dr] (backward)
  float* dkr;                        // [C][H_kv][dr] (backward, +=)
};

// One warp per (b, t, kv head g): the query heads' inverse norms and their
// normalised sum u.
template <typename T>
__global__ void __launch_bounds__(256) loss_prep_kernel(const __grid_constant__ LossArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + warp;       // (b, t, g)
  if (row >= (int64_t)a.B * a.T * a.Hkv) return;
  const int g = (int)(row % a.Hkv);
  const int64_t bt = row / a.Hkv;
  const T* q = reinterpret_cast<const T*>(a.qr);
  for (int i0 = 0; i0 < a.dr; i0 += 128) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int hh = 0; hh < a.G; ++hh) {
      const int h = g * a.G + hh;
      const T* qh = q + (bt * a.Hq + h) * a.dr;
      float nn = 0.f;
      for (int i = lane; i < a.dr; i += 32) nn += to_f32(qh[i]) * to_f32(qh[i]);
      nn = warp_sum(nn);
      const float inv = 1.0f / fmaxf(sqrtf(nn), 1e-12f);
      if (lane == 0 && i0 == 0) a.qinv[bt * a.Hq + h] = inv;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = i0 + lane + 32 * e;
        if (i < a.dr) acc[e] += to_f32(qh[i]) * inv;
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = i0 + lane + 32 * e;
      if (i < a.dr) a.u[row * a.dr + i] = acc[e];
    }
  }
}

constexpr int kLossChunks = 32;     // chunks per CTA of the score kernel
constexpr int kLossT = 64;          // query tokens per block
constexpr int kLossI = 64;          // elements of the H_kv * d_r dot product per stage

// Per (b, 32-chunk tile): S[t][c] = (1/H_q) sum_g u[t][g] . k^[c][g] for every
// query token, then the max over t and its first maximising token.  A
// register-tiled CUDA-core product: thread (tg, cg) owns tokens 4 tg .. +3 of
// a 64-token block and chunks 2 cg, 2 cg + 1; the operands are staged
// transposed in shared memory, 64 elements at a time, so that a step is one
// 16-byte and one 8-byte shared load for 8 fmas.  The per-head clamp of the
// cosine to [-1, 1] acts only on rounding excess and is left out here.
template <typename T>
__global__ void __launch_bounds__(256) loss_chunk_kernel(const __grid_constant__ LossArgs a) {
  __shared__ __align__(16) float us[kLossI][kLossT + 4];           // [element][token]
  __shared__ __align__(16) float ks[kLossI][kLossChunks + 4];      // [element][chunk]
  __shared__ float kinv[kLossChunks][16];
  const int HD = a.Hkv * a.dr;
  const int b = blockIdx.y;
  const int64_t c0 = (int64_t)blockIdx.x * kLossChunks;
  const int nc = (int)min64(kLossChunks, a.n_chunks - c0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const T* kr = reinterpret_cast<const T*>(a.kr);
  for (int rowi = warp; rowi < kLossChunks * a.Hkv; rowi += 8) {       // inverse norms of (chunk, kv head)
    const int cc = rowi / a.Hkv, g = rowi % a.Hkv;
    float nn = 0.f;
    if (cc < nc) {
      const T* src = kr + ((c0 + cc) * a.Hkv + g) * a.dr;
      for (int i = lane; i < a.dr; i += 32) nn += to_f32(src[i]) * to_f32(src[i]);
    }
    nn = warp_sum(nn);
    if (lane == 0) kinv[cc][g] = 1.0f / fmaxf(sqrtf(nn), 1e-12f);
  }
  const int tg = tid & 15, cg = tid >> 4;
  const float invH = 1.0f / (float)a.Hq;
  float best[2] = {-INFINITY, -INFINITY};
  int bt[2] = {0, 0};
  for (int t0 = 0; t0 < a.T; t0 += kLossT) {
    float acc[4][2];
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u][0] = acc[u][1] = 0.f;
    for (int i0 = 0; i0 < HD; i0 += kLossI) {
      __syncthreads();                           // norms ready / previous stage read
      for (int idx = tid; idx < kLossT * kLossI; idx += 256) {
        const int tt = idx / kLossI, ii = idx % kLossI;
        const int t = t0 + tt, i = i0 + ii;
        us[ii][tt] = (t < a.T && i < HD) ? a.u[((int64_t)b * a.T + t) * HD + i] : 0.f;
      }
      for (int idx = tid; idx < kLossChunks * kLossI; idx += 256) {
        const int cc = idx / kLossI, ii = idx % kLossI;
        const int i = i0 + ii;
        ks[ii][cc] = (cc < nc && i < HD) ? to_f32(kr[(c0 + cc) * HD + i]) * kinv[cc][i / a.dr] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int ii = 0; ii < kLossI; ++ii) {
        const float4 uv = *reinterpret_cast<const float4*>(&us[ii][4 * tg]);
        const float2 kv = *reinterpret_cast<const float2*>(&ks[ii][2 * cg]);
        acc[0][0] = fmaf(uv.x, kv.x, acc[0][0]); acc[0][1] = fmaf(uv.x, kv.y, acc[0][1]);
        acc[1][0] = fmaf(uv.y, kv.x, acc[1][0]); acc[1][1] = fmaf(uv.y, kv.y, acc[1][1]);
        acc[2][0] = fmaf(uv.z, kv.x, acc[2][0]); acc[2][1] = fmaf(uv.z, kv.y, acc[2][1]);
        acc[3][0] = fmaf(uv.w, kv.x, acc[3][0]); acc[3][1] = fmaf(uv.w, kv.y, acc[3][1]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = t0 + 4 * tg + u;
      if (t >= a.T) break;
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const float sc = acc[u][v] * invH;
        if (sc > best[v]) { best[v] = sc; bt[v] = t; }
      }
    }
  }
  // the 16 threads of a half-warp share their chunks: max, first token on ties
#pragma unroll
  for (int v = 0; v < 2; ++v) {
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best[v], o);
      const int ot = __shfl_xor_sync(0xffffffffu, bt[v], o);
      if (ob > best[v] || (ob == best[v] && ot < bt[v])) { best[v] = ob; bt[v] = ot; }
    }
  }
  if (tg == 0) {
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int cc = 2 * cg + v;
      if (cc < nc) {
        a.chunk_best[(int64_t)b * a.n_chunks + c0 + cc] = best[v];
        a.chunk_t[(int64_t)b * a.n_chunks + c0 + cc] = bt[v];
      }
    }
  }
}

// Per (b, document): the max over its chunks (first chunk on ties).
__global__ void __launch_bounds__(256) loss_doc_kernel(const __grid_constant__ LossArgs a) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)a.B * a.n_docs) return;
  const int b = (int)(idx / a.n_docs);
  const int64_t s = idx % a.n_docs;
  float best = -INFINITY;
  int64_t bc = a.doc_chunk_off[s];
  for (int64_t c = a.doc_chunk_off[s]; c < a.doc_chunk_off[s + 1]; ++c) {
    const float v = a.chunk_best[(int64_t)b * a.n_chunks + c];
    if (v > best) { best = v; bc = c; }
  }
  a.doc_score[idx] = best;
  a.doc_c[idx] = bc;
  a.doc_t[idx] = a.chunk_t[(int64_t)b * a.n_chunks + bc];
}

// One CTA per query: logsumexp of S / tau over all documents and over the
// query's positives; the loss is their difference.
__global__ void __launch_bounds__(256) loss_value_kernel(const __grid_constant__ LossArgs a) {
  __shared__ float red[8];
  __shared__ float bc;
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* sc = a.doc_score + (int64_t)b * a.n_docs;
  const float it = 1.0f / a.tau;
  auto block_reduce = [&](float v, bool is_max) -> float {
    v = is_max ? warp_max(v) : warp_sum(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
      float r = red[0];
      for (int w = 1; w < 8; ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
      bc = r;
    }
    __syncthreads();
    return bc;
  };
  const int p0 = a.pos_off[b], p1 = a.pos_off[b + 1];
  if (p1 <= p0 && threadIdx.x == 0) dev_flag(MSA_DEV_BAD_SHAPE);    // a query needs a relevant document
  float lse2[2];
  for (int which = 0; which < 2; ++which) {
    float m = -INFINITY;
    if (which == 0) {
      for (int64_t s = threadIdx.x; s < a.n_docs; s += 256) m = fmaxf(m, sc[s] * it);
    } else {
      for (int j = p0 + threadIdx.x; j < p1; j += 256) {
        int s = a.pos_doc[j];
        if (s < 0 || s >= a.n_docs) { dev_flag(MSA_DEV_BAD_DOC); continue; }
        m = fmaxf(m, sc[s] * it);
      }
    }
    m = block_reduce(m, true);
    float e = 0.f;
    if (which == 0) {
      for (int64_t s = threadIdx.x; s < a.n_docs; s += 256) e += expf(sc[s] * it - m);
    } else {
      for (int j = p0 + threadIdx.x; j < p1; j += 256) {
        const int s = a.pos_doc[j];
        if (s >= 0 && s < a.n_docs) e += expf(sc[s] * it - m);
      }
    }
    e = block_reduce(e, false);
    lse2[which] = m + logf(e);
  }
  if (threadIdx.x == 0) {
    a.lse[2 * b] = lse2[0];
    a.lse[2 * b + 1] = lse2[1];
    a.loss[b] = lse2[0] - lse2[1];
  }
}

// One warp per (b, document): dloss/dS_d, then through the maximising token
// t* and chunk c*: for each query head h of kv head g, with q^ = q/|q|,
// k^ = k/|k| and cos = q^ . k^,
//   dq[t*][h] += w/H_q (k^ - cos q^) / |q|,   dk[c*][g] += w/H_q (q^ - cos k^) / |k|.
template <typename T>
__global__ void __launch_bounds__(256) loss_bwd_kernel(const __grid_constant__ LossArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t idx = (int64_t)blockIdx.x * 8 + warp;
  if (idx >= (int64_t)a.B * a.n_docs) return;
  const int b = (int)(idx / a.n_docs);
  const int64_t s = idx % a.n_docs;
  const float it = 1.0f / a.tau;
  const float z = a.doc_score[idx] * it;
  float w = expf(z - a.lse[2 * b]);
  bool positive = false;
  for (int j = a.pos_off[b]; j < a.pos_off[b + 1]; ++j) positive |= a.pos_doc[j] == s;
  if (positive) w -= expf(z - a.lse[2 * b + 1]);
  w *= a.dloss[b] * it / (float)a.Hq;
  if (w == 0.f) return;
  const int t = a.doc_t[idx];
  const int64_t c = a.doc_c[idx];
  const T* q = reinterpret_cast<const T*>(a.qr);
  const T* kr = reinterpret_cast<const T*>(a.kr);
  for (int g = 0; g < a.Hkv; ++g) {
    const T* kp = kr + (c * a.Hkv + g) * a.dr;
    float nn = 0.f;
    for (int i = lane; i < a.dr; i += 32) nn += to_f32(kp[i]) * to_f32(kp[i]);
    nn = warp_sum(nn);
    const float kinv = 1.0f / fmaxf(sqrtf(nn), 1e-12f);
    float dk[4] = {0.f, 0.f, 0.f, 0.f};
    for (int hh = 0; hh < a.G; ++hh) {
      const int h = g * a.G + hh;
      const int64_t qrow = ((int64_t)b * a.T + t) * a.Hq + h;
      const T* qp = q + qrow * a.dr;
      const float qinv = a.qinv[qrow];
      float cs = 0.f;
      for (int i = lane; i < a.dr; i += 32) cs += to_f32(qp[i]) * to_f32(kp[i]);
      cs = warp_sum(cs) * qinv * kinv;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = lane + 32 * e;
        if (i >= a.dr) break;
        const float qh = to_f32(qp[i]) * qinv, kh = to_f32(kp[i]) * kinv;
        atomicAdd(a.dqr + qrow * a.dr + i, w * (kh - cs * qh) * qinv);
        dk[e] += w * (qh - cs * kh);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = lane + 32 * e;
      if (i < a.dr) atomicAdd(a.dkr + (c * a.Hkv + g) * a.dr + i, dk[e] * kinv);
    }
  }
}

}  // namespace msa
