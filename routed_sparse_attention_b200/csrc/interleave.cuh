// Memory Interleave: one context-expansion round on the GPU.
//
// "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts", section
// "How MSA compresses and routes documents", and "EverMind Releases
// Memory-Sparse Attention Code for Long-Context AI Models", section "Core
// Contributions", name the alternation of retrieval, context expansion and
// generation for multi-hop questions without a formula.  Read as: the
// selected set S of a query grows by the p best-scoring documents outside S,
// in (score desc, index asc) order.  Routing for the n + p best documents
// (n = |S|) always holds at least p documents outside S, and its first p such
// documents in rank order are exactly those; this kernel takes them.
#pragma once
#include <cstdint>

#include "msa_common.cuh"

namespace msa {

constexpr int kInterleaveMaxSet = 64;    // n + p, the routing's largest top_k

// One warp per query.  ranked: [B][n + p]; old_set: [B][n]; out: [B][n + p]
// (old set copied, then the first p ranked documents outside it).  A set that
// holds a document twice or out of range raises MSA_DEV_BAD_SET; unfilled
// slots are then written as -1.
__global__ void __launch_bounds__(128) interleave_expand_kernel(
    const int32_t* __restrict__ ranked, const int32_t* __restrict__ old_set, int32_t* __restrict__ out,
    int B, int n, int p, int64_t n_docs) {
  const unsigned full = 0xffffffffu;
  const int q = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
  if (q >= B) return;
  const int m = n + p;
  const int32_t* rk = ranked + (int64_t)q * m;
  const int32_t* od = old_set + (int64_t)q * n;
  int32_t* o = out + (int64_t)q * m;
  // each lane keeps entries lane and lane + 32 of the old set and of the ranking
  const int32_t s0 = lane < n ? od[lane] : -1, s1 = lane + 32 < n ? od[lane + 32] : -1;
  const int32_t r0 = lane < m ? rk[lane] : -1, r1 = lane + 32 < m ? rk[lane + 32] : -1;
  bool bad = (lane < n && (s0 < 0 || s0 >= n_docs)) || (lane + 32 < n && (s1 < 0 || s1 >= n_docs));
  bool fresh0 = lane < m && r0 >= 0 && r0 < n_docs;
  bool fresh1 = lane + 32 < m && r1 >= 0 && r1 < n_docs;
  for (int j = 0; j < n; ++j) {
    const int32_t sj = __shfl_sync(full, j < 32 ? s0 : s1, j & 31);
    bad |= (lane < n && j != lane && sj == s0) || (lane + 32 < n && j != lane + 32 && sj == s1);
    fresh0 &= r0 != sj;
    fresh1 &= r1 != sj;
  }
  // a ranked document already taken earlier in the ranking is not fresh either
  for (int j = 0; j < m; ++j) {
    const int32_t rj = __shfl_sync(full, j < 32 ? r0 : r1, j & 31);
    fresh0 &= !(j < lane && rj == r0);
    fresh1 &= !(j < lane + 32 && rj == r1);
  }
  for (int i = lane; i < n; i += 32) o[i] = od[i];
  const unsigned below = (1u << lane) - 1u;
  const unsigned m0 = __ballot_sync(full, fresh0), m1 = __ballot_sync(full, fresh1);
  const int pos0 = __popc(m0 & below), pos1 = __popc(m0) + __popc(m1 & below);
  if (fresh0 && pos0 < p) o[n + pos0] = r0;
  if (fresh1 && pos1 < p) o[n + pos1] = r1;
  const int filled = min(p, __popc(m0) + __popc(m1));
  for (int i = filled + lane; i < p; i += 32) o[n + i] = -1;
  if (__any_sync(full, bad || filled < p) && lane == 0) dev_flag(MSA_DEV_BAD_SET);
}

}  // namespace msa
