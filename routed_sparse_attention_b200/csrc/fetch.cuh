// Host-tier fetch on the device: the selected documents' pooled K/V rows
// gathered from pinned host memory into the staging buffer by one kernel.
//
// "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts", section
// "How MSA compresses and routes documents": at 100M tokens the content K/V
// stays in host DRAM and is fetched asynchronously when selected.  The copy
// path (msa_fetch_selected) needs the selection on the host first, so a layer
// whose decode waits for its own fetch pays a device -> host -> device round
// trip.  Here the GPU reads the selection itself and pulls each selected
// document's rows straight from the mapped host buffer over the host link, in
// stream order after the routing: nothing waits on the host.
//
// One CTA per (query, rank): the document's K chunks then V chunks are one
// contiguous run of 2 * n_c rows in the host tier, copied in 16-byte vectors
// into slot (b * top_k + r) of the staging buffer, the layout
// msa_fetch_selected writes.  Four loads per thread are in flight at a time,
// to cover the host link's latency.
#pragma once
#include <cstdint>

#include "msa_common.cuh"

namespace msa {

constexpr int kFetchThreads = 256;
constexpr int kFetchUnroll = 4;

struct FetchArgs {
  const int32_t* sel;             // (device) [B][top_k] selected documents
  const int64_t* doc_chunk_off;   // (device) [n_docs + 1]
  const uint4* host_kv;           // device address of the mapped host tier
  uint4* staging;                 // (device) [B * top_k][2 * max_doc_chunks][row]
  int64_t n_docs, n_chunks;
  int64_t row_vec;                // 16-byte vectors per pooled row of [H_kv][head_dim]
  int top_k, max_doc_chunks;
};

__global__ void __launch_bounds__(kFetchThreads) fetch_gather_kernel(const FetchArgs a) {
  const int64_t item = blockIdx.x;                          // b * top_k + r
  const int32_t doc = __ldg(a.sel + item);
  if (doc < 0 || doc >= a.n_docs) {
    if (threadIdx.x == 0) dev_flag(MSA_DEV_BAD_DOC);
    return;
  }
  const int64_t c0 = __ldg(a.doc_chunk_off + doc), c1 = __ldg(a.doc_chunk_off + doc + 1);
  const int64_t nc = c1 - c0;
  if (c0 < 0 || nc <= 0 || nc > a.max_doc_chunks || c1 > a.n_chunks) {
    if (threadIdx.x == 0) dev_flag(MSA_DEV_BAD_DOC);
    return;
  }
  const uint4* src = a.host_kv + 2 * c0 * a.row_vec;
  uint4* dst = a.staging + item * 2 * a.max_doc_chunks * a.row_vec;
  const int64_t n = 2 * nc * a.row_vec;
  for (int64_t i0 = threadIdx.x; i0 < n; i0 += kFetchUnroll * kFetchThreads) {
    uint4 v[kFetchUnroll];
#pragma unroll
    for (int u = 0; u < kFetchUnroll; ++u) {
      const int64_t i = i0 + (int64_t)u * kFetchThreads;
      if (i < n) v[u] = src[i];
    }
#pragma unroll
    for (int u = 0; u < kFetchUnroll; ++u) {
      const int64_t i = i0 + (int64_t)u * kFetchThreads;
      if (i < n) dst[i] = v[u];
    }
  }
}

}  // namespace msa
