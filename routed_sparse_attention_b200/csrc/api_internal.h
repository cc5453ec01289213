// Internal helpers shared by the host-side translation units of libmsa
// (hidden from the library's exported symbols).
#pragma once
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "msa.h"

namespace msa_host {

#define MSA_HIDDEN __attribute__((visibility("hidden")))

// Sets the thread's msa_last_error text (printf format) and returns s.
MSA_HIDDEN msa_status fail(msa_status s, const char* fmt, ...);
MSA_HIDDEN msa_status cuda_fail(cudaError_t e, const char* what);
MSA_HIDDEN msa_status check_layout(const msa_layout* L);
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int esize(const msa_layout* L) { return L->dtype == MSA_BF16 ? 2 : 4; }

// An NVTX range around one library call (route, fetch, decode, ...), so that
// profilers can attribute the kernels it launches; free when no tool listens.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace msa_host
