// Host layer of libmsa: argument checks, workspace carving and kernel
// launches behind the C ABI declared in include/msa.h.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <mutex>
#include <thread>
#include <vector>

#include "msa.h"
#include "msa_debug.h"
#include "api_internal.h"
#include "msa_common.cuh"
#include "encode.cuh"
#include "route.cuh"
#include "route_mma.cuh"
#include "decode.cuh"
#include "decode_mma.cuh"
#include "decode_tc.cuh"
#include "interleave.cuh"
#include "fetch.cuh"
#include "train.cuh"
#include "train_tc.cuh"

using namespace msa;

namespace msa_host {

thread_local std::string g_err;
thread_local int g_fail_copies = 0;     // test hook: copies to fail on purpose
thread_local cudaEvent_t g_scan_ev0 = nullptr, g_scan_ev1 = nullptr;   // scan timing hook

msa_status fail(msa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

msa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(MSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define MSA_CHECK_LAUNCH(what)                                   \
  do {                                                           \
    cudaError_t e_ = cudaGetLastError();                         \
    if (e_ != cudaSuccess) return cuda_fail(e_, what);           \
  } while (0)

// Launch with programmatic stream serialisation: the kernel may start while
// the kernel before it on the stream finishes, and waits for it in pdl_wait()
// before it reads that kernel's output.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
#define MSA_CHECK_PDL(call, what)                                \
  do {                                                           \
    cudaError_t e_ = (call);                                     \
    if (e_ != cudaSuccess) return cuda_fail(e_, what);           \
  } while (0)

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  return n;
}

msa_status check_layout(const msa_layout* L) {
  if (!L) return fail(MSA_ERR_INVALID_ARG, "layout is NULL");
  if (L->dtype != MSA_F32 && L->dtype != MSA_BF16) return fail(MSA_ERR_INVALID_ARG, "dtype %d", L->dtype);
  if (L->n_q_heads <= 0 || L->n_kv_heads <= 0 || L->n_q_heads % L->n_kv_heads)
    return fail(MSA_ERR_INVALID_ARG, "H_q=%d must be a positive multiple of H_kv=%d", L->n_q_heads, L->n_kv_heads);
  if (L->head_dim <= 0 || (L->head_dim & 1) || L->router_dim <= 0 || L->chunk_size <= 0)
    return fail(MSA_ERR_INVALID_ARG, "bad head_dim %d / router_dim %d / chunk_size %d", L->head_dim,
                L->router_dim, L->chunk_size);
  if (!(L->rope_theta > 0.0)) return fail(MSA_ERR_INVALID_ARG, "rope_theta must be > 0");
  return MSA_OK;
}

}  // namespace msa_host

using namespace msa_host;

namespace {

msa_status check_index(const msa_layout* L, const msa_index* I) {
  if (!I) return fail(MSA_ERR_INVALID_ARG, "index is NULL");
  if (I->n_docs <= 0 || I->n_chunks < I->n_docs || !I->doc_chunk_off || !I->kr)
    return fail(MSA_ERR_INVALID_ARG, "index: n_docs %lld, n_chunks %lld, CSR or Kr missing",
                (long long)I->n_docs, (long long)I->n_chunks);
  if (I->n_docs > INT_MAX - 1) return fail(MSA_ERR_UNSUPPORTED, "more than 2^31-2 documents");
  if (!aligned16(I->kr)) return fail(MSA_ERR_INVALID_ARG, "Kr not 16-byte aligned");
  if (!aligned16(I->kr_inv_norm)) return fail(MSA_ERR_INVALID_ARG, "kr_inv_norm not 16-byte aligned");
  if (I->kv_on_host) {
    if (!I->host_kv || !I->doc_chunk_off_host || I->max_doc_chunks <= 0)
      return fail(MSA_ERR_INVALID_ARG, "host tier needs host_kv, doc_chunk_off_host, max_doc_chunks");
  } else if (I->k && I->v && (!aligned16(I->k) || !aligned16(I->v))) {
    return fail(MSA_ERR_INVALID_ARG, "K/V not 16-byte aligned");
  }
  (void)L;
  return MSA_OK;
}

// Scan shapes the kernels implement: router_dim * element size == 256 bytes,
// H_kv in {4, 8}.
msa_status check_scan_shape(const msa_layout* L) {
  if (L->router_dim * esize(L) != 256)
    return fail(MSA_ERR_UNSUPPORTED, "router_dim * element size must be 256 bytes (got %d)",
                L->router_dim * esize(L));
  if (L->n_kv_heads != 4 && L->n_kv_heads != 8)
    return fail(MSA_ERR_UNSUPPORTED, "router scan supports H_kv = 4 or 8 (got %d)", L->n_kv_heads);
  return MSA_OK;
}

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename P> P* take(size_t bytes) {
    P* p = base ? reinterpret_cast<P*>(base + off) : nullptr;
    off += align_up(bytes);
    return p;
  }
};

// ------------------------------------------------------------ route plan
// Raises a kernel's dynamic shared-memory limit once per device.  `done` is
// that kernel's own bitmask of devices (one bit per device ordinal < 64).
template <typename K>
msa_status smem_attr_once(K kern, int bytes, std::atomic<uint64_t>& done, const char* what) {
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return MSA_OK;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e, what);
  done.fetch_or(bit, std::memory_order_release);
  return MSA_OK;
}

struct RoutePlan {
  int NQ, NQG, n_groups, n_cta, P;
  bool mma;                // tensor-core scan (many query rows, bf16 bank)
  int NQP, n_pass, n_tiles;
  __nv_bfloat16* ub;       // [n_pass][H_kv][2 NQP][d_r] hi / lo query rows
  double* qn2;             // [NQ][H_q] |Qr|^2 in fp64 for the re-scoring
  float* u;
  uint32_t* score;
  int* cta_first_doc;      // first document of each scan unit (CUDA-core scan) or tile (tensor cores)
  int64_t n_units;          // CUDA-core scan: units of unit_chunks chunks, claimed dynamically
  int unit_chunks;
  int* unit_counter;        // [n_groups] next unclaimed unit, zeroed by the prep kernel
  unsigned long long* cand;
  int* cand_cnt;
  int* band;
  int* band_cnt;
  unsigned long long* band_exact;
  int64_t* item_off;
  size_t bytes;
};

int scan_chunks_per_stage(const msa_layout* L) { return 32768 / (L->n_kv_heads * 256); }

RoutePlan plan_route(const msa_layout* L, int64_t D, int64_t C, int B, int T, int k, void* ws) {
  RoutePlan p{};
  p.NQ = B * T;
  p.NQG = p.NQ == 1 ? 1 : (p.NQ == 2 ? 2 : 4);
  p.n_groups = (p.NQ + p.NQG - 1) / p.NQG;
  const int64_t stages = (C + scan_chunks_per_stage(L) - 1) / scan_chunks_per_stage(L);
  p.n_cta = (int)std::max<int64_t>(1, std::min<int64_t>(2 * sm_count(), stages));
  // more than 4 query rows on a bf16 bank: one tensor-core pass per 128 rows
  // instead of one CUDA-core pass per 4
  p.mma = L->dtype == MSA_BF16 && p.NQ > 4;
  // rows per pass: 32, 64 or 128
  p.NQP = p.NQ <= 32 ? 32 : (p.NQ <= 64 ? 64 : kScanMaxRows);
  p.n_pass = (p.NQ + p.NQP - 1) / p.NQP;
  // the caller has checked that the tile count fits an int (check_route_args)
  p.n_tiles = (int)std::min<int64_t>((C + kScanTile - 1) / kScanTile, INT_MAX);
  if (p.mma) p.n_cta = std::max(1, std::min(sm_count(), p.n_tiles));
  p.P = (int)((D + kTopkSlice - 1) / kTopkSlice);
  // units of at least 4 stages, and at most 64 per CTA slot of the scan grid
  // (the unit table's size is then bounded whatever C is, which is what the
  // workspace size assumes)
  {
    const int64_t sch = scan_chunks_per_stage(L);
    const int64_t max_units = 64 * 2 * (int64_t)sm_count();
    int64_t uc = std::max<int64_t>(4 * sch, (C + max_units - 1) / max_units);
    uc = (uc + sch - 1) / sch * sch;
    p.unit_chunks = (int)std::min<int64_t>(uc, INT_MAX / 2);
    p.n_units = (C + p.unit_chunks - 1) / p.unit_chunks;
  }
  Carver c(ws);
  p.u = c.take<float>(sizeof(float) * p.NQ * L->n_kv_heads * L->router_dim);
  p.qn2 = c.take<double>(sizeof(double) * p.NQ * L->n_q_heads);
  p.score = c.take<uint32_t>(sizeof(uint32_t) * B * D);
  p.cta_first_doc = c.take<int>(sizeof(int) * (p.mma ? p.n_tiles : p.n_units));
  p.unit_counter = c.take<int>(sizeof(int) * p.n_groups);
  p.ub = p.mma ? c.take<__nv_bfloat16>(sizeof(__nv_bfloat16) * (size_t)p.n_pass * L->n_kv_heads * 2 *
                                       p.NQP * L->router_dim)
               : nullptr;
  p.cand = c.take<unsigned long long>(sizeof(unsigned long long) * (size_t)B * D);
  p.cand_cnt = c.take<int>(sizeof(int) * B);
  p.band = c.take<int>(sizeof(int) * B * D);
  p.band_cnt = c.take<int>(sizeof(int) * B);
  p.band_exact = c.take<unsigned long long>(sizeof(unsigned long long) * B * D);
  p.item_off = c.take<int64_t>(sizeof(int64_t) * B * (D + 1));
  p.bytes = c.off;
  return p;
}

template <typename T, int NQG, int HKV>
msa_status launch_scan_t(const RoutePlan& p, const msa_index* I, int T_tok, cudaStream_t st) {
  using Cfg = ScanCfg<T, NQG, HKV>;
  auto kern = kr_scan_kernel<T, NQG, HKV>;
  static std::atomic<uint64_t> attr_done{0};
  if (msa_status s = smem_attr_once(kern, Cfg::SMEM, attr_done, "scan smem attribute")) return s;
  dim3 grid(p.n_cta, p.n_groups);
  MSA_CHECK_PDL(launch_pdl(kern, grid, dim3(Cfg::THREADS), Cfg::SMEM, st, reinterpret_cast<const T*>(I->kr), p.u,
                           p.NQ, T_tok, I->doc_chunk_off, I->n_chunks, p.cta_first_doc, p.n_units, p.unit_chunks,
                           p.unit_counter, p.score, I->n_docs),
                "kr_scan_kernel");
  return MSA_OK;
}

template <typename T>
msa_status launch_scan_nqg(const msa_layout* L, const RoutePlan& p, const msa_index* I, int T_tok,
                           cudaStream_t st) {
  const int hkv = L->n_kv_heads;
#define MSA_SCAN_CASE(NQG_, HKV_) \
  if (p.NQG == NQG_ && hkv == HKV_) return launch_scan_t<T, NQG_, HKV_>(p, I, T_tok, st);
  MSA_SCAN_CASE(1, 4) MSA_SCAN_CASE(2, 4) MSA_SCAN_CASE(4, 4)
  MSA_SCAN_CASE(1, 8) MSA_SCAN_CASE(2, 8) MSA_SCAN_CASE(4, 8)
#undef MSA_SCAN_CASE
  return fail(MSA_ERR_UNSUPPORTED, "no scan kernel for H_kv %d", L->n_kv_heads);
}

msa_status make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                    const cuuint64_t* strides, const cuuint32_t* box,
                    CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B,
                    CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);

template <int NQP>
msa_status launch_scan_mma(const msa_layout* L, const msa_index* I, const RoutePlan& p, int T_tok, cudaStream_t st) {
  using Cfg = ScanMmaCfg<NQP>;
  ScanMmaArgs a;
  memset(&a, 0, sizeof a);
  const int dr = L->router_dim, H = L->n_kv_heads;
  const cuuint64_t kdims[3] = {(cuuint64_t)dr, (cuuint64_t)H, (cuuint64_t)I->n_chunks};
  const cuuint64_t kstr[2] = {(cuuint64_t)dr * 2, (cuuint64_t)H * dr * 2};
  const cuuint32_t kbox[3] = {64, 1, kScanTile};
  msa_status s = make_map(&a.tm_kr, I->kr, 3, kdims, kstr, kbox);
  if (s) return s;
  const cuuint64_t udims[2] = {(cuuint64_t)dr, (cuuint64_t)p.n_pass * H * Cfg::NP2};
  const cuuint64_t ustr[1] = {(cuuint64_t)dr * 2};
  const cuuint32_t ubox[2] = {64, (cuuint32_t)Cfg::NP2};
  if ((s = make_map(&a.tm_u, p.ub, 2, udims, ustr, ubox))) return s;
  a.doc_chunk_off = I->doc_chunk_off;
  a.tile_first_doc = p.cta_first_doc;
  a.score = p.score;
  a.rnorm = I->kr_inv_norm;
  a.P = (int64_t)p.n_tiles * kScanTile;
  a.C = I->n_chunks;
  a.D = I->n_docs;
  a.Hkv = H;
  a.NQ = p.NQ;
  a.Ttok = T_tok;
  a.n_tiles = p.n_tiles;
  auto kern = kr_scan_mma_kernel<NQP>;
  static std::atomic<uint64_t> attr_done{0};
  if (msa_status s = smem_attr_once(kern, Cfg::SMEM, attr_done, "tensor-core scan smem attribute")) return s;
  for (int pass = 0; pass < p.n_pass; ++pass) {
    a.pass = pass;
    kern<<<p.n_cta, kScanMmaThreads, Cfg::SMEM, st>>>(a);
    MSA_CHECK_LAUNCH("kr_scan_mma_kernel");
  }
  return MSA_OK;
}

template <typename T>
msa_status route_front(const msa_layout* L, const msa_index* I, int B, int T_tok, const void* qr,
                       const RoutePlan& p, cudaStream_t st) {
  const int prep_blocks = std::max(p.NQ * L->n_kv_heads, 2 * sm_count());
  const int G = L->n_q_heads / L->n_kv_heads;
  const size_t prep_smem = sizeof(float) * (G * L->router_dim + G);
  route_prep_kernel<T><<<prep_blocks, kPrepThreads, prep_smem, st>>>(
      reinterpret_cast<const T*>(qr), p.NQ, L->n_q_heads, L->n_kv_heads, L->router_dim, p.u, p.score,
      (int64_t)B * I->n_docs, I->doc_chunk_off, I->n_docs, I->n_chunks, p.mma ? (int)p.n_tiles : (int)p.n_units,
      p.cta_first_doc, p.cand_cnt, B, p.mma ? kScanTile : p.unit_chunks, p.qn2, p.unit_counter,
      p.mma ? 0 : p.n_groups);
  MSA_CHECK_LAUNCH("route_prep_kernel");
  if (p.mma) {
    const int64_t n = (int64_t)p.n_pass * L->n_kv_heads * p.NQP * L->router_dim;
    u_split_kernel<<<(int)std::min<int64_t>((n + 255) / 256, 1024), 256, 0, st>>>(
        p.u, p.NQ, L->n_kv_heads, L->router_dim, p.NQP, p.n_pass, p.ub);
    MSA_CHECK_LAUNCH("u_split_kernel");
  }
  const bool timed = g_scan_ev0 && g_scan_ev1;
  if (timed && cudaEventRecord(g_scan_ev0, st) != cudaSuccess) return fail(MSA_ERR_CUDA, "record scan start");
  msa_status s;
  if (p.mma) {
    if (p.NQP == 32) s = launch_scan_mma<32>(L, I, p, T_tok, st);
    else if (p.NQP == 64) s = launch_scan_mma<64>(L, I, p, T_tok, st);
    else s = launch_scan_mma<kScanMaxRows>(L, I, p, T_tok, st);
  } else {
    s = launch_scan_nqg<T>(L, p, I, T_tok, st);
  }
  if (s) return s;
  if (timed && cudaEventRecord(g_scan_ev1, st) != cudaSuccess) return fail(MSA_ERR_CUDA, "record scan stop");
  return MSA_OK;
}

template <typename T>
msa_status route_back(const msa_layout* L, const msa_index* I, int B, int T_tok, const void* qr, int k,
                      const RoutePlan& p, int32_t* out_idx, double* out_score, cudaStream_t st) {
  const int64_t D = I->n_docs;
  MSA_CHECK_PDL(launch_pdl(topk_local_kernel, dim3(p.P, B), dim3(kTopkThreads), 0, st, p.score, D, k, p.cand,
                           p.cand_cnt),
                "topk_local_kernel");
  MSA_CHECK_PDL(launch_pdl(merge_band_kernel, dim3(B), dim3(kMergeThreads), 0, st, D, k, T_tok, p.cand, p.cand_cnt,
                           I->doc_chunk_off, p.band, p.band_cnt, p.band_exact, p.item_off),
                "merge_band_kernel");
  const size_t smem = sizeof(double) * (kRescoreThreads / 32) * (L->n_q_heads + L->n_kv_heads) + sizeof(int64_t) * (B + 1) +
                      sizeof(int) * (2 * B + 2) + sizeof(int64_t) * kRescoreSmemItems;
  // enough warps for every band item of a typical call at once: each item is
  // one latency-bound fp64 chain per lane
  MSA_CHECK_PDL(launch_pdl(rescore_kernel<T>, dim3(8 * sm_count()), dim3(kRescoreThreads), smem, st,
                           reinterpret_cast<const T*>(qr), reinterpret_cast<const T*>(I->kr), B, T_tok, L->n_q_heads,
                           L->n_kv_heads, L->router_dim, D, I->doc_chunk_off, p.band, p.band_cnt, p.item_off, p.qn2,
                           p.band_exact),
                "rescore_kernel");
  MSA_CHECK_PDL(launch_pdl(final_select_kernel, dim3(B), dim3(kFinalThreads), 0, st, D, k, p.band, p.band_cnt,
                           p.band_exact, out_idx, out_score),
                "final_select_kernel");
  return MSA_OK;
}

msa_status check_route_args(const msa_layout* L, const msa_index* I, int B, int T, const void* qr) {
  msa_status s = check_layout(L);
  if (s) return s;
  if ((s = check_index(L, I))) return s;
  if ((s = check_scan_shape(L))) return s;
  if (B <= 0 || T <= 0) return fail(MSA_ERR_INVALID_ARG, "batch %d and T %d must be >= 1", B, T);
  if (B > kRouteMaxB) return fail(MSA_ERR_UNSUPPORTED, "batch %d (up to %d queries per call)", B, kRouteMaxB);
  if (!qr) return fail(MSA_ERR_INVALID_ARG, "qr is NULL");
  if ((int64_t)B * I->n_docs > (int64_t)INT_MAX * 8)
    return fail(MSA_ERR_UNSUPPORTED, "batch x documents too large");
  if ((I->n_chunks + kScanTile - 1) / kScanTile > INT_MAX)
    return fail(MSA_ERR_UNSUPPORTED, "%lld pooled chunks are too many", (long long)I->n_chunks);
  if ((int64_t)L->n_q_heads * (L->router_dim + 1) * 4 > 48 * 1024)
    return fail(MSA_ERR_UNSUPPORTED, "H_q x router_dim too large for the query prep");
  return MSA_OK;
}

// ------------------------------------------------------------ decode plan
struct DecodePlan {
  int S, n_rg, R, s_tot;
  std::vector<int64_t> len;  // live local tokens per query
  int rpc;                 // query rows per CTA
  int wr;                  // tensor-core path: m16 row blocks per CTA (0: CUDA-core kernel)
  bool tc;                 // 128-row CTAs on the 5th-generation tensor cores (decode_tc_kernel)
  int64_t max_ltot;
  std::vector<int32_t> split_off;
  int* counters;
  float* part_o;
  float* part_ml;
  size_t bytes;
};

msa_status plan_decode(const msa_layout* L, int B, int T, const int64_t* loff, const int64_t* llen, void* ws,
                       DecodePlan* p) {
  if (B <= 0 || B > kDecMaxB) return fail(MSA_ERR_UNSUPPORTED, "batch %d (1..%d supported)", B, kDecMaxB);
  if (T <= 0) return fail(MSA_ERR_INVALID_ARG, "T %d", T);
  if (!loff) return fail(MSA_ERR_INVALID_ARG, "local_off_host is NULL");
  p->R = (L->n_q_heads / L->n_kv_heads) * T;
  int64_t tot = 0;
  p->max_ltot = 0;
  p->len.assign(B, 0);
  if (loff[0] != 0) return fail(MSA_ERR_INVALID_ARG, "local_off_host[0] must be 0");
  for (int b = 0; b < B; ++b) {
    const int64_t cap = loff[b + 1] - loff[b];
    const int64_t lt = llen ? llen[b] : cap;
    if (lt < T) return fail(MSA_ERR_INVALID_ARG, "query %d holds %lld live local rows < T=%d", b, (long long)lt, T);
    if (lt > cap)
      return fail(MSA_ERR_INVALID_ARG, "query %d: live length %lld exceeds its capacity %lld", b, (long long)lt,
                  (long long)cap);
    p->len[b] = lt;
    tot += lt;
    p->max_ltot = std::max(p->max_ltot, lt);
  }
  // bf16 banks take the tensor-core kernel; its TMA row maps need at least one
  // whole 64-row box and int32 row coordinates
  const int64_t rows = loff[B] * L->n_kv_heads;
  p->wr = 0;
  p->tc = false;
  if (L->dtype == MSA_BF16 && rows >= kDecTile && rows + kDecTile < INT_MAX) {
    // many rows per kv head: M = 128 rows on tcgen05 (a CTA's rows are whole
    // tokens of at most 32, so G divides 128 and is at least 4)
    const int G = L->n_q_heads / L->n_kv_heads;
    if (L->head_dim == 128 && p->R > 64 && G >= 4 && kTcRows % G == 0) {
      p->tc = true;
      p->wr = kTcRows / 16;
    } else {
      p->wr = p->R <= 16 ? 1 : 2;
    }
  }
  p->rpc = p->wr ? 16 * p->wr : kDecRows;
  p->n_rg = (p->R + p->rpc - 1) / p->rpc;
  const int max_splits = kDecMaxSplits;
  // split size: local-key CTAs per SM over all (query, kv head, row group), in
  // whole 64-key tiles; each query's memory split comes on top.  A single
  // query is latency-bound and runs in one wave, its memory-split CTAs
  // counted: one CTA per SM at one token (4 rows per kv head; its last CTA
  // merges the splits, one L2 round trip per 16), two at several tokens
  // (T = 64: 58 us at one per SM, 38 us at two, 44-46 us at three or four).
  // Batches take six: with ragged local lengths the shorter splits even out
  // the CTAs' finish times (batch 32 over 1024..8192 tokens: 136 us at two
  // per SM, 124 us at six, the same at eight and twelve).
  const int64_t units = (int64_t)L->n_kv_heads * p->n_rg;
  // the tensor-core CTAs hold ~195 KB of shared memory: one per SM
  const int64_t per_sm = p->tc ? 1 : (B == 1 ? (p->R > 16 ? 2 : 1) : 6);
  const int64_t target = std::max<int64_t>(per_sm * sm_count(), units);
  int64_t S = (tot * units + target - 1) / target;
  S = (S + kDecTile - 1) / kDecTile * kDecTile;
  S = std::max<int64_t>(kDecTile, std::min<int64_t>(S, 16384));
  S = std::max<int64_t>(S, (p->max_ltot + max_splits - 2) / (max_splits - 1));   // splits per query within the cap
  S = (S + kDecTile - 1) / kDecTile * kDecTile;
  if (B == 1)                      // one wave: the memory split's CTAs count too
    while (S < 16384 && (1 + (p->len[0] + S - 1) / S) * units > target) S += kDecTile;
  p->S = (int)S;
  p->split_off.assign(B + 1, 0);
  for (int b = 0; b < B; ++b) {
    const int64_t lt = p->len[b];
    const int64_t ns = 1 + (lt + S - 1) / S;
    if (ns > max_splits) return fail(MSA_ERR_UNSUPPORTED, "query %d: %lld local rows are too many", b, (long long)lt);
    p->split_off[b + 1] = p->split_off[b] + (int)ns;
  }
  p->s_tot = p->split_off[B];
  Carver c(ws);
  p->counters = c.take<int>(sizeof(int) * (size_t)B * L->n_kv_heads * p->n_rg);
  p->part_o = c.take<float>(sizeof(float) * (size_t)p->s_tot * L->n_kv_heads * p->R * L->head_dim);
  p->part_ml = c.take<float>(sizeof(float) * (size_t)p->s_tot * L->n_kv_heads * p->R * 2);
  p->bytes = c.off;
  return MSA_OK;
}

template <typename T, int D>
msa_status launch_decode(const DecodeArgs& a, const DecodePlan& p, cudaStream_t st) {
  auto kern = decode_kernel<T, D>;
  const int smem = (int)sizeof(DecSmem<T, D>);
  static std::atomic<uint64_t> attr_done{0};
  if (msa_status s = smem_attr_once(kern, smem, attr_done, "decode smem attribute")) return s;
  dim3 grid(p.s_tot, a.Hkv * p.n_rg);
  kern<<<grid, kDecThreads, smem, st>>>(a);
  MSA_CHECK_LAUNCH("decode_kernel");
  return MSA_OK;
}

// ---- TMA row maps for the tensor-core decode
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn tensor_map_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Tensor of `rank` dims (innermost first), bf16 and the 128-byte swizzle
// unless told otherwise, zero fill outside the tensor.
msa_status make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                    const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swizzle,
                    CUtensorMapDataType dtype) {
  EncodeTiledFn fn = tensor_map_encoder();
  if (!fn) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, dtype, (cuuint32_t)rank, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MSA_OK;
}

// [rows][d] bf16 rows, boxes of 64 rows x 64 elements.
msa_status make_row_map(CUtensorMap* m, const void* base, int64_t rows, int d) {
  const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  const cuuint32_t box[2] = {64, 64};
  return make_map(m, base, 2, dims, strides, box);
}

template <int D, int WR>
msa_status launch_decode_mma(const DecodeMmaArgs& A, const DecodePlan& p, cudaStream_t st) {
  auto kern = decode_mma_kernel<D, WR>;
  const int smem = (int)sizeof(DecMmaSmem<D>) + 1024;      // + room to align the tiles to 1 KiB
  static std::atomic<uint64_t> attr_done{0};
  if (msa_status s = smem_attr_once(kern, smem, attr_done, "decode smem attribute")) return s;
  dim3 grid(p.s_tot, A.d.Hkv * p.n_rg);
  kern<<<grid, kMmaThreads, smem, st>>>(A);
  MSA_CHECK_LAUNCH("decode_mma_kernel");
  return MSA_OK;
}

msa_status launch_decode_tc(const DecodeMmaArgs& A, const DecodePlan& p, cudaStream_t st) {
  const int smem = (int)sizeof(DecTcSmem) + 1024;          // + room to align the tiles to 1 KiB
  static std::atomic<uint64_t> attr_done{0};
  if (msa_status s = smem_attr_once(decode_tc_kernel, smem, attr_done, "tensor-core decode smem attribute")) return s;
  dim3 grid(p.s_tot, A.d.Hkv * p.n_rg);
  decode_tc_kernel<<<grid, kTcThreads, smem, st>>>(A);
  MSA_CHECK_LAUNCH("decode_tc_kernel");
  const unsigned merge_ctas = (unsigned)((int64_t)A.d.B * A.d.Hkv * p.n_rg * (kTcRows / kTcMergeRows));
  MSA_CHECK_PDL(launch_pdl(decode_tc_merge_kernel, dim3(merge_ctas), dim3(kMmaThreads), 0, st, A.d),
                "decode_tc_merge_kernel");
  return MSA_OK;
}

template <int D>
msa_status launch_decode_mma_d(const DecodeArgs& a, const DecodePlan& p, int64_t rows, cudaStream_t st) {
  DecodeMmaArgs A;
  memset(&A, 0, sizeof A);
  msa_status s = make_row_map(&A.tm_k, a.lk, rows, D);
  if (s) return s;
  if ((s = make_row_map(&A.tm_v, a.lv, rows, D))) return s;
  A.d = a;
  if constexpr (D == 128)
    if (p.tc) {
      // Q [B * T][Hq][128] unswizzled; a box is one CTA's 128 rows (128 / G tokens x G heads)
      const cuuint64_t qdims[3] = {128, (cuuint64_t)a.Hq, (cuuint64_t)a.B * a.T};
      const cuuint64_t qstr[2] = {256, (cuuint64_t)a.Hq * 256};
      const cuuint32_t qbox[3] = {128, (cuuint32_t)a.G, (cuuint32_t)(kTcRows / a.G)};
      if ((s = make_map(&A.tm_q, a.q, 3, qdims, qstr, qbox, CU_TENSOR_MAP_SWIZZLE_NONE))) return s;
      return launch_decode_tc(A, p, st);
    }
  if (p.wr == 1) return launch_decode_mma<D, 1>(A, p, st);
  return launch_decode_mma<D, 2>(A, p, st);
}

}  // namespace

// =================================================================== C ABI
extern "C" {

int msa_version(void) { return 1; }

const char* msa_last_error(void) { return g_err.c_str(); }

const char* msa_status_string(msa_status s) {
  switch (s) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_ARG: return "invalid argument";
    case MSA_ERR_UNSUPPORTED: return "unsupported shape";
    case MSA_ERR_CUDA: return "CUDA error";
    case MSA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MSA_ERR_TIMEOUT: return "timeout";
    case MSA_ERR_INTERNAL: return "internal error";
  }
  return "unknown status";
}

msa_status msa_device_status(uint32_t* bits, cudaStream_t stream) {
  if (!bits) return fail(MSA_ERR_INVALID_ARG, "bits is NULL");
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream sync");
  unsigned int v = 0, z = 0;
  if ((e = cudaMemcpyFromSymbol(&v, g_dev_status, sizeof v)) != cudaSuccess) return cuda_fail(e, "read status");
  if ((e = cudaMemcpyToSymbol(g_dev_status, &z, sizeof z)) != cudaSuccess) return cuda_fail(e, "clear status");
  *bits = v;
  return MSA_OK;
}

msa_status msa_chunk_offsets(int64_t n_docs, const int64_t* tok, int32_t chunk, int64_t* out,
                             int32_t* max_doc_chunks, int64_t* max_doc_len) {
  if (n_docs <= 0 || !tok || !out || chunk <= 0)
    return fail(MSA_ERR_INVALID_ARG, "n_docs %lld, chunk %d", (long long)n_docs, chunk);
  if (tok[0] != 0) return fail(MSA_ERR_INVALID_ARG, "doc_tok_off[0] must be 0");
  int64_t mx = 0, mxl = 0;
  out[0] = 0;
  for (int64_t s = 0; s < n_docs; ++s) {
    const int64_t L = tok[s + 1] - tok[s];
    if (L <= 0) return fail(MSA_ERR_INVALID_ARG, "document %lld holds %lld tokens", (long long)s, (long long)L);
    const int64_t n = (L + chunk - 1) / chunk;
    out[s + 1] = out[s] + n;
    mx = std::max(mx, n);
    mxl = std::max(mxl, L);
  }
  if (mx > INT_MAX) return fail(MSA_ERR_UNSUPPORTED, "document too long");
  if (max_doc_chunks) *max_doc_chunks = (int32_t)mx;
  if (max_doc_len) *max_doc_len = mxl;
  return MSA_OK;
}

msa_status msa_rope_table(const msa_layout* L, int32_t n_pos, float* table, cudaStream_t stream) {
  msa_status s = check_layout(L);
  if (s) return s;
  if (n_pos <= 0 || !table || !aligned16(table)) return fail(MSA_ERR_INVALID_ARG, "n_pos %d / table", n_pos);
  const long long n = (long long)n_pos * (L->head_dim / 2);
  const int blocks = (int)std::min<long long>((n + 255) / 256, 4096);
  rope_table_kernel<<<blocks, 256, 0, stream>>>(n_pos, L->head_dim, L->rope_theta, reinterpret_cast<float2*>(table));
  MSA_CHECK_LAUNCH("rope_table_kernel");
  return MSA_OK;
}

static msa_status encode_common(const msa_layout* L, int64_t n_docs, int64_t n_chunks, const int64_t* tok_off,
                                const int64_t* chunk_off, int64_t max_doc_len, const void* k_tok, const void* v_tok,
                                const void* kr_tok, const float* rope, int32_t rope_rows, void* k_pool, void* v_pool,
                                void* kr_pool, int kv_interleaved, cudaStream_t stream) {
  msa_status s = check_layout(L);
  if (s) return s;
  if (n_docs <= 0 || n_chunks < n_docs || !tok_off || !chunk_off || !k_tok || !v_tok || !kr_tok || !rope ||
      !k_pool || !v_pool || !kr_pool)
    return fail(MSA_ERR_INVALID_ARG, "encode: missing pointer or empty bank");
  if (n_docs > INT_MAX) return fail(MSA_ERR_UNSUPPORTED, "too many documents");
  const void* ptrs[] = {k_tok, v_tok, kr_tok, rope, k_pool, v_pool, kr_pool};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(MSA_ERR_INVALID_ARG, "encode: pointer not 16-byte aligned");
  if (max_doc_len <= 0 || rope_rows < max_doc_len)
    return fail(MSA_ERR_INVALID_ARG, "rope_rows %d < longest document %lld", rope_rows, (long long)max_doc_len);
  const int V = L->dtype == MSA_BF16 ? 8 : 4;
  if ((L->head_dim / 2) % V || (L->router_dim / 2) % V)
    return fail(MSA_ERR_UNSUPPORTED, "head_dim/2 and router_dim/2 must be multiples of %d", V);
  const int TK = L->n_kv_heads * (L->head_dim / 2) / V, TR = L->n_kv_heads * (L->router_dim / 2) / V;
  const int threads = 2 * TK + TR;
  if (threads > kEncThreads - 32)
    return fail(MSA_ERR_UNSUPPORTED, "encode: %d consumer threads per CTA (> %d)", threads, kEncThreads - 32);
  EncodeArgs a{};
  a.doc_tok_off = tok_off; a.doc_chunk_off = chunk_off; a.k_tok = k_tok; a.v_tok = v_tok; a.kr_tok = kr_tok;
  a.rope = reinterpret_cast<const float2*>(rope); a.k_pool = k_pool; a.v_pool = v_pool; a.kr_pool = kr_pool;
  a.n_docs = n_docs; a.rope_rows = rope_rows; a.H = L->n_kv_heads; a.d = L->head_dim; a.dr = L->router_dim;
  a.chunk = L->chunk_size; a.kv_interleaved = kv_interleaved;
  a.stage_bytes = kEncStageTok * ((2 * L->n_kv_heads * L->head_dim + L->n_kv_heads * L->router_dim) * esize(L) +
                                  (L->head_dim / 2) * (int)sizeof(float2));     // + the stage's rotary rows
  a.stage_bytes = (a.stage_bytes + 127) / 128 * 128;
  const int budget = 72 * 1024;                  // three CTAs per SM
  a.n_stages = std::min(kEncMaxStages, budget / a.stage_bytes);
  if (a.n_stages < 2) return fail(MSA_ERR_UNSUPPORTED, "encode: %d-byte stages too large", a.stage_bytes);
  const int smem = a.n_stages * a.stage_bytes + 2 * kEncMaxStages * 8 + kEncMaxStages * 32;
  const unsigned grid = (unsigned)std::min<int64_t>(n_docs, 3 * sm_count());
  static std::atomic<uint64_t> attr_done[2];
  if (L->dtype == MSA_BF16) {
    if ((s = smem_attr_once(encode_pool_kernel<__nv_bfloat16>, smem, attr_done[0], "encode smem"))) return s;
    encode_pool_kernel<__nv_bfloat16><<<grid, kEncThreads, smem, stream>>>(a);
  } else {
    if ((s = smem_attr_once(encode_pool_kernel<float>, smem, attr_done[1], "encode smem"))) return s;
    encode_pool_kernel<float><<<grid, kEncThreads, smem, stream>>>(a);
  }
  MSA_CHECK_LAUNCH("encode_pool_kernel");
  return MSA_OK;
}

msa_status msa_encode_memory(const msa_layout* L, int64_t n_docs, int64_t n_chunks, const int64_t* tok_off,
                             const int64_t* chunk_off, int64_t max_doc_len, const void* k_tok,
                             const void* v_tok, const void* kr_tok, const float* rope, int32_t rope_rows,
                             void* k_pool, void* v_pool, void* kr_pool, cudaStream_t stream) {
  NvtxRange nvtx_("msa_encode_memory");
  return encode_common(L, n_docs, n_chunks, tok_off, chunk_off, max_doc_len, k_tok, v_tok, kr_tok, rope, rope_rows,
                       k_pool, v_pool, kr_pool, 0, stream);
}

msa_status msa_encode_memory_kv_interleaved(const msa_layout* L, int64_t n_docs, int64_t n_chunks,
                                            const int64_t* tok_off, const int64_t* chunk_off, int64_t max_doc_len,
                                            const void* k_tok, const void* v_tok, const void* kr_tok,
                                            const float* rope, int32_t rope_rows, void* kv_pool, void* kr_pool,
                                            cudaStream_t stream) {
  NvtxRange nvtx_("msa_encode_memory_kv_interleaved");
  return encode_common(L, n_docs, n_chunks, tok_off, chunk_off, max_doc_len, k_tok, v_tok, kr_tok, rope, rope_rows,
                       kv_pool, kv_pool, kr_pool, 1, stream);
}

size_t msa_route_workspace_size(const msa_layout* L, int64_t n_docs, int64_t n_chunks, int32_t batch, int32_t T,
                                int32_t top_k) {
  if (!L || n_docs <= 0 || n_chunks < n_docs || batch <= 0 || T <= 0 || top_k <= 0 || L->n_kv_heads <= 0) return 0;
  if ((n_chunks + kScanTile - 1) / kScanTile > INT_MAX) return 0;
  // the tensor-core scan keeps one entry per 128-chunk tile, so the size
  // depends on the chunk count as well as on the documents
  RoutePlan p = plan_route(L, n_docs, n_chunks, batch, T, top_k, nullptr);
  return p.bytes;
}

msa_status msa_route(const msa_layout* L, const msa_index* I, int32_t B, int32_t T, const void* qr,
                     int32_t k, int32_t* out_idx, double* out_score, int32_t* out_idx_host, void* ws,
                     size_t ws_bytes, cudaStream_t st) {
  NvtxRange nvtx_("msa_route");
  msa_status s = check_route_args(L, I, B, T, qr);
  if (s) return s;
  if (k < 1 || k > kMaxTopK || k > I->n_docs)
    return fail(MSA_ERR_INVALID_ARG, "top_k %d must be in [1, min(n_docs, %d)]", k, kMaxTopK);
  if (!out_idx) return fail(MSA_ERR_INVALID_ARG, "out_doc_idx is NULL");
  // the plan that carves the workspace is the one checked against its size
  RoutePlan p = plan_route(L, I->n_docs, I->n_chunks, B, T, k, ws);
  if (!ws || ws_bytes < p.bytes)
    return fail(MSA_ERR_WORKSPACE_TOO_SMALL, "route workspace %zu < %zu bytes", ws_bytes, p.bytes);
  if (L->dtype == MSA_BF16) {
    if ((s = route_front<__nv_bfloat16>(L, I, B, T, qr, p, st))) return s;
    if ((s = route_back<__nv_bfloat16>(L, I, B, T, qr, k, p, out_idx, out_score, st))) return s;
  } else {
    if ((s = route_front<float>(L, I, B, T, qr, p, st))) return s;
    if ((s = route_back<float>(L, I, B, T, qr, k, p, out_idx, out_score, st))) return s;
  }
  if (out_idx_host) {
    cudaError_t e = cudaMemcpyAsync(out_idx_host, out_idx, sizeof(int32_t) * B * k, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(e, "copy selected indices to host");
  }
  return MSA_OK;
}

}  // extern "C"

// ----------------------------------------------------------- no-alloc routing
// Built-in routing scratch for callers that may not allocate device memory.
// Host code must not pass the array's name to a kernel (on the host it is only
// a stand-in); its device address is looked up once per device below.
static __device__ __align__(256) unsigned char g_route_scratch[MSA_ROUTE_NOALLOC_MAX_BYTES];

namespace {
constexpr int kMaxScratchDevices = 64;
void* g_scratch_dev_ptr[kMaxScratchDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_route_scratch on the current device (looked up on the
// first call per device, with that device current).
msa_status route_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxScratchDevices) return fail(MSA_ERR_UNSUPPORTED, "device %d beyond %d", dev, kMaxScratchDevices);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_dev_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess || !p) return cuda_fail(e, "cudaGetSymbolAddress(route scratch)");
    g_scratch_dev_ptr[dev] = p;
  }
  *out = g_scratch_dev_ptr[dev];
  return MSA_OK;
}
}  // namespace

extern "C" {

msa_status msa_route_noalloc(const msa_layout* L, const msa_index* I, int32_t B, int32_t T, const void* qr,
                             int32_t k, int32_t* out_idx, double* out_score, int32_t* out_idx_host,
                             cudaStream_t st) {
  msa_status s = check_route_args(L, I, B, T, qr);
  if (s) return s;
  if (k < 1 || k > kMaxTopK || k > I->n_docs)
    return fail(MSA_ERR_INVALID_ARG, "top_k %d must be in [1, min(n_docs, %d)]", k, kMaxTopK);
  const size_t need = plan_route(L, I->n_docs, I->n_chunks, B, T, k, nullptr).bytes;
  if (need > MSA_ROUTE_NOALLOC_MAX_BYTES)
    return fail(MSA_ERR_WORKSPACE_TOO_SMALL,
                "routing %lld documents x %d queries needs %zu bytes of scratch; the built-in scratch "
                "holds %zu -- use msa_route with a caller workspace", (long long)I->n_docs, B, need,
                (size_t)MSA_ROUTE_NOALLOC_MAX_BYTES);
  void* ws = nullptr;
  if ((s = route_scratch(&ws))) return s;
  return msa_route(L, I, B, T, qr, k, out_idx, out_score, out_idx_host, ws, MSA_ROUTE_NOALLOC_MAX_BYTES, st);
}

msa_status msa_route_scores(const msa_layout* L, const msa_index* I, int32_t B, int32_t T, const void* qr,
                            float* out, void* ws, size_t ws_bytes, cudaStream_t st) {
  msa_status s = check_route_args(L, I, B, T, qr);
  if (s) return s;
  if (!out) return fail(MSA_ERR_INVALID_ARG, "out_doc_score is NULL");
  RoutePlan p = plan_route(L, I->n_docs, I->n_chunks, B, T, 1, ws);
  if (!ws || ws_bytes < p.bytes)
    return fail(MSA_ERR_WORKSPACE_TOO_SMALL, "route workspace %zu < %zu bytes", ws_bytes, p.bytes);
  if (L->dtype == MSA_BF16) s = route_front<__nv_bfloat16>(L, I, B, T, qr, p, st);
  else s = route_front<float>(L, I, B, T, qr, p, st);
  if (s) return s;
  scores_to_float_kernel<<<2 * sm_count(), 256, 0, st>>>(p.score, (int64_t)B * I->n_docs, out);
  MSA_CHECK_LAUNCH("scores_to_float_kernel");
  return MSA_OK;
}

size_t msa_fetch_staging_size(const msa_layout* L, const msa_index* I, int32_t B, int32_t k) {
  if (!L || !I || B <= 0 || k <= 0 || I->max_doc_chunks <= 0) return 0;
  return (size_t)B * k * 2 * I->max_doc_chunks * L->n_kv_heads * L->head_dim * esize(L);
}

void msa_debug_fail_next_copies(int32_t n) { g_fail_copies = n; }

void msa_debug_scan_events(cudaEvent_t start, cudaEvent_t stop) {
  g_scan_ev0 = start;
  g_scan_ev1 = stop;
}

msa_status msa_fetch_selected(const msa_layout* L, const msa_index* I, int32_t B, int32_t k,
                              const int32_t* sel_host, cudaEvent_t sel_ready, int32_t timeout_ms,
                              void* staging, size_t staging_bytes, cudaStream_t fetch_stream,
                              cudaEvent_t fetch_done) {
  NvtxRange nvtx_("msa_fetch_selected");
  msa_status s = check_layout(L);
  if (s) return s;
  if ((s = check_index(L, I))) return s;
  if (!I->kv_on_host) return fail(MSA_ERR_INVALID_ARG, "index is not host-resident");
  if (B <= 0 || k <= 0 || !sel_host || !staging) return fail(MSA_ERR_INVALID_ARG, "fetch arguments");
  const size_t need = msa_fetch_staging_size(L, I, B, k);
  if (staging_bytes < need) return fail(MSA_ERR_WORKSPACE_TOO_SMALL, "staging %zu < %zu bytes", staging_bytes, need);
  if (sel_ready) {
    const auto t0 = std::chrono::steady_clock::now();
    for (;;) {
      cudaError_t e = cudaEventQuery(sel_ready);
      if (e == cudaSuccess) break;
      if (e != cudaErrorNotReady) return cuda_fail(e, "query sel_ready");
      const auto ms = std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0).count();
      if (ms >= timeout_ms) return fail(MSA_ERR_TIMEOUT, "selected indices not ready after %d ms", timeout_ms);
      std::this_thread::yield();
    }
  }
  const size_t row = (size_t)L->n_kv_heads * L->head_dim * esize(L);
  const char* host = static_cast<const char*>(I->host_kv);
  char* dst = static_cast<char*>(staging);
  // validate every selection before enqueueing anything
  for (size_t i = 0; i < (size_t)B * k; ++i) {
    const int32_t doc = sel_host[i];
    if (doc < 0 || doc >= I->n_docs) return fail(MSA_ERR_INVALID_ARG, "selected document %d out of range", doc);
    const int64_t nc = I->doc_chunk_off_host[doc + 1] - I->doc_chunk_off_host[doc];
    if (nc <= 0 || nc > I->max_doc_chunks) return fail(MSA_ERR_INVALID_ARG, "document %d: %lld chunks", doc, (long long)nc);
  }
  for (int b = 0; b < B; ++b) {
    for (int r = 0; r < k; ++r) {
      const int32_t doc = sel_host[(size_t)b * k + r];
      const int64_t c0 = I->doc_chunk_off_host[doc], nc = I->doc_chunk_off_host[doc + 1] - c0;
      const size_t bytes = 2 * (size_t)nc * row;
      const size_t slot = ((size_t)b * k + r) * 2 * I->max_doc_chunks * row;
      cudaError_t e;
      if (g_fail_copies > 0) {
        --g_fail_copies;
        e = cudaErrorInvalidValue;
      } else {
        e = cudaMemcpyAsync(dst + slot, host + 2 * (size_t)c0 * row, bytes, cudaMemcpyHostToDevice, fetch_stream);
      }
      if (e != cudaSuccess) return cuda_fail(e, "fetch copy");
    }
  }
  if (fetch_done) {
    cudaError_t e = cudaEventRecord(fetch_done, fetch_stream);
    if (e != cudaSuccess) return cuda_fail(e, "record fetch_done");
  }
  return MSA_OK;
}

}  // extern "C"

// The device fetch behind msa_fetch_selected_device and msa_sparse_decode_raw.
static msa_status fetch_device_impl(const msa_layout* L, const msa_index* I, int32_t B, int32_t k,
                                    const int32_t* sel, void* staging, size_t staging_bytes, cudaStream_t st) {
  msa_status s = check_layout(L);
  if (s) return s;
  if ((s = check_index(L, I))) return s;
  if (!I->kv_on_host) return fail(MSA_ERR_INVALID_ARG, "index is not host-resident");
  if (B <= 0 || B > kRouteMaxB || k < 1 || k > kMaxTopK || k > I->n_docs)
    return fail(MSA_ERR_INVALID_ARG, "fetch: batch %d, top_k %d", B, k);
  if (!sel || !staging || !aligned16(staging)) return fail(MSA_ERR_INVALID_ARG, "fetch: sel_idx or staging");
  const size_t need = msa_fetch_staging_size(L, I, B, k);
  if (staging_bytes < need) return fail(MSA_ERR_WORKSPACE_TOO_SMALL, "staging %zu < %zu bytes", staging_bytes, need);
  const size_t row = (size_t)L->n_kv_heads * L->head_dim * esize(L);
  if (row % 16) return fail(MSA_ERR_UNSUPPORTED, "pooled rows of %zu bytes (a multiple of 16 needed)", row);
  // the kernel reads the host tier through its device mapping: both ends of
  // the array must be page-locked host memory the device can address
  const size_t bytes = 2 * (size_t)I->n_chunks * row;
  const char* h = static_cast<const char*>(I->host_kv);
  cudaPointerAttributes a0{}, a1{};
  cudaError_t e = cudaPointerGetAttributes(&a0, h);
  if (e == cudaSuccess) e = cudaPointerGetAttributes(&a1, h + bytes - 1);
  if (e != cudaSuccess) return cuda_fail(e, "host_kv attributes");
  if (a0.type != cudaMemoryTypeHost || a1.type != cudaMemoryTypeHost || !a0.devicePointer || !a1.devicePointer ||
      static_cast<const char*>(a1.devicePointer) - static_cast<const char*>(a0.devicePointer) != (ptrdiff_t)(bytes - 1))
    return fail(MSA_ERR_INVALID_ARG, "host_kv is not page-locked host memory mapped for the device");
  if (!aligned16(a0.devicePointer)) return fail(MSA_ERR_INVALID_ARG, "host_kv not 16-byte aligned");
  FetchArgs a{};
  a.sel = sel;
  a.doc_chunk_off = I->doc_chunk_off;
  a.host_kv = static_cast<const uint4*>(a0.devicePointer);
  a.staging = static_cast<uint4*>(staging);
  a.n_docs = I->n_docs;
  a.n_chunks = I->n_chunks;
  a.row_vec = (int64_t)(row / 16);
  a.top_k = k;
  a.max_doc_chunks = I->max_doc_chunks;
  fetch_gather_kernel<<<(unsigned)((int64_t)B * k), kFetchThreads, 0, st>>>(a);
  MSA_CHECK_LAUNCH("fetch_gather_kernel");
  return MSA_OK;
}

extern "C" {

msa_status msa_fetch_selected_device(const msa_layout* L, const msa_index* I, int32_t B, int32_t k,
                                     const int32_t* sel, void* staging, size_t staging_bytes, cudaStream_t st) {
  NvtxRange nvtx_("msa_fetch_selected_device");
  return fetch_device_impl(L, I, B, k, sel, staging, staging_bytes, st);
}

msa_status msa_rope_local(const msa_layout* L, int32_t B, const int64_t* loff, const int64_t* llen,
                          const int64_t* first, int32_t k, const void* src, void* dst, const float* rope,
                          int32_t rope_rows, cudaStream_t st) {
  NvtxRange nvtx_("msa_rope_local");
  msa_status s = check_layout(L);
  if (s) return s;
  if (B <= 0 || B > kRopeLocalMaxB) return fail(MSA_ERR_UNSUPPORTED, "batch %d (1..%d supported)", B, kRopeLocalMaxB);
  if (!loff || !src || !dst || !rope) return fail(MSA_ERR_INVALID_ARG, "rope_local: missing pointer");
  if (!aligned16(src) || !aligned16(dst) || !aligned16(rope))
    return fail(MSA_ERR_INVALID_ARG, "rope_local: pointer not 16-byte aligned");
  if ((L->head_dim / 2) % (16 / esize(L))) return fail(MSA_ERR_UNSUPPORTED, "head_dim %d", L->head_dim);
  if (k < 0) return fail(MSA_ERR_INVALID_ARG, "top_k %d", k);
  if (loff[0] != 0) return fail(MSA_ERR_INVALID_ARG, "local_off_host[0] must be 0");
  RopeLocalArgs a{};
  int64_t max_ltot = 0, max_rot = 0;
  for (int b = 0; b < B; ++b) {
    const int64_t cap = loff[b + 1] - loff[b];
    if (cap < 0) return fail(MSA_ERR_INVALID_ARG, "local_off_host must not decrease");
    const int64_t lt = llen ? llen[b] : cap;
    if (lt < 0 || lt > cap)
      return fail(MSA_ERR_INVALID_ARG, "query %d: live length %lld outside [0, %lld]", b, (long long)lt, (long long)cap);
    const int64_t f = first ? first[b] : 0;
    if (f < 0 || f > lt) return fail(MSA_ERR_INVALID_ARG, "query %d: first %lld outside [0, %lld]", b, (long long)f, (long long)lt);
    a.local_off[b] = loff[b];
    a.len[b] = lt;
    a.first[b] = f;
    max_ltot = std::max(max_ltot, lt);
    max_rot = std::max(max_rot, lt - f);
  }
  a.local_off[B] = loff[B];
  if ((int64_t)rope_rows < (int64_t)k + max_ltot)
    return fail(MSA_ERR_INVALID_ARG, "rope_rows %d < top_k + longest local context %lld", rope_rows,
                (long long)(k + max_ltot));
  const int64_t bytes = loff[B] * L->n_kv_heads * L->head_dim * esize(L);
  const char* ps = static_cast<const char*>(src);
  const char* pd = static_cast<const char*>(dst);
  if (ps != pd && ps < pd + bytes && pd < ps + bytes)
    return fail(MSA_ERR_INVALID_ARG, "rope_local: src and dst overlap without being equal");
  if (max_rot == 0) return MSA_OK;
  a.src = src; a.dst = dst; a.rope = reinterpret_cast<const float2*>(rope);
  a.d = L->head_dim; a.Hkv = L->n_kv_heads; a.top_k = k; a.rope_rows = rope_rows;
  const int64_t items = max_rot * L->n_kv_heads * (L->head_dim / 2) / (16 / esize(L));
  const int gx = (int)std::min<int64_t>((items + 255) / 256, 2 * sm_count());
  dim3 grid(gx, B);
  if (L->dtype == MSA_BF16) rope_local_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
  else rope_local_kernel<float><<<grid, 256, 0, st>>>(a);
  MSA_CHECK_LAUNCH("rope_local_kernel");
  return MSA_OK;
}

// A barrier that nothing arrives at: every lane's bounded wait must give up
// after limit_ns, flag MSA_DEV_PIPE_TIMEOUT and let the kernel finish.
__global__ void wait_probe_kernel(unsigned long long limit_ns, int* result) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const bool ok = limit_ns ? mbar_wait_for(&bar, 0u, limit_ns) : mbar_wait(&bar, 0u);
  const int gave_up = __syncthreads_count(!ok);
  if (threadIdx.x == 0) *result = gave_up;
}

msa_status msa_debug_expire_wait(int64_t limit_us, int32_t* lanes_gave_up, cudaStream_t st) {
  if (limit_us < 0 || limit_us > 10000000) return fail(MSA_ERR_INVALID_ARG, "limit %lld us", (long long)limit_us);
  if (!lanes_gave_up) return fail(MSA_ERR_INVALID_ARG, "debug_expire_wait: NULL result");
  int* d = nullptr;
  cudaError_t e = cudaMallocAsync(&d, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "probe result");
  wait_probe_kernel<<<1, 64, 0, st>>>((unsigned long long)limit_us * 1000ull, d);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaMemcpyAsync(lanes_gave_up, d, sizeof(int), cudaMemcpyDeviceToHost, st);
  cudaFreeAsync(d, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "wait probe");
  return MSA_OK;
}

msa_status msa_interleave_expand(int64_t n_docs, int32_t B, int32_t n, int32_t p, const int32_t* ranked,
                                 const int32_t* old_set, int32_t* out, int32_t* out_host, cudaStream_t st) {
  NvtxRange nvtx_("msa_interleave_expand");
  if (B <= 0 || B > kRouteMaxB) return fail(MSA_ERR_UNSUPPORTED, "batch %d (1..%d supported)", B, kRouteMaxB);
  if (n_docs <= 0 || n < 0 || p < 1) return fail(MSA_ERR_INVALID_ARG, "n_docs %lld, n_sel %d, per_round %d",
                                                  (long long)n_docs, n, p);
  const int64_t m = (int64_t)n + p;
  if (m > kInterleaveMaxSet || m > n_docs)
    return fail(MSA_ERR_INVALID_ARG, "n_sel + per_round = %lld exceeds min(n_docs, %d)", (long long)m,
                kInterleaveMaxSet);
  if (!ranked || !out || (n > 0 && !old_set)) return fail(MSA_ERR_INVALID_ARG, "interleave_expand: missing pointer");
  const int64_t nb = (int64_t)B * m * 4, ob = (int64_t)B * n * 4;
  const char* po = reinterpret_cast<const char*>(out);
  const char* pr = reinterpret_cast<const char*>(ranked);
  const char* ps = reinterpret_cast<const char*>(old_set);
  if ((pr < po + nb && po < pr + nb) || (n > 0 && ps < po + nb && po < ps + ob))
    return fail(MSA_ERR_INVALID_ARG, "interleave_expand: sel_new overlaps ranked or sel_old");
  interleave_expand_kernel<<<(B + 3) / 4, 128, 0, st>>>(ranked, old_set, out, B, n, p, n_docs);
  MSA_CHECK_LAUNCH("interleave_expand_kernel");
  if (out_host) {
    cudaError_t e = cudaMemcpyAsync(out_host, out, (size_t)nb, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(e, "copy the expanded set to the host");
  }
  return MSA_OK;
}

msa_status msa_append_local(const msa_layout* L, int32_t B, const int64_t* loff, const int64_t* llen,
                            const void* k_new, const void* v_new, int32_t k, const float* rope, int32_t rope_rows,
                            void* k_raw, void* k_rot, void* v, cudaStream_t st) {
  NvtxRange nvtx_("msa_append_local");
  msa_status s = check_layout(L);
  if (s) return s;
  if (B <= 0 || B > kRopeLocalMaxB) return fail(MSA_ERR_UNSUPPORTED, "batch %d (1..%d supported)", B, kRopeLocalMaxB);
  if (!loff || !llen || !k_new || !v_new || !rope || !k_rot || !v)
    return fail(MSA_ERR_INVALID_ARG, "append_local: missing pointer");
  const void* ptrs[] = {k_new, v_new, rope, k_rot, v};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(MSA_ERR_INVALID_ARG, "append_local: pointer not 16-byte aligned");
  if (k_raw && !aligned16(k_raw)) return fail(MSA_ERR_INVALID_ARG, "append_local: pointer not 16-byte aligned");
  if ((L->head_dim / 2) % (16 / esize(L)) || L->head_dim / 2 / (16 / esize(L)) > 64)
    return fail(MSA_ERR_UNSUPPORTED, "head_dim %d", L->head_dim);
  if (k < 0) return fail(MSA_ERR_INVALID_ARG, "top_k %d", k);
  if (loff[0] != 0) return fail(MSA_ERR_INVALID_ARG, "local_off_host[0] must be 0");
  AppendLocalArgs a{};
  int64_t max_pos = 0;
  for (int b = 0; b < B; ++b) {
    const int64_t cap = loff[b + 1] - loff[b];
    if (llen[b] < 0 || llen[b] >= cap)
      return fail(MSA_ERR_INVALID_ARG, "query %d: no room to append (live length %lld, capacity %lld)", b,
                  (long long)llen[b], (long long)cap);
    a.local_off[b] = loff[b];
    a.len[b] = llen[b];
    max_pos = std::max(max_pos, (int64_t)k + llen[b]);
  }
  a.local_off[B] = loff[B];
  if ((int64_t)rope_rows <= max_pos)
    return fail(MSA_ERR_INVALID_ARG, "rope_rows %d <= top_k + live length %lld", rope_rows, (long long)max_pos);
  a.k_new = k_new; a.v_new = v_new; a.k_raw = k_raw; a.k_rot = k_rot; a.v = v;
  a.rope = reinterpret_cast<const float2*>(rope);
  a.d = L->head_dim; a.Hkv = L->n_kv_heads; a.top_k = k; a.rope_rows = rope_rows;
  dim3 grid((unsigned)L->n_kv_heads, (unsigned)B);
  if (L->dtype == MSA_BF16) append_local_kernel<__nv_bfloat16><<<grid, 64, 0, st>>>(a);
  else append_local_kernel<float><<<grid, 64, 0, st>>>(a);
  MSA_CHECK_LAUNCH("append_local_kernel");
  return MSA_OK;
}

msa_status msa_append_local_devlen(const msa_layout* L, int32_t B, const int64_t* loff, const int64_t* llen_dev,
                                   const void* k_new, const void* v_new, int32_t k, const float* rope,
                                   int32_t rope_rows, void* k_raw, void* k_rot, void* v, cudaStream_t st) {
  NvtxRange nvtx_("msa_append_local_devlen");
  msa_status s = check_layout(L);
  if (s) return s;
  if (B <= 0 || B > kRopeLocalMaxB) return fail(MSA_ERR_UNSUPPORTED, "batch %d (1..%d supported)", B, kRopeLocalMaxB);
  if (!loff || !llen_dev || !k_new || !v_new || !rope || !k_rot || !v)
    return fail(MSA_ERR_INVALID_ARG, "append_local: missing pointer");
  const void* ptrs[] = {k_new, v_new, rope, k_rot, v};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(MSA_ERR_INVALID_ARG, "append_local: pointer not 16-byte aligned");
  if (k_raw && !aligned16(k_raw)) return fail(MSA_ERR_INVALID_ARG, "append_local: pointer not 16-byte aligned");
  if ((L->head_dim / 2) % (16 / esize(L)) || L->head_dim / 2 / (16 / esize(L)) > 64)
    return fail(MSA_ERR_UNSUPPORTED, "head_dim %d", L->head_dim);
  if (k < 0) return fail(MSA_ERR_INVALID_ARG, "top_k %d", k);
  if (loff[0] != 0) return fail(MSA_ERR_INVALID_ARG, "local_off_host[0] must be 0");
  AppendLocalArgs a{};
  int64_t max_cap = 0;
  for (int b = 0; b < B; ++b) {
    const int64_t cap = loff[b + 1] - loff[b];
    if (cap < 1) return fail(MSA_ERR_INVALID_ARG, "query %d: capacity %lld", b, (long long)cap);
    a.local_off[b] = loff[b];
    max_cap = std::max(max_cap, cap);
  }
  a.local_off[B] = loff[B];
  if ((int64_t)rope_rows < (int64_t)k + max_cap)
    return fail(MSA_ERR_INVALID_ARG, "rope_rows %d < top_k + largest capacity %lld", rope_rows,
                (long long)(k + max_cap));
  a.len_dev = llen_dev;
  a.k_new = k_new; a.v_new = v_new; a.k_raw = k_raw; a.k_rot = k_rot; a.v = v;
  a.rope = reinterpret_cast<const float2*>(rope);
  a.d = L->head_dim; a.Hkv = L->n_kv_heads; a.top_k = k; a.rope_rows = rope_rows;
  dim3 grid((unsigned)L->n_kv_heads, (unsigned)B);
  if (L->dtype == MSA_BF16) append_local_kernel<__nv_bfloat16><<<grid, 64, 0, st>>>(a);
  else append_local_kernel<float><<<grid, 64, 0, st>>>(a);
  MSA_CHECK_LAUNCH("append_local_kernel");
  return MSA_OK;
}

msa_status msa_advance_local_len(int32_t B, int64_t* llen_dev, int64_t by, cudaStream_t st) {
  if (B <= 0 || !llen_dev) return fail(MSA_ERR_INVALID_ARG, "advance_local_len: batch %d or NULL", B);
  advance_len_kernel<<<(B + 127) / 128, 128, 0, st>>>(llen_dev, B, by);
  MSA_CHECK_LAUNCH("advance_len_kernel");
  return MSA_OK;
}

size_t msa_kr_inv_norm_count(const msa_layout* L, int64_t n_chunks) {
  if (!L || check_layout(L) || n_chunks <= 0) return 0;
  return (size_t)L->n_kv_heads * (size_t)((n_chunks + kScanTile - 1) / kScanTile) * kScanTile;
}

msa_status msa_kr_inv_norms(const msa_layout* L, const msa_index* I, float* out, cudaStream_t st) {
  NvtxRange nvtx_("msa_kr_inv_norms");
  msa_status s = check_layout(L);
  if (s) return s;
  if ((s = check_index(L, I))) return s;
  if ((s = check_scan_shape(L))) return s;
  if (!out || !aligned16(out)) return fail(MSA_ERR_INVALID_ARG, "kr_inv_norms: out NULL or not 16-byte aligned");
  const int64_t P = (I->n_chunks + kScanTile - 1) / kScanTile * kScanTile;
  const int64_t n = P * L->n_kv_heads;
  const int blocks = (int)std::min<int64_t>((n + 255) / 256, 8 * sm_count());
  if (L->dtype == MSA_BF16)
    kr_inv_norms_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(I->kr), I->n_chunks, L->n_kv_heads, L->router_dim, P, out);
  else
    kr_inv_norms_kernel<float><<<blocks, 256, 0, st>>>(reinterpret_cast<const float*>(I->kr), I->n_chunks,
                                                      L->n_kv_heads, L->router_dim, P, out);
  MSA_CHECK_LAUNCH("kr_inv_norms_kernel");
  return MSA_OK;
}

size_t msa_decode_workspace_size(const msa_layout* L, int32_t B, int32_t T, const int64_t* loff,
                                 const int64_t* llen) {
  if (!L || check_layout(L)) return 0;
  DecodePlan p;
  if (plan_decode(L, B, T, loff, llen, nullptr, &p)) return 0;
  return p.bytes;
}

static msa_status decode_impl(const msa_layout* L, const msa_index* I, int32_t B, int32_t T, const void* q,
                              const void* lk, const void* lv, const int64_t* loff, const int64_t* llen,
                              const int32_t* sel, int32_t k, const void* staging, const float* rope,
                              int32_t rope_rows, void* out, float* lse, void* ws, size_t ws_bytes,
                              cudaEvent_t wait_event, cudaStream_t st, const int64_t* llen_dev = nullptr) {
  NvtxRange nvtx_("msa_sparse_decode");
  msa_status s = check_layout(L);
  if (s) return s;
  if ((s = check_index(L, I))) return s;
  if (L->head_dim != 64 && L->head_dim != 128) return fail(MSA_ERR_UNSUPPORTED, "head_dim %d (64 or 128)", L->head_dim);
  if (!q || !lk || !lv || !sel || !rope || !out) return fail(MSA_ERR_INVALID_ARG, "decode: missing pointer");
  const void* ptrs[] = {q, lk, lv, rope, out};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(MSA_ERR_INVALID_ARG, "decode: pointer not 16-byte aligned");
  if (k < 1 || k > kMaxTopK || k > I->n_docs) return fail(MSA_ERR_INVALID_ARG, "top_k %d", k);
  if (I->kv_on_host) {
    if (!staging || !aligned16(staging)) return fail(MSA_ERR_INVALID_ARG, "host tier needs the staging buffer");
  } else if (!I->k || !I->v) {
    return fail(MSA_ERR_INVALID_ARG, "index K/V missing");
  }
  DecodePlan p;
  if ((s = plan_decode(L, B, T, loff, llen, ws, &p))) return s;
  if (!ws || ws_bytes < p.bytes) return fail(MSA_ERR_WORKSPACE_TOO_SMALL, "decode workspace %zu < %zu bytes", ws_bytes, p.bytes);
  if ((int64_t)rope_rows < (int64_t)k + p.max_ltot)
    return fail(MSA_ERR_INVALID_ARG, "rope_rows %d < top_k + longest local context %lld", rope_rows,
                (long long)(k + p.max_ltot));
  if (wait_event) {
    cudaError_t e = cudaStreamWaitEvent(st, wait_event, 0);
    if (e != cudaSuccess) return cuda_fail(e, "wait event");
  }
  DecodeArgs a{};
  a.B = B; a.T = T; a.Hq = L->n_q_heads; a.Hkv = L->n_kv_heads; a.G = a.Hq / a.Hkv;
  a.R = p.R; a.n_rg = p.n_rg; a.S = p.S; a.top_k = k; a.rope_rows = rope_rows;
  a.kv_on_host = I->kv_on_host; a.max_doc_chunks = I->kv_on_host ? I->max_doc_chunks : INT_MAX;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)L->head_dim));
  a.q = q; a.lk = lk; a.lv = lv; a.sel = sel; a.doc_chunk_off = I->doc_chunk_off; a.n_docs = I->n_docs;
  a.mem_k = I->kv_on_host ? staging : I->k;
  a.mem_v = I->kv_on_host ? staging : I->v;
  a.rope = reinterpret_cast<const float2*>(rope);
  a.part_o = p.part_o; a.part_ml = p.part_ml; a.counters = p.counters; a.out = out; a.lse = lse;
  a.local_len_dev = llen_dev;
  for (int b = 0; b <= B; ++b) { a.split_off[b] = p.split_off[b]; a.local_off[b] = loff[b]; }
  for (int b = 0; b < B; ++b) a.local_len[b] = p.len[b];
  if (p.wr) {
    const int64_t rows = loff[B] * L->n_kv_heads;
    if (L->head_dim == 128) return launch_decode_mma_d<128>(a, p, rows, st);
    return launch_decode_mma_d<64>(a, p, rows, st);
  }
  const bool bf = L->dtype == MSA_BF16;
  if (L->head_dim == 128) {
    if (bf) return launch_decode<__nv_bfloat16, 128>(a, p, st);
    return launch_decode<float, 128>(a, p, st);
  }
  if (bf) return launch_decode<__nv_bfloat16, 64>(a, p, st);
  return launch_decode<float, 64>(a, p, st);
}

msa_status msa_sparse_decode(const msa_layout* L, const msa_index* I, int32_t B, int32_t T, const void* q,
                             const void* lk, const void* lv, const int64_t* loff, const int64_t* llen,
                             const int32_t* sel, int32_t k, const void* staging, const float* rope,
                             int32_t rope_rows, void* out, void* ws, size_t ws_bytes, cudaEvent_t wait_event,
                             cudaStream_t st) {
  return decode_impl(L, I, B, T, q, lk, lv, loff, llen, sel, k, staging, rope, rope_rows, out, nullptr, ws,
                     ws_bytes, wait_event, st);
}

msa_status msa_sparse_decode_devlen(const msa_layout* L, const msa_index* I, int32_t B, int32_t T, const void* q,
                                    const void* lk, const void* lv, const int64_t* loff, const int64_t* llen_dev,
                                    const int32_t* sel, int32_t k, const void* staging, const float* rope,
                                    int32_t rope_rows, void* out, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!llen_dev) return fail(MSA_ERR_INVALID_ARG, "decode_devlen: local_len_dev is NULL");
  return decode_impl(L, I, B, T, q, lk, lv, loff, nullptr, sel, k, staging, rope, rope_rows, out, nullptr, ws,
                     ws_bytes, nullptr, st, llen_dev);
}

// Workspace of msa_sparse_decode_raw: [decode workspace | rotated local keys |
// host-tier staging], each part a multiple of 256 bytes.
struct RawDecodeParts {
  size_t dec, keys, staging;
};
static bool raw_decode_parts(const msa_layout* L, const msa_index* I, int32_t B, int32_t T, int32_t k,
                             const int64_t* loff, const int64_t* llen, RawDecodeParts* p) {
  if (!L || !I || !loff || B <= 0 || check_layout(L)) return false;
  p->dec = msa_decode_workspace_size(L, B, T, loff, llen);
  if (!p->dec) return false;
  p->keys = align_up((size_t)loff[B] * L->n_kv_heads * L->head_dim * esize(L));
  p->staging = I->kv_on_host ? align_up(msa_fetch_staging_size(L, I, B, k)) : 0;
  return !I->kv_on_host || p->staging > 0;
}

size_t msa_sparse_decode_raw_workspace_size(const msa_layout* L, const msa_index* I, int32_t B, int32_t T,
                                            int32_t k, const int64_t* loff, const int64_t* llen) {
  RawDecodeParts p{};
  if (!raw_decode_parts(L, I, B, T, k, loff, llen, &p)) return 0;
  return p.dec + p.keys + p.staging;
}

msa_status msa_sparse_decode_raw(const msa_layout* L, const msa_index* I, int32_t B, int32_t T, const void* q,
                                 const void* lk_raw, const void* lv, const int64_t* loff, const int64_t* llen,
                                 const int32_t* sel, int32_t k, const float* rope, int32_t rope_rows, void* out,
                                 void* ws, size_t ws_bytes, cudaStream_t st) {
  NvtxRange nvtx_("msa_sparse_decode_raw");
  msa_status s = check_layout(L);
  if (s) return s;
  if ((s = check_index(L, I))) return s;
  if (!lk_raw || !lv || !sel || !ws) return fail(MSA_ERR_INVALID_ARG, "decode_raw: missing pointer");
  RawDecodeParts p{};
  if (!raw_decode_parts(L, I, B, T, k, loff, llen, &p))
    return fail(MSA_ERR_INVALID_ARG, "decode_raw: batch %d, T %d or local lengths rejected by the decode plan", B, T);
  if (ws_bytes < p.dec + p.keys + p.staging)
    return fail(MSA_ERR_WORKSPACE_TOO_SMALL, "decode_raw workspace %zu < %zu bytes", ws_bytes,
                p.dec + p.keys + p.staging);
  char* w = static_cast<char*>(ws);
  void* keys = w + p.dec;
  void* staging = I->kv_on_host ? w + p.dec + p.keys : nullptr;
  if (I->kv_on_host && (s = fetch_device_impl(L, I, B, k, sel, staging, p.staging, st))) return s;
  if ((s = msa_rope_local(L, B, loff, llen, nullptr, k, lk_raw, keys, rope, rope_rows, st))) return s;
  return decode_impl(L, I, B, T, q, keys, lv, loff, llen, sel, k, staging, rope, rope_rows, out, nullptr, ws, p.dec,
                     nullptr, st);
}

msa_status msa_sparse_attention_forward(const msa_layout* L, const msa_index* I, int32_t B, int32_t T,
                                        const void* q, const void* lk, const void* lv, const int64_t* loff,
                                        const int64_t* llen, const int32_t* sel, int32_t k, const float* rope,
                                        int32_t rope_rows, void* out, float* lse, void* ws, size_t ws_bytes,
                                        cudaStream_t st) {
  if (!lse) return fail(MSA_ERR_INVALID_ARG, "attention_forward: lse is NULL");
  if (I && I->kv_on_host) return fail(MSA_ERR_UNSUPPORTED, "training runs on a device-tier bank");
  return decode_impl(L, I, B, T, q, lk, lv, loff, llen, sel, k, nullptr, rope, rope_rows, out, lse, ws, ws_bytes,
                     nullptr, st);
}

size_t msa_attention_backward_workspace_size(const msa_layout* L, int32_t B, int32_t T) {
  if (!L || check_layout(L) || B <= 0 || T <= 0) return 0;
  Carver c(nullptr);
  c.take<float>(sizeof(float) * (size_t)B * T * L->n_q_heads * L->head_dim);
  c.take<float>(sizeof(float) * (size_t)B * T * L->n_q_heads);
  return c.off;
}

msa_status msa_sparse_attention_backward(const msa_layout* L, const msa_index* I, int32_t B, int32_t T,
                                         const void* q, const void* lk, const void* lv, const int64_t* loff,
                                         const int64_t* llen, const int32_t* sel, int32_t k, const float* rope,
                                         int32_t rope_rows, const void* out, const float* lse, const void* dout,
                                         float* dq, float* dmem_k, float* dmem_v, float* dlk, float* dlv, void* ws,
                                         size_t ws_bytes, cudaStream_t st) {
  NvtxRange nvtx_("msa_sparse_attention_backward");
  msa_status s = check_layout(L);
  if (s) return s;
  if ((s = check_index(L, I))) return s;
  if (I->kv_on_host || !I->k || !I->v) return fail(MSA_ERR_UNSUPPORTED, "training runs on a device-tier bank");
  if (I->max_doc_chunks <= 0) return fail(MSA_ERR_INVALID_ARG, "attention_backward: index max_doc_chunks needed");
  if (B <= 0 || B > kBwdMaxB) return fail(MSA_ERR_UNSUPPORTED, "batch %d (1..%d supported)", B, kBwdMaxB);
  if (T <= 0) return fail(MSA_ERR_INVALID_ARG, "T %d", T);
  if (L->head_dim != 64 && L->head_dim != 128) return fail(MSA_ERR_UNSUPPORTED, "head_dim %d", L->head_dim);
  if (k < 1 || k > kMaxTopKDecode || k > I->n_docs) return fail(MSA_ERR_INVALID_ARG, "top_k %d", k);
  const void* ptrs[] = {q, lk, lv, sel, rope, out, lse, dout, dq, dmem_k, dmem_v, dlk, dlv};
  for (const void* p : ptrs)
    if (!p) return fail(MSA_ERR_INVALID_ARG, "attention_backward: missing pointer");
  const void* al[] = {q, lk, lv, rope, out, dout, dq, dmem_k, dmem_v, dlk, dlv};
  for (const void* p : al)
    if (!aligned16(p)) return fail(MSA_ERR_INVALID_ARG, "attention_backward: pointer not 16-byte aligned");
  if (!loff || loff[0] != 0) return fail(MSA_ERR_INVALID_ARG, "local_off_host missing or not starting at 0");
  const size_t need = msa_attention_backward_workspace_size(L, B, T);
  if (!ws || ws_bytes < need) return fail(MSA_ERR_WORKSPACE_TOO_SMALL, "backward workspace %zu < %zu bytes", ws_bytes, need);
  BwdArgs a{};
  a.B = B; a.T = T; a.Hq = L->n_q_heads; a.Hkv = L->n_kv_heads; a.G = a.Hq / a.Hkv; a.R = a.G * T;
  a.top_k = k; a.rope_rows = rope_rows;
  const bool bf = L->dtype == MSA_BF16;
  // bf16 with head_dim 128 runs on tcgen05 (128-key tiles, a query box of
  // 128 / G tokens x G heads: G divides 128); the rest on mma.sync / CUDA cores
  const bool tc = bf && L->head_dim == 128 && kBwtRows % a.G == 0;
  const int64_t key_tile = tc ? kBwtKeys : kBwdTile;
  a.mem_tiles = (int)(((int64_t)k * I->max_doc_chunks + key_tile - 1) / key_tile);
  int64_t max_ltot = 0;
  a.tile_off[0] = 0;
  for (int b = 0; b < B; ++b) {
    const int64_t cap = loff[b + 1] - loff[b];
    const int64_t lt = llen ? llen[b] : cap;
    if (lt < T || lt > cap)
      return fail(MSA_ERR_INVALID_ARG, "query %d: live length %lld outside [T, capacity %lld]", b, (long long)lt,
                  (long long)cap);
    a.local_off[b] = loff[b];
    a.local_len[b] = lt;
    max_ltot = std::max(max_ltot, lt);
    const int64_t tiles = a.tile_off[b] + a.mem_tiles + (lt + key_tile - 1) / key_tile;
    if (tiles > INT_MAX / 2) return fail(MSA_ERR_UNSUPPORTED, "too many key tiles");
    a.tile_off[b + 1] = (int32_t)tiles;
  }
  a.local_off[B] = loff[B];
  if ((int64_t)rope_rows < (int64_t)k + max_ltot)
    return fail(MSA_ERR_INVALID_ARG, "rope_rows %d < top_k + longest local context %lld", rope_rows,
                (long long)(k + max_ltot));
  a.scale = (float)(1.0 / std::sqrt((double)L->head_dim));
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)L->head_dim));
  a.q = q; a.lk = lk; a.lv = lv; a.sel = sel; a.doc_chunk_off = I->doc_chunk_off; a.n_docs = I->n_docs;
  a.mem_k = I->k; a.mem_v = I->v; a.rope = reinterpret_cast<const float2*>(rope);
  a.out = out; a.dout = dout; a.lse = lse; a.dq = dq; a.dmem_k = dmem_k; a.dmem_v = dmem_v; a.dlk = dlk; a.dlv = dlv;
  Carver c(ws);
  a.qrot = c.take<float>(sizeof(float) * (size_t)B * T * a.Hq * L->head_dim);
  a.drow = c.take<float>(sizeof(float) * (size_t)B * T * a.Hq);
  const int64_t rows = (int64_t)B * T * a.Hq;
  const unsigned prep_blocks = (unsigned)((rows + 7) / 8);
  const dim3 grid((unsigned)a.tile_off[B], (unsigned)a.Hkv);
  static std::atomic<uint64_t> attr_done[5];
  if (tc) {
    BwdTcArgs T_;
    memset(&T_, 0, sizeof T_);
    // rotated queries (the prep kernel writes them in bf16) and dO: [B * T][Hq][128],
    // boxes of 64 dims x G heads x 128 / G tokens
    const cuuint64_t dims[3] = {128, (cuuint64_t)a.Hq, (cuuint64_t)B * T};
    const cuuint64_t str[2] = {256, (cuuint64_t)a.Hq * 256};
    const cuuint32_t box[3] = {64, (cuuint32_t)a.G, (cuuint32_t)(kBwtRows / a.G)};
    if ((s = make_map(&T_.tm_q, a.qrot, 3, dims, str, box))) return s;
    if ((s = make_map(&T_.tm_do, dout, 3, dims, str, box))) return s;
    // local key / value caches [loff[B] * H_kv rows][128], boxes of 64 dims x 128 rows
    const int64_t cache_rows = loff[B] * a.Hkv;
    if (cache_rows + kBwtKeys >= INT_MAX) return fail(MSA_ERR_UNSUPPORTED, "local cache of %lld rows", (long long)cache_rows);
    const cuuint64_t kdims[2] = {128, (cuuint64_t)cache_rows};
    const cuuint64_t kstr[1] = {256};
    const cuuint32_t kbox[2] = {64, (cuuint32_t)kBwtKeys};
    if ((s = make_map(&T_.tm_k, lk, 2, kdims, kstr, kbox))) return s;
    if ((s = make_map(&T_.tm_v, lv, 2, kdims, kstr, kbox))) return s;
    // the fp32 dq~ [B * T][Hq][128] for the tile reduce-adds: boxes of 32 dims x G heads x 128 / G tokens
    const cuuint64_t qdims[3] = {128, (cuuint64_t)a.Hq, (cuuint64_t)B * T};
    const cuuint64_t qstr[2] = {512, (cuuint64_t)a.Hq * 512};
    const cuuint32_t qbox[3] = {32, (cuuint32_t)a.G, (cuuint32_t)(kBwtRows / a.G)};
    if ((s = make_map(&T_.tm_dq, dq, 3, qdims, qstr, qbox, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_DATA_TYPE_FLOAT32)))
      return s;
    T_.a = a;
    attn_bwd_prep_kernel<__nv_bfloat16, 128><<<prep_blocks, 256, 0, st>>>(a);
    MSA_CHECK_LAUNCH("attn_bwd_prep_kernel");
    const int smem = (int)sizeof(BwdTcSmem) + 1024;          // + room to align the tiles to 1 KiB
    if ((s = smem_attr_once(attn_bwd_tc_kernel, smem, attr_done[4], "attn_bwd_tc smem"))) return s;
    attn_bwd_tc_kernel<<<grid, kBwtThreads, smem, st>>>(T_);
    MSA_CHECK_LAUNCH("attn_bwd_tc_kernel");
    const int64_t n = rows * 64;
    attn_bwd_rotq_kernel<128><<<(unsigned)std::min<int64_t>((n + 255) / 256, 4 * sm_count()), 256, 0, st>>>(a);
    MSA_CHECK_LAUNCH("attn_bwd_rotq_kernel");
    return MSA_OK;
  }
#define MSA_BWD_LAUNCH(TT, DD, KERN, SMEM, THREADS, IDX)                                                \
  do {                                                                                                   \
    attn_bwd_prep_kernel<TT, DD><<<prep_blocks, 256, 0, st>>>(a);                                        \
    MSA_CHECK_LAUNCH("attn_bwd_prep_kernel");                                                            \
    const int smem = (int)sizeof(SMEM);                                                                  \
    if ((s = smem_attr_once(KERN, smem, attr_done[IDX], "attn_bwd smem"))) return s;                     \
    KERN<<<grid, THREADS, smem, st>>>(a);                                                                \
    MSA_CHECK_LAUNCH("attn_bwd_kernel");                                                                 \
    const int64_t n = rows * (DD / 2);                                                                   \
    attn_bwd_rotq_kernel<DD><<<(unsigned)std::min<int64_t>((n + 255) / 256, 4 * sm_count()), 256, 0, st>>>(a); \
    MSA_CHECK_LAUNCH("attn_bwd_rotq_kernel");                                                            \
  } while (0)
  if (L->head_dim == 128) {
    if (bf) MSA_BWD_LAUNCH(__nv_bfloat16, 128, attn_bwd_mma_kernel<128>, BwdMmaSmem<128>, kBwdMmaThreads, 0);
    else MSA_BWD_LAUNCH(float, 128, (attn_bwd_kernel<float, 128>), BwdSmem<128>, kBwdThreads, 1);
  } else {
    if (bf) MSA_BWD_LAUNCH(__nv_bfloat16, 64, attn_bwd_mma_kernel<64>, BwdMmaSmem<64>, kBwdMmaThreads, 2);
    else MSA_BWD_LAUNCH(float, 64, (attn_bwd_kernel<float, 64>), BwdSmem<64>, kBwdThreads, 3);
  }
#undef MSA_BWD_LAUNCH
  return MSA_OK;
}

// ---------------------------------------------------- auxiliary routing loss

static msa_status plan_loss(const msa_layout* L, const msa_index* I, int B, int T, void* ws, LossArgs* a,
                            size_t* bytes) {
  msa_status s = check_layout(L);
  if (s) return s;
  if ((s = check_index(L, I))) return s;
  if (B <= 0 || T <= 0) return fail(MSA_ERR_INVALID_ARG, "batch %d, T %d", B, T);
  if (L->router_dim > 128) return fail(MSA_ERR_UNSUPPORTED, "routing loss: router_dim %d > 128", L->router_dim);
  const int64_t HD = (int64_t)L->n_kv_heads * L->router_dim;
  if (L->n_kv_heads > 16) return fail(MSA_ERR_UNSUPPORTED, "routing loss: H_kv %d > 16", L->n_kv_heads);
  a->B = B; a->T = T; a->Hq = L->n_q_heads; a->Hkv = L->n_kv_heads; a->G = a->Hq / a->Hkv; a->dr = L->router_dim;
  a->n_docs = I->n_docs; a->n_chunks = I->n_chunks;
  a->kr = I->kr; a->doc_chunk_off = I->doc_chunk_off;
  Carver c(ws);
  a->qinv = c.take<float>(sizeof(float) * (size_t)B * T * a->Hq);
  a->u = c.take<float>(sizeof(float) * (size_t)B * T * HD);
  a->chunk_best = c.take<float>(sizeof(float) * (size_t)B * I->n_chunks);
  a->chunk_t = c.take<int32_t>(sizeof(int32_t) * (size_t)B * I->n_chunks);
  a->doc_score = c.take<float>(sizeof(float) * (size_t)B * I->n_docs);
  a->doc_t = c.take<int32_t>(sizeof(int32_t) * (size_t)B * I->n_docs);
  a->doc_c = c.take<int64_t>(sizeof(int64_t) * (size_t)B * I->n_docs);
  a->lse = c.take<float>(sizeof(float) * (size_t)B * 2);
  *bytes = c.off;
  return MSA_OK;
}

size_t msa_route_loss_workspace_size(const msa_layout* L, const msa_index* I, int32_t B, int32_t T) {
  LossArgs a{};
  size_t bytes = 0;
  if (plan_loss(L, I, B, T, nullptr, &a, &bytes)) return 0;
  return bytes;
}

msa_status msa_route_loss_forward(const msa_layout* L, const msa_index* I, int32_t B, int32_t T, const void* qr,
                                  const int32_t* pos_off, const int32_t* pos_doc, float tau, float* loss,
                                  float* doc_score, void* ws, size_t ws_bytes, cudaStream_t st) {
  NvtxRange nvtx_("msa_route_loss_forward");
  LossArgs a{};
  size_t need = 0;
  msa_status s = plan_loss(L, I, B, T, ws, &a, &need);
  if (s) return s;
  if (!qr || !pos_off || !pos_doc || !loss) return fail(MSA_ERR_INVALID_ARG, "route_loss: missing pointer");
  if (!(tau > 0.f)) return fail(MSA_ERR_INVALID_ARG, "route_loss: tau must be > 0");
  if (!ws || ws_bytes < need) return fail(MSA_ERR_WORKSPACE_TOO_SMALL, "route_loss workspace %zu < %zu bytes", ws_bytes, need);
  a.qr = qr; a.pos_off = pos_off; a.pos_doc = pos_doc; a.tau = tau; a.loss = loss;
  const bool bf = L->dtype == MSA_BF16;
  const int64_t prow = (int64_t)B * T * a.Hkv;
  if (bf) loss_prep_kernel<__nv_bfloat16><<<(unsigned)((prow + 7) / 8), 256, 0, st>>>(a);
  else loss_prep_kernel<float><<<(unsigned)((prow + 7) / 8), 256, 0, st>>>(a);
  MSA_CHECK_LAUNCH("loss_prep_kernel");
  const dim3 grid((unsigned)((I->n_chunks + kLossChunks - 1) / kLossChunks), (unsigned)B);
  if (bf) loss_chunk_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
  else loss_chunk_kernel<float><<<grid, 256, 0, st>>>(a);
  MSA_CHECK_LAUNCH("loss_chunk_kernel");
  const int64_t nd = (int64_t)B * I->n_docs;
  loss_doc_kernel<<<(unsigned)((nd + 255) / 256), 256, 0, st>>>(a);
  MSA_CHECK_LAUNCH("loss_doc_kernel");
  loss_value_kernel<<<(unsigned)B, 256, 0, st>>>(a);
  MSA_CHECK_LAUNCH("loss_value_kernel");
  if (doc_score) {
    cudaError_t e = cudaMemcpyAsync(doc_score, a.doc_score, sizeof(float) * (size_t)nd, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "copy the document scores");
  }
  return MSA_OK;
}

msa_status msa_route_loss_backward(const msa_layout* L, const msa_index* I, int32_t B, int32_t T, const void* qr,
                                   const int32_t* pos_off, const int32_t* pos_doc, float tau, const float* dloss,
                                   float* dqr, float* dkr, void* ws, size_t ws_bytes, cudaStream_t st) {
  NvtxRange nvtx_("msa_route_loss_backward");
  LossArgs a{};
  size_t need = 0;
  msa_status s = plan_loss(L, I, B, T, ws, &a, &need);
  if (s) return s;
  if (!qr || !pos_off || !pos_doc || !dloss || !dqr || !dkr)
    return fail(MSA_ERR_INVALID_ARG, "route_loss_backward: missing pointer");
  if (!(tau > 0.f)) return fail(MSA_ERR_INVALID_ARG, "route_loss: tau must be > 0");
  if (!ws || ws_bytes < need) return fail(MSA_ERR_WORKSPACE_TOO_SMALL, "route_loss workspace %zu < %zu bytes", ws_bytes, need);
  a.qr = qr; a.pos_off = pos_off; a.pos_doc = pos_doc; a.tau = tau; a.dloss = dloss; a.dqr = dqr; a.dkr = dkr;
  cudaError_t e = cudaMemsetAsync(dqr, 0, sizeof(float) * (size_t)B * T * a.Hq * a.dr, st);
  if (e != cudaSuccess) return cuda_fail(e, "zero dqr");
  const int64_t nd = (int64_t)B * I->n_docs;
  if (L->dtype == MSA_BF16) loss_bwd_kernel<__nv_bfloat16><<<(unsigned)((nd + 7) / 8), 256, 0, st>>>(a);
  else loss_bwd_kernel<float><<<(unsigned)((nd + 7) / 8), 256, 0, st>>>(a);
  MSA_CHECK_LAUNCH("loss_bwd_kernel");
  return MSA_OK;
}

}  // extern "C"
