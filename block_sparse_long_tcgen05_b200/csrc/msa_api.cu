// C ABI of the MSA library: argument validation, workspace layout, TMA descriptors and
// the launch sequence of every entry point declared in include/msa.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/msa.h"
#include "common.cuh"
#include "csr.cuh"
#include "index_blockmax.cuh"
#include "index_topk.cuh"
#include "kl.cuh"
#include "kvouter.cuh"
#include "merge.cuh"
#include "decode.cuh"
#include "topk.cuh"

using namespace msa;

namespace {

thread_local char g_detail[512] = "";

msa_status_t fail(msa_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
  return st;
}

#define MSA_CHECK_CUDA(expr)                                                                     \
  do {                                                                                           \
    cudaError_t e_ = (expr);                                                                     \
    if (e_ != cudaSuccess) return fail(MSA_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
  } while (0)

#define MSA_CHECK_LAUNCH()                                                                        \
  do {                                                                                            \
    cudaError_t e_ = cudaGetLastError();                                                          \
    if (e_ != cudaSuccess) return fail(MSA_ERR_CUDA, "launch failed: %s", cudaGetErrorString(e_)); \
  } while (0)

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Sub-allocation of the caller's workspace (sizes only when base == nullptr).
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  void* take(size_t bytes) {
    void* p = base ? base + off : nullptr;
    off = align_up(off + bytes);
    return p;
  }
};

// ------------------------------- limits / policy -------------------------------
constexpr int64_t kMaxN = (int64_t(1) << 26) - 1;
// Maxima buffer of one index launch (bytes). The index branch is cut into query-block
// ranges whose packed block maxima fit this cap.
constexpr size_t kMaximaCap = size_t(4) << 30;
constexpr int64_t kDefaultQueryChunk = 16384;
constexpr int kDefaultMergeSms = 0;

int64_t tri(int64_t x) { return x * (x - 1) / 2; }

size_t maxima_bytes(int64_t qb0, int64_t qb1, int G) { return size_t(4) * G * 128 * size_t(tri(qb1) - tri(qb0)); }

// [qb0, qb1) ranges of the index branch
std::vector<std::pair<int, int>> index_chunks(int64_t nb, int G, size_t cap = kMaximaCap) {
  std::vector<std::pair<int, int>> out;
  int64_t qb0 = 0;
  while (qb0 < nb) {
    int64_t qb1 = qb0 + 1;
    // grow while within the cap and within the run table
    int64_t lo = qb0 + 1, hi = nb;
    while (lo < hi) {
      const int64_t mid = (lo + hi + 1) / 2;
      if (maxima_bytes(qb0, mid, G) <= cap && (mid + kIdxKbRun - 1) / kIdxKbRun <= kIdxMaxRuns) lo = mid;
      else hi = mid - 1;
    }
    qb1 = lo;
    out.emplace_back(int(qb0), int(qb1));
    qb0 = qb1;
  }
  return out;
}

bool supported_r(int R) { return R == 1 || R == 2 || R == 4 || R == 8 || R == 16; }

// Longest sequence of the two-kernel Index Branch: one launch's key runs must fit the run
// table passed to index_blockmax_kernel (kIdxMaxRuns runs of kIdxKbRun key blocks).
constexpr int64_t kTwoKernelMaxBlocks = int64_t(kIdxMaxRuns) * kIdxKbRun;
// Longest sequence of the Main Branch: the CSR build keeps one 128-bit membership mask per
// key block of the chunk's causal range in shared memory (227 KB per CTA).
constexpr int64_t kCsrMaxBlocks = (227 * 1024) / 16;

msa_status_t check_common(int64_t n, int32_t g, int32_t bk, int32_t k) {
  if (n < 1 || n > kMaxN) return fail(MSA_ERR_INVALID_ARG, "n=%lld out of range [1, %lld]", (long long)n, (long long)kMaxN);
  if (g < 1 || g > 64) return fail(MSA_ERR_INVALID_ARG, "g=%d out of range [1, 64]", g);
  if (k < 1 || k > 32) return fail(MSA_ERR_UNSUPPORTED, "k=%d unsupported (1..32)", k);
  if (bk != 128 && bk != 64 && bk != 32) return fail(MSA_ERR_UNSUPPORTED, "bk=%d unsupported (32, 64, 128)", bk);
  return MSA_OK;
}

msa_status_t check_ptr(const void* p, const char* name) {
  if (p == nullptr) return fail(MSA_ERR_INVALID_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return fail(MSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return MSA_OK;
}

// ------------------------------- TMA descriptors -------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D bf16 tensor map: dims {d0, d1, d2} (d0 innermost), byte strides of dims 1 and 2.
msa_status_t make_map_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                         uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {s1, s2};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return MSA_OK;
}

// 4-D bf16 tensor map: dims {d0..d3} (d0 innermost), byte strides of dims 1..3 (any order).
msa_status_t make_map_4d(CUtensorMap* map, const void* base, const uint64_t (&dims)[4], const uint64_t (&strides)[3],
                         const uint32_t (&box)[4], CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t d[4] = {dims[0], dims[1], dims[2], dims[3]};
  const cuuint64_t s[3] = {strides[0], strides[1], strides[2]};
  const cuuint32_t b[4] = {box[0], box[1], box[2], box[3]};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), d, s, b, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled (4-D) failed (%d)", int(r));
  return MSA_OK;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

template <typename K>
msa_status_t set_smem(K kernel, int bytes) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return fail(MSA_ERR_CUDA, "cudaFuncSetAttribute(smem=%d): %s", bytes, cudaGetErrorString(e));
  return MSA_OK;
}


// ------------------------------- per-kernel timing -------------------------------
enum ProfKind {
  kPIndex, kPTopkPrefill, kPCsrCount, kPCsrScan, kPCsrOffsets, kPCsrScatter, kPCsrItems, kPKvOuter, kPMerge,
  kPDecodeScan, kPTopkDecode, kPDecodeAttn, kPIndexTopk, kPKl, kPKlMerge, kPNumKinds
};
const char* const kProfNames[kPNumKinds] = {"index_blockmax", "topk_prefill", "csr_count", "csr_scan",
                                            "csr_offsets", "csr_scatter", "csr_items", "kvouter", "merge",
                                            "decode_scan", "topk_decode", "decode_attn", "index_topk", "kl",
                                            "kl_merge"};
struct ProfRec {
  int kind;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t prof_event() {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Records a CUDA event before and after the launches of its scope when profiling is on.
struct ProfScope {
  ProfRec r{};
  cudaStream_t st;
  bool on;
  ProfScope(int kind, cudaStream_t s) : st(s), on(g_prof_on) {
    if (on) {
      r.kind = kind;
      r.a = prof_event();
      r.b = prof_event();
      cudaEventRecord(r.a, st);
    }
  }
  ~ProfScope() {
    if (on) {
      cudaEventRecord(r.b, st);
      std::lock_guard<std::mutex> lk(g_prof_mu);
      g_prof.push_back(r);
    }
  }
};

// ------------------------------- index branch -------------------------------
struct IndexLayout {
  uint32_t* maxima = nullptr;
  size_t bytes = 0;
  size_t cap = kMaximaCap;   // largest maxima buffer one index launch may fill
};

IndexLayout index_layout(void* ws, int64_t n, int32_t g) {
  const int64_t nb = (n + 127) / 128;
  size_t mx = 0;
  for (auto& c : index_chunks(nb, g)) mx = std::max(mx, maxima_bytes(c.first, c.second, g));
  Carver cv(ws);
  IndexLayout L;
  L.maxima = static_cast<uint32_t*>(cv.take(std::max<size_t>(mx, 16)));
  L.bytes = cv.off;
  return L;
}

template <int KM>
void launch_topk_prefill(const TopkPrefillParams& tp, dim3 grid, cudaStream_t st) {
  topk_prefill_kernel<KM><<<grid, 128, 0, st>>>(tp);
}

msa_status_t dispatch_topk_prefill(int k, const TopkPrefillParams& tp, dim3 grid, cudaStream_t st) {
  switch (k - 1) {
#define MSA_TOPK_CASE(KM) \
  case KM:                \
    launch_topk_prefill<KM>(tp, grid, st); break;
    MSA_TOPK_CASE(0) MSA_TOPK_CASE(1) MSA_TOPK_CASE(2) MSA_TOPK_CASE(3) MSA_TOPK_CASE(4) MSA_TOPK_CASE(5)
    MSA_TOPK_CASE(6) MSA_TOPK_CASE(7) MSA_TOPK_CASE(8) MSA_TOPK_CASE(9) MSA_TOPK_CASE(10) MSA_TOPK_CASE(11)
    MSA_TOPK_CASE(12) MSA_TOPK_CASE(13) MSA_TOPK_CASE(14) MSA_TOPK_CASE(15) MSA_TOPK_CASE(16) MSA_TOPK_CASE(17)
    MSA_TOPK_CASE(18) MSA_TOPK_CASE(19) MSA_TOPK_CASE(20) MSA_TOPK_CASE(21) MSA_TOPK_CASE(22) MSA_TOPK_CASE(23)
    MSA_TOPK_CASE(24) MSA_TOPK_CASE(25) MSA_TOPK_CASE(26) MSA_TOPK_CASE(27) MSA_TOPK_CASE(28) MSA_TOPK_CASE(29)
    MSA_TOPK_CASE(30) MSA_TOPK_CASE(31)
#undef MSA_TOPK_CASE
    default:
      return fail(MSA_ERR_UNSUPPORTED, "k=%d", k);
  }
  return MSA_OK;
}

template <int KM>
void launch_topk_decode(const TopkDecodeParams& tp, cudaStream_t st) {
  const int rows = tp.B * tp.G;
  topk_decode_kernel<KM><<<(rows + 7) / 8, 256, 0, st>>>(tp);   // one warp per row
}

msa_status_t dispatch_topk_decode(int k, const TopkDecodeParams& tp, cudaStream_t st) {
  switch (k - 1) {
#define MSA_TOPK_CASE(KM) \
  case KM:                \
    launch_topk_decode<KM>(tp, st); break;
    MSA_TOPK_CASE(0) MSA_TOPK_CASE(1) MSA_TOPK_CASE(2) MSA_TOPK_CASE(3) MSA_TOPK_CASE(4) MSA_TOPK_CASE(5)
    MSA_TOPK_CASE(6) MSA_TOPK_CASE(7) MSA_TOPK_CASE(8) MSA_TOPK_CASE(9) MSA_TOPK_CASE(10) MSA_TOPK_CASE(11)
    MSA_TOPK_CASE(12) MSA_TOPK_CASE(13) MSA_TOPK_CASE(14) MSA_TOPK_CASE(15) MSA_TOPK_CASE(16) MSA_TOPK_CASE(17)
    MSA_TOPK_CASE(18) MSA_TOPK_CASE(19) MSA_TOPK_CASE(20) MSA_TOPK_CASE(21) MSA_TOPK_CASE(22) MSA_TOPK_CASE(23)
    MSA_TOPK_CASE(24) MSA_TOPK_CASE(25) MSA_TOPK_CASE(26) MSA_TOPK_CASE(27) MSA_TOPK_CASE(28) MSA_TOPK_CASE(29)
    MSA_TOPK_CASE(30) MSA_TOPK_CASE(31)
#undef MSA_TOPK_CASE
    default:
      return fail(MSA_ERR_UNSUPPORTED, "k=%d", k);
  }
  return MSA_OK;
}

template <int DI>
msa_status_t launch_index(const void* q_idx, const void* k_idx, int64_t n, int32_t g, const IndexLayout& L,
                          int32_t* block_ids, int32_t k, cudaStream_t st) {
  using C = IdxCfg<DI>;
  static std::once_flag once;
  static msa_status_t attr = MSA_OK;
  std::call_once(once, [] { attr = set_smem(index_blockmax_kernel<DI>, C::kSmemBytes); });
  if (attr != MSA_OK) return attr;
  const int64_t nb = (n + 127) / 128;
  const uint64_t row_stride = uint64_t(g) * DI * 2;
  CUtensorMap tq, tk;
  const uint32_t box0 = C::kSw64 ? 32 : 64;
  const CUtensorMapSwizzle sw = C::kSw64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  msa_status_t s;
  if ((s = make_map_3d(&tq, q_idx, DI, g, n, DI * 2, row_stride, box0, 1, 128, sw)) != MSA_OK) return s;
  if ((s = make_map_3d(&tk, k_idx, DI, g, n, DI * 2, row_stride, box0, 1, 128, sw)) != MSA_OK) return s;
  const int sms = num_sms();
  for (auto& ch : index_chunks(nb, g, L.cap)) {
    const int qb0 = ch.first, qb1 = ch.second;
    IdxParams P{};
    P.qb0 = qb0;
    P.qb1 = qb1;
    P.npairs = (qb1 - qb0 + 1) / 2;
    P.G = g;
    P.maxima = L.maxima;
    P.region_per_group = 128 * (tri(qb1) - tri(qb0));
    IdxRunTable T{};
    // kbend(p) = qa + 1 with a partner tile, qa without; nondecreasing in p
    auto kbend = [&](int p) { const int qa = qb0 + 2 * p; return (qa + 1 < qb1) ? qa + 1 : qa; };
    const int maxend = P.npairs > 0 ? kbend(P.npairs - 1) : 0;
    P.nruns = (maxend + kIdxKbRun - 1) / kIdxKbRun;
    if (P.nruns > kIdxMaxRuns)   // excluded by check_index_n before anything is enqueued
      return fail(MSA_ERR_UNSUPPORTED, "index launch needs %d key runs (at most %d)", P.nruns, kIdxMaxRuns);
    int acc = 0;
    for (int c = 0; c < P.nruns; ++c) {
      int p = 0;
      while (p < P.npairs && kbend(p) <= c * kIdxKbRun) ++p;
      T.pmin[c] = p;
      T.prefix[c] = acc;
      acc += P.npairs - p;
    }
    T.prefix[P.nruns] = acc;
    P.items_per_group = acc;
    const int64_t total = int64_t(acc) * g;
    if (total > 0) {
      const int grid = int(std::min<int64_t>(sms, total));
      ProfScope ps(kPIndex, st);
      index_blockmax_kernel<DI><<<grid, kIdxThreads, C::kSmemBytes, st>>>(tq, tk, P, T);
      MSA_CHECK_LAUNCH();
    }
    TopkPrefillParams tp{};
    tp.maxima = L.maxima;
    tp.block_ids = block_ids;
    tp.N = n;
    tp.G = g;
    tp.k = k;
    tp.qb0 = qb0;
    tp.region_per_group = P.region_per_group;
    {
      ProfScope ps(kPTopkPrefill, st);
      if ((s = dispatch_topk_prefill(k, tp, dim3(qb1 - qb0, g), st)) != MSA_OK) return s;
    }
    MSA_CHECK_LAUNCH();
  }
  return MSA_OK;
}

// The one-kernel Index Branch (Top-k fused into the score epilogue, no block maxima in
// memory) serves the common k at every length: its CTAs sweep the key blocks of one group in
// near lockstep (each item starts at key block 0, and the items of a round have nearly equal
// lengths), so the key tiles they stream are shared through L2 even when the group's index
// keys are larger than L2. Anything else takes the two-kernel path.
#ifndef MSA_FUSED_INDEX_MAX_N
#define MSA_FUSED_INDEX_MAX_N ((int64_t(1) << 26) - 1)
#endif
constexpr int64_t kFusedIndexMaxN = MSA_FUSED_INDEX_MAX_N;
bool fused_index_ok(int64_t n, int32_t k) {
  return n <= kFusedIndexMaxN && (k == 4 || k == 8 || k == 16 || k == 32);
}

// Sequence-length limit of the Index Branch path that serves (n, k); checked before anything
// is enqueued.
msa_status_t check_index_n(int64_t n, int32_t bk, int32_t k) {
  const int64_t nb = (n + 127) / 128;
  if (bk != 128 && !fused_index_ok(n, k))
    return fail(MSA_ERR_UNSUPPORTED, "bk=%d takes the one-kernel Index Branch only (k in 4, 8, 16, 32; got k=%d)", bk, k);
  if (!fused_index_ok(n, k) && nb > kTwoKernelMaxBlocks)
    return fail(MSA_ERR_UNSUPPORTED, "n=%lld with k=%d takes the two-kernel Index Branch, which serves at most %lld tokens",
                (long long)n, k, (long long)(kTwoKernelMaxBlocks * 128));
  return MSA_OK;
}

// Sequence-length limit of the Main Branch (CSR build); checked before anything is enqueued.
msa_status_t check_attn_n(int64_t n, int32_t bk) {
  const int64_t nb = (n + bk - 1) / bk;
  if (nb > kCsrMaxBlocks)
    return fail(MSA_ERR_UNSUPPORTED, "n=%lld with bk=%d: the Main Branch serves at most %lld blocks (%lld tokens)",
                (long long)n, bk, (long long)kCsrMaxBlocks, (long long)(kCsrMaxBlocks * bk));
  return MSA_OK;
}

size_t index_ws_bytes(int64_t n, int32_t g, int32_t k) {
  return fused_index_ok(n, k) ? kAlign : index_layout(nullptr, n, g).bytes;
}

template <int DI, int KM, int BK>
msa_status_t launch_index_topk_km(const CUtensorMap& tq, const CUtensorMap& tk, const IdxTopkParams& P,
                                  cudaStream_t st) {
  using C = IdxTopkCfg<DI, KM>;
  static std::once_flag once;
  static msa_status_t attr = MSA_OK;
  std::call_once(once, [] { attr = set_smem(index_topk_kernel<DI, KM, BK>, C::kSmemBytes); });
  if (attr != MSA_OK) return attr;
  const int total = P.G * P.nt;
  const int grid = std::min(num_sms(), total);
  ProfScope ps(kPIndexTopk, st);
  index_topk_kernel<DI, KM, BK><<<grid, kIdxThreads, C::kSmemBytes, st>>>(tq, tk, P);
  MSA_CHECK_LAUNCH();
  return MSA_OK;
}

template <int DI, int BK>
msa_status_t launch_index_topk_bk(const CUtensorMap& tq, const CUtensorMap& tk, const IdxTopkParams& P, int32_t k,
                                  cudaStream_t st) {
  switch (k) {
    case 4: return launch_index_topk_km<DI, 3, BK>(tq, tk, P, st);
    case 8: return launch_index_topk_km<DI, 7, BK>(tq, tk, P, st);
    case 16: return launch_index_topk_km<DI, 15, BK>(tq, tk, P, st);
    default: return launch_index_topk_km<DI, 31, BK>(tq, tk, P, st);
  }
}

template <int DI>
msa_status_t launch_index_topk(const void* q_idx, const void* k_idx, int64_t n, int32_t g, int32_t* block_ids,
                               int32_t bk, int32_t k, cudaStream_t st) {
  using C = IdxCfg<DI>;
  const uint64_t row_stride = uint64_t(g) * DI * 2;
  CUtensorMap tq, tk;
  const uint32_t box0 = C::kSw64 ? 32 : 64;
  const CUtensorMapSwizzle sw = C::kSw64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  msa_status_t s;
  if ((s = make_map_3d(&tq, q_idx, DI, g, n, DI * 2, row_stride, box0, 1, 128, sw)) != MSA_OK) return s;
  if ((s = make_map_3d(&tk, k_idx, DI, g, n, DI * 2, row_stride, box0, 1, 128, sw)) != MSA_OK) return s;
  IdxTopkParams P{};
  P.nt = int((n + 127) / 128);
  P.G = g;
  P.k = k;
  P.N = n;
  P.block_ids = block_ids;
  if (bk == 128) return launch_index_topk_bk<DI, 128>(tq, tk, P, k, st);
  if (bk == 64) return launch_index_topk_bk<DI, 64>(tq, tk, P, k, st);
  return launch_index_topk_bk<DI, 32>(tq, tk, P, k, st);
}

msa_status_t run_index_select(const void* q_idx, const void* k_idx, int64_t n, int32_t g, int32_t d_idx, int32_t bk,
                              int32_t k, int32_t* block_ids, void* ws, cudaStream_t st) {
  if (fused_index_ok(n, k)) {
    switch (d_idx) {
      case 32: return launch_index_topk<32>(q_idx, k_idx, n, g, block_ids, bk, k, st);
      case 64: return launch_index_topk<64>(q_idx, k_idx, n, g, block_ids, bk, k, st);
      default: return launch_index_topk<128>(q_idx, k_idx, n, g, block_ids, bk, k, st);
    }
  }
  if (bk != 128) return fail(MSA_ERR_UNSUPPORTED, "bk=%d needs the one-kernel Index Branch", bk);
  IndexLayout L = index_layout(ws, n, g);
  switch (d_idx) {
    case 32: return launch_index<32>(q_idx, k_idx, n, g, L, block_ids, k, st);
    case 64: return launch_index<64>(q_idx, k_idx, n, g, L, block_ids, k, st);
    case 128: return launch_index<128>(q_idx, k_idx, n, g, L, block_ids, k, st);
    default: return fail(MSA_ERR_UNSUPPORTED, "d_idx=%d", d_idx);
  }
}

// ------------------------ Index Branch without caller workspace ------------------------
// Scratch for msa_index_select_static: the packed block maxima of one index launch live in
// this file-scope device array instead of a caller-provided workspace. It is part of the
// library's device image, so every GPU that loads the library holds it until the process
// exits; calls on one device share it.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_static_mu;
constexpr int kMaxDevices = 128;
void* g_static_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device, looked up once per device (host
// code only sees a host-side stand-in for the symbol; that stand-in must never reach a
// kernel). The first call on a device does the lookup.
msa_status_t static_scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(MSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(MSA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (g_static_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(MSA_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(e));
    g_static_addr[dev] = p;
  }
  *out = g_static_addr[dev];
  return MSA_OK;
}

// ------------------------------- main branch (prefill) -------------------------------
// Chunk overlap. The KV-outer pass of chunk c + 1 (bound by the exp unit and the MMA chain)
// runs on the caller's stream while the merge of chunk c (bound by HBM) runs on a second
// stream, each on its own share of the SMs: kvouter launches sms - merge_sms persistent CTAs
// and the merge merge_sms, so both are resident at once. The partials and (m, l) pairs are
// double-buffered by chunk parity. The first KV-outer pass and the last merge run alone and
// take every SM. MSA_MERGE_SMS overrides the merge's share (0 runs the chunks back to back).
int merge_sm_count(int sms) {
  static int v = [] {
    const char* e = std::getenv("MSA_MERGE_SMS");
    return e ? std::atoi(e) : kDefaultMergeSms;
  }();
  return std::max(0, std::min(v, sms / 2));
}

struct AttnLayout {
  int64_t chunk_tiles = 0;    // 128-query tiles per chunk
  int64_t chunks = 0;
  uint32_t *hist = nullptr, *totals = nullptr, *bstart = nullptr, *istart = nullptr;
  int32_t* entries = nullptr;
  int4* items = nullptr;
  void* opart[2] = {nullptr, nullptr};   // chunk c uses buffer c % 2 (one buffer for one chunk)
  float2* ml[2] = {nullptr, nullptr};
  CsrChunkTable table{};                  // per-chunk regions of the inverted index
  float* kl_part = nullptr;               // msa_index_kl: one chunk's (query, group, slot) partial sums
  size_t bytes = 0;
};

int rows_per_query(int R) { return R < 8 ? 8 : R; }

// Tiles per chunk: the requested query chunk (a multiple of 128; 0 = the default), raised if
// needed so that the sequence has at most kCsrMaxChunks chunks.
int64_t chunk_tiles(int64_t n, int64_t query_chunk) {
  const int64_t nt = (n + 127) / 128;
  int64_t cq = (query_chunk > 0 ? query_chunk : kDefaultQueryChunk) / 128;
  cq = std::max<int64_t>(cq, (nt + kCsrMaxChunks - 1) / kCsrMaxChunks);
  return std::max<int64_t>(1, std::min(cq, nt));
}

// kl = true: the layout of msa_index_kl (the inverted index and one chunk's KL partials
// instead of the attention partials).
AttnLayout attn_layout(void* ws, int64_t n, int32_t hq, int32_t g, int32_t d, int32_t bk, int32_t k,
                       int64_t query_chunk, bool kl = false) {
  const int64_t nt = (n + 127) / 128;
  const int64_t nblocks = (n + bk - 1) / bk;
  const int64_t bpt = 128 / bk;
  const int R = hq / g;
  const int TQ = 128 / rows_per_query(R);
  AttnLayout L;
  L.chunk_tiles = chunk_tiles(n, query_chunk);
  L.chunks = (nt + L.chunk_tiles - 1) / L.chunk_tiles;
  int64_t hist = 0, buckets = 0, entries = 0, items = 0;
  for (int64_t c = 0; c < L.chunks; ++c) {
    const int64_t t0 = c * L.chunk_tiles, ntc = std::min(L.chunk_tiles, nt - t0);
    const int64_t nbk = std::min(nblocks, (t0 + ntc) * bpt);
    const int64_t rows = std::min(n, (t0 + ntc) * 128) - t0 * 128;
    L.table.hist[c] = hist;
    L.table.bucket[c] = buckets;
    L.table.entry[c] = entries;
    L.table.item[c] = items;
    hist += int64_t(g) * nbk * ntc;
    buckets += int64_t(g) * nbk;
    entries += rows * g * k;
    items += rows * g * k / (int64_t(TQ) * kKvItemTiles) + int64_t(g) * nbk + 1;
  }
  L.table.bucket[L.chunks] = buckets;
  const int64_t rows = L.chunk_tiles * 128;
  const int64_t max_entries = rows * g * k;   // of one chunk
  Carver cv(ws);
  L.hist = static_cast<uint32_t*>(cv.take(size_t(hist) * 4));
  L.totals = static_cast<uint32_t*>(cv.take(size_t(buckets) * 4));
  L.bstart = static_cast<uint32_t*>(cv.take(size_t(buckets + L.chunks) * 4));
  L.istart = static_cast<uint32_t*>(cv.take(size_t(buckets + L.chunks) * 4));
  L.entries = static_cast<int32_t*>(cv.take(size_t(entries) * 4));
  L.items = static_cast<int4*>(cv.take(size_t(items) * 16));
  if (kl) {
    L.kl_part = static_cast<float*>(cv.take(size_t(max_entries) * 32));
    L.bytes = cv.off;
    return L;
  }
  const int nbuf = (L.chunks > 1 && merge_sm_count(num_sms()) > 0) ? 2 : 1;   // overlap needs two
  for (int i = 0; i < nbuf; ++i) {
    L.opart[i] = cv.take(size_t(max_entries) * R * d * 2);
    L.ml[i] = static_cast<float2*>(cv.take(size_t(max_entries) * R * 8));
  }
  if (nbuf == 1) { L.opart[1] = L.opart[0]; L.ml[1] = L.ml[0]; }
  L.bytes = cv.off;
  return L;
}

template <int D, int RP, int BK>
msa_status_t launch_kvouter(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                            const KvParams& kp, int grid, cudaStream_t st) {
  using C = KvCfg<D, RP, BK>;
  static std::once_flag once;
  static msa_status_t attr = MSA_OK;
  std::call_once(once, [] { attr = set_smem(kvouter_kernel<D, RP, BK>, C::kSmemBytes); });
  if (attr != MSA_OK) return attr;
  ProfScope ps(kPKvOuter, st);
  kvouter_kernel<D, RP, BK><<<grid, kKvThreads, C::kSmemBytes, st>>>(tq, tk, tv, to, kp);
  MSA_CHECK_LAUNCH();
  return MSA_OK;
}

template <int D, int BK>
msa_status_t dispatch_kvouter_r(int R, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& to, const KvParams& kp, int grid, cudaStream_t st) {
  if (R <= 8) return launch_kvouter<D, 8, BK>(tq, tk, tv, to, kp, grid, st);
  return launch_kvouter<D, 16, BK>(tq, tk, tv, to, kp, grid, st);
}

msa_status_t dispatch_kvouter(int d, int R, int bk, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const CUtensorMap& to, const KvParams& kp, int grid, cudaStream_t st) {
  if (d == 128) {
    if (bk == 128) return dispatch_kvouter_r<128, 128>(R, tq, tk, tv, to, kp, grid, st);
    if (bk == 64) return dispatch_kvouter_r<128, 64>(R, tq, tk, tv, to, kp, grid, st);
    return dispatch_kvouter_r<128, 32>(R, tq, tk, tv, to, kp, grid, st);
  }
  if (bk == 128) return dispatch_kvouter_r<64, 128>(R, tq, tk, tv, to, kp, grid, st);
  if (bk == 64) return dispatch_kvouter_r<64, 64>(R, tq, tk, tv, to, kp, grid, st);
  return dispatch_kvouter_r<64, 32>(R, tq, tk, tv, to, kp, grid, st);
}

// The streaming merge: a ring of shared-memory stages, each holding one (query, group) slab
// of partials plus its (m, l) pairs, ids and weights; as many stages as fit ~210 KB (8 at
// most), rounded down to a multiple of the consumer groups that run.
msa_status_t launch_merge_stream(const MergeParams& mp, int d, int max_grid, cudaStream_t st) {
  MergeStreamLayout L{};
  const int kR = mp.k * mp.R;
  L.slab_bytes = kR * d * 2;
  L.ml_off = (L.slab_bytes + 15) / 16 * 16;
  L.ids_off = (L.ml_off + kR * 8 + 15) / 16 * 16;
  L.w_off = (L.ids_off + mp.k * 4 + 15) / 16 * 16;
  L.stage_bytes = (L.w_off + kR * 4 + 127) / 128 * 128;
  const int fit = std::min(8, (210 * 1024) / L.stage_bytes);
  L.groups = std::max(1, std::min(kMergeGroups, fit));
  L.stages = std::max(1, fit / L.groups * L.groups);
  L.bulk_meta = (kR % 2 == 0 && mp.k % 4 == 0) ? 1 : 0;
  const int smem = L.stages * L.stage_bytes + L.stages * 16 + 16 + 128;
  if (smem > 227 * 1024) return fail(MSA_ERR_UNSUPPORTED, "merge stage of %d bytes too large", L.stage_bytes);
  static std::once_flag once;
  static msa_status_t attr = MSA_OK;
  std::call_once(once, [] {
    attr = set_smem(merge_stream_kernel<128, false>, 227 * 1024);
    if (attr == MSA_OK) attr = set_smem(merge_stream_kernel<64, false>, 227 * 1024);
    if (attr == MSA_OK) attr = set_smem(merge_stream_kernel<128, true>, 227 * 1024);
    if (attr == MSA_OK) attr = set_smem(merge_stream_kernel<64, true>, 227 * 1024);
  });
  if (attr != MSA_OK) return attr;
  const int64_t units = mp.rows * mp.G;
  const int grid = int(std::min<int64_t>(max_grid, units));
  {
    ProfScope ps(kPMerge, st);
    const bool lse = mp.lse != nullptr;
    if (d == 128) {
      if (lse) merge_stream_kernel<128, true><<<grid, kMergeThreads, smem, st>>>(mp, L);
      else merge_stream_kernel<128, false><<<grid, kMergeThreads, smem, st>>>(mp, L);
    } else {
      if (lse) merge_stream_kernel<64, true><<<grid, kMergeThreads, smem, st>>>(mp, L);
      else merge_stream_kernel<64, false><<<grid, kMergeThreads, smem, st>>>(mp, L);
    }
  }
  MSA_CHECK_LAUNCH();
  return MSA_OK;
}

msa_status_t set_csr_smem() {
  static std::once_flag once;
  static msa_status_t attr = MSA_OK;
  std::call_once(once, [] {
    attr = set_smem(csr_count_kernel, 227 * 1024);
    if (attr == MSA_OK) attr = set_smem(csr_scatter_kernel, 227 * 1024);
  });
  return attr;
}

// Extra streams of the calling device, created once per device and kept: kind 0 runs the
// overlapped merges, kind 1 the host-to-device copies and kind 2 the device-to-host copies of
// msa_forward_host.
cudaStream_t aux_stream(int kind) {
  static std::mutex mu;
  static cudaStream_t streams[3][64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  if (dev < 0 || dev >= 64 || kind < 0 || kind > 2) return nullptr;
  cudaStream_t& s = streams[kind][dev];
  if (s == nullptr && cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) s = nullptr;
  return s;
}
cudaStream_t side_stream() { return aux_stream(0); }

// Events of one call, destroyed when the call returns (CUDA releases them once they complete).
struct EventSet {
  std::vector<cudaEvent_t> ev;
  bool make(size_t n) {
    ev.assign(n, nullptr);
    for (auto& e : ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return false;
    return true;
  }
  ~EventSet() {
    for (auto e : ev)
      if (e) cudaEventDestroy(e);
  }
};

// Joins the side stream back into the caller's stream when a call returns, on success or
// after an error, so that no merge is still in flight on memory the caller may reuse.
struct SideJoin {
  cudaStream_t st = nullptr, side = nullptr;
  ~SideJoin() {
    if (side == nullptr) return;
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      cudaStreamSynchronize(side);
      return;
    }
    cudaEventRecord(e, side);
    cudaStreamWaitEvent(st, e, 0);
    cudaEventDestroy(e);
  }
};

// The inverted index of every query chunk, in five launches (see csr.cuh).
msa_status_t build_csr(const AttnLayout& L, const int32_t* block_ids, int64_t n, int32_t g, int32_t bk, int32_t k,
                       int TQ, cudaStream_t st) {
  CsrParams cp{};
  cp.block_ids = block_ids;
  cp.N = n;
  cp.G = g;
  cp.k = k;
  cp.bk = bk;
  cp.bpt = 128 / bk;
  cp.ntiles = int((n + 127) / 128);
  cp.nblocks = int((n + bk - 1) / bk);
  cp.ct = int(L.chunk_tiles);
  cp.nchunks = int(L.chunks);
  cp.tq = TQ;
  cp.item_tiles = kKvItemTiles;
  cp.hist = L.hist;
  cp.totals = L.totals;
  cp.bucket_start = L.bstart;
  cp.item_start = L.istart;
  cp.entries = L.entries;
  cp.items = L.items;
  const int64_t buckets = L.table.bucket[L.chunks];
  const size_t bm_bytes = size_t(cp.nblocks) * 16;   // masks of the last tile (checked by check_attn_n)
  if (bm_bytes > 227 * 1024) return fail(MSA_ERR_UNSUPPORTED, "sequence too long for the CSR build (%d blocks)", cp.nblocks);
  const dim3 tiles(unsigned(cp.ntiles), unsigned(g));
  { ProfScope ps(kPCsrCount, st); csr_count_kernel<<<tiles, 128, bm_bytes, st>>>(cp, L.table); }
  MSA_CHECK_LAUNCH();
  { ProfScope ps(kPCsrScan, st); csr_scan_kernel<<<unsigned((buckets + 7) / 8), 256, 0, st>>>(cp, L.table); }
  MSA_CHECK_LAUNCH();
  { ProfScope ps(kPCsrOffsets, st); csr_offsets_kernel<<<unsigned(L.chunks), 1024, 0, st>>>(cp, L.table); }
  MSA_CHECK_LAUNCH();
  { ProfScope ps(kPCsrScatter, st); csr_scatter_kernel<<<tiles, 128, bm_bytes, st>>>(cp, L.table); }
  MSA_CHECK_LAUNCH();
  { ProfScope ps(kPCsrItems, st); csr_items_kernel<<<unsigned((buckets + 255) / 256), 256, 0, st>>>(cp, L.table); }
  MSA_CHECK_LAUNCH();
  return MSA_OK;
}

// chunk_in (optional, one event per chunk): the caller's stream waits for chunk_in[c] before
// chunk c's attention kernels (its query rows and the key/value rows up to its end must be
// resident; the inverted index needs only the block ids).
// chunk_out (optional): recorded after chunk c's merge, once o's rows of chunk c are final.
msa_status_t run_sparse_attn(const void* q, const void* kk, const void* v, const int32_t* block_ids, int64_t n,
                             int32_t hq, int32_t g, int32_t d, int32_t bk, int32_t k, float scale, void* o, void* ws,
                             int64_t query_chunk, cudaStream_t st, const cudaEvent_t* chunk_in = nullptr,
                             const cudaEvent_t* chunk_out = nullptr, float* lse = nullptr) {
  msa_status_t s;
  if ((s = set_csr_smem()) != MSA_OK) return s;
  const int R = hq / g;
  const int RP = rows_per_query(R);
  const int TQ = 128 / RP;
  AttnLayout L = attn_layout(ws, n, hq, g, d, bk, k, query_chunk);
  const int64_t nt = (n + 127) / 128;
  const int64_t nblocks = (n + bk - 1) / bk;
  if (scale == 0.0f) scale = 1.0f / std::sqrt(float(d));
  CUtensorMap tq, tk, tv, to[2];
  const uint64_t panels = uint64_t(d) / 64;
  // q as (64 elems, hq heads, panels, n): one box = 8 heads x all panels of one query
  if ((s = make_map_4d(&tq, q, {64, uint64_t(hq), panels, uint64_t(n)},
                       {uint64_t(d) * 2, 128, uint64_t(hq) * d * 2}, {64, 8, uint32_t(panels), 1},
                       CU_TENSOR_MAP_SWIZZLE_128B)) != MSA_OK)
    return s;
  if ((s = make_map_3d(&tk, kk, d, g, n, uint64_t(d) * 2, uint64_t(g) * d * 2, 64, 1, uint32_t(bk),
                       CU_TENSOR_MAP_SWIZZLE_128B)) != MSA_OK)
    return s;
  if ((s = make_map_3d(&tv, v, d, g, n, uint64_t(d) * 2, uint64_t(g) * d * 2, 64, 1, uint32_t(bk),
                       CU_TENSOR_MAP_SWIZZLE_128B)) != MSA_OK)
    return s;
  const int64_t slot_rows = L.chunk_tiles * 128 * g * k;
  // partials [rows][R][d] as (64 elems, R heads, panels, rows); R >= 8: one box per 8 heads
  // covering all panels, R < 8: one box per panel
  for (int i = 0; i < 2; ++i)
    if ((s = make_map_4d(&to[i], L.opart[i], {64, uint64_t(R), panels, uint64_t(slot_rows)},
                         {uint64_t(d) * 2, 128, uint64_t(R) * d * 2},
                         {64, uint32_t(std::min(R, 8)), R >= 8 ? uint32_t(panels) : 1u, 1},
                         CU_TENSOR_MAP_SWIZZLE_128B)) != MSA_OK)
      return s;
  if ((s = build_csr(L, block_ids, n, g, bk, k, TQ, st)) != MSA_OK) return s;
  const int sms = num_sms();
  const int msms = (L.chunks > 1 && L.opart[1] != L.opart[0]) ? merge_sm_count(sms) : 0;
  cudaStream_t side = msms > 0 ? side_stream() : nullptr;
  const bool overlap = side != nullptr;
  EventSet kv_done, m_done;   // per chunk: KV-outer pass done (caller's stream), merge done (side stream)
  if (overlap && (!kv_done.make(size_t(L.chunks)) || !m_done.make(size_t(L.chunks))))
    return fail(MSA_ERR_CUDA, "cudaEventCreateWithFlags failed");
  SideJoin join;   // declared after the events: it runs first when the call returns
  if (overlap) { join.st = st; join.side = side; }
  for (int64_t ci = 0; ci < L.chunks; ++ci) {
    const int64_t t0 = ci * L.chunk_tiles, t1 = std::min(nt, t0 + L.chunk_tiles);
    const int64_t nbk = std::min(nblocks, t1 * (128 / bk));
    const int buf = int(ci & 1);
    if (chunk_in && cudaStreamWaitEvent(st, chunk_in[ci], 0) != cudaSuccess)
      return fail(MSA_ERR_CUDA, "cudaStreamWaitEvent failed");
    KvParams kp{};
    kp.entries = L.entries + L.table.entry[ci];
    kp.items = L.items + L.table.item[ci];
    kp.n_items = L.istart + L.table.bucket[ci] + ci + int64_t(g) * nbk;
    kp.G = g;
    kp.R = R;
    kp.k = k;
    kp.nbk = int(nbk);
    kp.row0 = t0 * 128;
    kp.scale_log2 = scale * 1.4426950408889634f;
    kp.ml = L.ml[buf];
    // buffer `buf` was last read by the merge of chunk ci - 2
    if (overlap && ci >= 2 && cudaStreamWaitEvent(st, m_done.ev[ci - 2], 0) != cudaSuccess)
      return fail(MSA_ERR_CUDA, "cudaStreamWaitEvent failed");
    const int kv_grid = (overlap && ci > 0) ? sms - msms : sms;
    if ((s = dispatch_kvouter(d, R, bk, tq, tk, tv, to[buf], kp, kv_grid, st)) != MSA_OK) return s;
    cudaStream_t mst = st;
    if (overlap) {
      if (cudaEventRecord(kv_done.ev[ci], st) != cudaSuccess || cudaStreamWaitEvent(side, kv_done.ev[ci], 0) != cudaSuccess)
        return fail(MSA_ERR_CUDA, "cross-stream event failed");
      mst = side;
    }
    MergeParams mp{};
    mp.opart = static_cast<const __nv_bfloat16*>(L.opart[buf]);
    mp.ml = L.ml[buf];
    mp.block_ids = block_ids;
    mp.o = static_cast<__nv_bfloat16*>(o);
    mp.lse = lse;
    mp.row0 = t0 * 128;
    mp.rows = std::min<int64_t>(n, t1 * 128) - t0 * 128;
    mp.G = g;
    mp.R = R;
    mp.k = k;
    const int m_grid = (!overlap || ci == L.chunks - 1) ? sms : msms;
    if ((s = launch_merge_stream(mp, d, m_grid, mst)) != MSA_OK) return s;
    if (overlap && cudaEventRecord(m_done.ev[ci], side) != cudaSuccess)
      return fail(MSA_ERR_CUDA, "cudaEventRecord failed");
    if (chunk_out && cudaEventRecord(chunk_out[ci], mst) != cudaSuccess)
      return fail(MSA_ERR_CUDA, "cudaEventRecord failed");
  }
  return MSA_OK;   // the caller's stream resumes once the last merge is done (SideJoin)
}

// ------------------------------- decode -------------------------------
struct DecodeLayout {
  uint32_t* maxima = nullptr;
  int32_t* block_ids = nullptr;
  void* opart = nullptr;
  float2* ml = nullptr;
  size_t bytes = 0;
};

DecodeLayout decode_layout(void* ws, const msa_params* p, bool need_ids) {
  const int64_t B = p->n;
  const int64_t nbmax = (p->lmax + p->bk - 1) / p->bk;
  const int R = p->hq / p->g;
  Carver cv(ws);
  DecodeLayout L;
  L.maxima = static_cast<uint32_t*>(cv.take(size_t(B) * p->g * nbmax * 4));
  if (need_ids) L.block_ids = static_cast<int32_t*>(cv.take(size_t(B) * p->g * p->k * 4));
  L.opart = cv.take(size_t(B) * p->g * p->k * R * p->d * 2);
  L.ml = static_cast<float2*>(cv.take(size_t(B) * p->g * p->k * R * 8));
  L.bytes = cv.off;
  return L;
}

msa_status_t run_decode(const msa_params* p, const void* q, const void* kc, const void* vc, const void* q_idx,
                        const void* k_idx, int32_t* block_ids_out, void* o, void* ws, cudaStream_t st) {
  DecodeLayout L = decode_layout(ws, p, block_ids_out == nullptr);
  int32_t* ids = block_ids_out ? block_ids_out : L.block_ids;
  const int B = int(p->n);
  const int nbmax = int((p->lmax + p->bk - 1) / p->bk);
  const int R = p->hq / p->g;
  const float scale = p->scale == 0.0f ? 1.0f / std::sqrt(float(p->d)) : p->scale;
  DecodeScanParams sp{};
  sp.q_idx = static_cast<const __nv_bfloat16*>(q_idx);
  sp.k_idx = static_cast<const __nv_bfloat16*>(k_idx);
  sp.seqlens = p->seqlens;
  sp.maxima = L.maxima;
  sp.B = B;
  sp.G = p->g;
  sp.nbmax = nbmax;
  sp.bk = p->bk;
  sp.Lmax = p->lmax;
  const dim3 sgrid(unsigned((p->lmax + 127) / 128), B);
  {
    ProfScope ps(kPDecodeScan, st);
    switch (p->d_idx) {
      case 32: decode_scan_kernel<32><<<sgrid, 256, 0, st>>>(sp); break;
      case 64: decode_scan_kernel<64><<<sgrid, 256, 0, st>>>(sp); break;
      case 128: decode_scan_kernel<128><<<sgrid, 256, 0, st>>>(sp); break;
      default: return fail(MSA_ERR_UNSUPPORTED, "d_idx=%d", p->d_idx);
    }
  }
  MSA_CHECK_LAUNCH();
  TopkDecodeParams tp{};
  tp.maxima = L.maxima;
  tp.block_ids = ids;
  tp.seqlens = p->seqlens;
  tp.B = B;
  tp.G = p->g;
  tp.k = p->k;
  tp.nbmax = nbmax;
  tp.bk = p->bk;
  msa_status_t s;
  {
    ProfScope ps(kPTopkDecode, st);
    if ((s = dispatch_topk_decode(p->k, tp, st)) != MSA_OK) return s;
  }
  MSA_CHECK_LAUNCH();
  DecodeAttnParams ap{};
  ap.q = static_cast<const __nv_bfloat16*>(q);
  ap.kc = static_cast<const __nv_bfloat16*>(kc);
  ap.vc = static_cast<const __nv_bfloat16*>(vc);
  ap.seqlens = p->seqlens;
  ap.block_ids = ids;
  ap.opart = static_cast<__nv_bfloat16*>(L.opart);
  ap.ml = L.ml;
  ap.B = B;
  ap.G = p->g;
  ap.R = R;
  ap.k = p->k;
  ap.bk = p->bk;
  ap.Lmax = p->lmax;
  ap.scale_log2 = scale * 1.4426950408889634f;
  const int smem = 2 * 128 * (p->d + 8) * 2 + R * 128 * 4 + R * 8;
  const dim3 agrid(p->k, p->g, B);
  if (p->d == 128) {
    static std::once_flag once;
    static msa_status_t attr = MSA_OK;
    std::call_once(once, [] { attr = set_smem(decode_attn_kernel<128>, 200 * 1024); });
    if (attr != MSA_OK) return attr;
    ProfScope ps(kPDecodeAttn, st);
    decode_attn_kernel<128><<<agrid, 128, smem, st>>>(ap);
  } else {
    static std::once_flag once;
    static msa_status_t attr = MSA_OK;
    std::call_once(once, [] { attr = set_smem(decode_attn_kernel<64>, 200 * 1024); });
    if (attr != MSA_OK) return attr;
    ProfScope ps(kPDecodeAttn, st);
    decode_attn_kernel<64><<<agrid, 128, smem, st>>>(ap);
  }
  MSA_CHECK_LAUNCH();
  MergeParams mp{};
  mp.opart = static_cast<const __nv_bfloat16*>(L.opart);
  mp.ml = L.ml;
  mp.block_ids = ids;
  mp.o = static_cast<__nv_bfloat16*>(o);
  mp.row0 = 0;
  mp.rows = B;
  mp.G = p->g;
  mp.R = R;
  mp.k = p->k;
  const int hpw = 32 / (p->d / 8);
  const int64_t warps = (int64_t(B) * p->g * R + hpw - 1) / hpw;
  const unsigned blocks = unsigned((warps + 7) / 8);
  {
    ProfScope ps(kPMerge, st);
    if (p->d == 128) merge_kernel<128><<<blocks, 256, 0, st>>>(mp);
    else merge_kernel<64><<<blocks, 256, 0, st>>>(mp);
  }
  MSA_CHECK_LAUNCH();
  return MSA_OK;
}

msa_status_t check_main_dims(int32_t hq, int32_t g, int32_t d) {
  if (hq < 1 || hq % g != 0) return fail(MSA_ERR_INVALID_ARG, "hq=%d is not a positive multiple of g=%d", hq, g);
  if (!supported_r(hq / g)) return fail(MSA_ERR_UNSUPPORTED, "hq/g=%d unsupported (1, 2, 4, 8, 16)", hq / g);
  if (d != 64 && d != 128) return fail(MSA_ERR_UNSUPPORTED, "d=%d unsupported (64, 128)", d);
  return MSA_OK;
}

msa_status_t check_d_idx(int32_t d_idx) {
  if (d_idx != 32 && d_idx != 64 && d_idx != 128) return fail(MSA_ERR_UNSUPPORTED, "d_idx=%d unsupported (32, 64, 128)", d_idx);
  return MSA_OK;
}

size_t prefill_ids_bytes(int64_t n, int32_t g, int32_t k) { return align_up(size_t(n) * g * k * 4); }

// ------------------------------- index-branch KL loss -------------------------------
template <int D, int BK, int DI>
msa_status_t launch_kl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tki, const KlParams& kp,
                       int grid, cudaStream_t st) {
  using C = KlCfg<D, 8, BK, DI>;
  static std::once_flag once;
  static msa_status_t attr = MSA_OK;
  std::call_once(once, [] { attr = set_smem(kl_kernel<D, 8, BK, DI>, C::kSmemBytes); });
  if (attr != MSA_OK) return attr;
  ProfScope ps(kPKl, st);
  kl_kernel<D, 8, BK, DI><<<grid, kKlThreads, C::kSmemBytes, st>>>(tq, tk, tki, kp);
  MSA_CHECK_LAUNCH();
  return MSA_OK;
}

template <int D, int BK>
msa_status_t dispatch_kl_di(int di, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tki,
                            const KlParams& kp, int grid, cudaStream_t st) {
  if (di == 128) return launch_kl<D, BK, 128>(tq, tk, tki, kp, grid, st);
  if (di == 64) return launch_kl<D, BK, 64>(tq, tk, tki, kp, grid, st);
  return launch_kl<D, BK, 32>(tq, tk, tki, kp, grid, st);
}

msa_status_t dispatch_kl(int d, int bk, int di, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tki,
                         const KlParams& kp, int grid, cudaStream_t st) {
  if (d == 128) {
    if (bk == 128) return dispatch_kl_di<128, 128>(di, tq, tk, tki, kp, grid, st);
    if (bk == 64) return dispatch_kl_di<128, 64>(di, tq, tk, tki, kp, grid, st);
    return dispatch_kl_di<128, 32>(di, tq, tk, tki, kp, grid, st);
  }
  if (bk == 128) return dispatch_kl_di<64, 128>(di, tq, tk, tki, kp, grid, st);
  if (bk == 64) return dispatch_kl_di<64, 64>(di, tq, tk, tki, kp, grid, st);
  return dispatch_kl_di<64, 32>(di, tq, tk, tki, kp, grid, st);
}

msa_status_t run_index_kl(const msa_params* p, const void* q, const void* kk, const void* q_idx, const void* k_idx,
                          const int32_t* block_ids, const float* lse, float idx_scale, float* kl, void* ws,
                          cudaStream_t st) {
  msa_status_t s;
  if ((s = set_csr_smem()) != MSA_OK) return s;
  const int64_t n = p->n;
  const int g = p->g, hq = p->hq, d = p->d, di = p->d_idx, bk = p->bk, k = p->k;
  const int R = hq / g;
  const AttnLayout L = attn_layout(ws, n, hq, g, d, bk, k, p->query_chunk, true);
  const int64_t nt = (n + 127) / 128;
  const int64_t nblocks = (n + bk - 1) / bk;
  const float scale = p->scale == 0.0f ? 1.0f / std::sqrt(float(d)) : p->scale;
  if (idx_scale == 0.0f) idx_scale = 1.0f / std::sqrt(float(di));
  CUtensorMap tq, tk, tki;
  const uint64_t panels = uint64_t(d) / 64;
  if ((s = make_map_4d(&tq, q, {64, uint64_t(hq), panels, uint64_t(n)},
                       {uint64_t(d) * 2, 128, uint64_t(hq) * d * 2}, {64, 8, uint32_t(panels), 1},
                       CU_TENSOR_MAP_SWIZZLE_128B)) != MSA_OK)
    return s;
  if ((s = make_map_3d(&tk, kk, d, g, n, uint64_t(d) * 2, uint64_t(g) * d * 2, 64, 1, uint32_t(bk),
                       CU_TENSOR_MAP_SWIZZLE_128B)) != MSA_OK)
    return s;
  const bool sw64 = (di == 32);
  if ((s = make_map_3d(&tki, k_idx, di, g, n, uint64_t(di) * 2, uint64_t(g) * di * 2, sw64 ? 32 : 64, 1, uint32_t(bk),
                       sw64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B)) != MSA_OK)
    return s;
  if ((s = build_csr(L, block_ids, n, g, bk, k, 16, st)) != MSA_OK) return s;
  const int sms = num_sms();
  for (int64_t ci = 0; ci < L.chunks; ++ci) {
    const int64_t t0 = ci * L.chunk_tiles, t1 = std::min(nt, t0 + L.chunk_tiles);
    const int64_t nbk = std::min(nblocks, t1 * (128 / bk));
    KlParams kp{};
    kp.entries = L.entries + L.table.entry[ci];
    kp.items = L.items + L.table.item[ci];
    kp.n_items = L.istart + L.table.bucket[ci] + ci + int64_t(g) * nbk;
    kp.q_idx = static_cast<const __nv_bfloat16*>(q_idx);
    kp.lse = lse;
    kp.G = g;
    kp.R = R;
    kp.k = k;
    kp.nbk = int(nbk);
    kp.row0 = t0 * 128;
    kp.scale_log2 = scale * 1.4426950408889634f;
    kp.idx_scale_log2 = idx_scale * 1.4426950408889634f;
    kp.part = L.kl_part;
    if ((s = dispatch_kl(d, bk, di, tq, tk, tki, kp, sms, st)) != MSA_OK) return s;
    KlMergeParams mp{};
    mp.part = L.kl_part;
    mp.block_ids = block_ids;
    mp.kl = kl;
    mp.row0 = t0 * 128;
    mp.rows = std::min<int64_t>(n, t1 * 128) - t0 * 128;
    mp.G = g;
    mp.k = k;
    mp.idx_scale = idx_scale;
    {
      ProfScope ps(kPKlMerge, st);
      kl_merge_kernel<<<unsigned((mp.rows * g + 255) / 256), 256, 0, st>>>(mp);
    }
    MSA_CHECK_LAUNCH();
  }
  return MSA_OK;
}

msa_status_t check_kl_params(const msa_params* p) {
  msa_status_t s;
  if (!p) return fail(MSA_ERR_INVALID_ARG, "params is NULL");
  if (p->mode != MSA_MODE_PREFILL) return fail(MSA_ERR_UNSUPPORTED, "msa_index_kl takes prefill shapes only");
  if ((s = check_common(p->n, p->g, p->bk, p->k)) != MSA_OK) return s;
  if ((s = check_main_dims(p->hq, p->g, p->d)) != MSA_OK) return s;
  if ((s = check_d_idx(p->d_idx)) != MSA_OK) return s;
  if ((s = check_attn_n(p->n, p->bk)) != MSA_OK) return s;
  if (p->hq / p->g > 8) return fail(MSA_ERR_UNSUPPORTED, "msa_index_kl takes hq/g <= 8 (got %d)", p->hq / p->g);
  if (!(p->scale >= 0.0f) || std::isinf(p->scale)) return fail(MSA_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if (p->query_chunk < 0 || p->query_chunk % 128 != 0)
    return fail(MSA_ERR_INVALID_ARG, "query_chunk=%lld must be a non-negative multiple of 128", (long long)p->query_chunk);
  return MSA_OK;
}

}  // namespace

// =====================================================================================
// C ABI
// =====================================================================================
extern "C" {

const char* msa_status_string(msa_status_t s) {
  switch (s) {
    case MSA_OK: return "MSA_OK";
    case MSA_ERR_INVALID_ARG: return "MSA_ERR_INVALID_ARG";
    case MSA_ERR_UNSUPPORTED: return "MSA_ERR_UNSUPPORTED";
    case MSA_ERR_WORKSPACE: return "MSA_ERR_WORKSPACE";
    case MSA_ERR_CUDA: return "MSA_ERR_CUDA";
    case MSA_ERR_TIMEOUT: return "MSA_ERR_TIMEOUT";
    case MSA_ERR_DEVICE_BOUNDS: return "MSA_ERR_DEVICE_BOUNDS";
  }
  return "MSA_ERR_UNKNOWN";
}

const char* msa_last_error_detail(void) { return g_detail; }

size_t msa_index_select_workspace(int64_t n, int32_t g, int32_t d_idx, int32_t bk, int32_t k) {
  if (check_common(n, g, bk, k) != MSA_OK || check_d_idx(d_idx) != MSA_OK || check_index_n(n, bk, k) != MSA_OK) return 0;
  return index_ws_bytes(n, g, k);
}

msa_status_t msa_index_select(const void* q_idx, const void* k_idx, int64_t n, int32_t g, int32_t d_idx, int32_t bk,
                              int32_t k, int32_t* block_ids, void* workspace, size_t workspace_bytes, void* stream) {
  g_detail[0] = 0;
  msa_status_t s;
  if ((s = check_common(n, g, bk, k)) != MSA_OK) return s;
  if ((s = check_d_idx(d_idx)) != MSA_OK) return s;
  if ((s = check_index_n(n, bk, k)) != MSA_OK) return s;
  if ((s = check_ptr(q_idx, "q_idx")) != MSA_OK || (s = check_ptr(k_idx, "k_idx")) != MSA_OK ||
      (s = check_ptr(block_ids, "block_ids")) != MSA_OK || (s = check_ptr(workspace, "workspace")) != MSA_OK)
    return s;
  const size_t need = index_ws_bytes(n, g, k);
  if (workspace_bytes < need)
    return fail(MSA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, need);
  return run_index_select(q_idx, k_idx, n, g, d_idx, bk, k, block_ids, workspace, static_cast<cudaStream_t>(stream));
}

msa_status_t msa_index_select_static(const void* q_idx, const void* k_idx, int64_t n, int32_t g, int32_t d_idx,
                                     int32_t bk, int32_t k, int32_t* block_ids, void* stream) {
  g_detail[0] = 0;
  msa_status_t s;
  if ((s = check_common(n, g, bk, k)) != MSA_OK) return s;
  if ((s = check_d_idx(d_idx)) != MSA_OK) return s;
  if ((s = check_ptr(q_idx, "q_idx")) != MSA_OK || (s = check_ptr(k_idx, "k_idx")) != MSA_OK ||
      (s = check_ptr(block_ids, "block_ids")) != MSA_OK)
    return s;
  if ((s = check_index_n(n, bk, k)) != MSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the one-kernel Index Branch keeps no block maxima in memory: no scratch at all
  if (fused_index_ok(n, k)) return run_index_select(q_idx, k_idx, n, g, d_idx, bk, k, block_ids, nullptr, st);
  // the two-kernel path: the launches are cut so that each fits the static scratch; the last
  // query block alone needs 4 * g * 128 * (blocks - 1) bytes
  const int64_t nb = (n + 127) / 128;
  const size_t need = maxima_bytes(nb - 1, nb, g);
  if (need > kStaticScratchBytes)
    return fail(MSA_ERR_UNSUPPORTED,
                "n=%lld with g=%d needs %zu bytes of block-maxima scratch per query block; the static scratch "
                "holds %zu (use msa_index_select with a workspace)",
                (long long)n, g, need, kStaticScratchBytes);
  void* scratch = nullptr;
  if ((s = static_scratch_address(&scratch)) != MSA_OK) return s;
  IndexLayout L;
  L.maxima = static_cast<uint32_t*>(scratch);
  L.bytes = kStaticScratchBytes;
  L.cap = kStaticScratchBytes;
  switch (d_idx) {
    case 32: return launch_index<32>(q_idx, k_idx, n, g, L, block_ids, k, st);
    case 64: return launch_index<64>(q_idx, k_idx, n, g, L, block_ids, k, st);
    default: return launch_index<128>(q_idx, k_idx, n, g, L, block_ids, k, st);
  }
}

size_t msa_sparse_attn_workspace(int64_t n, int32_t hq, int32_t g, int32_t d, int32_t bk, int32_t k) {
  if (check_common(n, g, bk, k) != MSA_OK || check_main_dims(hq, g, d) != MSA_OK || check_attn_n(n, bk) != MSA_OK) return 0;
  return attn_layout(nullptr, n, hq, g, d, bk, k, 0).bytes;
}

msa_status_t msa_sparse_attn(const void* q, const void* k, const void* v, const int32_t* block_ids, int64_t n,
                             int32_t hq, int32_t g, int32_t d, int32_t bk, int32_t kk, float scale, void* o,
                             void* workspace, size_t workspace_bytes, void* stream) {
  g_detail[0] = 0;
  msa_status_t s;
  if ((s = check_common(n, g, bk, kk)) != MSA_OK) return s;
  if ((s = check_main_dims(hq, g, d)) != MSA_OK) return s;
  if ((s = check_attn_n(n, bk)) != MSA_OK) return s;
  if (!(scale >= 0.0f) || std::isinf(scale)) return fail(MSA_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if ((s = check_ptr(q, "q")) != MSA_OK || (s = check_ptr(k, "k")) != MSA_OK || (s = check_ptr(v, "v")) != MSA_OK ||
      (s = check_ptr(block_ids, "block_ids")) != MSA_OK || (s = check_ptr(o, "o")) != MSA_OK ||
      (s = check_ptr(workspace, "workspace")) != MSA_OK)
    return s;
  const size_t need = attn_layout(nullptr, n, hq, g, d, bk, kk, 0).bytes;
  if (workspace_bytes < need)
    return fail(MSA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, need);
  return run_sparse_attn(q, k, v, block_ids, n, hq, g, d, bk, kk, scale, o, workspace, 0,
                         static_cast<cudaStream_t>(stream));
}

size_t msa_forward_workspace(const msa_params* p) {
  if (!p) return 0;
  if (p->mode == MSA_MODE_PREFILL) {
    if (check_common(p->n, p->g, p->bk, p->k) != MSA_OK || check_main_dims(p->hq, p->g, p->d) != MSA_OK ||
        check_d_idx(p->d_idx) != MSA_OK || check_index_n(p->n, p->bk, p->k) != MSA_OK ||
        check_attn_n(p->n, p->bk) != MSA_OK)
      return 0;
    if (p->query_chunk < 0 || p->query_chunk % 128 != 0) return 0;
    const size_t a = attn_layout(nullptr, p->n, p->hq, p->g, p->d, p->bk, p->k, p->query_chunk).bytes;
    const size_t b = index_ws_bytes(p->n, p->g, p->k);
    return prefill_ids_bytes(p->n, p->g, p->k) + std::max(a, b);
  }
  if (p->mode == MSA_MODE_DECODE) {
    if (check_common(p->n, p->g, p->bk, p->k) != MSA_OK || check_main_dims(p->hq, p->g, p->d) != MSA_OK ||
        check_d_idx(p->d_idx) != MSA_OK || p->lmax < 1)
      return 0;
    return decode_layout(nullptr, p, true).bytes;
  }
  return 0;
}

msa_status_t msa_forward(const msa_params* p, const void* q, const void* k, const void* v, const void* q_idx,
                         const void* k_idx, int32_t* block_ids_out, void* o, void* workspace, size_t workspace_bytes,
                         void* stream) {
  g_detail[0] = 0;
  if (!p) return fail(MSA_ERR_INVALID_ARG, "params is NULL");
  msa_status_t s;
  if ((s = check_common(p->n, p->g, p->bk, p->k)) != MSA_OK) return s;
  if ((s = check_main_dims(p->hq, p->g, p->d)) != MSA_OK) return s;
  if ((s = check_d_idx(p->d_idx)) != MSA_OK) return s;
  if (!(p->scale >= 0.0f) || std::isinf(p->scale)) return fail(MSA_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if ((s = check_ptr(q, "q")) != MSA_OK || (s = check_ptr(k, "k")) != MSA_OK || (s = check_ptr(v, "v")) != MSA_OK ||
      (s = check_ptr(q_idx, "q_idx")) != MSA_OK || (s = check_ptr(k_idx, "k_idx")) != MSA_OK ||
      (s = check_ptr(o, "o")) != MSA_OK || (s = check_ptr(workspace, "workspace")) != MSA_OK)
    return s;
  if (block_ids_out && (s = check_ptr(block_ids_out, "block_ids_out")) != MSA_OK) return s;
  if (p->lse_out && (s = check_ptr(p->lse_out, "lse_out")) != MSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p->mode == MSA_MODE_PREFILL) {
    if ((s = check_index_n(p->n, p->bk, p->k)) != MSA_OK || (s = check_attn_n(p->n, p->bk)) != MSA_OK) return s;
    if (p->query_chunk < 0 || p->query_chunk % 128 != 0)
      return fail(MSA_ERR_INVALID_ARG, "query_chunk=%lld must be a non-negative multiple of 128", (long long)p->query_chunk);
    const size_t need = msa_forward_workspace(p);
    if (workspace_bytes < need)
      return fail(MSA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, need);
    uint8_t* w = static_cast<uint8_t*>(workspace);
    int32_t* ids = block_ids_out ? block_ids_out : reinterpret_cast<int32_t*>(w);
    void* rest = w + prefill_ids_bytes(p->n, p->g, p->k);
    if ((s = run_index_select(q_idx, k_idx, p->n, p->g, p->d_idx, p->bk, p->k, ids, rest, st)) != MSA_OK) return s;
    return run_sparse_attn(q, k, v, ids, p->n, p->hq, p->g, p->d, p->bk, p->k, p->scale, o, rest, p->query_chunk, st,
                           nullptr, nullptr, p->lse_out);
  }
  if (p->mode == MSA_MODE_DECODE) {
    if (p->lse_out) return fail(MSA_ERR_UNSUPPORTED, "lse_out is written by prefill only (pass NULL for decode)");
    if (p->lmax < 1 || p->lmax > kMaxN) return fail(MSA_ERR_INVALID_ARG, "lmax=%lld out of range", (long long)p->lmax);
    if ((s = check_ptr(p->seqlens, "seqlens")) != MSA_OK) return s;
    const int cpt = p->g * p->d_idx / 32;
    if (cpt > 32 || (cpt & (cpt - 1)) != 0)
      return fail(MSA_ERR_UNSUPPORTED, "decode needs g*d_idx/32 a power of two <= 32 (got %d)", cpt);
    if (p->n > 65535) return fail(MSA_ERR_UNSUPPORTED, "decode batch %lld > 65535", (long long)p->n);
    const size_t need = msa_forward_workspace(p);
    if (workspace_bytes < need)
      return fail(MSA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, need);
    return run_decode(p, q, k, v, q_idx, k_idx, block_ids_out, o, workspace, st);
  }
  return fail(MSA_ERR_INVALID_ARG, "mode=%d", p->mode);
}

// Device buffer of msa_forward_host: device copies of the five inputs and of o, then the
// msa_forward workspace (whose first bytes hold the block ids).
struct HostLayout {
  void *q, *k, *v, *qi, *ki, *o, *ws;
  size_t ws_bytes, bytes;
};
static HostLayout host_layout(void* base, const msa_params* p) {
  Carver cv(base);
  HostLayout H{};
  const size_t n = size_t(p->n);
  H.q = cv.take(n * p->hq * p->d * 2);
  H.k = cv.take(n * p->g * p->d * 2);
  H.v = cv.take(n * p->g * p->d * 2);
  H.qi = cv.take(n * p->g * p->d_idx * 2);
  H.ki = cv.take(n * p->g * p->d_idx * 2);
  H.o = cv.take(n * p->hq * p->d * 2);
  H.ws_bytes = msa_forward_workspace(p);
  H.ws = cv.take(H.ws_bytes);
  H.bytes = cv.off;
  return H;
}

size_t msa_forward_host_device_bytes(const msa_params* p) {
  if (!p || p->mode != MSA_MODE_PREFILL || msa_forward_workspace(p) == 0) return 0;
  return host_layout(nullptr, p).bytes;
}

msa_status_t msa_forward_host(const msa_params* p, const void* q, const void* k, const void* v, const void* q_idx,
                              const void* k_idx, int32_t* block_ids_out, void* o, void* device_buf,
                              size_t device_bytes, void* stream) {
  g_detail[0] = 0;
  if (!p) return fail(MSA_ERR_INVALID_ARG, "params is NULL");
  if (p->mode != MSA_MODE_PREFILL) return fail(MSA_ERR_UNSUPPORTED, "msa_forward_host takes prefill only");
  if (p->lse_out) return fail(MSA_ERR_UNSUPPORTED, "msa_forward_host does not write lse_out (pass NULL)");
  msa_status_t s;
  if ((s = check_common(p->n, p->g, p->bk, p->k)) != MSA_OK) return s;
  if ((s = check_main_dims(p->hq, p->g, p->d)) != MSA_OK) return s;
  if ((s = check_d_idx(p->d_idx)) != MSA_OK) return s;
  if ((s = check_index_n(p->n, p->bk, p->k)) != MSA_OK || (s = check_attn_n(p->n, p->bk)) != MSA_OK) return s;
  if (!(p->scale >= 0.0f) || std::isinf(p->scale)) return fail(MSA_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if (p->query_chunk < 0 || p->query_chunk % 128 != 0)
    return fail(MSA_ERR_INVALID_ARG, "query_chunk=%lld must be a non-negative multiple of 128", (long long)p->query_chunk);
  if ((s = check_ptr(q, "q")) != MSA_OK || (s = check_ptr(k, "k")) != MSA_OK || (s = check_ptr(v, "v")) != MSA_OK ||
      (s = check_ptr(q_idx, "q_idx")) != MSA_OK || (s = check_ptr(k_idx, "k_idx")) != MSA_OK ||
      (s = check_ptr(o, "o")) != MSA_OK || (s = check_ptr(device_buf, "device_buf")) != MSA_OK)
    return s;
  if (block_ids_out && (s = check_ptr(block_ids_out, "block_ids_out")) != MSA_OK) return s;
  const size_t need = msa_forward_host_device_bytes(p);
  if (device_bytes < need) return fail(MSA_ERR_WORKSPACE, "device buffer %zu bytes < %zu needed", device_bytes, need);
  const HostLayout H = host_layout(device_buf, p);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStream_t cin = aux_stream(1), cout = aux_stream(2);
  if (cin == nullptr || cout == nullptr) return fail(MSA_ERR_CUDA, "could not create the copy streams");
  const int64_t n = p->n;
  const AttnLayout L = attn_layout(nullptr, n, p->hq, p->g, p->d, p->bk, p->k, p->query_chunk);
  const int64_t rows_per_chunk = L.chunk_tiles * 128;
  EventSet ev;   // 0 start, 1 index inputs in, 2 selection done, then per chunk: rows in, rows out
  if (!ev.make(size_t(3 + 2 * L.chunks))) return fail(MSA_ERR_CUDA, "cudaEventCreateWithFlags failed");
  const cudaEvent_t* chunk_in = ev.ev.data() + 3;
  const cudaEvent_t* chunk_out = ev.ev.data() + 3 + L.chunks;
  SideJoin join_in, join_out;   // whatever happens, `stream` waits for both copy streams
  join_in.st = st; join_in.side = cin;
  join_out.st = st; join_out.side = cout;
  auto cuda_ok = [](cudaError_t e) { return e == cudaSuccess; };
  // the device buffer may still be in use by earlier work on `stream`
  if (!cuda_ok(cudaEventRecord(ev.ev[0], st)) || !cuda_ok(cudaStreamWaitEvent(cin, ev.ev[0], 0)) ||
      !cuda_ok(cudaStreamWaitEvent(cout, ev.ev[0], 0)))
    return fail(MSA_ERR_CUDA, "stream ordering failed");
  // index inputs first, alone on the link, so the Index Branch starts as early as possible
  const size_t idx_bytes = size_t(n) * p->g * p->d_idx * 2;
  if (!cuda_ok(cudaMemcpyAsync(H.qi, q_idx, idx_bytes, cudaMemcpyHostToDevice, st)) ||
      !cuda_ok(cudaMemcpyAsync(H.ki, k_idx, idx_bytes, cudaMemcpyHostToDevice, st)) ||
      !cuda_ok(cudaEventRecord(ev.ev[1], st)) || !cuda_ok(cudaStreamWaitEvent(cin, ev.ev[1], 0)))
    return fail(MSA_ERR_CUDA, "index input copy failed");
  // then the rows of q, k and v chunk by chunk, behind the Index Branch
  const size_t qrow = size_t(p->hq) * p->d * 2, krow = size_t(p->g) * p->d * 2;
  for (int64_t c = 0; c < L.chunks; ++c) {
    const int64_t r0 = c * rows_per_chunk, r1 = std::min(n, r0 + rows_per_chunk);
    const size_t nr = size_t(r1 - r0);
    if (!cuda_ok(cudaMemcpyAsync(static_cast<uint8_t*>(H.q) + r0 * qrow, static_cast<const uint8_t*>(q) + r0 * qrow,
                                 nr * qrow, cudaMemcpyHostToDevice, cin)) ||
        !cuda_ok(cudaMemcpyAsync(static_cast<uint8_t*>(H.k) + r0 * krow, static_cast<const uint8_t*>(k) + r0 * krow,
                                 nr * krow, cudaMemcpyHostToDevice, cin)) ||
        !cuda_ok(cudaMemcpyAsync(static_cast<uint8_t*>(H.v) + r0 * krow, static_cast<const uint8_t*>(v) + r0 * krow,
                                 nr * krow, cudaMemcpyHostToDevice, cin)) ||
        !cuda_ok(cudaEventRecord(chunk_in[c], cin)))
      return fail(MSA_ERR_CUDA, "input copy failed");
  }
  int32_t* ids = reinterpret_cast<int32_t*>(H.ws);
  void* rest = static_cast<uint8_t*>(H.ws) + prefill_ids_bytes(n, p->g, p->k);
  if ((s = run_index_select(H.qi, H.ki, n, p->g, p->d_idx, p->bk, p->k, ids, rest, st)) != MSA_OK) return s;
  if (block_ids_out) {
    if (!cuda_ok(cudaEventRecord(ev.ev[2], st)) || !cuda_ok(cudaStreamWaitEvent(cout, ev.ev[2], 0)) ||
        !cuda_ok(cudaMemcpyAsync(block_ids_out, ids, size_t(n) * p->g * p->k * 4, cudaMemcpyDeviceToHost, cout)))
      return fail(MSA_ERR_CUDA, "block id copy failed");
  }
  if ((s = run_sparse_attn(H.q, H.k, H.v, ids, n, p->hq, p->g, p->d, p->bk, p->k, p->scale, H.o, rest, p->query_chunk, st,
                           chunk_in, chunk_out, nullptr)) != MSA_OK)
    return s;
  // each chunk's output rows go back as soon as its merge is done
  for (int64_t c = 0; c < L.chunks; ++c) {
    const int64_t r0 = c * rows_per_chunk, r1 = std::min(n, r0 + rows_per_chunk);
    if (!cuda_ok(cudaStreamWaitEvent(cout, chunk_out[c], 0)) ||
        !cuda_ok(cudaMemcpyAsync(static_cast<uint8_t*>(o) + r0 * qrow, static_cast<const uint8_t*>(H.o) + r0 * qrow,
                                 size_t(r1 - r0) * qrow, cudaMemcpyDeviceToHost, cout)))
      return fail(MSA_ERR_CUDA, "output copy failed");
  }
  return MSA_OK;   // `stream` resumes once both copy streams are done (SideJoin)
}

size_t msa_index_kl_workspace(const msa_params* p) {
  if (check_kl_params(p) != MSA_OK) return 0;
  return attn_layout(nullptr, p->n, p->hq, p->g, p->d, p->bk, p->k, p->query_chunk, true).bytes;
}

msa_status_t msa_index_kl(const msa_params* p, const void* q, const void* k, const void* q_idx, const void* k_idx,
                          const int32_t* block_ids, const float* lse, float idx_scale, float* kl, void* workspace,
                          size_t workspace_bytes, void* stream) {
  g_detail[0] = 0;
  msa_status_t s;
  if ((s = check_kl_params(p)) != MSA_OK) return s;
  if (!(idx_scale >= 0.0f) || std::isinf(idx_scale)) return fail(MSA_ERR_INVALID_ARG, "idx_scale must be finite and >= 0");
  if ((s = check_ptr(q, "q")) != MSA_OK || (s = check_ptr(k, "k")) != MSA_OK || (s = check_ptr(q_idx, "q_idx")) != MSA_OK ||
      (s = check_ptr(k_idx, "k_idx")) != MSA_OK || (s = check_ptr(block_ids, "block_ids")) != MSA_OK ||
      (s = check_ptr(lse, "lse")) != MSA_OK || (s = check_ptr(kl, "kl")) != MSA_OK ||
      (s = check_ptr(workspace, "workspace")) != MSA_OK)
    return s;
  const size_t need = msa_index_kl_workspace(p);
  if (workspace_bytes < need) return fail(MSA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, need);
  return run_index_kl(p, q, k, q_idx, k_idx, block_ids, lse, idx_scale, kl, workspace, static_cast<cudaStream_t>(stream));
}

msa_status_t msa_profile_start(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = true;
  return MSA_OK;
}

int32_t msa_profile_stop(msa_kernel_stat* out, int32_t max_out) {
  std::vector<ProfRec> recs;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_on = false;
    recs.swap(g_prof);
  }
  int launches[kPNumKinds] = {0};
  double ms[kPNumKinds] = {0.0};
  bool ok = true;
  for (auto& r : recs) {
    float t = 0.0f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) ok = false;
    launches[r.kind] += 1;
    ms[r.kind] += t;
  }
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    for (auto& r : recs) {
      g_event_pool.push_back(r.a);
      g_event_pool.push_back(r.b);
    }
  }
  if (!ok) return -1;
  int32_t n = 0;
  for (int k = 0; k < kPNumKinds; ++k) {
    if (launches[k] == 0) continue;
    if (out && n < max_out) {
      out[n].name = kProfNames[k];
      out[n].launches = launches[k];
      out[n].total_ms = ms[k];
    }
    ++n;
  }
  return n;
}

msa_status_t msa_set_wait_limit_ns(uint64_t ns) {
  g_detail[0] = 0;
  const uint64_t v = (ns == 0) ? kWaitLimitNs : std::min<uint64_t>(ns, kWaitLimitNs);
  cudaError_t e = cudaMemcpyToSymbol(msa::g_msa_wait_limit_ns, &v, sizeof(v));
  if (e != cudaSuccess) return fail(MSA_ERR_CUDA, "set wait limit: %s", cudaGetErrorString(e));
  return MSA_OK;
}

msa_status_t msa_get_device_error(void* stream) {
  g_detail[0] = 0;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(MSA_ERR_CUDA, "stream sync: %s", cudaGetErrorString(e));
  unsigned int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, msa::g_msa_error, sizeof(v));
  if (e != cudaSuccess) return fail(MSA_ERR_CUDA, "read error word: %s", cudaGetErrorString(e));
  if (v != 0) {
    e = cudaMemcpyToSymbol(msa::g_msa_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return fail(MSA_ERR_CUDA, "clear error word: %s", cudaGetErrorString(e));
    fail(static_cast<msa_status_t>(v & 0xFF), "device error %s in kernel %u", msa_status_string(static_cast<msa_status_t>(v & 0xFF)),
         (v >> 8) & 0xFF);
    return static_cast<msa_status_t>(v & 0xFF);
  }
  return MSA_OK;
}

}  // extern "C"
