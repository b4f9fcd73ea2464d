// Host side of the fused linear cross-entropy C ABI (include/flce.h):
// argument checks, workspace layout, TMA tensor-map encoding and launches.
//
// bf16 path, forward:   tc_gemm<FwdStatsEpi> over all (128-token x 256-vocab)
//                       tiles -> fwd_merge -> row_loss -> finalize.
// bf16 path, backward:  the [N, V] problem is cut into chunks of at most
//                       kChunkTokens x kChunkVocab; per chunk
//                         tc_gemm<DzEpi>    dZ block (bf16, in the workspace)
//                         tc_gemm<StoreEpi> dHidden[chunk rows] (+)= dZ . W[chunk]
//                         tc_gemm<StoreEpi> dWeight[chunk rows] (+)= dZ^T . hidden[chunk]
//                       The first chunk along the reduced dimension stores,
//                       later ones TMA-reduce-add into the fp32 outputs.
// fp32 path:            simt_fwd / simt_dh / simt_dw (CUDA cores).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/flce.h"
#include "small_kernels.cuh"

namespace flce {
namespace {

constexpr int kChunkTokens = 4096;  // multiple of BM
constexpr int kChunkVocab = 8192;   // multiple of BN
constexpr int kGroupM = 16;
constexpr size_t kHeaderBytes = 256;
constexpr int64_t kMaxDim = (int64_t{1} << 31) - 1024;
constexpr int kSimtMaxH = 12288;

// ---------------------------------------------------------------- errors
thread_local char g_last_error[256];

flce_status cuda_fail(cudaError_t e) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s", cudaGetErrorString(e));
  return FLCE_ERR_CUDA;
}

// ---------------------------------------------------------------- profiling
constexpr int kKinds = 7;
enum Kind { kFwdGemm = 0, kFwdMerge = 1, kBwdDz = 2, kBwdDh = 3, kBwdDw = 4, kHelper = 5, kSimt = 6 };

struct ProfRec {
  int kind;
  cudaEvent_t a, b;
};

std::mutex g_prof_mu;
bool g_prof = false;
std::vector<ProfRec> g_recs;
std::atomic<uint64_t> g_launches{0};

template <class F>
cudaError_t launch(int kind, cudaStream_t st, F&& f) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  bool prof;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    prof = g_prof;
  }
  if (!prof) {
    f();
    return cudaGetLastError();
  }
  cudaEvent_t a, b;
  cudaEventCreate(&a);
  cudaEventCreate(&b);
  cudaEventRecord(a, st);
  f();
  cudaError_t e = cudaGetLastError();
  cudaEventRecord(b, st);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_recs.push_back({kind, a, b});
  return e;
}

// ---------------------------------------------------------------- device info
struct DevInfo {
  bool init = false;
  bool ok = false;
  int sms = 0;
  bool attr_set[8] = {false, false, false, false, false, false, false, false};
};
std::mutex g_dev_mu;
DevInfo g_dev[64];

flce_status device_info(DevInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return FLCE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (!d.init) {
    cudaDeviceProp p;
    e = cudaGetDeviceProperties(&p, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    d.ok = (p.major == 10);
    d.sms = p.multiProcessorCount;
    d.init = true;
  }
  if (!d.ok) return FLCE_ERR_UNSUPPORTED;
  *out = &d;
  return FLCE_OK;
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major 2-D tensor [outer, inner] with a 128-byte-swizzled box.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
              uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- workspace
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct FwdLayout {
  size_t part_m, part_s, label_logit, block_loss, block_cnt, end;
};

FwdLayout fwd_layout(int64_t N, int64_t V, bool bf16) {
  FwdLayout L{};
  size_t off = kHeaderBytes;
  const size_t n_vt = bf16 ? static_cast<size_t>((V + BN - 1) / BN) : 0;
  const size_t nblk = static_cast<size_t>((N + kLossThreads - 1) / kLossThreads);
  L.part_m = off;
  off = align_up(off + n_vt * N * sizeof(float), 256);
  L.part_s = off;
  off = align_up(off + n_vt * N * sizeof(float), 256);
  L.label_logit = off;
  off = align_up(off + N * sizeof(float), 256);
  L.block_loss = off;
  off = align_up(off + nblk * sizeof(double), 256);
  L.block_cnt = off;
  off = align_up(off + nblk * sizeof(long long), 256);
  L.end = off;
  return L;
}

struct Chunking {
  int tc, vc;  // chunk sizes (tokens, vocab)
};

Chunking chunking(int64_t N, int64_t V) {
  Chunking c;
  c.tc = static_cast<int>(std::min<int64_t>(kChunkTokens, align_up(std::max<int64_t>(N, 1), BM)));
  c.vc = static_cast<int>(std::min<int64_t>(kChunkVocab, align_up(V, BN)));
  return c;
}

size_t bwd_bytes(int64_t N, int64_t V, bool bf16) {
  if (!bf16) return kHeaderBytes;
  const Chunking c = chunking(N, V);
  return align_up(kHeaderBytes, 1024) + static_cast<size_t>(c.tc) * c.vc * 2 + 1024;
}

size_t ws_bytes(int64_t N, int64_t V, bool bf16) {
  return align_up(std::max(fwd_layout(N, V, bf16).end, bwd_bytes(N, V, bf16)), 256);
}

unsigned int* ws_status(void* ws) { return reinterpret_cast<unsigned int*>(ws); }
long long* ws_nvalid(void* ws) {
  return reinterpret_cast<long long*>(reinterpret_cast<char*>(ws) + 8);
}

unsigned long long timeout_ns() {
  static unsigned long long t = [] {
    const char* s = std::getenv("FLCE_WAIT_TIMEOUT_MS");
    long long ms = s ? std::atoll(s) : 1000;
    if (ms < 10) ms = 10;
    if (ms > 60000) ms = 60000;
    return static_cast<unsigned long long>(ms) * 1000000ull;
  }();
  return t;
}

// ---------------------------------------------------------------- checks
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

flce_status check_common(const void* hidden, const void* weight, const int64_t* labels,
                         int64_t N, int64_t H, int64_t V, float softcap, int32_t reduction,
                         int32_t dtype, void* ws, size_t ws_size) {
  if (reduction != FLCE_SUM && reduction != FLCE_MEAN) return FLCE_ERR_ARG;
  if (dtype != FLCE_BF16 && dtype != FLCE_FP32) return FLCE_ERR_ARG;
  if (!(softcap >= 0.f) || !(softcap < INFINITY)) return FLCE_ERR_ARG;
  if (N < 0 || V < 1 || H < 8 || N > kMaxDim || V > kMaxDim || H > kMaxDim) return FLCE_ERR_SHAPE;
  if (dtype == FLCE_BF16 && (H % 8) != 0) return FLCE_ERR_SHAPE;
  if (dtype == FLCE_FP32 && H > kSimtMaxH) return FLCE_ERR_SHAPE;
  if (N > 0 && (hidden == nullptr || labels == nullptr)) return FLCE_ERR_ARG;
  if (weight == nullptr || ws == nullptr) return FLCE_ERR_ARG;
  if (!aligned16(hidden) || !aligned16(weight) || !aligned16(ws)) return FLCE_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(labels) & 7u) != 0) return FLCE_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return FLCE_ERR_ARG;
  if (ws_size < ws_bytes(N, V, dtype == FLCE_BF16)) return FLCE_ERR_WORKSPACE;
  return FLCE_OK;
}

template <class Kern>
cudaError_t set_smem_attr(DevInfo* d, int slot, Kern k, size_t bytes) {
  if (d->attr_set[slot]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(bytes));
  if (e == cudaSuccess) d->attr_set[slot] = true;
  return e;
}

// Kernel instantiation slots for the shared-memory attribute cache.
enum Slot { kSlotFwd = 0, kSlotFwdCap, kSlotDz, kSlotDzCap, kSlotDh, kSlotDw, kSlotSimtDh, kSlotSimtDw };

template <class Epi, bool kAMn, bool kBMn>
cudaError_t run_gemm(DevInfo* d, int slot, int kind, const CUtensorMap& a, const CUtensorMap& b,
                     const CUtensorMap& out, const GemmArgs& g, const typename Epi::Params& ep,
                     cudaStream_t st) {
  auto k = tc_gemm_kernel<Epi, kAMn, kBMn>;
  cudaError_t e = set_smem_attr(d, slot, k, kGemmSmemBytes);
  if (e != cudaSuccess) return e;
  const int tiles = g.m_tiles * g.n_tiles;
  const int grid = std::max(1, std::min(tiles, d->sms));
  return launch(kind, st, [&] { k<<<grid, kThreads, kGemmSmemBytes, st>>>(a, b, out, g, ep); });
}

// ---------------------------------------------------------------- forward
flce_status forward_bf16(DevInfo* d, const void* hidden, const void* weight,
                         const int64_t* labels, int64_t N, int64_t H, int64_t V,
                         int64_t ignore_index, float softcap, int32_t reduction, float* loss,
                         int64_t* num_tokens, float* lse, void* ws, cudaStream_t st) {
  char* w = static_cast<char*>(ws);
  const FwdLayout L = fwd_layout(N, V, true);
  float* part_m = reinterpret_cast<float*>(w + L.part_m);
  float* part_s = reinterpret_cast<float*>(w + L.part_s);
  float* label_logit = reinterpret_cast<float*>(w + L.label_logit);
  double* block_loss = reinterpret_cast<double*>(w + L.block_loss);
  long long* block_cnt = reinterpret_cast<long long*>(w + L.block_cnt);

  CUtensorMap ta, tb;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, hidden, H, N, H * 2, BK, BM) ||
      !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, weight, H, V, H * 2, BK, BN))
    return FLCE_ERR_CUDA;

  GemmArgs g{};
  g.m_tiles = static_cast<int>((N + BM - 1) / BM);
  g.n_tiles = static_cast<int>((V + BN - 1) / BN);
  g.k_blocks = static_cast<int>((H + BK - 1) / BK);
  g.group_m = kGroupM;
  g.a_off = 0;
  g.b_off = 0;
  g.status = ws_status(ws);
  g.timeout_ns = timeout_ns();

  cudaError_t e;
  if (softcap > 0.f) {
    FwdStatsEpi<true>::Params ep{labels, static_cast<int>(N), static_cast<int>(V), softcap,
                                 1.0f / softcap, part_m, part_s, label_logit};
    e = run_gemm<FwdStatsEpi<true>, false, false>(d, kSlotFwdCap, kFwdGemm, ta, tb, ta, g, ep, st);
  } else {
    FwdStatsEpi<false>::Params ep{labels, static_cast<int>(N), static_cast<int>(V), 0.f, 0.f,
                                  part_m, part_s, label_logit};
    e = run_gemm<FwdStatsEpi<false>, false, false>(d, kSlotFwd, kFwdGemm, ta, tb, ta, g, ep, st);
  }
  if (e != cudaSuccess) return cuda_fail(e);

  const int n = static_cast<int>(N);
  const int n_vt = g.n_tiles;
  e = launch(kFwdMerge, st, [&] {
    fwd_merge_kernel<<<(n + kMergeRows - 1) / kMergeRows, dim3(kMergeRows, kMergeSplit), 0, st>>>(
        part_m, part_s, n_vt, n, lse);
  });
  if (e != cudaSuccess) return cuda_fail(e);
  const int nblk = (n + kLossThreads - 1) / kLossThreads;
  e = launch(kFwdMerge, st, [&] {
    row_loss_kernel<<<nblk, kLossThreads, 0, st>>>(lse, label_logit, labels, n, ignore_index, V,
                                                   block_loss, block_cnt, ws_status(ws));
  });
  if (e != cudaSuccess) return cuda_fail(e);
  e = launch(kFwdMerge, st, [&] {
    finalize_kernel<<<1, kFinalThreads, 0, st>>>(block_loss, block_cnt, nblk,
                                                 reduction == FLCE_MEAN, loss, num_tokens,
                                                 ws_nvalid(ws));
  });
  if (e != cudaSuccess) return cuda_fail(e);
  return FLCE_OK;
}

flce_status forward_fp32(DevInfo* d, const void* hidden, const void* weight,
                         const int64_t* labels, int64_t N, int64_t H, int64_t V,
                         int64_t ignore_index, float softcap, int32_t reduction, float* loss,
                         int64_t* num_tokens, float* lse, void* ws, cudaStream_t st) {
  (void)d;
  char* w = static_cast<char*>(ws);
  const FwdLayout L = fwd_layout(N, V, false);
  float* label_logit = reinterpret_cast<float*>(w + L.label_logit);
  double* block_loss = reinterpret_cast<double*>(w + L.block_loss);
  long long* block_cnt = reinterpret_cast<long long*>(w + L.block_cnt);
  const int n = static_cast<int>(N), h = static_cast<int>(H), v = static_cast<int>(V);
  cudaError_t e;
  if (h * sizeof(float) > 48 * 1024) {
    e = cudaFuncSetAttribute(simt_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(h * sizeof(float)));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  e = launch(kSimt, st, [&] {
    simt_fwd_kernel<<<n, kSimtThreads, h * sizeof(float), st>>>(
        static_cast<const float*>(hidden), static_cast<const float*>(weight), labels, n, h, v,
        softcap, lse, label_logit);
  });
  if (e != cudaSuccess) return cuda_fail(e);
  const int nblk = (n + kLossThreads - 1) / kLossThreads;
  e = launch(kFwdMerge, st, [&] {
    row_loss_kernel<<<nblk, kLossThreads, 0, st>>>(lse, label_logit, labels, n, ignore_index, V,
                                                   block_loss, block_cnt, ws_status(ws));
  });
  if (e != cudaSuccess) return cuda_fail(e);
  e = launch(kFwdMerge, st, [&] {
    finalize_kernel<<<1, kFinalThreads, 0, st>>>(block_loss, block_cnt, nblk,
                                                 reduction == FLCE_MEAN, loss, num_tokens,
                                                 ws_nvalid(ws));
  });
  if (e != cudaSuccess) return cuda_fail(e);
  return FLCE_OK;
}

// ---------------------------------------------------------------- backward
flce_status backward_bf16(DevInfo* d, const void* hidden, const void* weight,
                          const int64_t* labels, const float* lse, int64_t N, int64_t H,
                          int64_t V, int64_t ignore_index, float softcap, int32_t reduction,
                          const float* grad_output, float grad_scale, const long long* n_valid,
                          float* d_hidden, float* d_weight, void* ws, cudaStream_t st) {
  const Chunking ck = chunking(N, V);
  char* w = static_cast<char*>(ws);
  void* gbuf = w + align_up(kHeaderBytes, 1024);

  CUtensorMap t_hid_k, t_hid_mn, t_w_k, t_w_mn, t_dh, t_dw;
  if (!make_map(&t_hid_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, hidden, H, N, H * 2, BK, BM) ||
      !make_map(&t_hid_mn, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, hidden, H, N, H * 2, 64, BK) ||
      !make_map(&t_w_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, weight, H, V, H * 2, BK, BN) ||
      !make_map(&t_w_mn, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, weight, H, V, H * 2, 64, BK) ||
      !make_map(&t_dh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, d_hidden, H, N, H * 4, 32, 32) ||
      !make_map(&t_dw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, d_weight, H, V, H * 4, 32, 32))
    return FLCE_ERR_CUDA;

  const int n_tiles_h = static_cast<int>((H + BN - 1) / BN);
  const int k_blocks_h = static_cast<int>((H + BK - 1) / BK);
  const unsigned long long tmo = timeout_ns();
  const int mean = reduction == FLCE_MEAN;

  for (int64_t t0 = 0; t0 < N; t0 += ck.tc) {
    const int rows = static_cast<int>(std::min<int64_t>(ck.tc, N - t0));
    for (int64_t v0 = 0; v0 < V; v0 += ck.vc) {
      const int cols = static_cast<int>(std::min<int64_t>(ck.vc, V - v0));
      // dZ block [rows, cols] bf16, row stride ck.vc elements.
      CUtensorMap t_g_store, t_g_k, t_g_mn;
      if (!make_map(&t_g_store, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gbuf, cols, rows,
                    static_cast<uint64_t>(ck.vc) * 2, 64, 32) ||
          !make_map(&t_g_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gbuf, cols, rows,
                    static_cast<uint64_t>(ck.vc) * 2, BK, BM) ||
          !make_map(&t_g_mn, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gbuf, cols, rows,
                    static_cast<uint64_t>(ck.vc) * 2, 64, BK))
        return FLCE_ERR_CUDA;

      // 1) dZ = f(hidden[t0:] . W[v0:]^T) -> bf16 block
      GemmArgs gz{};
      gz.m_tiles = (rows + BM - 1) / BM;
      gz.n_tiles = (cols + BN - 1) / BN;
      gz.k_blocks = k_blocks_h;
      gz.group_m = kGroupM;
      gz.a_off = static_cast<int>(t0);
      gz.b_off = static_cast<int>(v0);
      gz.status = ws_status(ws);
      gz.timeout_ns = tmo;
      cudaError_t e;
      if (softcap > 0.f) {
        DzEpi<true>::Params ep{labels, lse, ignore_index, static_cast<int>(t0), rows,
                               static_cast<int>(v0), cols, softcap, 1.0f / softcap};
        e = run_gemm<DzEpi<true>, false, false>(d, kSlotDzCap, kBwdDz, t_hid_k, t_w_k, t_g_store,
                                                gz, ep, st);
      } else {
        DzEpi<false>::Params ep{labels, lse, ignore_index, static_cast<int>(t0), rows,
                                static_cast<int>(v0), cols, 0.f, 0.f};
        e = run_gemm<DzEpi<false>, false, false>(d, kSlotDz, kBwdDz, t_hid_k, t_w_k, t_g_store,
                                                 gz, ep, st);
      }
      if (e != cudaSuccess) return cuda_fail(e);

      // 2) dHidden[t0:t0+rows] (+)= dZ . W[v0:v0+cols]
      GemmArgs gh{};
      gh.m_tiles = (rows + BM - 1) / BM;
      gh.n_tiles = n_tiles_h;
      gh.k_blocks = (cols + BK - 1) / BK;
      gh.group_m = kGroupM;
      gh.a_off = 0;
      gh.b_off = static_cast<int>(v0);
      gh.a_mn_extent = 0;
      gh.b_mn_extent = static_cast<int>(H);
      gh.status = ws_status(ws);
      gh.timeout_ns = tmo;
      StoreEpi::Params eh{static_cast<int>(t0), v0 > 0 ? 1 : 0, static_cast<int>(H),
                          static_cast<int>(N), grad_output, grad_scale, n_valid, mean};
      e = run_gemm<StoreEpi, false, true>(d, kSlotDh, kBwdDh, t_g_k, t_w_mn, t_dh, gh, eh, st);
      if (e != cudaSuccess) return cuda_fail(e);

      // 3) dWeight[v0:v0+cols] (+)= dZ^T . hidden[t0:t0+rows]
      GemmArgs gw{};
      gw.m_tiles = (cols + BM - 1) / BM;
      gw.n_tiles = n_tiles_h;
      gw.k_blocks = (rows + BK - 1) / BK;
      gw.group_m = kGroupM;
      gw.a_off = 0;
      gw.b_off = static_cast<int>(t0);
      gw.a_mn_extent = cols;
      gw.b_mn_extent = static_cast<int>(H);
      gw.status = ws_status(ws);
      gw.timeout_ns = tmo;
      StoreEpi::Params ew{static_cast<int>(v0), t0 > 0 ? 1 : 0, static_cast<int>(H),
                          static_cast<int>(V), grad_output, grad_scale, n_valid, mean};
      e = run_gemm<StoreEpi, true, true>(d, kSlotDw, kBwdDw, t_g_mn, t_hid_mn, t_dw, gw, ew, st);
      if (e != cudaSuccess) return cuda_fail(e);
    }
  }
  return FLCE_OK;
}

flce_status backward_fp32(DevInfo* d, const void* hidden, const void* weight,
                          const int64_t* labels, const float* lse, int64_t N, int64_t H,
                          int64_t V, int64_t ignore_index, float softcap, int32_t reduction,
                          const float* grad_output, float grad_scale, const long long* n_valid,
                          float* d_hidden, float* d_weight, cudaStream_t st) {
  const int n = static_cast<int>(N), h = static_cast<int>(H), v = static_cast<int>(V);
  const int mean = reduction == FLCE_MEAN;
  const size_t sh_dh = (2 * static_cast<size_t>(h) + kSimtChunk) * sizeof(float);
  const size_t sh_dw = (2 * static_cast<size_t>(h) + kSimtThreads) * sizeof(float);
  cudaError_t e = set_smem_attr(d, kSlotSimtDh, simt_dh_kernel, 2 * kSimtMaxH * 4 + kSimtChunk * 4);
  if (e != cudaSuccess) return cuda_fail(e);
  e = set_smem_attr(d, kSlotSimtDw, simt_dw_kernel, 2 * kSimtMaxH * 4 + kSimtThreads * 4);
  if (e != cudaSuccess) return cuda_fail(e);
  if (n > 0) {
    e = launch(kSimt, st, [&] {
      simt_dh_kernel<<<n, kSimtThreads, sh_dh, st>>>(
          static_cast<const float*>(hidden), static_cast<const float*>(weight), labels, lse, n, h,
          v, ignore_index, softcap, grad_output, grad_scale, n_valid, mean, d_hidden);
    });
    if (e != cudaSuccess) return cuda_fail(e);
  }
  e = launch(kSimt, st, [&] {
    simt_dw_kernel<<<v, kSimtThreads, sh_dw, st>>>(
        static_cast<const float*>(hidden), static_cast<const float*>(weight), labels, lse, n, h, v,
        ignore_index, softcap, grad_output, grad_scale, n_valid, mean, d_weight);
  });
  if (e != cudaSuccess) return cuda_fail(e);
  return FLCE_OK;
}

}  // namespace
}  // namespace flce

using namespace flce;

extern "C" {

size_t flce_workspace_bytes(int64_t N, int64_t H, int64_t V, int32_t dtype) {
  if (N < 0 || V < 1 || H < 8 || N > kMaxDim || V > kMaxDim) return 0;
  if (dtype != FLCE_BF16 && dtype != FLCE_FP32) return 0;
  return ws_bytes(N, V, dtype == FLCE_BF16);
}

flce_status flce_forward(const void* hidden, const void* weight, const int64_t* labels,
                         int64_t N, int64_t H, int64_t V, int64_t ignore_index, float softcap,
                         int32_t reduction, int32_t dtype, float* loss, int64_t* num_tokens,
                         float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  flce_status s = check_common(hidden, weight, labels, N, H, V, softcap, reduction, dtype,
                               workspace, workspace_bytes);
  if (s != FLCE_OK) return s;
  if (loss == nullptr || num_tokens == nullptr || (N > 0 && lse == nullptr)) return FLCE_ERR_ARG;
  DevInfo* d = nullptr;
  s = device_info(&d);
  if (s != FLCE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // status word and n_valid
  cudaError_t e = cudaMemsetAsync(workspace, 0, 16, st);
  if (e != cudaSuccess) return cuda_fail(e);
  if (N == 0) {
    if ((e = cudaMemsetAsync(loss, 0, sizeof(float), st)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaMemsetAsync(num_tokens, 0, sizeof(int64_t), st)) != cudaSuccess)
      return cuda_fail(e);
    return FLCE_OK;
  }
  if (dtype == FLCE_BF16)
    return forward_bf16(d, hidden, weight, labels, N, H, V, ignore_index, softcap, reduction,
                        loss, num_tokens, lse, workspace, st);
  return forward_fp32(d, hidden, weight, labels, N, H, V, ignore_index, softcap, reduction, loss,
                      num_tokens, lse, workspace, st);
}

flce_status flce_backward(const void* hidden, const void* weight, const int64_t* labels,
                          const float* lse, int64_t N, int64_t H, int64_t V,
                          int64_t ignore_index, float softcap, int32_t reduction, int32_t dtype,
                          const float* grad_output, float grad_scale, const int64_t* num_valid,
                          float* d_hidden, float* d_weight, void* workspace,
                          size_t workspace_bytes, void* stream) {
  flce_status s = check_common(hidden, weight, labels, N, H, V, softcap, reduction, dtype,
                               workspace, workspace_bytes);
  if (s != FLCE_OK) return s;
  if (d_weight == nullptr || (N > 0 && (d_hidden == nullptr || lse == nullptr)))
    return FLCE_ERR_ARG;
  if (!aligned16(d_hidden) || !aligned16(d_weight)) return FLCE_ERR_ARG;
  if (!(grad_scale == grad_scale) || grad_scale == INFINITY || grad_scale == -INFINITY)
    return FLCE_ERR_ARG;
  DevInfo* d = nullptr;
  s = device_info(&d);
  if (s != FLCE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (N == 0) {
    e = cudaMemsetAsync(d_weight, 0, static_cast<size_t>(V) * H * sizeof(float), st);
    return e == cudaSuccess ? FLCE_OK : cuda_fail(e);
  }
  const long long* nv = reinterpret_cast<const long long*>(num_valid);
  if (nv == nullptr) {
    long long* out = ws_nvalid(workspace);
    e = launch(kHelper, st, [&] {
      count_valid_kernel<<<1, kFinalThreads, 0, st>>>(labels, static_cast<int>(N), ignore_index,
                                                      out);
    });
    if (e != cudaSuccess) return cuda_fail(e);
    nv = out;
  }
  if (dtype == FLCE_BF16)
    return backward_bf16(d, hidden, weight, labels, lse, N, H, V, ignore_index, softcap,
                         reduction, grad_output, grad_scale, nv, d_hidden, d_weight, workspace,
                         st);
  return backward_fp32(d, hidden, weight, labels, lse, N, H, V, ignore_index, softcap, reduction,
                       grad_output, grad_scale, nv, d_hidden, d_weight, st);
}

flce_status flce_get_status(const void* workspace, void* stream) {
  if (workspace == nullptr) return FLCE_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned int word = 0;
  e = cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  if (word & kStatusLabelRange) return FLCE_ERR_LABEL_RANGE;
  if (word & kStatusTimeout) return FLCE_ERR_TIMEOUT;
  return FLCE_OK;
}

const char* flce_status_string(int32_t status) {
  switch (status) {
    case FLCE_OK: return "FLCE_OK";
    case FLCE_ERR_ARG: return "FLCE_ERR_ARG";
    case FLCE_ERR_SHAPE: return "FLCE_ERR_SHAPE";
    case FLCE_ERR_LABEL_RANGE: return "FLCE_ERR_LABEL_RANGE";
    case FLCE_ERR_CUDA: return "FLCE_ERR_CUDA";
    case FLCE_ERR_UNSUPPORTED: return "FLCE_ERR_UNSUPPORTED";
    case FLCE_ERR_TIMEOUT: return "FLCE_ERR_TIMEOUT";
    case FLCE_ERR_WORKSPACE: return "FLCE_ERR_WORKSPACE";
    default: return "FLCE_ERR_UNKNOWN";
  }
}

int32_t flce_version(void) { return 100; }

uint64_t flce_launch_count(void) { return g_launches.load(); }

flce_status flce_profile_enable(int32_t enable) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof = enable != 0;
  return FLCE_OK;
}

flce_status flce_profile_read(int32_t kind, double* total_ms, int64_t* launches) {
  if (kind < 0 || kind >= kKinds || total_ms == nullptr || launches == nullptr)
    return FLCE_ERR_ARG;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  double ms = 0.0;
  int64_t n = 0;
  std::vector<ProfRec> keep;
  for (ProfRec& r : g_recs) {
    if (r.kind != kind) {
      keep.push_back(r);
      continue;
    }
    cudaError_t e = cudaEventSynchronize(r.b);
    float t = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
    if (e != cudaSuccess) {
      g_recs.swap(keep);
      return cuda_fail(e);
    }
    ms += t;
    ++n;
  }
  g_recs.swap(keep);
  *total_ms = ms;
  *launches = n;
  return FLCE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- no-alloc forward
// flce_forward_noalloc: the bf16 / fp32 forward of flce_forward with its
// scratch in a static device buffer instead of a caller workspace, for callers
// that cannot allocate device memory (see include/flce.h).
namespace flce {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FLCE_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[64] = {};

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device with that device current.
flce_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return FLCE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return FLCE_OK;
}

}  // namespace
}  // namespace flce

extern "C" flce_status flce_forward_noalloc(const void* hidden, const void* weight,
                                            const int64_t* labels, int64_t N, int64_t H,
                                            int64_t V, int64_t ignore_index, float softcap,
                                            int32_t reduction, int32_t dtype, float* loss,
                                            int64_t* num_tokens, float* lse, uint32_t* status,
                                            void* stream) {
  if (reduction != FLCE_SUM && reduction != FLCE_MEAN) return FLCE_ERR_ARG;
  if (dtype != FLCE_BF16 && dtype != FLCE_FP32) return FLCE_ERR_ARG;
  if (!(softcap >= 0.f) || !(softcap < INFINITY)) return FLCE_ERR_ARG;
  if (N < 0 || V < 1 || H < 8 || N > kMaxDim || V > kMaxDim || H > kMaxDim) return FLCE_ERR_SHAPE;
  if (dtype == FLCE_BF16 && (H % 8) != 0) return FLCE_ERR_SHAPE;
  if (dtype == FLCE_FP32 && H > kSimtMaxH) return FLCE_ERR_SHAPE;
  if (N > 0 && (hidden == nullptr || labels == nullptr || lse == nullptr)) return FLCE_ERR_ARG;
  if (weight == nullptr || loss == nullptr || num_tokens == nullptr) return FLCE_ERR_ARG;
  if (!aligned16(hidden) || !aligned16(weight)) return FLCE_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(labels) & 7u) != 0) return FLCE_ERR_ARG;
  // the forward's scratch must fit the static buffer
  if (fwd_layout(N, V, dtype == FLCE_BF16).end > FLCE_NOALLOC_SCRATCH_BYTES) return FLCE_ERR_SHAPE;
  DevInfo* d = nullptr;
  flce_status s = device_info(&d);
  if (s != FLCE_OK) return s;
  void* ws = nullptr;
  s = noalloc_scratch(&ws);
  if (s != FLCE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // status word and n_valid start at zero
  cudaError_t e = cudaMemsetAsync(ws, 0, 16, st);
  if (e != cudaSuccess) return cuda_fail(e);
  if (N == 0) {
    if ((e = cudaMemsetAsync(loss, 0, sizeof(float), st)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaMemsetAsync(num_tokens, 0, sizeof(int64_t), st)) != cudaSuccess)
      return cuda_fail(e);
  } else {
    s = (dtype == FLCE_BF16)
            ? forward_bf16(d, hidden, weight, labels, N, H, V, ignore_index, softcap, reduction,
                           loss, num_tokens, lse, ws, st)
            : forward_fp32(d, hidden, weight, labels, N, H, V, ignore_index, softcap, reduction,
                           loss, num_tokens, lse, ws, st);
    if (s != FLCE_OK) return s;
  }
  if (status != nullptr) {
    e = cudaMemcpyAsync(status, ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return FLCE_OK;
}
