// Host side of the fused linear cross-entropy C ABI (include/flce.h):
// argument checks, workspace layout, TMA tensor-map encoding and launches.
//
// bf16 path, forward:   row compaction (the rows in the loss first) ->
//                       tc_gemm<FwdStatsEpi> over the valid rows' tiles ->
//                       fwd_merge (lse back through the permutation) ->
//                       row_loss -> finalize.
// bf16 path, backward:  row compaction and label sort, then the [n, V]
//                       problem is cut into chunks of at most chunk_tokens x
//                       chunk_vocab (options); per chunk
//                         tc_gemm<DzEpi>    dZ block (bf16, in the workspace)
//                         tc_gemm<StoreEpi> (one launch, two GEMMs)
//                           dHidden[chunk rows] (+)= dZ . W[chunk]
//                           dWeight[chunk rows] (+)= dZ^T . hidden[chunk]
//                       The first chunk along the reduced dimension stores,
//                       later ones add (TMA reduce-add) into fp32 outputs:
//                       dWeight itself, and a compact-order dHidden block per
//                       token chunk, which dh_scatter moves to token order
//                       with the exact fp32 label term once the chunk's last
//                       vocab chunk is done; at the end the exact fp32 label
//                       term of dWeight.
// fp32 path:            simt_fwd / simt_dh / simt_dw (CUDA cores).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>
#include <vector>

#include "../../include/flce.h"
#include "small_kernels.cuh"

namespace flce {
namespace {

// Backward chunk: kChunkTokens x kChunkVocab (dZ block 512 MiB bf16, 1/8 of
// the [16384, 131072] dZ of the bench problem).  Longer tiles along the
// reduced dimensions (K = 16384 for dHidden, up to 16384 for dWeight), fewer
// launches and fewer fp32 read-add-write passes over dHidden and dWeight: one
// token chunk writes dWeight once.  Measured at the power cap (interleaved
// A/B): 16384 x 16384 chunks 0.5% faster than 8192 x 16384, which was 6%
// faster than an L2-sized 4096 x 8192 block.
constexpr int kChunkTokens = 16384;
constexpr int kChunkVocab = 16384;
constexpr int kGroupM = 16;     // forward and dZ
constexpr int kGroupMGrad = 8;  // dHidden and dWeight: their long-K panels (8 MiB at the bench
                                // size) make a 16-tile group's panels overflow L2 (ncu: 2.4 vs
                                // 2.8 GB of DRAM reads per launch)
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
enum Kind { kFwdGemm = 0, kFwdMerge = 1, kBwdDz = 2, kBwdDhDw = 3, kHelper = 5, kSimt = 6 };

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

// The 3-D chunk view of a row-major bf16 matrix [k_rows, mn] (row pitch
// row_bytes) for MN-major operand loads: x = 64 elements within a chunk, y =
// row, z = 64-element chunk, box {64, BK, 2}.  mn must be a multiple of 64 and
// every chunk must lie inside the allocation (x is not clipped per row).
bool make_map_mn3d(CUtensorMap* m, const void* base, uint64_t mn, uint64_t k_rows,
                   uint64_t row_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr || mn % 64 != 0) return false;
  cuuint64_t dims[3] = {64, k_rows, mn / 64};
  cuuint64_t strides[2] = {row_bytes, 128};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(BK), 2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- workspace
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Forward workspace: header | softmax partials m, s [ceil(V/256), N] | label
// logits [N] | per-block loss partials | and, when the rows are compacted
// (bf16 path), the permutation, compact labels and lse, per-block counts, the
// valid count and the compact hidden copy [N, H] bf16.
struct FwdLayout {
  size_t part_m, part_s, label_logit, block_loss, block_cnt, end;
  size_t perm, labels_c, lse_c, block_valid, n_valid_c, hidden_c, end_compact;
};

FwdLayout fwd_layout(int64_t N, int64_t V, bool bf16, int64_t H = 0) {
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
  const size_t cblk = static_cast<size_t>((N + kCompactThreads - 1) / kCompactThreads);
  L.perm = off;
  off = align_up(off + 4 * static_cast<size_t>(N), 256);
  L.labels_c = off;
  off = align_up(off + 8 * static_cast<size_t>(N), 256);
  L.lse_c = off;
  off = align_up(off + 4 * static_cast<size_t>(N), 256);
  L.block_valid = off;
  off = align_up(off + 4 * cblk, 256);
  L.n_valid_c = off;
  off = align_up(off + 8, 1024);
  L.hidden_c = off;
  off = align_up(off + 2 * static_cast<size_t>(N) * static_cast<size_t>(H), 256);
  L.end_compact = off;
  return L;
}

// ---------------------------------------------------------------- options
// Process-wide settings (flce_set_option).  Every call takes one snapshot of
// them at its start, so a concurrent flce_set_option never changes a call
// half-way; flce_workspace_bytes and the calls that use the workspace must see
// the same chunk sizes.
struct OptSpec {
  int64_t dflt, lo, hi;
};
constexpr int kNumOpts = FLCE_OPT_COUNT_;
constexpr OptSpec kOptSpec[kNumOpts] = {
    {2, 1, 2},                 // FLCE_OPT_CTA_GROUP
    {1, 0, 1},                 // FLCE_OPT_BWD_COMPACT
    {1, 0, 1},                 // FLCE_OPT_BWD_FUSE
    {1, 0, 1},                 // FLCE_OPT_MN3D
    {kChunkTokens, 256, 1 << 20},  // FLCE_OPT_CHUNK_TOKENS
    {kChunkVocab, 256, 1 << 20},   // FLCE_OPT_CHUNK_VOCAB
    {1000, 10, 60000},         // FLCE_OPT_WAIT_TIMEOUT_MS
    {512, 256, 512},           // FLCE_OPT_GRAD_TILE_N
    {0, 0, 512},               // FLCE_OPT_DZ_TILE_N (0: by softcap)
    {512, 256, 512},           // FLCE_OPT_FWD_TILE_N
    {kGroupM, 1, 64},          // FLCE_OPT_FWD_GROUP_M
    {kGroupM, 1, 64},          // FLCE_OPT_DZ_GROUP_M
    {kGroupMGrad, 1, 64},      // FLCE_OPT_GRAD_GROUP_M
    {1, 0, 1},                 // FLCE_OPT_FWD_DYNAMIC
    {1, 1, 2},                 // FLCE_OPT_DZ_BUFFERS
    {1, 0, 1},                 // FLCE_OPT_FWD_COMPACT
};
std::atomic<int64_t> g_opt[kNumOpts] = {
    {kOptSpec[0].dflt}, {kOptSpec[1].dflt}, {kOptSpec[2].dflt}, {kOptSpec[3].dflt},
    {kOptSpec[4].dflt}, {kOptSpec[5].dflt}, {kOptSpec[6].dflt}, {kOptSpec[7].dflt},
    {kOptSpec[8].dflt}, {kOptSpec[9].dflt}, {kOptSpec[10].dflt}, {kOptSpec[11].dflt},
    {kOptSpec[12].dflt}, {kOptSpec[13].dflt}, {kOptSpec[14].dflt}, {kOptSpec[15].dflt}};

struct Opts {
  int cta_group;          // 2: CTA pairs with 256-row tiles; 1: single CTAs, 128-row tiles
  bool compact;           // backward leaves ignored rows out of its GEMMs
  bool fuse;              // dHidden and dWeight GEMMs of a chunk share one launch
  bool mn3d;              // MN-major operands load through 3-D chunk views
  int64_t chunk_tokens;   // backward chunk (multiples of 256)
  int64_t chunk_vocab;
  unsigned long long timeout_ns;  // limit of every bounded wait inside a kernel
  int grad_bn;            // columns of a dHidden / dWeight tile (512 needs CTA pairs)
  int dz_bn;              // columns of a dZ tile; 0: 512 without softcap, 256 with
  int fwd_bn;             // columns of a forward tile
  int fwd_group, dz_group, grad_group;  // row tiles per raster group (L2 reuse)
  bool fwd_dynamic;       // forward tiles handed out by an atomic counter (else round-robin)
  int dz_buffers;         // backward dZ blocks: 2 lets a chunk's dZ run beside the previous
                          // chunk's gradient GEMMs
  bool fwd_compact;       // the bf16 forward leaves rows outside the loss out of its GEMM
};

Opts opts() {
  Opts o;
  o.cta_group = static_cast<int>(g_opt[FLCE_OPT_CTA_GROUP].load());
  o.compact = g_opt[FLCE_OPT_BWD_COMPACT].load() != 0;
  o.fuse = g_opt[FLCE_OPT_BWD_FUSE].load() != 0;
  o.mn3d = g_opt[FLCE_OPT_MN3D].load() != 0;
  o.chunk_tokens = align_up(static_cast<size_t>(g_opt[FLCE_OPT_CHUNK_TOKENS].load()), 256);
  o.chunk_vocab = align_up(static_cast<size_t>(g_opt[FLCE_OPT_CHUNK_VOCAB].load()), 256);
  o.timeout_ns = static_cast<unsigned long long>(g_opt[FLCE_OPT_WAIT_TIMEOUT_MS].load()) * 1000000ull;
  o.grad_bn = (o.cta_group == 2) ? static_cast<int>(g_opt[FLCE_OPT_GRAD_TILE_N].load()) : 256;
  o.dz_bn = (o.cta_group == 2) ? static_cast<int>(g_opt[FLCE_OPT_DZ_TILE_N].load()) : 256;
  o.fwd_bn = (o.cta_group == 2) ? static_cast<int>(g_opt[FLCE_OPT_FWD_TILE_N].load()) : 256;
  o.fwd_group = static_cast<int>(g_opt[FLCE_OPT_FWD_GROUP_M].load());
  o.dz_group = static_cast<int>(g_opt[FLCE_OPT_DZ_GROUP_M].load());
  o.grad_group = static_cast<int>(g_opt[FLCE_OPT_GRAD_GROUP_M].load());
  o.fwd_dynamic = g_opt[FLCE_OPT_FWD_DYNAMIC].load() != 0;
  o.dz_buffers = static_cast<int>(g_opt[FLCE_OPT_DZ_BUFFERS].load());
  o.fwd_compact = g_opt[FLCE_OPT_FWD_COMPACT].load() != 0;
  return o;
}

// Divisor of a 'sum' loss (and of its gradient) normalised by the global
// number of label tokens: max(num_label_tokens, 1), the clamp that keeps an
// all-ignored batch at 0 instead of NaN; 1 when no count is given (< 0) or for
// 'mean', which divides by its own count.
double label_token_divisor(int32_t reduction, int64_t num_label_tokens) {
  if (reduction != FLCE_SUM || num_label_tokens < 0) return 1.0;
  return static_cast<double>(num_label_tokens > 0 ? num_label_tokens : 1);
}

struct Chunking {
  int tc, vc;  // chunk sizes (tokens, vocab)
};

Chunking chunking(const Opts& o, int64_t N, int64_t V) {
  Chunking c;
  c.tc = static_cast<int>(std::min<int64_t>(o.chunk_tokens, align_up(std::max<int64_t>(N, 1), BM)));
  c.vc = static_cast<int>(std::min<int64_t>(o.chunk_vocab, align_up(V, BN)));
  return c;
}

int64_t bwd_chunks(const Opts& o, int64_t N, int64_t V) {
  const Chunking c = chunking(o, N, V);
  return ((N + c.tc - 1) / c.tc) * ((V + c.vc - 1) / c.vc);
}

// Backward counters of one call, zeroed at its start: a dynamic tile counter
// for each GEMM launch (at most three per chunk), then one per chunk that the
// CTAs of its gradient launches count themselves out on.
int64_t bwd_counters(const Opts& o, int64_t N, int64_t V) { return 4 * bwd_chunks(o, N, V); }

// Backward workspace: header | tile counters | row compaction (permutation,
// compact labels and lse, per-block counts, valid count) | label sort (two
// key/value buffers, digit counts) | label residuals | compact hidden [N, H]
// bf16 | dZ block, whose space the dWeight label correction's run pieces
// reuse once the GEMMs are done | compact-order dHidden of one token chunk
// [chunk_tokens, H] fp32 (row compaction only).
struct BwdLayout {
  size_t counters, perm, labels_c, lse_c, block_valid, n_valid_c, keys0, keys1, vals0, vals1,
      hist, resid, hidden_c, gblock, gblock_bytes, part, dh_c, end;
};

BwdLayout bwd_layout(const Opts& o, int64_t N, int64_t H, int64_t V) {
  BwdLayout L{};
  const Chunking c = chunking(o, N, V);
  const size_t nblk = static_cast<size_t>((N + kCompactThreads - 1) / kCompactThreads);
  size_t off = kHeaderBytes;
  L.counters = off;
  off = align_up(off + 4 * static_cast<size_t>(bwd_counters(o, N, V)), 256);
  L.perm = off;
  off = align_up(off + 4 * static_cast<size_t>(N), 256);
  L.labels_c = off;
  off = align_up(off + 8 * static_cast<size_t>(N), 256);
  L.lse_c = off;
  off = align_up(off + 4 * static_cast<size_t>(N), 256);
  L.block_valid = off;
  off = align_up(off + 4 * nblk, 256);
  L.n_valid_c = off;
  off = align_up(off + 8, 256);
  for (size_t* b : {&L.keys0, &L.keys1, &L.vals0, &L.vals1, &L.resid}) {
    *b = off;
    off = align_up(off + 4 * static_cast<size_t>(N), 256);
  }
  L.hist = off;
  off = align_up(off + 4 * static_cast<size_t>(kRadixBuckets) * nblk, 1024);
  L.hidden_c = off;
  off = align_up(off + 2 * static_cast<size_t>(N) * static_cast<size_t>(H), 1024);
  L.gblock = off;
  L.gblock_bytes = align_up(static_cast<size_t>(c.tc) * c.vc * 2 + 1024, 1024);
  L.part = off;
  const size_t nseg = static_cast<size_t>((N + kFixSeg - 1) / kFixSeg);
  off += std::max(L.gblock_bytes * static_cast<size_t>(o.dz_buffers),
                  nseg * 2 * static_cast<size_t>(H) * 4);
  off = align_up(off, 1024);
  L.dh_c = off;
  if (o.compact) off += static_cast<size_t>(c.tc) * static_cast<size_t>(H) * 4;
  L.end = off;
  return L;
}

size_t bwd_bytes(const Opts& o, int64_t N, int64_t H, int64_t V, bool bf16) {
  if (!bf16) return kHeaderBytes;
  return bwd_layout(o, N, H, V).end;
}

size_t ws_bytes(const Opts& o, int64_t N, int64_t H, int64_t V, bool bf16) {
  const FwdLayout F = fwd_layout(N, V, bf16, H);
  const size_t fwd = (bf16 && o.fwd_compact) ? F.end_compact : F.end;
  return align_up(std::max(fwd, bwd_bytes(o, N, H, V, bf16)), 256);
}

// bf16 gradient outputs: fp32 scratch for dHidden and/or dWeight after the
// shape's own workspace.
constexpr int32_t kBf16OutFlags = FLCE_DHIDDEN_BF16 | FLCE_DWEIGHT_BF16;
constexpr int32_t kAllBwdFlags = FLCE_ACCUMULATE_DHIDDEN | FLCE_ACCUMULATE_DWEIGHT | kBf16OutFlags;

struct GradScratch {
  size_t dh, dw, end;  // byte offsets (dh / dw meaningful only with their flag)
};

GradScratch grad_scratch(const Opts& o, int64_t N, int64_t H, int64_t V, bool bf16,
                         int32_t flags) {
  GradScratch g{};
  size_t off = align_up(ws_bytes(o, N, H, V, bf16), 256);
  g.dh = off;
  if (flags & FLCE_DHIDDEN_BF16) off = align_up(off + 4 * static_cast<size_t>(N) * H, 256);
  g.dw = off;
  if (flags & FLCE_DWEIGHT_BF16) off = align_up(off + 4 * static_cast<size_t>(V) * H, 256);
  g.end = off;
  return g;
}

// Workspace header (256 B; its first 16 bytes are zeroed by every forward):
// status word at 0, the forward's tile counter at 4, n_valid at 8.
unsigned int* ws_status(void* ws) { return reinterpret_cast<unsigned int*>(ws); }
int* ws_fwd_counter(void* ws) { return reinterpret_cast<int*>(static_cast<char*>(ws) + 4); }
long long* ws_nvalid(void* ws) {
  return reinterpret_cast<long long*>(reinterpret_cast<char*>(ws) + 8);
}


// ---------------------------------------------------------------- checks
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

flce_status check_common(const Opts& o, const void* hidden, const void* weight,
                         const int64_t* labels, int64_t N, int64_t H, int64_t V, float softcap,
                         int32_t reduction, int32_t dtype, void* ws, size_t ws_size) {
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
  if (ws_size < ws_bytes(o, N, H, V, dtype == FLCE_BF16)) return FLCE_ERR_WORKSPACE;
  return FLCE_OK;
}

// Opt a kernel in to `bytes` of dynamic shared memory, once per (device, kernel).
std::mutex g_attr_mu;
std::set<std::pair<int, const void*>> g_attr_done;

template <class Kern>
cudaError_t set_smem_attr(Kern k, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const auto key = std::make_pair(dev, reinterpret_cast<const void*>(k));
  {
    std::lock_guard<std::mutex> lk(g_attr_mu);
    if (g_attr_done.count(key)) return cudaSuccess;
  }
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) {
    std::lock_guard<std::mutex> lk(g_attr_mu);
    g_attr_done.insert(key);
  }
  return e;
}

// One GEMM of a launch: operand / output tensor maps, output rows M (tiled by
// 128 * kCG), output columns Ncols (tiled by the launch's tile width) and the
// rest of its GemmArgs.
struct GemmProblem {
  const CUtensorMap* a;
  const CUtensorMap* b;
  const CUtensorMap* out;
  int64_t M;
  int64_t Ncols;
  GemmArgs g;
};

// One tensor-core launch over one GEMM (p1 == nullptr) or two independent
// GEMMs with the same epilogue.  kCG = 2 launches clusters of two CTAs.
template <class Epi, int kCG, int kBN, bool kAMn0, bool kBMn0, bool kAMn1, bool kBMn1>
cudaError_t run_gemm_cg(DevInfo* d, int kind, const GemmProblem& p0,
                        const typename Epi::Params& ep0, const GemmProblem* p1,
                        const typename Epi::Params& ep1, cudaStream_t st, int* ctas_out) {
  using Cfg = TileCfg<kCG, kBN>;
  auto k = tc_gemm_kernel<Epi, kCG, kBN, kAMn0, kBMn0, kAMn1, kBMn1>;
  constexpr size_t kSmem = gemm_smem_bytes<Epi, kCG, kBN>();
  static_assert(kSmem <= 227 * 1024 - 512, "shared memory");
  cudaError_t e = set_smem_attr(k, kSmem);
  if (e != cudaSuccess) return e;
  GemmArgs g0 = p0.g;
  g0.m_tiles = static_cast<int>((p0.M + Cfg::kUnitRows - 1) / Cfg::kUnitRows);
  g0.n_tiles = static_cast<int>((p0.Ncols + kBN - 1) / kBN);
  GemmArgs g1 = p1 ? p1->g : p0.g;
  if (p1) {
    g1.m_tiles = static_cast<int>((p1->M + Cfg::kUnitRows - 1) / Cfg::kUnitRows);
    g1.n_tiles = static_cast<int>((p1->Ncols + kBN - 1) / kBN);
  } else {
    g1.m_tiles = g1.n_tiles = 0;
  }
  const GemmProblem& q1 = p1 ? *p1 : p0;
  const int tiles = g0.m_tiles * g0.n_tiles + g1.m_tiles * g1.n_tiles;
  const int units = std::max(1, std::min(tiles, d->sms / kCG));
  if (ctas_out != nullptr) *ctas_out = units * kCG;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(units * kCG, 1, 1);
  cfg.blockDim = dim3(gemm_threads<Epi>(), 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int nattr = 0;
  if (kCG > 1) {
    attr[nattr].id = cudaLaunchAttributeClusterDimension;
    attr[nattr].val.clusterDim.x = kCG;
    attr[nattr].val.clusterDim.y = 1;
    attr[nattr].val.clusterDim.z = 1;
    ++nattr;
  }
  if (g0.dep_wait != kDepNone) {
    // may start while the previous kernel drains; it waits where it depends on it
    attr[nattr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[nattr].val.programmaticStreamSerializationAllowed = 1;
    ++nattr;
  }
  cfg.attrs = attr;
  cfg.numAttrs = nattr;
  cudaError_t le = cudaSuccess;
  cudaError_t e2 = launch(kind, st, [&] {
    le = cudaLaunchKernelEx(&cfg, k, *p0.a, *p0.b, *p0.out, *q1.a, *q1.b, *q1.out, g0, g1, ep0,
                            ep1);
  });
  return le != cudaSuccess ? le : e2;
}

// The launch in the CTA group of `o` with tiles of `bn` columns (512 only
// with CTA pairs; opts() guarantees it).  *ctas_out (if given) receives the
// number of CTAs launched.
template <class Epi, bool kAMn0, bool kBMn0, bool kAMn1 = false, bool kBMn1 = false>
cudaError_t run_gemm(DevInfo* d, const Opts& o, int bn, int kind, const GemmProblem& p0,
                     const typename Epi::Params& ep0, const GemmProblem* p1,
                     const typename Epi::Params& ep1, cudaStream_t st,
                     int* ctas_out = nullptr) {
  if (o.cta_group == 1)
    return run_gemm_cg<Epi, 1, 256, kAMn0, kBMn0, kAMn1, kBMn1>(d, kind, p0, ep0, p1, ep1, st,
                                                                ctas_out);
  if (bn == 512)
    return run_gemm_cg<Epi, 2, 512, kAMn0, kBMn0, kAMn1, kBMn1>(d, kind, p0, ep0, p1, ep1, st,
                                                                ctas_out);
  return run_gemm_cg<Epi, 2, 256, kAMn0, kBMn0, kAMn1, kBMn1>(d, kind, p0, ep0, p1, ep1, st,
                                                              ctas_out);
}

// Rows of B (K-major) one CTA stages per bank and K-block.
uint32_t b_box_rows(const Opts& o) { return static_cast<uint32_t>(BN / o.cta_group); }

// ---------------------------------------------------------------- forward
// `compact`: the rows outside the loss (ignore_index, or a label outside
// [0, V)) are left out of the GEMM: the valid rows are compacted first (the
// backward's stable compaction and hidden-row gather), the GEMM's token rows
// are bounded by the device-side count, and the merge writes each lse back
// through the permutation.  Either way such rows get lse 0.
flce_status forward_bf16(DevInfo* d, const Opts& o, const void* hidden, const void* weight,
                         const int64_t* labels, int64_t N, int64_t H, int64_t V,
                         int64_t ignore_index, float softcap, int32_t reduction,
                         double loss_scale, double loss_div, float* loss, int64_t* num_tokens,
                         float* lse, void* ws, cudaStream_t st, bool compact) {
  char* w = static_cast<char*>(ws);
  const FwdLayout L = fwd_layout(N, V, true, H);
  float* part_m = reinterpret_cast<float*>(w + L.part_m);
  float* part_s = reinterpret_cast<float*>(w + L.part_s);
  float* label_logit = reinterpret_cast<float*>(w + L.label_logit);
  double* block_loss = reinterpret_cast<double*>(w + L.block_loss);
  long long* block_cnt = reinterpret_cast<long long*>(w + L.block_cnt);
  const int n = static_cast<int>(N);
  cudaError_t e;

  const void* hid = hidden;
  const int64_t* lab = labels;
  int* perm = nullptr;
  long long* n_valid_c = nullptr;
  float* lse_c = nullptr;
  if (compact) {
    perm = reinterpret_cast<int*>(w + L.perm);
    int64_t* labels_c = reinterpret_cast<int64_t*>(w + L.labels_c);
    lse_c = reinterpret_cast<float*>(w + L.lse_c);
    int* block_valid = reinterpret_cast<int*>(w + L.block_valid);
    n_valid_c = reinterpret_cast<long long*>(w + L.n_valid_c);
    void* hidden_c = w + L.hidden_c;
    const int cblk = (n + kCompactThreads - 1) / kCompactThreads;
    e = launch(kHelper, st, [&] {
      compact_count_kernel<<<cblk, kCompactThreads, 0, st>>>(labels, n, ignore_index, V,
                                                             ws_status(ws), block_valid);
    });
    if (e == cudaSuccess)
      e = launch(kHelper, st, [&] {
        exclusive_scan_kernel<<<1, kCompactThreads, 0, st>>>(block_valid, cblk, n_valid_c);
      });
    if (e == cudaSuccess)
      e = launch(kHelper, st, [&] {
        compact_scatter_kernel<<<cblk, kCompactThreads, 0, st>>>(
            labels, nullptr, n, ignore_index, block_valid, n_valid_c, perm, labels_c, nullptr, V,
            nullptr, nullptr);
      });
    if (e == cudaSuccess)
      e = launch(kHelper, st, [&] {
        gather_rows_kernel<<<n, 256, 0, st>>>(static_cast<const uint4*>(hidden),
                                              static_cast<int>(H / 8), n, perm, n_valid_c,
                                              static_cast<uint4*>(hidden_c), nullptr,
                                              static_cast<int>(H / 4), 0);
      });
    if (e != cudaSuccess) return cuda_fail(e);
    hid = hidden_c;
    lab = labels_c;
  }

  CUtensorMap ta, tb;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, hid, H, N, H * 2, BK, BM) ||
      !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, weight, H, V, H * 2, BK, b_box_rows(o)))
    return FLCE_ERR_CUDA;

  GemmArgs g{};
  g.k_blocks = static_cast<int>((H + BK - 1) / BK);
  g.group_m = o.fwd_group;
  g.a_off = 0;
  g.b_off = 0;
  g.status = ws_status(ws);
  g.timeout_ns = o.timeout_ns;
  // dynamic hand-out keeps the pairs in step across the raster's waves, so the
  // weight panels a wave shares are still in L2 when its last pair reads them
  g.tile_counter = o.fwd_dynamic ? ws_fwd_counter(ws) : nullptr;
  if (compact) {  // only the valid (compacted) rows are worked on
    g.rows_valid = n_valid_c;
    g.rows_base = 0;
    g.rows_host = n;
    g.rows_dim = kRowsM;
  }

  const GemmProblem prob{&ta, &tb, &ta, N, V, g};
  if (softcap > 0.f) {
    FwdStatsEpi<true>::Params ep{lab, n, static_cast<int>(V), softcap, 1.0f / softcap, part_m,
                                 part_s, label_logit};
    e = run_gemm<FwdStatsEpi<true>, false, false>(d, o, o.fwd_bn, kFwdGemm, prob, ep, nullptr,
                                                  ep, st);
  } else {
    FwdStatsEpi<false>::Params ep{lab, n, static_cast<int>(V), 0.f, 0.f, part_m, part_s,
                                  label_logit};
    e = run_gemm<FwdStatsEpi<false>, false, false>(d, o, o.fwd_bn, kFwdGemm, prob, ep, nullptr,
                                                   ep, st);
  }
  if (e != cudaSuccess) return cuda_fail(e);

  const int n_vt = static_cast<int>((V + BN - 1) / BN);  // (m, s) partials per row
  e = launch(kFwdMerge, st, [&] {
    fwd_merge_kernel<<<(n + kMergeRows - 1) / kMergeRows, dim3(kMergeRows, kMergeSplit), 0, st>>>(
        part_m, part_s, n_vt, n, lse, labels, ignore_index, V, perm, n_valid_c, lse_c);
  });
  if (e != cudaSuccess) return cuda_fail(e);
  // per-row losses in compact order when compacted (the rows past the valid
  // ones carry ignore_index and add nothing)
  const int nblk = (n + kLossThreads - 1) / kLossThreads;
  e = launch(kFwdMerge, st, [&] {
    row_loss_kernel<<<nblk, kLossThreads, 0, st>>>(compact ? lse_c : lse, label_logit, lab, n,
                                                   ignore_index, V, block_loss, block_cnt,
                                                   ws_status(ws));
  });
  if (e != cudaSuccess) return cuda_fail(e);
  e = launch(kFwdMerge, st, [&] {
    finalize_kernel<<<1, kFinalThreads, 0, st>>>(block_loss, block_cnt, nblk,
                                                 reduction == FLCE_MEAN, loss_scale, loss_div,
                                                 loss, num_tokens, ws_nvalid(ws));
  });
  if (e != cudaSuccess) return cuda_fail(e);
  return FLCE_OK;
}

flce_status forward_fp32(DevInfo* d, const void* hidden, const void* weight,
                         const int64_t* labels, int64_t N, int64_t H, int64_t V,
                         int64_t ignore_index, float softcap, int32_t reduction,
                         double loss_scale, double loss_div, float* loss, int64_t* num_tokens,
                         float* lse, void* ws, cudaStream_t st) {
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
        softcap, ignore_index, lse, label_logit);
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
                                                 reduction == FLCE_MEAN, loss_scale, loss_div,
                                                 loss, num_tokens, ws_nvalid(ws));
  });
  if (e != cudaSuccess) return cuda_fail(e);
  return FLCE_OK;
}

// ---------------------------------------------------------------- backward
flce_status backward_bf16(DevInfo* d, const Opts& o, const void* hidden, const void* weight,
                          const int64_t* labels, const float* lse, int64_t N, int64_t H,
                          int64_t V, int64_t ignore_index, float softcap, int32_t reduction,
                          const float* grad_output, float grad_scale, const long long* n_valid,
                          bool n_valid_is_count, float* d_hidden, float* d_weight,
                          int32_t flags, void* ws, cudaStream_t st) {
  const bool acc_dh = (flags & FLCE_ACCUMULATE_DHIDDEN) != 0;
  const bool acc_dw = (flags & FLCE_ACCUMULATE_DWEIGHT) != 0;
  const bool want_dh = d_hidden != nullptr;  // a NULL output is not computed
  const bool want_dw = d_weight != nullptr;
  const Chunking ck = chunking(o, N, V);
  const BwdLayout BL = bwd_layout(o, N, H, V);
  char* w = static_cast<char*>(ws);
  int* counters = reinterpret_cast<int*>(w + BL.counters);
  int next_counter = 0;
  const int nchunks = static_cast<int>(bwd_chunks(o, N, V));
  int* done = counters + 3 * nchunks;  // per chunk: CTAs of its gradient launches that finished
  std::vector<int> readers(nchunks, 0);  // per chunk: CTAs of its gradient launches
  {
    const cudaError_t e = cudaMemsetAsync(counters, 0, 4 * bwd_counters(o, N, V), st);
    if (e != cudaSuccess) return cuda_fail(e);
  }

  // Row compaction: the GEMMs see the valid token rows first (compact hidden,
  // labels and lse), the device-side count bounds their token-row dimension,
  // and dHidden rows are scattered back through the permutation.
  const bool compact = o.compact;
  const void* hid = hidden;
  const int64_t* lab = labels;
  const float* lsev = lse;
  int* perm = nullptr;
  const long long* rows_valid = nullptr;
  float* resid = nullptr;  // label-entry residuals (compact mode: label-sorted rows)
  if (compact) {
    perm = reinterpret_cast<int*>(w + BL.perm);
    int64_t* labels_c = reinterpret_cast<int64_t*>(w + BL.labels_c);
    float* lse_c = reinterpret_cast<float*>(w + BL.lse_c);
    int* block_valid = reinterpret_cast<int*>(w + BL.block_valid);
    long long* n_valid_c = reinterpret_cast<long long*>(w + BL.n_valid_c);
    void* hidden_c = w + BL.hidden_c;
    const int n = static_cast<int>(N);
    const int nblk = (n + kCompactThreads - 1) / kCompactThreads;
    cudaError_t e = launch(kHelper, st, [&] {
      compact_count_kernel<<<nblk, kCompactThreads, 0, st>>>(labels, n, ignore_index, V,
                                                             ws_status(ws), block_valid);
    });
    if (e == cudaSuccess)
      e = launch(kHelper, st, [&] {
        exclusive_scan_kernel<<<1, kCompactThreads, 0, st>>>(block_valid, nblk, n_valid_c);
      });
    uint32_t* keys[2] = {reinterpret_cast<uint32_t*>(w + BL.keys0),
                         reinterpret_cast<uint32_t*>(w + BL.keys1)};
    int* vals[2] = {reinterpret_cast<int*>(w + BL.vals0), reinterpret_cast<int*>(w + BL.vals1)};
    if (e == cudaSuccess)
      e = launch(kHelper, st, [&] {
        compact_scatter_kernel<<<nblk, kCompactThreads, 0, st>>>(
            labels, lse, n, ignore_index, block_valid, n_valid_c, perm, labels_c, lse_c, V,
            keys[0], vals[0]);
      });
    // Valid rows in (label, token) order: keys are labels in [0, V), so
    // ceil(bits(V - 1) / 8) passes of 8 bits sort them.
    int key_bits = 0;
    while (((V - 1) >> key_bits) != 0) ++key_bits;
    const int passes = (key_bits + 7) / 8;
    int* hist = reinterpret_cast<int*>(w + BL.hist);
    for (int ps = 0; ps < passes && e == cudaSuccess; ++ps) {
      const int src = ps & 1, shift = 8 * ps;
      e = launch(kHelper, st, [&] {
        radix_hist_kernel<<<nblk, kCompactThreads, 0, st>>>(keys[src], n_valid_c, shift, nblk,
                                                              hist);
      });
      if (e == cudaSuccess)
        e = launch(kHelper, st, [&] {
          exclusive_scan_kernel<<<1, kCompactThreads, 0, st>>>(hist, kRadixBuckets * nblk,
                                                               nullptr);
        });
      if (e == cudaSuccess)
        e = launch(kHelper, st, [&] {
          radix_scatter_kernel<<<nblk, kCompactThreads, 0, st>>>(
              keys[src], vals[src], keys[src ^ 1], vals[src ^ 1], n_valid_c, shift, nblk, hist);
        });
    }
    if (e == cudaSuccess)
      e = launch(kHelper, st, [&] {
        apply_label_order_kernel<<<nblk, kCompactThreads, 0, st>>>(
            keys[passes & 1], vals[passes & 1], lse, n_valid_c, perm, labels_c, lse_c);
      });
    if (e == cudaSuccess)
      e = launch(kHelper, st, [&] {
        gather_rows_kernel<<<n, 256, 0, st>>>(
            static_cast<const uint4*>(hidden), static_cast<int>(H / 8), n, perm, n_valid_c,
            static_cast<uint4*>(hidden_c), reinterpret_cast<float4*>(d_hidden),
            static_cast<int>(H / 4), (want_dh && !acc_dh) ? 1 : 0);
      });
    if (e != cudaSuccess) return cuda_fail(e);
    hid = hidden_c;
    lab = labels_c;
    lsev = lse_c;
    resid = reinterpret_cast<float*>(w + BL.resid);
    rows_valid = n_valid_c;
    if (n_valid_is_count) n_valid = n_valid_c;  // the library's own count serves both
  }

  // dHidden GEMM output: with row compaction a chunk-local compact-order fp32
  // block (TMA stores and reduce-adds, then dh_scatter to token order),
  // else d_hidden itself.
  float* dh_c = compact ? reinterpret_cast<float*>(w + BL.dh_c) : nullptr;
  float* dh_out = compact ? dh_c : d_hidden;
  const int64_t dh_rows = compact ? ck.tc : N;
  CUtensorMap t_hid_k, t_hid_mn, t_w_k, t_w_mn, t_dh, t_dw;
  if (!make_map(&t_hid_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, hid, H, N, H * 2, BK, BM) ||
      !make_map(&t_hid_mn, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, hid, H, N, H * 2, 64, BK) ||
      !make_map(&t_w_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, weight, H, V, H * 2, BK, b_box_rows(o)) ||
      !make_map(&t_w_mn, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, weight, H, V, H * 2, 64, BK) ||
      (want_dh && !make_map(&t_dh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, dh_out, H, dh_rows, H * 4,
                            32, 32)) ||
      (want_dw &&
       !make_map(&t_dw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, d_weight, H, V, H * 4, 32, 32)))
    return FLCE_ERR_CUDA;
  // H a multiple of 64: the MN-major hidden and weight operands use the 3-D view
  // (FLCE_OPT_MN3D = 0: every MN-major operand uses the 2-D view)
  const bool mn3d = o.mn3d;
  const bool h3d = mn3d && (H % 64 == 0);
  if (h3d && (!make_map_mn3d(&t_hid_mn, hid, H, N, H * 2) ||
              !make_map_mn3d(&t_w_mn, weight, H, V, H * 2)))
    return FLCE_ERR_CUDA;

  const int k_blocks_h = static_cast<int>((H + BK - 1) / BK);
  const unsigned long long tmo = o.timeout_ns;
  // dZ tile width: by default 512 columns (fewer operand bytes per FLOP), but
  // 256 with softcap, whose tanh-heavy epilogue a 512-column tile exposes
  // (measured at the power cap: -1.2% vs +0.5% step time)
  const int dz_bn = o.dz_bn != 0 ? o.dz_bn : (softcap > 0.f ? 256 : 512);
  const int mean = reduction == FLCE_MEAN;

  int ci = 0;  // chunk index
  for (int64_t t0 = 0; t0 < N; t0 += ck.tc) {
    const int rows = static_cast<int>(std::min<int64_t>(ck.tc, N - t0));
    for (int64_t v0 = 0; v0 < V; v0 += ck.vc, ++ci) {
      const int cols = static_cast<int>(std::min<int64_t>(ck.vc, V - v0));
      // dZ block [rows, cols] bf16, row stride ck.vc elements (one of dz_buffers
      // blocks, used by chunks in turn)
      void* gbuf = w + BL.gblock + static_cast<size_t>(ci % o.dz_buffers) * BL.gblock_bytes;
      CUtensorMap t_g_store, t_g_k, t_g_mn;
      if (!make_map(&t_g_store, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gbuf, cols, rows,
                    static_cast<uint64_t>(ck.vc) * 2, 64, 32) ||
          !make_map(&t_g_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gbuf, cols, rows,
                    static_cast<uint64_t>(ck.vc) * 2, BK, BM) ||
          !(mn3d ? make_map_mn3d(&t_g_mn, gbuf, ck.vc, rows, static_cast<uint64_t>(ck.vc) * 2)
                 : make_map(&t_g_mn, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gbuf, cols, rows,
                            static_cast<uint64_t>(ck.vc) * 2, 64, BK)))
        return FLCE_ERR_CUDA;
      // (the dZ block's 3-D view spans its full row pitch: columns past `cols`
      // hold stale values that reach only dWeight rows past V, which the
      // output map clips)

      // 1) dZ = f(hidden[t0:] . W[v0:]^T) -> bf16 block
      GemmArgs gz{};
      gz.k_blocks = k_blocks_h;
      gz.group_m = o.dz_group;
      gz.a_off = static_cast<int>(t0);
      gz.b_off = static_cast<int>(v0);
      gz.status = ws_status(ws);
      gz.timeout_ns = tmo;
      gz.tile_counter = counters + next_counter++;
      gz.rows_valid = rows_valid;
      gz.rows_base = static_cast<int>(t0);
      gz.rows_host = rows;
      gz.rows_dim = kRowsM;
      if (ci == 0) {
        gz.dep_wait = kDepNone;
      } else if (o.dz_buffers == 1) {
        // dZ overwrites the block the previous chunk's dHidden/dWeight GEMMs
        // read: its main loop may start early, its first store waits for them
        gz.dep_wait = kDepBeforeStores;
      } else {
        // two blocks: dZ runs beside the previous chunk's gradient GEMMs (in
        // their last wave), stores once the chunk before that, which read this
        // block, has counted all its CTAs out, and completes only after the
        // previous launch, so the next gradient launch, which waits for this
        // one, also follows the previous one
        gz.dep_wait = kDepBeforeExit;
        if (ci >= 2) {
          gz.wait_counter = done + (ci - 2);
          gz.wait_target = readers[ci - 2];
        }
      }
      cudaError_t e;
      const GemmProblem pz{&t_hid_k, &t_w_k, &t_g_store, rows, cols, gz};
      if (softcap > 0.f) {
        DzEpi<true>::Params ep{lab,  lsev,    ignore_index, static_cast<int>(t0),
                               rows, static_cast<int>(v0), cols, softcap, 1.0f / softcap,
                               resid, V};
        e = run_gemm<DzEpi<true>, false, false>(d, o, dz_bn, kBwdDz, pz, ep, nullptr, ep, st);
      } else {
        DzEpi<false>::Params ep{lab,  lsev, ignore_index, static_cast<int>(t0), rows,
                                static_cast<int>(v0), cols, 0.f, 0.f, resid, V};
        e = run_gemm<DzEpi<false>, false, false>(d, o, dz_bn, kBwdDz, pz, ep, nullptr, ep, st);
      }
      if (e != cudaSuccess) return cuda_fail(e);

      // 2) dHidden[t0:t0+rows] (+)= dZ . W[v0:v0+cols]
      GemmArgs gh{};
      gh.k_blocks = (cols + BK - 1) / BK;
      gh.group_m = o.grad_group;
      gh.a_off = 0;
      gh.b_off = static_cast<int>(v0);
      gh.status = ws_status(ws);
      gh.timeout_ns = tmo;
      gh.tile_counter = counters + next_counter++;
      gh.rows_valid = rows_valid;
      gh.rows_base = static_cast<int>(t0);
      gh.rows_host = rows;
      gh.rows_dim = kRowsM;
      gh.dep_wait = kDepBeforeLoads;  // reads the dZ block written just before
      gh.b_mn3d = h3d ? 1 : 0;
      if (o.dz_buffers > 1) gh.done_counter = done + ci;
      const bool last_v = v0 + ck.vc >= V;
      StoreEpi::Params eh{compact ? 0 : static_cast<int>(t0),
                          (v0 > 0 || (acc_dh && !compact)) ? 1 : 0, static_cast<int>(H),
                          compact ? rows : static_cast<int>(N), grad_output, grad_scale,
                          n_valid, mean};

      // 3) dWeight[v0:v0+cols] (+)= dZ^T . hidden[t0:t0+rows]
      GemmArgs gw{};
      gw.k_blocks = (rows + BK - 1) / BK;
      gw.group_m = o.grad_group;
      gw.a_off = 0;
      gw.b_off = static_cast<int>(t0);
      gw.status = ws_status(ws);
      gw.timeout_ns = tmo;
      gw.tile_counter = counters + next_counter++;
      gw.rows_valid = rows_valid;
      gw.rows_base = static_cast<int>(t0);
      gw.rows_host = rows;
      gw.rows_dim = kRowsK;
      gw.zero_if_empty = (t0 == 0 && !acc_dw) ? 1 : 0;  // the first chunk overwrites dWeight
      gw.dep_wait = kDepBeforeLoads;
      gw.a_mn3d = mn3d ? 1 : 0;
      gw.b_mn3d = h3d ? 1 : 0;
      if (o.dz_buffers > 1) gw.done_counter = done + ci;
      StoreEpi::Params ew{static_cast<int>(v0), (t0 > 0 || acc_dw) ? 1 : 0, static_cast<int>(H),
                          static_cast<int>(V), grad_output, grad_scale, n_valid, mean};

      const GemmProblem ph{&t_g_k, &t_w_mn, &t_dh, rows, H, gh};
      const GemmProblem pw{&t_g_mn, &t_hid_mn, &t_dw, cols, H, gw};
      const int gbn = o.grad_bn;
      int ctas = 0;
      if (want_dh && want_dw && o.fuse) {
        // 2) + 3) in one launch: the dWeight tiles fill the dHidden grid's last wave
        e = run_gemm<StoreEpi, false, true, true, true>(d, o, gbn, kBwdDhDw, ph, eh, &pw, ew, st,
                                                        &ctas);
        readers[ci] += ctas;
      } else {
        if (want_dh) {
          e = run_gemm<StoreEpi, false, true>(d, o, gbn, kBwdDhDw, ph, eh, nullptr, eh, st, &ctas);
          readers[ci] += ctas;
        }
        if (want_dw && e == cudaSuccess) {
          e = run_gemm<StoreEpi, true, true>(d, o, gbn, kBwdDhDw, pw, ew, nullptr, ew, st, &ctas);
          readers[ci] += ctas;
        }
      }
      if (e != cudaSuccess) return cuda_fail(e);

      if (compact && want_dh && last_v) {
        // the token chunk's dHidden is complete: add the exact label term and
        // move it to token order
        e = launch(kHelper, st, [&] {
          dh_scatter_kernel<<<rows, 256, 0, st>>>(
              reinterpret_cast<const float4*>(dh_c), static_cast<int>(t0), rows, perm,
              rows_valid, lab, resid, static_cast<const __nv_bfloat16*>(weight), V,
              static_cast<int>(H / 4), reinterpret_cast<float4*>(d_hidden), acc_dh ? 1 : 0,
              grad_output, grad_scale, n_valid, mean);
        });
        if (e != cudaSuccess) return cuda_fail(e);
      }
    }
  }

  if (compact && want_dw) {
    // dWeight's exact label term, per label run (dHidden's was added above).
    float* part = reinterpret_cast<float*>(w + BL.part);
    const dim3 grid(static_cast<unsigned>((N + kFixSeg - 1) / kFixSeg),
                    static_cast<unsigned>((H + kFixCols - 1) / kFixCols));
    const int64_t* labels_c = lab;
    cudaError_t e = launch(kHelper, st, [&] {
      dw_fix_segments_kernel<<<grid, kFixThreads, 0, st>>>(
          labels_c, resid, rows_valid, static_cast<const __nv_bfloat16*>(hid),
          static_cast<int>(H), V, d_weight, part, grad_output, grad_scale, n_valid, mean);
    });
    if (e == cudaSuccess)
      e = launch(kHelper, st, [&] {
        dw_fix_runs_kernel<<<grid, kFixThreads, 0, st>>>(labels_c, rows_valid,
                                                         static_cast<int>(H), V, d_weight, part,
                                                         grad_output, grad_scale, n_valid, mean);
      });
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return FLCE_OK;
}

flce_status backward_fp32(DevInfo* d, const void* hidden, const void* weight,
                          const int64_t* labels, const float* lse, int64_t N, int64_t H,
                          int64_t V, int64_t ignore_index, float softcap, int32_t reduction,
                          const float* grad_output, float grad_scale, const long long* n_valid,
                          float* d_hidden, float* d_weight, int32_t flags, cudaStream_t st) {
  const int acc_dh = (flags & FLCE_ACCUMULATE_DHIDDEN) ? 1 : 0;
  const int acc_dw = (flags & FLCE_ACCUMULATE_DWEIGHT) ? 1 : 0;
  const int n = static_cast<int>(N), h = static_cast<int>(H), v = static_cast<int>(V);
  const int mean = reduction == FLCE_MEAN;
  const size_t sh_dh = (2 * static_cast<size_t>(h) + kSimtChunk) * sizeof(float);
  const size_t sh_dw = (2 * static_cast<size_t>(h) + kSimtThreads) * sizeof(float);
  (void)d;
  cudaError_t e = set_smem_attr(simt_dh_kernel, 2 * kSimtMaxH * 4 + kSimtChunk * 4);
  if (e != cudaSuccess) return cuda_fail(e);
  e = set_smem_attr(simt_dw_kernel, 2 * kSimtMaxH * 4 + kSimtThreads * 4);
  if (e != cudaSuccess) return cuda_fail(e);
  if (n > 0 && d_hidden != nullptr) {
    e = launch(kSimt, st, [&] {
      simt_dh_kernel<<<n, kSimtThreads, sh_dh, st>>>(
          static_cast<const float*>(hidden), static_cast<const float*>(weight), labels, lse, n, h,
          v, ignore_index, softcap, grad_output, grad_scale, n_valid, mean, acc_dh, d_hidden);
    });
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (d_weight == nullptr) return FLCE_OK;
  e = launch(kSimt, st, [&] {
    simt_dw_kernel<<<v, kSimtThreads, sh_dw, st>>>(
        static_cast<const float*>(hidden), static_cast<const float*>(weight), labels, lse, n, h, v,
        ignore_index, softcap, grad_output, grad_scale, n_valid, mean, acc_dw, d_weight);
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
  return ws_bytes(opts(), N, H, V, dtype == FLCE_BF16);
}

size_t flce_workspace_bytes_ex(int64_t N, int64_t H, int64_t V, int32_t dtype, int32_t flags) {
  if ((flags & ~kAllBwdFlags) != 0) return 0;
  if (flce_workspace_bytes(N, H, V, dtype) == 0) return 0;
  return grad_scratch(opts(), N, H, V, dtype == FLCE_BF16, flags).end;
}

flce_status flce_forward(const void* hidden, const void* weight, const int64_t* labels,
                         int64_t N, int64_t H, int64_t V, int64_t ignore_index, float softcap,
                         int32_t reduction, int32_t dtype, float* loss, int64_t* num_tokens,
                         float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  return flce_forward_ex2(hidden, weight, labels, N, H, V, ignore_index, softcap, reduction,
                          dtype, 1.0f, -1, loss, num_tokens, lse, workspace, workspace_bytes,
                          stream);
}

flce_status flce_forward_ex(const void* hidden, const void* weight, const int64_t* labels,
                            int64_t N, int64_t H, int64_t V, int64_t ignore_index, float softcap,
                            int32_t reduction, int32_t dtype, float loss_scale, float* loss,
                            int64_t* num_tokens, float* lse, void* workspace,
                            size_t workspace_bytes, void* stream) {
  return flce_forward_ex2(hidden, weight, labels, N, H, V, ignore_index, softcap, reduction,
                          dtype, loss_scale, -1, loss, num_tokens, lse, workspace,
                          workspace_bytes, stream);
}

flce_status flce_forward_ex2(const void* hidden, const void* weight, const int64_t* labels,
                             int64_t N, int64_t H, int64_t V, int64_t ignore_index, float softcap,
                             int32_t reduction, int32_t dtype, float loss_scale,
                             int64_t num_label_tokens, float* loss, int64_t* num_tokens,
                             float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  if (!(loss_scale == loss_scale) || loss_scale == INFINITY || loss_scale == -INFINITY)
    return FLCE_ERR_ARG;
  const Opts o = opts();
  flce_status s = check_common(o, hidden, weight, labels, N, H, V, softcap, reduction, dtype,
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
  const double div = label_token_divisor(reduction, num_label_tokens);
  if (dtype == FLCE_BF16)
    return forward_bf16(d, o, hidden, weight, labels, N, H, V, ignore_index, softcap, reduction,
                        loss_scale, div, loss, num_tokens, lse, workspace, st, o.fwd_compact);
  return forward_fp32(d, hidden, weight, labels, N, H, V, ignore_index, softcap, reduction,
                      loss_scale, div, loss, num_tokens, lse, workspace, st);
}

flce_status flce_backward(const void* hidden, const void* weight, const int64_t* labels,
                          const float* lse, int64_t N, int64_t H, int64_t V,
                          int64_t ignore_index, float softcap, int32_t reduction, int32_t dtype,
                          const float* grad_output, float grad_scale, const int64_t* num_valid,
                          float* d_hidden, float* d_weight, int32_t flags, void* workspace,
                          size_t workspace_bytes, void* stream) {
  return flce_backward_ex(hidden, weight, labels, lse, N, H, V, ignore_index, softcap, reduction,
                          dtype, grad_output, grad_scale, -1, num_valid, d_hidden, d_weight,
                          flags, workspace, workspace_bytes, stream);
}

flce_status flce_backward_ex(const void* hidden, const void* weight, const int64_t* labels,
                             const float* lse, int64_t N, int64_t H, int64_t V,
                             int64_t ignore_index, float softcap, int32_t reduction,
                             int32_t dtype, const float* grad_output, float grad_scale,
                             int64_t num_label_tokens, const int64_t* num_valid,
                             float* d_hidden, float* d_weight, int32_t flags, void* workspace,
                             size_t workspace_bytes, void* stream) {
  if ((flags & ~kAllBwdFlags) != 0) return FLCE_ERR_ARG;
  const Opts o = opts();
  flce_status s = check_common(o, hidden, weight, labels, N, H, V, softcap, reduction, dtype,
                               workspace, workspace_bytes);
  if (s != FLCE_OK) return s;
  const GradScratch gs = grad_scratch(o, N, H, V, dtype == FLCE_BF16, flags);
  if (workspace_bytes < gs.end) return FLCE_ERR_WORKSPACE;
  // a NULL d_hidden or d_weight is not computed; one of them must be given
  if ((d_hidden == nullptr && d_weight == nullptr) || (N > 0 && lse == nullptr))
    return FLCE_ERR_ARG;
  if (!aligned16(d_hidden) || !aligned16(d_weight)) return FLCE_ERR_ARG;
  if (!(grad_scale == grad_scale) || grad_scale == INFINITY || grad_scale == -INFINITY)
    return FLCE_ERR_ARG;
  // the gradient of a 'sum' loss normalised by max(num_label_tokens, 1)
  const float gscale =
      static_cast<float>(static_cast<double>(grad_scale) /
                         label_token_divisor(reduction, num_label_tokens));
  DevInfo* d = nullptr;
  s = device_info(&d);
  if (s != FLCE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(unsigned int), st);  // status word
  if (e != cudaSuccess) return cuda_fail(e);
  if (N == 0) {
    if (d_weight == nullptr || (flags & FLCE_ACCUMULATE_DWEIGHT)) return FLCE_OK;  // adds nothing
    const size_t elem = (flags & FLCE_DWEIGHT_BF16) ? 2 : sizeof(float);  // +0.0 in both
    e = cudaMemsetAsync(d_weight, 0, static_cast<size_t>(V) * H * elem, st);
    return e == cudaSuccess ? FLCE_OK : cuda_fail(e);
  }
  // bf16 outputs: the gradient is computed into fp32 scratch (overwritten, not
  // accumulated) and rounded once into the caller's buffer afterwards.
  char* wsb = static_cast<char*>(workspace);
  float* dh32 = (d_hidden != nullptr && (flags & FLCE_DHIDDEN_BF16))
                    ? reinterpret_cast<float*>(wsb + gs.dh) : d_hidden;
  float* dw32 = (d_weight != nullptr && (flags & FLCE_DWEIGHT_BF16))
                    ? reinterpret_cast<float*>(wsb + gs.dw) : d_weight;
  int32_t inner = flags & (FLCE_ACCUMULATE_DHIDDEN | FLCE_ACCUMULATE_DWEIGHT);
  if (flags & FLCE_DHIDDEN_BF16) inner &= ~FLCE_ACCUMULATE_DHIDDEN;
  if (flags & FLCE_DWEIGHT_BF16) inner &= ~FLCE_ACCUMULATE_DWEIGHT;
  const bool compacts = (dtype == FLCE_BF16 && o.compact);
  if (!compacts) {  // the compaction checks the labels itself
    e = launch(kHelper, st, [&] {
      label_range_kernel<<<static_cast<unsigned>((N + 255) / 256), 256, 0, st>>>(
          labels, static_cast<int>(N), ignore_index, V, ws_status(workspace));
    });
    if (e != cudaSuccess) return cuda_fail(e);
  }
  const long long* nv = reinterpret_cast<const long long*>(num_valid);
  const bool own_count = (nv == nullptr);
  if (nv == nullptr && !compacts) {
    long long* out = ws_nvalid(workspace);
    e = launch(kHelper, st, [&] {
      count_valid_kernel<<<1, kFinalThreads, 0, st>>>(labels, static_cast<int>(N), ignore_index,
                                                      V, out);
    });
    if (e != cudaSuccess) return cuda_fail(e);
    nv = out;
  }
  if (dtype == FLCE_BF16)
    s = backward_bf16(d, o, hidden, weight, labels, lse, N, H, V, ignore_index, softcap,
                      reduction, grad_output, gscale, nv, own_count, dh32, dw32, inner, workspace,
                      st);
  else
    s = backward_fp32(d, hidden, weight, labels, lse, N, H, V, ignore_index, softcap, reduction,
                      grad_output, gscale, nv, dh32, dw32, inner, st);
  if (s != FLCE_OK) return s;
  const struct {
    int32_t flag, acc;
    const float* src;
    void* dst;
    size_t n;
  } outs[2] = {{FLCE_DHIDDEN_BF16, FLCE_ACCUMULATE_DHIDDEN, dh32, d_hidden,
                static_cast<size_t>(N) * H},
               {FLCE_DWEIGHT_BF16, FLCE_ACCUMULATE_DWEIGHT, dw32, d_weight,
                static_cast<size_t>(V) * H}};
  for (const auto& out : outs) {
    if (!(flags & out.flag) || out.dst == nullptr) continue;
    const unsigned blocks = static_cast<unsigned>(
        std::min<size_t>((out.n / 8 + 255) / 256 + 1, static_cast<size_t>(d->sms) * 8));
    e = launch(kHelper, st, [&] {
      f32_to_bf16_kernel<<<blocks, 256, 0, st>>>(out.src, static_cast<__nv_bfloat16*>(out.dst),
                                                 out.n, (flags & out.acc) ? 1 : 0);
    });
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return FLCE_OK;
}

flce_status flce_set_option(int32_t option, int64_t value) {
  if (option < 0 || option >= kNumOpts) return FLCE_ERR_ARG;
  const OptSpec& sp = kOptSpec[option];
  if (value < sp.lo || value > sp.hi) return FLCE_ERR_ARG;
  if ((option == FLCE_OPT_GRAD_TILE_N || option == FLCE_OPT_DZ_TILE_N ||
       option == FLCE_OPT_FWD_TILE_N) && value != 256 && value != 512 &&
      !(option == FLCE_OPT_DZ_TILE_N && value == 0))
    return FLCE_ERR_ARG;
  g_opt[option].store(value);
  return FLCE_OK;
}

flce_status flce_get_option(int32_t option, int64_t* value) {
  if (option < 0 || option >= kNumOpts || value == nullptr) return FLCE_ERR_ARG;
  *value = g_opt[option].load();
  return FLCE_OK;
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

flce_status flce_selftest_wait_timeout(void* workspace, int32_t timeout_ms, void* stream) {
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FLCE_ERR_ARG;
  if (timeout_ms < 1 || timeout_ms > 10000) return FLCE_ERR_ARG;
  DevInfo* d = nullptr;
  flce_status s = device_info(&d);
  if (s != FLCE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int* status = ws_status(workspace);
  const unsigned long long ns = static_cast<unsigned long long>(timeout_ms) * 1000000ull;
  const cudaError_t e = launch(kHelper, st, [&] { selftest_wait_kernel<<<1, 32, 0, st>>>(status, ns); });
  return e == cudaSuccess ? FLCE_OK : cuda_fail(e);
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
            ? forward_bf16(d, opts(), hidden, weight, labels, N, H, V, ignore_index, softcap,
                           reduction, 1.0, 1.0, loss, num_tokens, lse, ws, st, false)
            : forward_fp32(d, hidden, weight, labels, N, H, V, ignore_index, softcap, reduction,
                           1.0, 1.0, loss, num_tokens, lse, ws, st);
    if (s != FLCE_OK) return s;
  }
  if (status != nullptr) {
    e = cudaMemcpyAsync(status, ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return FLCE_OK;
}
