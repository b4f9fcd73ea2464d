// Persistent tcgen05 GEMM for the fused linear cross-entropy (FLCE).
//
// One CTA per SM (192 threads, ~225 KB shared memory, all 512 TMEM columns).
// Warp roles:
//   warp 0  TMA producer   (one thread): K-blocks of A and B into a 4-stage ring
//   warp 1  MMA issuer     (one thread): tcgen05.mma M=128 N=256 K=16, fp32 in TMEM;
//                                        two 256-column accumulators so the
//                                        epilogue of tile i overlaps the MMAs of i+1
//   warps 2-5 epilogue     (128 threads, thread = accumulator row): tcgen05.ld
//                                        then an operation-specific epilogue
// Output tile 128 x 256, K-block 64 (one 128-byte swizzle row of bf16).
//
// Operands may be K-major (row-major [rows, K], the usual "TN" GEMM) or
// MN-major (row-major [K, rows]); both are staged with 128-byte swizzle and
// described to the tensor core by UMMA shared-memory descriptors.
//
// The three epilogues implement the steps of the fused linear cross-entropy:
//   FwdStatsEpi  softcap, per-row online max / sum of exp over the tile's 256
//                vocab columns, label-logit capture (forward)
//   DzEpi        softcap, dZ = g*(exp(L-lse) - onehot)*softcap' -> bf16 block
//                of dZ in global memory via TMA store (backward)
//   StoreEpi     fp32 tile -> TMA store or TMA reduce-add (dHidden, dWeight)
// The GEMM itself is the LM-head projection logits = hidden . weight^T
// (NeMo AutoModel linear_ce API: lm_weight is [vocab, hidden]) and, in the
// backward, dZ . weight and dZ^T . hidden.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "ptx.cuh"

namespace flce {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK * 2;  // 16 KB
constexpr int kBBytes = BN * BK * 2;  // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kEpiWarps = 4;
constexpr int kStagingBuf = 4096;                 // 32 rows x 128 bytes
constexpr int kStagingPerWarp = 2 * kStagingBuf;  // double buffered
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr size_t kGemmSmemBytes =
    1024 + static_cast<size_t>(kStages) * kStageBytes + kEpiWarps * kStagingPerWarp;

constexpr uint32_t kStatusLabelRange = 1u;
constexpr uint32_t kStatusTimeout = 2u;

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct GemmArgs {
  int m_tiles;
  int n_tiles;
  int k_blocks;
  int group_m;    // tiles are walked in groups of group_m row-tiles (L2 reuse)
  int a_off;      // added to A's outer (row) TMA coordinate
  int b_off;      // added to B's outer (row) TMA coordinate
  int a_mn_extent;  // MN-major A: extent of its inner (M) dimension
  int b_mn_extent;  // MN-major B: extent of its inner (N) dimension
  unsigned int* status;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void tile_coords(int tile, const GemmArgs& g, int& mb, int& nb) {
  const int per_group = g.group_m * g.n_tiles;
  const int grp = tile / per_group;
  const int first_m = grp * g.group_m;
  const int gm = min(g.group_m, g.m_tiles - first_m);
  const int r = tile - grp * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

__device__ __forceinline__ void release_tmem(uint32_t tempty_bar, int lane) {
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(tempty_bar);
}

// Write 128 bytes (8 x 16 B) of row `lane` into a 32-row staging buffer laid
// out as the TMA 128-byte swizzle expects: 16-byte chunk j of row r lives at
// chunk position j ^ (r % 8).  Rows r and r+8 share banks, so a warp's store
// takes the minimum four wavefronts.
__device__ __forceinline__ void stage_row_128b(uint8_t* buf, int lane, const uint32_t (&w)[32]) {
  uint8_t* row = buf + lane * 128;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint4 v = make_uint4(w[4 * j + 0], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
    *reinterpret_cast<uint4*>(row + ((j ^ (lane & 7)) << 4)) = v;
  }
}

// ------------------------------------------------------------------ forward
// Per tile: L = softcap(Z) over 256 vocab columns; per row the maximum m and
// s = sum exp(L - m) (both in the log2 domain), written to partials
// [n_tile][N]; the label logit L[i, y_i] is written by the tile holding y_i.
template <bool kSoftcap>
struct FwdStatsEpi {
  struct Params {
    const int64_t* labels;
    int N;
    int V;
    float softcap;
    float inv_softcap;
    float* part_m;       // [n_tiles][N], log2 domain
    float* part_s;       // [n_tiles][N]
    float* label_logit;  // [N]
  };

  __device__ static void tile(const Params& p, const GemmArgs&, int mb, int nb, uint32_t taddr,
                              int q, int lane, uint8_t*, const CUtensorMap*, uint32_t tempty,
                              int&) {
    const int row = mb * BM + q * 32 + lane;
    const bool row_ok = row < p.N;
    const int col0 = nb * BN;
    int y_local = -1;
    if (row_ok) {
      const int64_t y = p.labels[row];
      if (y >= col0 && y < static_cast<int64_t>(col0) + BN) y_local = static_cast<int>(y - col0);
    }
    const int ncols = min(BN, p.V - col0);
    float m = -CUDART_INF_F;
    float s = 0.f;
    float ly = 0.f;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      tmem_ld_x32(taddr + c * 32, r);
      tmem_ld_wait();
      if (c == BN / 32 - 1) release_tmem(tempty, lane);
      float t[32];
      float cmax = -CUDART_INF_F;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float z = __uint_as_float(r[j]);
        const float L = kSoftcap ? p.softcap * tanhf(z * p.inv_softcap) : z;
        const int col = c * 32 + j;
        if (col == y_local) ly = L;
        t[j] = (col < ncols) ? L * kLog2e : -CUDART_INF_F;
        cmax = fmaxf(cmax, t[j]);
      }
      const float mn = fmaxf(m, cmax);
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) acc += exp2f(t[j] - mn);
      s = (m == -CUDART_INF_F) ? acc : s * exp2f(m - mn) + acc;
      m = mn;
    }
    if (row_ok) {
      const size_t idx = static_cast<size_t>(nb) * p.N + row;
      p.part_m[idx] = m;
      p.part_s[idx] = s;
      if (y_local >= 0) p.label_logit[row] = ly;
    }
  }
};

// ------------------------------------------------------------------ dZ
// Per tile of a (token-block x vocab-block) chunk: recompute L from Z, form
// dZ/g = (exp(L - lse) - [v == y])*(softcap ? 1 - (L/s)^2 : 1) in fp32
// registers, round to bf16 and TMA-store into the chunk's dZ block
// [rows x cols] (block-local coordinates).  Ignored rows get exact zeros.
// The scalar g = grad_output * grad_scale (/ n for 'mean') is applied later,
// in fp32, by the dHidden / dWeight epilogues: folding an arbitrary g into
// the bf16 value would move the dominant label entry (p - 1 ~ -1, which
// rounds to -1 almost exactly) off the bf16 grid.
template <bool kSoftcap>
struct DzEpi {
  struct Params {
    const int64_t* labels;
    const float* lse;
    int64_t ignore_index;
    int t0;     // global token row of the block's row 0
    int rows;   // valid token rows in this block
    int v0;     // global vocab id of the block's column 0
    int cols;   // valid vocab columns in this block
    float softcap;
    float inv_softcap;
  };

  __device__ static void tile(const Params& p, const GemmArgs&, int mb, int nb, uint32_t taddr,
                              int q, int lane, uint8_t* stg, const CUtensorMap* out,
                              uint32_t tempty, int& nstore) {
    // 64-column chunks whose store box starts inside the block (warp-uniform)
    const int y0 = mb * BM + q * 32;
    const int rem = p.cols - nb * BN;
    const int nch = (y0 >= p.rows || rem <= 0) ? 0 : min(BN / 64, (rem + 63) / 64);
    if (nch == 0) {
      release_tmem(tempty, lane);
      return;
    }
    const int row_l = y0 + lane;
    bool valid = false;
    int y_local = -1;
    float lse2 = 0.f;
    if (row_l < p.rows) {
      const int row = p.t0 + row_l;
      const int64_t y = p.labels[row];
      valid = (y != p.ignore_index);
      const int64_t c0 = static_cast<int64_t>(p.v0) + static_cast<int64_t>(nb) * BN;
      if (valid && y >= c0 && y < c0 + BN) y_local = static_cast<int>(y - c0);
      lse2 = p.lse[row] * kLog2e;
    }
    const uint32_t stg_u32 = smem_u32(stg);
#pragma unroll 1
    for (int c2 = 0; c2 < nch; ++c2) {
      uint32_t r0[32], r1[32];
      tmem_ld_x32(taddr + c2 * 64, r0);
      tmem_ld_x32(taddr + c2 * 64 + 32, r1);
      tmem_ld_wait();
      if (c2 == nch - 1) release_tmem(tempty, lane);
      uint32_t packed[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float gv[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int jj = 2 * j + h;
          const float z = __uint_as_float(jj < 32 ? r0[jj] : r1[jj - 32]);
          const float L = kSoftcap ? p.softcap * tanhf(z * p.inv_softcap) : z;
          float d = exp2f(fmaf(L, kLog2e, -lse2));
          if (c2 * 64 + jj == y_local) d -= 1.0f;
          if (kSoftcap) {
            const float u = L * p.inv_softcap;
            d *= fmaf(-u, u, 1.0f);
          }
          gv[h] = valid ? d : 0.0f;
        }
        __nv_bfloat162 b2 = __floats2bfloat162_rn(gv[0], gv[1]);
        packed[j] = *reinterpret_cast<uint32_t*>(&b2);
      }
      // Buffer = parity of this warp's store count: the store that last read
      // this buffer is the one before the most recent, which wait_read<1>
      // has retired.
      const int b = nstore & 1;
      if (lane == 0) bulk_wait_group_read<1>();
      __syncwarp();
      stage_row_128b(stg + b * kStagingBuf, lane, packed);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(out, stg_u32 + b * kStagingBuf, nb * BN + c2 * 64, y0);
        bulk_commit_group();
      }
      ++nstore;
    }
  }
};

// ------------------------------------------------------------------ fp32 out
// Tile * g -> fp32 output rows [out_row0 + m]: TMA store, or TMA reduce-add
// when `reduce` (accumulation across chunks of the split reduction dimension).
// g = grad_output * grad_scale, divided by max(n, 1) for 'mean'.
struct StoreEpi {
  struct Params {
    int out_row0;
    int reduce;
    int x_limit;  // output columns
    int y_limit;  // output rows
    const float* grad_output;  // may be null (1.0)
    float grad_scale;
    const long long* n_valid;  // device count of non-ignored rows
    int mean;
  };

  __device__ static float grad_factor(const Params& p) {
    float g = (p.grad_output != nullptr ? p.grad_output[0] : 1.0f) * p.grad_scale;
    if (p.mean) {
      const long long n = *p.n_valid;
      g = g / static_cast<float>(n > 0 ? n : 1);
    }
    return g;
  }

  __device__ static void tile(const Params& p, const GemmArgs&, int mb, int nb, uint32_t taddr,
                              int q, int lane, uint8_t* stg, const CUtensorMap* out,
                              uint32_t tempty, int& nstore) {
    // 32-column chunks whose store box starts inside the output (warp-uniform)
    const int y = p.out_row0 + mb * BM + q * 32;
    const int rem = p.x_limit - nb * BN;
    const int nch = (y >= p.y_limit || rem <= 0) ? 0 : min(BN / 32, (rem + 31) / 32);
    if (nch == 0) {
      release_tmem(tempty, lane);
      return;
    }
    const uint32_t stg_u32 = smem_u32(stg);
    const float g = grad_factor(p);
#pragma unroll 1
    for (int c = 0; c < nch; ++c) {
      uint32_t r[32];
      tmem_ld_x32(taddr + c * 32, r);
      tmem_ld_wait();
      if (c == nch - 1) release_tmem(tempty, lane);
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * g);
      const int b = nstore & 1;  // see DzEpi
      if (lane == 0) bulk_wait_group_read<1>();
      __syncwarp();
      stage_row_128b(stg + b * kStagingBuf, lane, r);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int x = nb * BN + c * 32;
        if (p.reduce)
          tma_reduce_add_2d(out, stg_u32 + b * kStagingBuf, x, y);
        else
          tma_store_2d(out, stg_u32 + b * kStagingBuf, x, y);
        bulk_commit_group();
      }
      ++nstore;
    }
  }
};

// ------------------------------------------------------------------ kernel
__device__ __forceinline__ void record_timeout(const GemmArgs& g, volatile int* abort) {
  *abort = 1;
  if (g.status != nullptr) atomicOr(g.status, kStatusTimeout);
}

template <class Epi, bool kAMn, bool kBMn>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmOut, const GemmArgs g,
                   const typename Epi::Params ep) {
  extern __shared__ uint8_t smem_dyn[];
  __shared__ __align__(8) uint64_t bar_full[kStages];
  __shared__ __align__(8) uint64_t bar_empty[kStages];
  __shared__ __align__(8) uint64_t bar_tfull[2];
  __shared__ __align__(8) uint64_t bar_tempty[2];
  __shared__ __align__(8) uint64_t bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  // 1024-byte alignment of the operand ring (required by the 128-byte swizzle).
  const uint32_t pad = (1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u;
  uint8_t* smem = smem_dyn + pad;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&bar_tfull[a]), 1);
      mbar_init(smem_u32(&bar_tempty[a]), kEpiWarps);
    }
    mbar_init(smem_u32(&bar_drain), 1);
    abort_sh = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmOut);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  const int num_tiles = g.m_tiles * g.n_tiles;
  volatile int* abort_flag = &abort_sh;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      uint32_t stage = 0, phase = 0;
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, g, mb, nb);
        for (int kb = 0; kb < g.k_blocks; ++kb) {
          if (!mbar_wait(smem_u32(&bar_empty[stage]), phase ^ 1u, abort_flag, g.timeout_ns)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&bar_full[stage]);
          const uint32_t sa = smem_u32(smem + stage * kStageBytes);
          const uint32_t sb = sa + kABytes;
          // An MN-major operand is loaded as 64-wide chunks along M/N.  A chunk
          // that starts at or past the tensor's extent is not loaded at all:
          // its shared-memory columns only feed output rows/columns that are
          // never stored, and a box lying wholly outside the tensor is avoided.
          uint32_t bytes = kStageBytes;
          if (kAMn) {
#pragma unroll
            for (int c = 0; c < BM / 64; ++c)
              if (mb * BM + c * 64 >= g.a_mn_extent) bytes -= 8192;
          }
          if (kBMn) {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              if (nb * BN + c * 64 >= g.b_mn_extent) bytes -= 8192;
          }
          mbar_arrive_expect_tx(fb, bytes);
          if (kAMn) {
#pragma unroll
            for (int c = 0; c < BM / 64; ++c)
              if (mb * BM + c * 64 < g.a_mn_extent)
                tma_load_2d(sa + c * 8192, &tmA, fb, mb * BM + c * 64, g.a_off + kb * BK);
          } else {
            tma_load_2d(sa, &tmA, fb, kb * BK, g.a_off + mb * BM);
          }
          if (kBMn) {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              if (nb * BN + c * 64 < g.b_mn_extent)
                tma_load_2d(sb + c * 8192, &tmB, fb, nb * BN + c * 64, g.b_off + kb * BK);
          } else {
            tma_load_2d(sb, &tmB, fb, kb * BK, g.b_off + nb * BN);
          }
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        record_timeout(g, abort_flag);
        // Let every load already issued land before the CTA can exit.
        for (int s = 0; s < kStages; ++s)
          if ((issued_mask >> s) & 1u)
            mbar_wait(smem_u32(&bar_full[s]), (issued_par >> s) & 1u, nullptr, g.timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t idesc = umma_idesc_bf16(BM, BN, kAMn, kBMn);
      uint32_t stage = 0, phase = 0;
      int it = 0;
      bool ok = true;
      bool issued = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const uint32_t acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(smem_u32(&bar_tempty[acc]), aph ^ 1u, abort_flag, g.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < g.k_blocks; ++kb) {
          if (!mbar_wait(smem_u32(&bar_full[stage]), phase, abort_flag, g.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int j = 0; j < BK / 16; ++j) {
            const uint64_t ad = kAMn ? umma_desc_sw128(sa + j * 2048, 8192, 1024)
                                     : umma_desc_sw128(sa + j * 32, 16, 1024);
            const uint64_t bd = kBMn ? umma_desc_sw128(sb + j * 2048, 8192, 1024)
                                     : umma_desc_sw128(sb + j * 32, 16, 1024);
            tc_mma_bf16(d_tmem, ad, bd, idesc, (kb > 0 || j > 0) ? 1u : 0u);
          }
          issued = true;
          tc_commit(smem_u32(&bar_empty[stage]));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(smem_u32(&bar_tfull[acc]));
      }
      if (!ok) {
        record_timeout(g, abort_flag);
        if (issued) {
          // Wait for the MMAs in flight before TMEM is released.
          tc_commit(smem_u32(&bar_drain));
          mbar_wait(smem_u32(&bar_drain), 0, nullptr, g.timeout_ns);
        }
      }
    }
  } else {
    // ---------------- epilogue warps
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    uint8_t* stg = smem + kStages * kStageBytes + (warp - 2) * kStagingPerWarp;
    int it = 0;
    int nstore = 0;  // TMA stores issued by this warp (selects the staging buffer)
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      int mb, nb;
      tile_coords(tile, g, mb, nb);
      const uint32_t acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      bool w = mbar_wait(smem_u32(&bar_tfull[acc]), aph, abort_flag, g.timeout_ns);
      w = __all_sync(0xffffffffu, w);
      if (!w) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + acc * BN + (static_cast<uint32_t>(q * 32) << 16);
      Epi::tile(ep, g, mb, nb, taddr, q, lane, stg, &tmOut, smem_u32(&bar_tempty[acc]), nstore);
    }
    if (lane == 0) {
      bulk_wait_group_all();
      if (!ok) record_timeout(g, abort_flag);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace flce
