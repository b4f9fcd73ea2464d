// Persistent tcgen05 GEMM for the fused linear cross-entropy (FLCE).
//
// One CTA per SM (320 threads, up to ~225 KB shared memory, all 512 TMEM
// columns).  Warp roles:
//   warp 0  TMA producer   (one thread): K-blocks of A and B into a stage ring
//   warp 1  MMA issuer     (one thread): tcgen05.mma K=16 steps, fp32 in TMEM
//   warps 2-9 epilogue     (a count the epilogue type sets), thread =
//                          accumulator row.  A warp may read only its TMEM lane
//                          quadrant (warp % 4), so two warps share a quadrant
//                          and each takes half of a bank's columns: it loads
//                          its 128 columns into registers, hands the TMEM bank
//                          back at once (the next tile's MMAs wait for it), and
//                          then runs the operation-specific epilogue.
// Tile shapes (template parameters kCG, the CTA group, and kBN, the columns of
// a tile):
//   kCG = 1, kBN = 256  one CTA computes a 128 x 256 tile
//            (tcgen05.mma.cta_group::1, M=128 N=256), 4 stages of 48 KiB;
//   kCG = 2, kBN = 256  a cluster of two CTAs computes a 256 x 256 tile with one
//            tcgen05.mma.cta_group::2 (M=256 N=256) issued by the pair's
//            leader: each CTA stages its own 128 rows of A and 128 rows of B
//            (32 KiB a stage, 6 stages) and holds its own 128 x 256
//            accumulator rows in TMEM, so each SM moves half the operand bytes
//            per FLOP of the 1-CTA shape (64 B per clock at the MMA rate);
//   kCG = 2, kBN = 512  the pair computes a 256 x 512 tile as two M=256 N=256
//            MMAs per K step that share the A operand: each CTA stages 128
//            rows of A and 2 x 128 rows of B (48 KiB a stage, 4 stages), 48 B
//            per clock at the MMA rate.  The accumulator fills all 512 TMEM
//            columns; the epilogue drains it as two 256-column banks, and the
//            next tile's MMAs start on bank 0 (for up to kStages - 1 K-blocks,
//            whose stages stay held) while bank 1 is still being drained.
// TMEM is treated as two banks of 256 columns.  A 256-column tile uses one
// bank (tiles alternate, so the epilogue of one overlaps the MMAs of the next);
// a 512-column tile uses both.  K-block 64 (one 128-byte swizzle row of bf16).
//
// Operands may be K-major (row-major [rows, K], the usual "TN" GEMM) or
// MN-major (row-major [K, rows]); both are staged with 128-byte swizzle and
// described to the tensor core by UMMA shared-memory descriptors.
//
// The three epilogues implement the steps of the fused linear cross-entropy:
//   FwdStatsEpi  softcap, per-row online max / sum of exp over the tile's 256
//                vocab columns, label-logit capture (forward)
//   DzEpi        softcap, dZ/g = (exp(L-lse) - onehot)*softcap' -> bf16 block
//                of dZ in global memory via TMA store (backward)
//   StoreEpi     g * fp32 tile -> TMA store or TMA reduce-add (dHidden, dWeight)
// The GEMM itself is the LM-head projection logits = hidden . weight^T
// (NeMo AutoModel linear_ce API: lm_weight is [vocab, hidden]) and, in the
// backward, dZ . weight and dZ^T . hidden.
#pragma once

#include <cuda_bf16.h>
#include <type_traits>
#include <math_constants.h>

#include "ptx.cuh"

namespace flce {

constexpr int BM = 128;  // accumulator rows held by one CTA
constexpr int BN = 256;  // accumulator columns
constexpr int BK = 64;
constexpr int kABytes = BM * BK * 2;  // 16 KB
constexpr int kStagingBuf = 4096;                 // 32 rows x 128 bytes
constexpr uint32_t kTmemCols = 512;

template <int kCG, int kBN = 256>
struct TileCfg {
  static_assert(kBN == 256 || (kBN == 512 && kCG == 2), "512-column tiles need CTA pairs");
  static constexpr int kBanks = kBN / BN;          // 256-column TMEM banks of one tile
  static constexpr int kBankRows = BN / kCG;       // B rows of one bank staged by one CTA
  static constexpr int kBankBytes = kBankRows * BK * 2;
  static constexpr int kBRows = kBanks * kBankRows;  // B rows (N index) staged by one CTA
  static constexpr int kBBytes = kBRows * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (kCG == 1 || kBN == 512) ? 4 : 6;
  static constexpr int kUnitRows = BM * kCG;  // output rows of one tile
  static constexpr size_t kRingBytes = 1024 + static_cast<size_t>(kStages) * kStageBytes;
};

// Threads and dynamic shared memory of a GEMM CTA with epilogue Epi (its
// warps and per-warp staging bytes are traits of the epilogue).
template <class Epi>
constexpr int gemm_threads() {
  return 64 + 32 * Epi::kEpiWarps;
}
template <class Epi, int kCG, int kBN>
constexpr size_t gemm_smem_bytes() {
  return TileCfg<kCG, kBN>::kRingBytes +
         static_cast<size_t>(Epi::kEpiWarps) * Epi::kStagingPerWarp;
}

constexpr int kRing = 8;  // tile indices in flight between the fetcher and the other roles

constexpr uint32_t kStatusLabelRange = 1u;
constexpr uint32_t kStatusTimeout = 2u;

constexpr float kLog2e = 1.4426950408889634f;

// tanh from one SFU exp2 and one fast division, by the identity
// tanh(x) = sign(x) * (1 - e^{-2|x|}) / (1 + e^{-2|x|}).  e^{-2|x|} lies in
// (0, 1] with relative (so also absolute) error about 2^-22, and the division
// by a value in [1, 2] adds about as much: the absolute error of the result
// stays near 2^-21 for every x, which the softcap s scales to s * 2^-21 in the
// capped logit (1.4e-5 at s = 30).
__device__ __forceinline__ float tanh_exp2(float x) {
  const float e = ex2_approx(-2.0f * kLog2e * fabsf(x));
  return copysignf(__fdividef(1.0f - e, 1.0f + e), x);
}
constexpr float kLn2 = 0.6931471805599453f;

struct GemmArgs {
  int m_tiles;    // tiles of kUnitRows output rows
  int n_tiles;    // tiles of kBN output columns
  int k_blocks;
  int group_m;    // tiles are walked in groups of group_m row-tiles (L2 reuse)
  int a_off;      // added to A's outer (row) TMA coordinate
  int b_off;      // added to B's outer (row) TMA coordinate
  unsigned int* status;
  unsigned long long timeout_ns;
  int* tile_counter;  // zeroed device counter: tiles are handed out dynamically;
                      // nullptr: static round-robin over the CTAs (or CTA pairs)
  int dep_wait;       // what waits for the previous kernel on the stream (launched
                      // as a programmatic dependent): kDepNone, kDepBeforeLoads
                      // (operands it produced), kDepBeforeStores (an output it reads),
                      // kDepBeforeExit (only completion order: the grid does not
                      // complete before the previous one)
  // Before its first store the epilogue waits (bounded) until *wait_counter
  // reaches wait_target: the CTAs of an earlier launch that read what this
  // launch overwrites count themselves out there.  Null: no wait.
  const int* wait_counter;
  int wait_target;
  int* done_counter;  // every CTA adds 1 here when it has finished (null: none)
  // Token rows bounded on the device: when rows_valid is set, only the first
  // clamp(*rows_valid - rows_base, 0, rows_host) token rows of this launch are
  // worked on.  rows_dim says which GEMM dimension they are (kRowsM, kRowsK);
  // with kRowsK an empty range drops the tiles, or (zero_if_empty) makes them
  // write zeros.
  const long long* rows_valid;
  int rows_base;
  int rows_host;
  int rows_dim;
  int zero_if_empty;
  // An MN-major operand whose map is the 3-D chunk view (x = 64 elements of a
  // 64-wide MN chunk, y = K row, z = chunk; one 16 KiB box = two chunks of 64 K
  // rows) instead of the 2-D view (one 8 KiB box per chunk).  Fewer, larger
  // TMA requests: 76.7 vs 68.9 B/clk per SM measured into shared memory.
  int a_mn3d, b_mn3d;
};

constexpr int kRowsNone = 0;
constexpr int kRowsM = 1;
constexpr int kRowsK = 2;

constexpr int kDepNone = 0;
constexpr int kDepBeforeLoads = 1;
constexpr int kDepBeforeStores = 2;
constexpr int kDepBeforeExit = 3;

__device__ __forceinline__ void tile_coords(int tile, const GemmArgs& g, int& mb, int& nb) {
  const int per_group = g.group_m * g.n_tiles;
  const int grp = tile / per_group;
  const int first_m = grp * g.group_m;
  const int gm = min(g.group_m, g.m_tiles - first_m);
  const int r = tile - grp * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

// Hand the accumulator back to the MMA issuer: `tempty_bar` is the
// shared::cluster address of the (leader CTA's) accumulator-empty barrier.
__device__ __forceinline__ void release_tmem(uint32_t tempty_bar, int lane) {
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive_cluster(tempty_bar);
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

// The same row from two halves: words 0-15 of `lo`, then words 0-15 of `hi`.
__device__ __forceinline__ void stage_row_128b(uint8_t* buf, int lane, const uint32_t (&lo)[32],
                                               const uint32_t (&hi)[32]) {
  uint8_t* row = buf + lane * 128;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t(&w)[32] = j < 4 ? lo : hi;
    const int b = 4 * (j & 3);
    uint4 v = make_uint4(w[b + 0], w[b + 1], w[b + 2], w[b + 3]);
    *reinterpret_cast<uint4*>(row + ((j ^ (lane & 7)) << 4)) = v;
  }
}

// ------------------------------------------------------------------ forward
// Per tile: L = softcap(Z) over 256 vocab columns; per row the maximum m and
// s = sum exp(L - m) (both in the log2 domain), written to partials
// [n_tile][N]; the label logit L[i, y_i] is written by the tile holding y_i.
// Eight epilogue warps: the two warps of a TMEM lane quadrant each reduce 128
// of the bank's columns, and the second hands its (m, s) to the first through
// shared memory (two slots used in turn, each with a full and an empty
// mbarrier; bounded waits), which merges and writes them.
template <bool kSoftcap>
struct FwdStatsEpi {
  static constexpr int kEpiWarps = 8;
  // first warp of a quadrant: its mbarriers full[2], empty[2]; second warp:
  // the two (m[32], s[32]) slots
  static constexpr int kStagingPerWarp = 2 * 64 * 4;
  __device__ static void init_smem(uint8_t* staging) {
    for (int w = 0; w < 4; ++w) {
      uint64_t* b = reinterpret_cast<uint64_t*>(staging + w * kStagingPerWarp);
      for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&b[i]), 1);
    }
  }
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

  // The row's label, read before the accumulator is ready.
  struct Pre {
    int64_t y;
  };
  __device__ static Pre prepare(const Params& p, int m_base, int q, int lane) {
    const int row = m_base + q * 32 + lane;
    return Pre{row < p.N ? p.labels[row] : int64_t{-1}};
  }

  __device__ static bool tile(const Params& p, const Pre& pre, int m_base, int col0,
                              uint32_t taddr, int q, int lane, int part, uint8_t* stg,
                              const CUtensorMap*, uint32_t tempty, int& nbank, bool,
                              const volatile int* abort, unsigned long long timeout_ns) {
    if (col0 >= p.V) {  // the second bank of a 512-column tile past the vocabulary
      release_tmem(tempty, lane);
      return true;
    }
    const int slot = nbank & 1;
    const uint32_t use = static_cast<uint32_t>(nbank >> 1);  // earlier uses of this slot
    ++nbank;
    const int row = m_base + q * 32 + lane;
    const bool row_ok = row < p.N;
    const int h0 = col0 + part * (BN / 2);  // this warp's first column
    int y_local = -1;
    if (row_ok && pre.y >= h0 && pre.y < static_cast<int64_t>(h0) + BN / 2)
      y_local = static_cast<int>(pre.y - h0);
    const int ncols = max(0, min(BN / 2, p.V - h0));
    // warp-uniform: does any row's label fall in these columns?
    const bool any_label = __any_sync(0xffffffffu, y_local >= 0);
    float m = -CUDART_INF_F;  // log2 domain
    float s = 0.f;
    float ly = 0.f;
    const uint32_t ta = taddr + part * (BN / 2);
    if constexpr (!kSoftcap) {
      // all 128 columns into registers, the TMEM half released at once (the
      // next tile's MMAs wait for it), then one max and one sum over them
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_x32(ta + c * 32, r[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(r[c]);
      release_tmem(tempty, lane);
      if (any_label) {
#pragma unroll
        for (int j = 0; j < 128; ++j)
          if (j == y_local) ly = __uint_as_float(r[j / 32][j % 32]);
      }
      if (ncols < BN / 2) {  // the vocabulary ends inside (or before) these columns
#pragma unroll
        for (int j = 0; j < 128; ++j)
          if (j >= ncols) r[j / 32][j % 32] = __float_as_uint(-CUDART_INF_F);
      }
      float mx[32];
#pragma unroll
      for (int j = 0; j < 32; ++j)
        mx[j] = fmaxf(fmaxf(__uint_as_float(r[0][j]), __uint_as_float(r[1][j])),
                      fmaxf(__uint_as_float(r[2][j]), __uint_as_float(r[3][j])));
#pragma unroll
      for (int w = 16; w >= 1; w /= 2)
#pragma unroll
        for (int j = 0; j < w; ++j) mx[j] = fmaxf(mx[j], mx[j + w]);
      if (mx[0] != -CUDART_INF_F) {
        m = mx[0] * kLog2e;
        float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 128; ++j)
          a8[j & 7] += ex2_approx(fmaf(__uint_as_float(r[j / 32][j % 32]), kLog2e, -m));
        s = ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
      }
    } else {
      // softcapped: 32-column chunks with an online max, the next chunk's
      // TMEM load in flight; the tanh body is kept rolled to bound code size
      auto chunk = [&](int c, const uint32_t(&r)[32]) {
        float L[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
          L[j] = p.softcap * tanh_exp2(__uint_as_float(r[j]) * p.inv_softcap);
        if (any_label) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c * 32 + j == y_local) ly = L[j];
        }
        if (c * 32 + 32 > ncols) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c * 32 + j >= ncols) L[j] = -CUDART_INF_F;
        }
        float mx[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) mx[j] = fmaxf(L[j], L[j + 16]);
#pragma unroll
        for (int w = 8; w >= 1; w /= 2)
#pragma unroll
          for (int j = 0; j < w; ++j) mx[j] = fmaxf(mx[j], mx[j + w]);
        const float mn = fmaxf(m, mx[0] * kLog2e);
        if (mn == -CUDART_INF_F) return;  // nothing in range yet
        float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 32; ++j) a4[j & 3] += ex2_approx(fmaf(L[j], kLog2e, -mn));
        const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
        s = (m == -CUDART_INF_F) ? acc : fmaf(s, ex2_approx(m - mn), acc);
        m = mn;
      };
      constexpr int kChunks = BN / 2 / 32;
      uint32_t buf[2][32];
      tmem_ld_x32(ta, buf[0]);
      tmem_ld_wait(buf[0]);
#pragma unroll 1
      for (int c = 0; c < kChunks; c += 2) {
        tmem_ld_x32(ta + (c + 1) * 32, buf[1]);
        chunk(c, buf[0]);
        tmem_ld_wait(buf[1]);
        if (c + 2 < kChunks)
          tmem_ld_x32(ta + (c + 2) * 32, buf[0]);
        else
          release_tmem(tempty, lane);  // every column of this half is in registers
        chunk(c + 1, buf[1]);
        if (c + 2 < kChunks) tmem_ld_wait(buf[0]);
      }
    }
    if (row_ok && y_local >= 0) p.label_logit[row] = ly;
    // the quadrant's second warp hands (m, s) to the first
    uint64_t* bars = reinterpret_cast<uint64_t*>(part == 0 ? stg : stg - 4 * kStagingPerWarp);
    float* x = reinterpret_cast<float*>(part == 1 ? stg : stg + 4 * kStagingPerWarp) + slot * 64;
    const uint32_t full = smem_u32(&bars[slot]), empty = smem_u32(&bars[2 + slot]);
    if (part == 1) {
      if (use > 0 && !__all_sync(0xffffffffu, mbar_wait(empty, (use - 1) & 1u, abort, timeout_ns)))
        return false;
      x[lane] = m;
      x[32 + lane] = s;
      __syncwarp();
      if (lane == 0) mbar_arrive(full);
      return true;
    }
    if (!__all_sync(0xffffffffu, mbar_wait(full, use & 1u, abort, timeout_ns))) return false;
    const float m1 = x[lane], s1 = x[32 + lane];
    __syncwarp();
    if (lane == 0) mbar_arrive(empty);
    if (row_ok) {
      if (m1 != -CUDART_INF_F) {  // the second half has columns in range
        const float mm = fmaxf(m, m1);
        s = s * ex2_approx(m - mm) + s1 * ex2_approx(m1 - mm);
        m = mm;
      }
      const size_t idx = static_cast<size_t>(col0 / BN) * p.N + row;
      p.part_m[idx] = m;
      p.part_s[idx] = s;
    }
    return true;
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
// With `resid` set, the label entry's rounding residual d - bf16(d) (exact in
// fp32) is recorded per row, for the fp32 corrections that make the label
// term of dHidden and dWeight exact.
template <bool kSoftcap>
struct DzEpi {
  // Eight warps: the two warps of a TMEM lane quadrant each take 128 of a
  // bank's columns.  One 4 KiB staging buffer per warp (32 rows x 64 bf16).
  static constexpr int kEpiWarps = 8;
  static constexpr int kStagingPerWarp = kStagingBuf;
  __device__ static void init_smem(uint8_t*) {}
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
    float* resid;      // [token rows] or null
    int64_t v_total;   // V: a label outside [0, V) counts as ignored
  };

  // The row's label and lse, read before the accumulator is ready.
  struct Pre {
    int64_t y;
    float lse;
  };
  __device__ static Pre prepare(const Params& p, int m_base, int q, int lane) {
    const int row_l = m_base + q * 32 + lane;
    if (row_l >= p.rows) return Pre{0, 0.f};
    return Pre{p.labels[p.t0 + row_l], p.lse[p.t0 + row_l]};
  }

  __device__ static bool tile(const Params& p, const Pre& pre, int m_base, int col0,
                              uint32_t taddr, int q, int lane, int part, uint8_t* stg,
                              const CUtensorMap* out, uint32_t tempty, int& nstore, bool,
                              const volatile int*, unsigned long long) {
    // this warp's columns: [h0, h0 + 128) of the block; 64-column stores whose
    // box starts inside the block (warp-uniform)
    const int h0 = col0 + part * (BN / 2);
    const int y0 = m_base + q * 32;
    const int rem = p.cols - h0;
    const int nch = (y0 >= p.rows || rem <= 0) ? 0 : min(BN / 2 / 64, (rem + 63) / 64);
    if (nch == 0) {
      release_tmem(tempty, lane);
      return true;
    }
    const int row_l = y0 + lane;
    bool valid = false;
    int y_local = -1;
    float lse2 = 0.f;
    if (row_l < p.rows) {
      const int64_t y = pre.y;
      valid = (y != p.ignore_index) && y >= 0 && y < p.v_total;
      const int64_t c0 = static_cast<int64_t>(p.v0) + h0;
      if (valid && y >= c0 && y < c0 + BN / 2) y_local = static_cast<int>(y - c0);
      lse2 = pre.lse * kLog2e;
    }
    const uint32_t stg_u32 = smem_u32(stg);
    // warp-uniform: does any row's label fall in these columns?
    const bool any_label = __any_sync(0xffffffffu, y_local >= 0);
    // dZ/g of 32 columns (local columns c0l..c0l+31 of this warp), packed as
    // 16 bf16 pairs into r[0..15] (in place: no second register array)
    auto dz32 = [&](int c0l, uint32_t(&r)[32]) {
      // d overwrites the logit it comes from
      if constexpr (kSoftcap) {
        float f[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float L = p.softcap * tanh_exp2(__uint_as_float(r[j]) * p.inv_softcap);
          const float u = L * p.inv_softcap;
          f[j] = fmaf(-u, u, 1.0f);
          r[j] = __float_as_uint(ex2_approx(fmaf(L, kLog2e, -lse2)));
        }
        if (any_label) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0l + j == y_local) r[j] = __float_as_uint(__uint_as_float(r[j]) - 1.0f);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * f[j]);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          r[j] = __float_as_uint(ex2_approx(fmaf(__uint_as_float(r[j]), kLog2e, -lse2)));
        if (any_label) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0l + j == y_local) r[j] = __float_as_uint(__uint_as_float(r[j]) - 1.0f);
        }
      }
      if (any_label && p.resid != nullptr) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0l + j == y_local) {
            const float d = __uint_as_float(r[j]);
            p.resid[p.t0 + row_l] = d - __bfloat162float(__float2bfloat16_rn(d));
          }
      }
      // pairs (2j, 2j+1) -> word j; word j is written after words 2j, 2j+1
      // (>= j) are read
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(valid ? __uint_as_float(r[2 * j]) : 0.0f,
                                                  valid ? __uint_as_float(r[2 * j + 1]) : 0.0f);
        r[j] = *reinterpret_cast<uint32_t*>(&b2);
      }
    };
    // 64 packed columns (local store index sidx) -> staging -> TMA store; the
    // buffer is reused once the previous store has read it
    auto store64 = [&](int sidx, const uint32_t(&lo)[32], const uint32_t(&hi)[32]) {
      if (lane == 0) bulk_wait_group_read<0>();
      __syncwarp();
      stage_row_128b(stg, lane, lo, hi);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(out, stg_u32, h0 + sidx * 64, y0);
        bulk_commit_group();
      }
      ++nstore;
    };
    if constexpr (!kSoftcap) {
      // all 128 columns into registers, the TMEM half released at once
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_x32(taddr + part * (BN / 2) + c * 32, r[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(r[c]);
      release_tmem(tempty, lane);
#pragma unroll
      for (int sidx = 0; sidx < 2; ++sidx) {
        if (sidx < nch) {
          dz32(sidx * 64, r[2 * sidx]);
          dz32(sidx * 64 + 32, r[2 * sidx + 1]);
          store64(sidx, r[2 * sidx], r[2 * sidx + 1]);
        }
      }
    } else {
      // softcapped: 32-column sub-chunks, the next one's TMEM load in flight;
      // the tanh body is kept rolled to bound code size
      const uint32_t ta = taddr + part * (BN / 2);
      uint32_t buf[2][32];
      tmem_ld_x32(ta, buf[0]);
      tmem_ld_wait(buf[0]);
#pragma unroll 1
      for (int sidx = 0; sidx < 2; ++sidx) {
        uint32_t lo[32];
        tmem_ld_x32(ta + (2 * sidx + 1) * 32, buf[1]);
        if (sidx < nch) {
          dz32(sidx * 64, buf[0]);
#pragma unroll
          for (int j = 0; j < 16; ++j) lo[j] = buf[0][j];
        }
        tmem_ld_wait(buf[1]);
        if (sidx == 0)
          tmem_ld_x32(ta + 64, buf[0]);
        else
          release_tmem(tempty, lane);  // every column of this half is in registers
        if (sidx < nch) {
          dz32(sidx * 64 + 32, buf[1]);
          store64(sidx, lo, buf[1]);
        }
        if (sidx == 0) tmem_ld_wait(buf[0]);
      }
    }
    return true;
  }
};

// ------------------------------------------------------------------ fp32 out
// Tile * g -> fp32 output rows [out_row0 + m]: TMA store, or TMA reduce-add
// when `reduce` (accumulation across chunks of the split reduction dimension).
// g = grad_output * grad_scale, divided by max(n, 1) for 'mean'.
struct StoreEpi {
  // Eight warps: the two warps of a TMEM lane quadrant each take 128 of a
  // bank's columns.  One 4 KiB staging buffer per warp (32 rows x 32 fp32).
  static constexpr int kEpiWarps = 8;
  static constexpr int kStagingPerWarp = kStagingBuf;
  __device__ static void init_smem(uint8_t*) {}
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

  // The scale g, read before the accumulator is ready.
  struct Pre {
    float g;
  };
  __device__ static Pre prepare(const Params& p, int, int, int) { return Pre{grad_factor(p)}; }

  __device__ static bool tile(const Params& p, const Pre& pre, int m_base, int col0,
                              uint32_t taddr, int q, int lane, int part, uint8_t* stg,
                              const CUtensorMap* out, uint32_t tempty, int& nstore,
                              bool empty, const volatile int*, unsigned long long) {
    // this warp's columns: [h0, h0 + 128); 32-column stores whose box starts
    // inside the output (warp-uniform)
    const int h0 = col0 + part * (BN / 2);
    const int y = p.out_row0 + m_base + q * 32;
    const int rem = p.x_limit - h0;
    const int nch = (y >= p.y_limit || rem <= 0) ? 0 : min(BN / 2 / 32, (rem + 31) / 32);
    if (nch == 0) {
      release_tmem(tempty, lane);
      return true;
    }
    // An empty K range contributes zeros: the accumulator was never written, so
    // its stale contents are not read (0 * stale could be NaN).
    const float g = empty ? 0.0f : pre.g;
    const uint32_t stg_u32 = smem_u32(stg);
    // all 128 columns into registers, the TMEM half released at once
    uint32_t r[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld_x32(taddr + part * (BN / 2) + c * 32, r[c]);
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < 4; ++c) reg_fence(r[c]);
    release_tmem(tempty, lane);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (c < nch) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          r[c][j] = empty ? 0u : __float_as_uint(__uint_as_float(r[c][j]) * g);
        // the buffer is reused once the previous store has read it
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
        stage_row_128b(stg, lane, r[c]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int x = h0 + c * 32;
          if (p.reduce)
            tma_reduce_add_2d(out, stg_u32, x, y);
          else
            tma_store_2d(out, stg_u32, x, y);
          bulk_commit_group();
        }
        ++nstore;
      }
    }
    return true;
  }
};

// ------------------------------------------------------------------ kernel
__device__ __forceinline__ void record_timeout(const GemmArgs& g, volatile int* abort) {
  *abort = 1;
  if (g.status != nullptr) atomicOr(g.status, kStatusTimeout);
}

template <int kCG>
__device__ __forceinline__ void load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                        int32_t x, int32_t y) {
  if constexpr (kCG == 1)
    tma_load_2d(dst, map, bar, x, y);
  else
    tma_load_2d_pair(dst, map, bar, x, y);
}

// An MN-major operand tile of `rows` MN elements x BK K rows starting at MN
// coordinate mn (a multiple of 128) and K row k: 64-element chunks 8 KiB apart.
template <int kCG>
__device__ __forceinline__ void load_mn(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                        int rows, int mn, int k, bool view3d) {
  if (view3d) {
    for (int c = 0; c < rows / 128; ++c) {
      if constexpr (kCG == 1)
        tma_load_3d(dst + c * 16384, map, bar, 0, k, mn / 64 + 2 * c);
      else
        tma_load_3d_pair(dst + c * 16384, map, bar, 0, k, mn / 64 + 2 * c);
    }
  } else {
    for (int c = 0; c < rows / 64; ++c) load_2d<kCG>(dst + c * 8192, map, bar, mn + c * 64, k);
  }
}

// One launch runs the tiles of one GEMM, or of two independent GEMMs that
// share the epilogue type (problem 0's tiles first, then problem 1's, so the
// last wave of one is filled by the other).  Operand majors are per problem.
template <class Epi, int kCG, int kBN, bool kAMn0, bool kBMn0, bool kAMn1 = false,
          bool kBMn1 = false>
__global__ void __launch_bounds__(gemm_threads<Epi>(), 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmOut0, const __grid_constant__ CUtensorMap tmA1,
                   const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmOut1,
                   const GemmArgs g0, const GemmArgs g1, const typename Epi::Params ep0,
                   const typename Epi::Params ep1) {
  using Cfg = TileCfg<kCG, kBN>;
  static_assert(Epi::kEpiWarps == 8, "two epilogue warps per TMEM lane quadrant, half a bank each");
  constexpr int kStages = Cfg::kStages;
  constexpr int kBanks = Cfg::kBanks;
  // K-blocks of a 512-column tile issued on bank 0 alone while bank 1 still
  // holds the previous tile (their stages stay held until bank 1 catches up)
  constexpr int kStagger = kStages - 1;
  extern __shared__ uint8_t smem_dyn[];
  __shared__ __align__(8) uint64_t bar_full[kStages];
  __shared__ __align__(8) uint64_t bar_empty[kStages];
  __shared__ __align__(8) uint64_t bar_tfull[2];
  __shared__ __align__(8) uint64_t bar_tempty[2];
  __shared__ __align__(8) uint64_t bar_drain;
  __shared__ __align__(8) uint64_t ring_full[kRing];
  __shared__ __align__(8) uint64_t ring_empty[kRing];
  __shared__ int tile_ring[kRing];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  // 1024-byte alignment of the operand ring (required by the 128-byte swizzle).
  const uint32_t pad = (1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u;
  uint8_t* smem = smem_dyn + pad;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = (kCG == 1) ? 0u : cluster_ctarank();
  const bool leader = (rank == 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&bar_tfull[a]), 1);
      mbar_init(smem_u32(&bar_tempty[a]), Epi::kEpiWarps * kCG);
    }
    mbar_init(smem_u32(&bar_drain), 1);
    // each tile index is read by: the MMA issuer and the epilogue warps of
    // the leader, and the producer and the epilogue warps of the peer
    for (int r = 0; r < kRing; ++r) {
      mbar_init(smem_u32(&ring_full[r]), 1);
      mbar_init(smem_u32(&ring_empty[r]), (1 + Epi::kEpiWarps) * kCG);
    }
    abort_sh = 0;
    Epi::init_smem(smem + kStages * Cfg::kStageBytes);
    fence_mbar_init();
    prefetch_tmap(&tmA0);
    prefetch_tmap(&tmB0);
    prefetch_tmap(&tmOut0);
    if (g1.m_tiles > 0) {
      prefetch_tmap(&tmA1);
      prefetch_tmap(&tmB1);
      prefetch_tmap(&tmOut1);
    }
  }
  if (warp == 1) {
    if constexpr (kCG == 1) {
      tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
      tmem_relinquish();
    } else {
      tmem_alloc_pair(smem_u32(&tmem_base_sh), kTmemCols);
      tmem_relinquish_pair();
    }
  }
  tc_fence_before();
  if constexpr (kCG == 1)
    __syncthreads();
  else
    cluster_sync();  // the leader's barriers are initialised before the peer uses them
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  // The next kernel on the stream may be scheduled as SMs free up; it waits
  // for this one wherever it depends on it.
  griddep_launch_dependents();
  // Token-row bounds known only on the device (the same in every thread).
  auto bound_rows = [](GemmArgs g) {
    if (g.rows_valid != nullptr && g.rows_dim != kRowsNone) {
      long long eff = *g.rows_valid - g.rows_base;
      eff = eff < 0 ? 0 : (eff > g.rows_host ? g.rows_host : eff);
      if (g.rows_dim == kRowsM) {
        g.m_tiles = static_cast<int>((eff + Cfg::kUnitRows - 1) / Cfg::kUnitRows);
      } else {
        g.k_blocks = static_cast<int>((eff + BK - 1) / BK);
        if (g.k_blocks == 0 && !g.zero_if_empty) g.m_tiles = 0;
      }
    }
    return g;
  };
  const GemmArgs a0 = bound_rows(g0);
  const GemmArgs a1 = bound_rows(g1);
  const int tiles0 = a0.m_tiles * a0.n_tiles;
  const int num_tiles = tiles0 + a1.m_tiles * a1.n_tiles;
  const int unit = blockIdx.x / kCG;  // CTA (kCG = 1) or CTA pair (kCG = 2)
  const int n_units = gridDim.x / kCG;
  volatile int* abort_flag = &abort_sh;

  // problem, its args and the tile's coordinates for global tile index t
  auto locate = [&](int t, int& prob, int& mb, int& nb) {
    prob = (t < tiles0) ? 0 : 1;
    tile_coords(prob ? t - tiles0 : t, prob ? a1 : a0, mb, nb);
  };

  // ---- tile hand-out.  The leader's producer thread picks each next tile
  // (an atomic on g0.tile_counter, or unit + k * n_units without one) and
  // publishes it in a ring slot of both CTAs; every other role reads the
  // same sequence from its own CTA's ring.  A value >= num_tiles ends it.
  auto ring_publish = [&](int slot, uint32_t rph, int t) -> bool {
    // the peer's consumers release the slot remotely: acquire at cluster scope
    const bool free = (kCG == 2)
        ? mbar_wait_cluster(smem_u32(&ring_empty[slot]), rph ^ 1u, abort_flag, g0.timeout_ns)
        : mbar_wait(smem_u32(&ring_empty[slot]), rph ^ 1u, abort_flag, g0.timeout_ns);
    if (!free) return false;
    tile_ring[slot] = t;
    if constexpr (kCG == 2) {
      const uint32_t peer_slot = mapa_shared(smem_u32(&tile_ring[slot]), 1);
      st_shared_cluster_u32(peer_slot, static_cast<uint32_t>(t));
      mbar_arrive_cluster(mapa_shared(smem_u32(&ring_full[slot]), 1));
    }
    mbar_arrive(smem_u32(&ring_full[slot]));
    return true;
  };
  // Read the next tile index (all lanes of the calling warp, or one thread).
  auto ring_take = [&](int slot, uint32_t rph, bool warp_wide, int& t) -> bool {
    // the peer's copy is written remotely: acquire at cluster scope
    bool w = (kCG == 2) ? mbar_wait_cluster(smem_u32(&ring_full[slot]), rph, abort_flag,
                                            g0.timeout_ns)
                        : mbar_wait(smem_u32(&ring_full[slot]), rph, abort_flag, g0.timeout_ns);
    if (warp_wide) w = __all_sync(0xffffffffu, w);
    if (!w) return false;
    t = *reinterpret_cast<volatile int*>(&tile_ring[slot]);
    if (warp_wide) __syncwarp();
    if (!warp_wide || lane == 0) {
      const uint32_t e = smem_u32(&ring_empty[slot]);
      if (kCG == 1 || leader)
        mbar_arrive(e);
      else
        mbar_arrive_cluster(mapa_shared(e, 0));  // the leader's slot
    }
    return true;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (every CTA loads its own halves)
      if (g0.dep_wait == kDepBeforeLoads) griddep_wait();
      uint32_t stage = 0, phase = 0;
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      int rslot = 0;
      uint32_t rph = 0;
      for (int k = 0; ok; ++k) {
        int tile;
        if (leader) {
          tile = (g0.tile_counter != nullptr) ? atomicAdd(g0.tile_counter, 1) : unit + k * n_units;
          if (tile > num_tiles) tile = num_tiles;
          ok = ring_publish(rslot, rph, tile);
        } else {
          ok = ring_take(rslot, rph, false, tile);
        }
        if (++rslot == kRing) {
          rslot = 0;
          rph ^= 1u;
        }
        if (!ok || tile >= num_tiles) break;
        int prob, mb, nb;
        locate(tile, prob, mb, nb);
        const GemmArgs& g = prob ? a1 : a0;
        const CUtensorMap* mA = prob ? &tmA1 : &tmA0;
        const CUtensorMap* mB = prob ? &tmB1 : &tmB0;
        const bool a_mn = prob ? kAMn1 : kAMn0;
        const bool b_mn = prob ? kBMn1 : kBMn0;
        const int m_cta = mb * Cfg::kUnitRows + static_cast<int>(rank) * BM;
        // bank h of the tile: B rows nb * kBN + h * BN + [rank * kBankRows, + kBankRows)
        const int n_cta = nb * kBN + static_cast<int>(rank) * Cfg::kBankRows;
        for (int kb = 0; kb < g.k_blocks; ++kb) {
          if (!mbar_wait(smem_u32(&bar_empty[stage]), phase ^ 1u, abort_flag, g0.timeout_ns)) {
            ok = false;
            break;
          }
          const uint32_t fb_local = smem_u32(&bar_full[stage]);
          uint32_t fb = fb_local;
          if constexpr (kCG == 1) {
            mbar_arrive_expect_tx(fb_local, Cfg::kStageBytes);
          } else {
            // the leader's barrier counts both CTAs' bytes
            if (leader) mbar_arrive_expect_tx(fb_local, 2 * Cfg::kStageBytes);
            fb = fb_local & kPairPeerBitMask;
          }
          const uint32_t sa = smem_u32(smem + stage * Cfg::kStageBytes);
          const uint32_t sb = sa + kABytes;
          if (a_mn) {
            load_mn<kCG>(sa, mA, fb, BM, m_cta, g.a_off + kb * BK, g.a_mn3d != 0);
          } else {
            load_2d<kCG>(sa, mA, fb, kb * BK, g.a_off + m_cta);
          }
#pragma unroll
          for (int h = 0; h < kBanks; ++h) {
            const uint32_t sbh = sb + h * Cfg::kBankBytes;
            if (b_mn) {
              load_mn<kCG>(sbh, mB, fb, Cfg::kBankRows, n_cta + h * BN, g.b_off + kb * BK,
                           g.b_mn3d != 0);
            } else {
              load_2d<kCG>(sbh, mB, fb, kb * BK, g.b_off + n_cta + h * BN);
            }
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
        record_timeout(g0, abort_flag);
        // Let every load already issued land before the CTA can exit (the
        // leader's full barriers also count the peer's bytes).
        if (kCG == 1 || leader)
          for (int s = 0; s < kStages; ++s)
            if ((issued_mask >> s) & 1u)
              mbar_wait(smem_u32(&bar_full[s]), (issued_par >> s) & 1u, nullptr, g0.timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (the pair's leader issues for both CTAs)
      const uint32_t idesc0 = umma_idesc_bf16(BM * kCG, BN, kAMn0, kBMn0);
      const uint32_t idesc1 = umma_idesc_bf16(BM * kCG, BN, kAMn1, kBMn1);
      uint32_t stage = 0, phase = 0;
      int it = 0;
      bool ok = true;
      bool issued = false;
      int rslot = 0;
      uint32_t rph = 0;
      // The 4 K=16 MMAs of one K-block of stage `st` with B part `part` of the
      // stage (the tile's bank `part`) into TMEM bank `bank`; `first`: the
      // K-block starts the accumulation.
      auto mma_kblock = [&](uint32_t st, int part, uint32_t bank, bool first, uint32_t idesc,
                            bool a_mn, bool b_mn) {
        const uint32_t sa = smem_u32(smem + st * Cfg::kStageBytes);
        const uint32_t sb = sa + kABytes + part * Cfg::kBankBytes;
        const uint32_t d_tmem = tmem_base + bank * BN;
#pragma unroll
        for (int j = 0; j < BK / 16; ++j) {
          const uint64_t ad = a_mn ? umma_desc_sw128(sa + j * 2048, 8192, 1024)
                                   : umma_desc_sw128(sa + j * 32, 16, 1024);
          const uint64_t bd = b_mn ? umma_desc_sw128(sb + j * 2048, 8192, 1024)
                                   : umma_desc_sw128(sb + j * 32, 16, 1024);
          const uint32_t accum = (!first || j > 0) ? 1u : 0u;
          if constexpr (kCG == 1)
            tc_mma_bf16(d_tmem, ad, bd, idesc, accum);
          else
            tc_mma_bf16_pair(d_tmem, ad, bd, idesc, accum);
        }
      };
      auto commit_to = [&](uint64_t* bar) {
        if constexpr (kCG == 1)
          tc_commit(smem_u32(bar));
        else
          tc_commit_pair_mc(smem_u32(bar), 0x3);
      };
      auto next_stage = [&]() {
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      };
      for (;; ++it) {
        int tile;
        ok = ring_take(rslot, rph, false, tile);
        if (++rslot == kRing) {
          rslot = 0;
          rph ^= 1u;
        }
        if (!ok || tile >= num_tiles) break;
        const int prob = (tile < tiles0) ? 0 : 1;
        const int k_blocks = prob ? a1.k_blocks : a0.k_blocks;
        const uint32_t idesc = prob ? idesc1 : idesc0;
        const bool a_mn = prob ? kAMn1 : kAMn0;
        const bool b_mn = prob ? kBMn1 : kBMn0;
        if constexpr (kBanks == 1) {
          // tiles alternate between the two banks
          const uint32_t acc = it & 1;
          const uint32_t aph = (it >> 1) & 1;
          if (!mbar_wait(smem_u32(&bar_tempty[acc]), aph ^ 1u, abort_flag, g0.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int kb = 0; kb < k_blocks; ++kb) {
            if (!mbar_wait(smem_u32(&bar_full[stage]), phase, abort_flag, g0.timeout_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            mma_kblock(stage, 0, acc, kb == 0, idesc, a_mn, b_mn);
            issued = true;
            commit_to(&bar_empty[stage]);
            next_stage();
          }
          if (!ok) break;
          commit_to(&bar_tfull[acc]);
        } else {
          // one tile spans both banks.  Bank 0 starts as soon as the epilogue
          // has drained it: its first d K-blocks run while bank 1 is still
          // drained, their stages held; then bank 1 catches up on those stages
          // and the rest of the K-blocks feed both banks.
          const uint32_t aph = it & 1;
          const int d = min(kStagger, k_blocks);
          if (!mbar_wait(smem_u32(&bar_tempty[0]), aph ^ 1u, abort_flag, g0.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st0 = stage;
          for (int kb = 0; kb < d; ++kb) {
            if (!mbar_wait(smem_u32(&bar_full[stage]), phase, abort_flag, g0.timeout_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            mma_kblock(stage, 0, 0, kb == 0, idesc, a_mn, b_mn);
            issued = true;
            next_stage();
          }
          if (!ok) break;
          if (!mbar_wait(smem_u32(&bar_tempty[1]), aph ^ 1u, abort_flag, g0.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t s1 = st0;
          for (int kb = 0; kb < d; ++kb) {
            mma_kblock(s1, 1, 1, kb == 0, idesc, a_mn, b_mn);
            commit_to(&bar_empty[s1]);
            s1 = (s1 + 1 == kStages) ? 0u : s1 + 1;
          }
          for (int kb = d; kb < k_blocks; ++kb) {
            if (!mbar_wait(smem_u32(&bar_full[stage]), phase, abort_flag, g0.timeout_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            mma_kblock(stage, 0, 0, false, idesc, a_mn, b_mn);
            mma_kblock(stage, 1, 1, false, idesc, a_mn, b_mn);
            issued = true;
            commit_to(&bar_empty[stage]);
            next_stage();
          }
          if (!ok) break;
          commit_to(&bar_tfull[0]);
        }
      }
      if (!ok) {
        record_timeout(g0, abort_flag);
        if (issued) {
          // Wait for the MMAs in flight before TMEM is released.
          if constexpr (kCG == 1)
            tc_commit(smem_u32(&bar_drain));
          else
            tc_commit_pair(smem_u32(&bar_drain));
          mbar_wait(smem_u32(&bar_drain), 0, nullptr, g0.timeout_ns);
        }
      }
    }
  } else {
    // ---------------- epilogue warps (they may read what the previous kernel
    // wrote, so they wait for it in either of the first two modes)
    if (g0.dep_wait == kDepBeforeLoads || g0.dep_wait == kDepBeforeStores) griddep_wait();
    const int q = warp & 3;             // TMEM lane quadrant this warp may access
    const int part = (warp - 2) >> 2;   // which half of a bank
    uint8_t* stg = smem + kStages * Cfg::kStageBytes + (warp - 2) * Epi::kStagingPerWarp;
    int it = 0;
    int nstore = 0;  // TMA stores issued by this warp (selects the staging buffer)
    bool ok = true;
    if (g0.wait_counter != nullptr) {
      // the launch that last read what this one overwrites has finished
      bool w = true;
      if (lane == 0) {
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu(g0.wait_counter) < g0.wait_target) {
          if (*abort_flag || globaltimer_ns() - t0 > g0.timeout_ns) {
            w = false;
            break;
          }
          __nanosleep(256);
        }
        fence_proxy_async_global();
      }
      ok = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
    }
    int rslot = 0;
    uint32_t rph = 0;
    for (; ok; ++it) {
      int tile;
      ok = ring_take(rslot, rph, true, tile);
      if (++rslot == kRing) {
        rslot = 0;
        rph ^= 1u;
      }
      if (!ok || tile >= num_tiles) break;
      int prob, mb, nb;
      locate(tile, prob, mb, nb);
      const int m_base = mb * Cfg::kUnitRows + static_cast<int>(rank) * BM;
      const GemmArgs& ga = prob ? a1 : a0;
      // per-row inputs of the epilogue, in flight while the MMAs finish
      const typename Epi::Pre pre = Epi::prepare(prob ? ep1 : ep0, m_base, q, lane);
      // the tile's first bank and the phase its full barrier completes
      const uint32_t acc = (kBanks == 1) ? (it & 1) : 0u;
      const uint32_t aph = (kBanks == 1) ? ((it >> 1) & 1) : (it & 1);
      bool w = mbar_wait(smem_u32(&bar_tfull[acc]), aph, abort_flag, g0.timeout_ns);
      w = __all_sync(0xffffffffu, w);
      if (!w) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < kBanks; ++h) {  // bank 0 first: the next tile starts on it
        const uint32_t bank = acc + h;
        const uint32_t taddr = tmem_base + bank * BN + (static_cast<uint32_t>(q * 32) << 16);
        const uint32_t tempty_local = smem_u32(&bar_tempty[bank]);
        const uint32_t tempty = (kCG == 1) ? tempty_local : mapa_shared(tempty_local, 0);
        if (!Epi::tile(prob ? ep1 : ep0, pre, m_base, nb * kBN + h * BN, taddr, q, lane, part,
                       stg, prob ? &tmOut1 : &tmOut0, tempty, nstore, ga.k_blocks == 0,
                       abort_flag, g0.timeout_ns)) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
    }
    if (lane == 0) {
      bulk_wait_group_all();
      if (!ok) record_timeout(g0, abort_flag);
    }
  }

  __syncthreads();
  if constexpr (kCG == 2) cluster_sync();  // neither CTA leaves while its peer may still use it
  if (warp == 1) {
    tc_fence_after();
    if constexpr (kCG == 1)
      tmem_dealloc(tmem_base, kTmemCols);
    else
      tmem_dealloc_pair(tmem_base, kTmemCols);
  }
  // every operand load of this CTA has been consumed and every store waited for
  if (g0.done_counter != nullptr && threadIdx.x == 0) red_release_gpu_add(g0.done_counter, 1);
  if (g0.dep_wait == kDepBeforeExit && threadIdx.x == 0) griddep_wait();
}

}  // namespace flce
