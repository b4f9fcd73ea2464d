// CUDA-core kernels of the fused linear cross-entropy: merging the forward's
// per-vocab-tile softmax statistics into lse, the per-row loss with a
// deterministic float64 reduction, the valid-row count, and the fp32 path
// (plain FFMA kernels for float32 inputs; a correctness path, not tuned).
#pragma once

#include <math_constants.h>

#include "tc_gemm.cuh"

namespace flce {

constexpr int kMergeRows = 32;
constexpr int kMergeSplit = 32;
constexpr int kLossThreads = 256;
constexpr int kFinalThreads = 1024;

// Merge (m, s) pairs of the log2-domain online softmax: returns the pair for
// the union of both column sets.  (-inf, 0) is the empty set.
__device__ __forceinline__ void merge_ms(float& M, float& S, float m, float s) {
  if (m == -CUDART_INF_F) return;
  if (m > M) {
    S = (M == -CUDART_INF_F) ? s : S * exp2f(M - m) + s;
    M = m;
  } else {
    S += s * exp2f(m - M);
  }
}

// lse = ln 2 * (M + log2 S) over all vocab tiles of a row, for the rows that
// take part in the loss; a row whose label is ignore_index (or outside
// [0, V)) gets lse 0 and no merge.  Block (32 rows, 32 splits); grid ceil(N/32).
//   perm == nullptr: the partials are indexed by row; a row's label decides.
//   perm != nullptr: the forward ran on compacted rows: partial column j is
//     compact row j, the original row perm[j]; the first *n_valid compact rows
//     take part.  lse_c[j] receives the value as well (compact order).
__global__ void __launch_bounds__(kMergeRows * kMergeSplit)
    fwd_merge_kernel(const float* __restrict__ part_m, const float* __restrict__ part_s,
                     int n_vt, int N, float* __restrict__ lse, const int64_t* __restrict__ labels,
                     int64_t ignore_index, int64_t V, const int* __restrict__ perm,
                     const long long* __restrict__ n_valid, float* __restrict__ lse_c) {
  __shared__ float sm[kMergeSplit][kMergeRows];
  __shared__ float ss[kMergeSplit][kMergeRows];
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int j = blockIdx.x * kMergeRows + tx;
  bool live = j < N;
  if (live) {
    if (perm != nullptr) {
      live = j < *n_valid;
    } else {
      const int64_t y = labels[j];
      live = (y != ignore_index) && y >= 0 && y < V;
    }
  }
  float M = -CUDART_INF_F, S = 0.f;
  if (live) {
    for (int vt = ty; vt < n_vt; vt += kMergeSplit) {
      const size_t idx = static_cast<size_t>(vt) * N + j;
      merge_ms(M, S, part_m[idx], part_s[idx]);
    }
  }
  sm[ty][tx] = M;
  ss[ty][tx] = S;
  __syncthreads();
  if (ty == 0 && j < N) {
    float v = 0.f;
    if (live) {
      float Mt = -CUDART_INF_F, St = 0.f;
      for (int k = 0; k < kMergeSplit; ++k) merge_ms(Mt, St, sm[k][tx], ss[k][tx]);
      v = (Mt + log2f(St)) * kLn2;
    }
    if (perm != nullptr) {
      lse[perm[j]] = v;
      lse_c[j] = v;
    } else {
      lse[j] = v;
    }
  }
}

// Per-row loss lse_i - L[i, y_i] for non-ignored rows, summed in float64 per
// block in a fixed order; rows with a label outside [0, V) that is not
// ignore_index set the label-range status bit and contribute nothing.
__global__ void __launch_bounds__(kLossThreads)
    row_loss_kernel(const float* __restrict__ lse, const float* __restrict__ label_logit,
                    const int64_t* __restrict__ labels, int N, int64_t ignore_index, int64_t V,
                    double* __restrict__ block_loss, long long* __restrict__ block_cnt,
                    unsigned int* status) {
  __shared__ double sl[kLossThreads];
  __shared__ long long sc[kLossThreads];
  const int t = threadIdx.x;
  const int row = blockIdx.x * kLossThreads + t;
  double l = 0.0;
  long long c = 0;
  if (row < N) {
    const int64_t y = labels[row];
    if (y != ignore_index) {
      if (y < 0 || y >= V) {
        atomicOr(status, kStatusLabelRange);
      } else {
        l = static_cast<double>(lse[row]) - static_cast<double>(label_logit[row]);
        c = 1;
      }
    }
  }
  sl[t] = l;
  sc[t] = c;
  __syncthreads();
  for (int w = kLossThreads / 2; w > 0; w >>= 1) {
    if (t < w) {
      sl[t] += sl[t + w];
      sc[t] += sc[t + w];
    }
    __syncthreads();
  }
  if (t == 0) {
    block_loss[blockIdx.x] = sl[0];
    block_cnt[blockIdx.x] = sc[0];
  }
}

// One block: fixed-order float64 sum of the block partials, then the
// reduction contract: 'sum' -> (sum, n); 'mean' -> (sum / max(n,1), 0).  The
// returned loss is also multiplied by loss_scale and divided by loss_div (a
// 'sum' loss normalised by a global token count), in float64.
__global__ void __launch_bounds__(kFinalThreads)
    finalize_kernel(const double* __restrict__ block_loss, const long long* __restrict__ block_cnt,
                    int nblk, int mean, double loss_scale, double loss_div, float* loss,
                    int64_t* num_tokens, long long* n_valid_out) {
  __shared__ double sl[kFinalThreads];
  __shared__ long long sc[kFinalThreads];
  const int t = threadIdx.x;
  double l = 0.0;
  long long c = 0;
  for (int b = t; b < nblk; b += kFinalThreads) {
    l += block_loss[b];
    c += block_cnt[b];
  }
  sl[t] = l;
  sc[t] = c;
  __syncthreads();
  for (int w = kFinalThreads / 2; w > 0; w >>= 1) {
    if (t < w) {
      sl[t] += sl[t + w];
      sc[t] += sc[t + w];
    }
    __syncthreads();
  }
  if (t == 0) {
    const long long n = sc[0];
    const double total = sl[0];
    if (mean) {
      loss[0] = static_cast<float>(total / static_cast<double>(n > 0 ? n : 1) * loss_scale /
                                   loss_div);
      num_tokens[0] = 0;
    } else {
      loss[0] = static_cast<float>(total * loss_scale / loss_div);
      num_tokens[0] = n;
    }
    if (n_valid_out != nullptr) *n_valid_out = n;
  }
}

// n = #rows whose label is neither ignore_index nor outside [0, V) (one block).
__global__ void __launch_bounds__(kFinalThreads)
    count_valid_kernel(const int64_t* __restrict__ labels, int N, int64_t ignore_index,
                       int64_t V, long long* n_valid_out) {
  __shared__ long long sc[kFinalThreads];
  const int t = threadIdx.x;
  long long c = 0;
  for (int i = t; i < N; i += kFinalThreads) {
    const int64_t y = labels[i];
    c += (y != ignore_index && y >= 0 && y < V) ? 1 : 0;
  }
  sc[t] = c;
  __syncthreads();
  for (int w = kFinalThreads / 2; w > 0; w >>= 1) {
    if (t < w) sc[t] += sc[t + w];
    __syncthreads();
  }
  if (t == 0) *n_valid_out = sc[0];
}

// Records a label outside [0, V) that is not ignore_index (backward paths that
// do not compact the rows).
__global__ void __launch_bounds__(256)
    label_range_kernel(const int64_t* __restrict__ labels, int N, int64_t ignore_index, int64_t V,
                       unsigned int* __restrict__ status) {
  const int i = blockIdx.x * 256 + threadIdx.x;
  if (i >= N) return;
  const int64_t y = labels[i];
  if (y != ignore_index && (y < 0 || y >= V)) atomicOr(status, kStatusLabelRange);
}

// ------------------------------------------------------------------ bf16 outputs
// dst[i] = bf16(src[i]) or, accumulating, bf16(float(dst[i]) + src[i]); one
// round-to-nearest-even per element.  8 elements per thread step when both
// pointers are 16-byte aligned, else one.
__global__ void __launch_bounds__(256)
    f32_to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, size_t n,
                       int accumulate) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const bool vec = ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u) == 0;
  size_t done = 0;
  if (vec) {
    const size_t n8 = n / 8;
    for (size_t i = t; i < n8; i += stride) {
      const float4 a = reinterpret_cast<const float4*>(src)[2 * i];
      const float4 b = reinterpret_cast<const float4*>(src)[2 * i + 1];
      float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      uint4 o;
      __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
      if (accumulate) {
        const uint4 old = reinterpret_cast<const uint4*>(dst)[i];
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&old);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(p2[k]);
          v[2 * k] += f.x;
          v[2 * k + 1] += f.y;
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) o2[k] = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
      reinterpret_cast<uint4*>(dst)[i] = o;
    }
    done = n8 * 8;
  }
  for (size_t i = done + t; i < n; i += stride) {
    const float v = src[i] + (accumulate ? __bfloat162float(dst[i]) : 0.0f);
    dst[i] = __float2bfloat16_rn(v);
  }
}

// ------------------------------------------------------------------ row compaction
// The backward skips token rows whose label is ignore_index (their gradient is
// exactly zero), and rows whose label lies outside [0, V) (an error the status
// word reports; the forward leaves them out of the loss and the count too).  A stable compaction puts the valid rows first, in order, then
// the ignored rows, in order: perm[j] is the original row of compact row j.
constexpr int kCompactThreads = 1024;

// Valid rows per block of kCompactThreads rows.
__global__ void __launch_bounds__(kCompactThreads)
    compact_count_kernel(const int64_t* __restrict__ labels, int N, int64_t ignore_index,
                         int64_t V, unsigned int* __restrict__ status,
                         int* __restrict__ block_valid) {
  __shared__ int warp_sum[kCompactThreads / 32];
  const int i = blockIdx.x * kCompactThreads + threadIdx.x;
  const int64_t y = (i < N) ? labels[i] : ignore_index;
  const bool in_range = y >= 0 && y < V;
  if (i < N && y != ignore_index && !in_range) atomicOr(status, kStatusLabelRange);
  const bool v = (i < N) && (y != ignore_index) && in_range;  // out of range: as ignored
  const unsigned m = __ballot_sync(0xffffffffu, v);
  if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = __popc(m);
  __syncthreads();
  if (threadIdx.x == 0) {
    int s = 0;
    for (int w = 0; w < kCompactThreads / 32; ++w) s += warp_sum[w];
    block_valid[blockIdx.x] = s;
  }
}

// One block: exclusive prefix sum of a[0..n) in place (the per-block valid
// counts, or a radix pass's digit counts), and the total when `total` is set.
__global__ void __launch_bounds__(kCompactThreads)
    exclusive_scan_kernel(int* __restrict__ a, int n, long long* __restrict__ total) {
  __shared__ int carry;
  __shared__ int warp_sum[kCompactThreads / 32];
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int base = 0; base < n; base += kCompactThreads) {
    const int b = base + threadIdx.x;
    const int x = (b < n) ? a[b] : 0;
    int incl = x;  // inclusive scan within the warp
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += warp_sum[w];
    const int excl = carry + before + incl - x;
    __syncthreads();
    if (b < n) a[b] = excl;
    if (threadIdx.x == kCompactThreads - 1) carry = excl + x;
    __syncthreads();
  }
  if (threadIdx.x == 0 && total != nullptr) *total = carry;
}

// perm[j], and the compact labels and lse of every compact row: valid rows keep
// theirs; ignored rows get ignore_index and lse 0.  lse / lse_c and the sort
// keys may be null (the forward's compaction has no lse yet and no sort).
__global__ void __launch_bounds__(kCompactThreads)
    compact_scatter_kernel(const int64_t* __restrict__ labels, const float* __restrict__ lse,
                           int N, int64_t ignore_index, const int* __restrict__ block_offset,
                           const long long* __restrict__ n_valid, int* __restrict__ perm,
                           int64_t* __restrict__ labels_c, float* __restrict__ lse_c,
                           int64_t V, uint32_t* __restrict__ sort_keys,
                           int* __restrict__ sort_vals) {
  __shared__ int warp_sum[kCompactThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i = blockIdx.x * kCompactThreads + threadIdx.x;
  const int64_t y = (i < N) ? labels[i] : ignore_index;
  const bool v = (i < N) && (y != ignore_index) && y >= 0 && y < V;
  const unsigned m = __ballot_sync(0xffffffffu, v);
  if (lane == 0) warp_sum[warp] = __popc(m);
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += warp_sum[w];
  const int rank_v = block_offset[blockIdx.x] + before + __popc(m & ((1u << lane) - 1u));
  if (i < N) {
    const int j = v ? rank_v : static_cast<int>(*n_valid) + (i - rank_v);
    perm[j] = i;
    labels_c[j] = v ? y : ignore_index;
    if (lse_c != nullptr) lse_c[j] = v ? lse[i] : 0.f;
    if (v && sort_keys != nullptr) {  // the key is the label (in [0, V) for every compacted row)
      sort_keys[j] = static_cast<uint32_t>(y);
      sort_vals[j] = i;
    }
  }
}

// ------------------------------------------------------------------ label sort
// The valid rows are then put in (label, row) order by a stable LSD radix sort
// on 8-bit digits of the label, so the rows of each label are contiguous and
// the per-label sums below have a fixed order.  Only the first *n_valid
// entries take part.
constexpr int kRadixBuckets = 256;

// Per-block digit counts, digit-major: hist[digit * nblk + block].
__global__ void __launch_bounds__(kCompactThreads)
    radix_hist_kernel(const uint32_t* __restrict__ keys, const long long* __restrict__ n_valid,
                      int shift, int nblk, int* __restrict__ hist) {
  __shared__ int h[kRadixBuckets];
  for (int t = threadIdx.x; t < kRadixBuckets; t += blockDim.x) h[t] = 0;
  __syncthreads();
  const long long j = static_cast<long long>(blockIdx.x) * kCompactThreads + threadIdx.x;
  if (j < *n_valid) atomicAdd(&h[(keys[j] >> shift) & (kRadixBuckets - 1)], 1);
  __syncthreads();
  for (int t = threadIdx.x; t < kRadixBuckets; t += blockDim.x) hist[t * nblk + blockIdx.x] = h[t];
}

// Stable scatter of one radix pass: an element's place is its digit's block
// offset plus the number of equal digits before it in the block (earlier
// warps, then earlier lanes of its warp).
__global__ void __launch_bounds__(kCompactThreads)
    radix_scatter_kernel(const uint32_t* __restrict__ keys_in, const int* __restrict__ vals_in,
                         uint32_t* __restrict__ keys_out, int* __restrict__ vals_out,
                         const long long* __restrict__ n_valid, int shift, int nblk,
                         const int* __restrict__ offsets) {
  __shared__ int wcnt[kCompactThreads / 32][kRadixBuckets];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int t = threadIdx.x; t < (kCompactThreads / 32) * kRadixBuckets; t += blockDim.x)
    (&wcnt[0][0])[t] = 0;
  __syncthreads();
  const long long j = static_cast<long long>(blockIdx.x) * kCompactThreads + threadIdx.x;
  const bool live = j < *n_valid;
  const uint32_t key = live ? keys_in[j] : 0u;
  const int dg = live ? static_cast<int>((key >> shift) & (kRadixBuckets - 1)) : kRadixBuckets;
  const unsigned peers = __match_any_sync(0xffffffffu, dg);
  const int rank_w = __popc(peers & ((1u << lane) - 1u));
  if (live && rank_w == 0) wcnt[warp][dg] = __popc(peers);
  __syncthreads();
  if (threadIdx.x < kRadixBuckets) {
    int run = 0;
    for (int w = 0; w < kCompactThreads / 32; ++w) {
      const int c = wcnt[w][threadIdx.x];
      wcnt[w][threadIdx.x] = run;
      run += c;
    }
  }
  __syncthreads();
  if (live) {
    const int dst = offsets[dg * nblk + blockIdx.x] + wcnt[warp][dg] + rank_w;
    keys_out[dst] = key;
    vals_out[dst] = vals_in[j];
  }
}

// The sorted valid rows become compact rows 0..n_valid-1.
__global__ void __launch_bounds__(kCompactThreads)
    apply_label_order_kernel(const uint32_t* __restrict__ keys, const int* __restrict__ vals,
                             const float* __restrict__ lse, const long long* __restrict__ n_valid,
                             int* __restrict__ perm, int64_t* __restrict__ labels_c,
                             float* __restrict__ lse_c) {
  const long long j = static_cast<long long>(blockIdx.x) * kCompactThreads + threadIdx.x;
  if (j >= *n_valid) return;
  const int i = vals[j];
  perm[j] = i;
  labels_c[j] = static_cast<int64_t>(keys[j]);
  lse_c[j] = lse[i];
}

// ------------------------------------------------------------------ label-entry residuals
// The dZ block holds bf16(dZ/g).  For the label entry of each valid row, which
// dominates the row's gradient, the rounding residual e = d - bf16(d) (exact in
// fp32) is recorded by the dZ epilogue and added back here in fp32:
//   dHidden[row]   += g * e * W[label]
//   dWeight[label] += g * sum over the label's rows (in order) of e * hidden[row]
__device__ __forceinline__ float backward_grad_factor(const float* grad_output, float grad_scale,
                                                      const long long* n_valid_for_mean,
                                                      int mean) {
  float g = (grad_output != nullptr ? grad_output[0] : 1.0f) * grad_scale;
  if (mean) {
    const long long n = *n_valid_for_mean;
    g = g / static_cast<float>(n > 0 ? n : 1);
  }
  return g;
}

// dWeight part, deterministic: the valid compact rows are in label order, so
// each label's rows form one run.  Phase 1 cuts the rows into segments of
// kFixSeg and sums e * hidden over each run piece in row order; a run that
// lies inside one segment is added to dWeight at once, a run crossing a
// segment boundary leaves its piece in part[seg][slot] (slot 0: the segment's
// first run, begun in an earlier segment; slot 1: its last run, going on into
// the next).  Phase 2 lets the segment where such a run begins add its pieces
// in segment order.  Blocks cover kFixCols columns, two per thread.
constexpr int kFixSeg = 64;
constexpr int kFixCols = 256;
constexpr int kFixThreads = kFixCols / 2;

// Each dWeight element receives at most one such addition (a label's rows form
// one run), so a reduction without a returned value (no thread waits on the
// old value) leaves the result as reproducible as a read-add-write.
__device__ __forceinline__ void dw_fix_add(float* d_weight, int64_t v, int64_t V, int H, int col,
                                           float g, float a0, float a1) {
  if (v < 0 || v >= V) return;  // a label the forward reported as out of range
  float* o = d_weight + static_cast<size_t>(v) * H + col;
  atomicAdd(o, g * a0);
  atomicAdd(o + 1, g * a1);
}

__global__ void __launch_bounds__(kFixThreads)
    dw_fix_segments_kernel(const int64_t* __restrict__ labels_c, const float* __restrict__ resid,
                           const long long* __restrict__ rows_valid,
                           const __nv_bfloat16* __restrict__ hidden_c, int H, int64_t V,
                           float* __restrict__ d_weight, float* __restrict__ part,
                           const float* grad_output, float grad_scale,
                           const long long* n_valid_for_mean, int mean) {
  const long long nv = *rows_valid;
  const long long s0 = static_cast<long long>(blockIdx.x) * kFixSeg;
  if (s0 >= nv) return;
  const int n = static_cast<int>(min(static_cast<long long>(kFixSeg), nv - s0));
  __shared__ int64_t lab[kFixSeg];
  __shared__ float es[kFixSeg];
  __shared__ int64_t lab_before, lab_after;
  for (int t = threadIdx.x; t < n; t += blockDim.x) {
    lab[t] = labels_c[s0 + t];
    es[t] = resid[s0 + t];
  }
  if (threadIdx.x == 0) {
    lab_before = s0 > 0 ? labels_c[s0 - 1] : INT64_MIN;
    lab_after = s0 + n < nv ? labels_c[s0 + n] : INT64_MIN;
  }
  __syncthreads();
  const int col = blockIdx.y * kFixCols + 2 * threadIdx.x;
  if (col >= H) return;  // H is even
  const float g = backward_grad_factor(grad_output, grad_scale, n_valid_for_mean, mean);
  float* part_seg = part + static_cast<size_t>(blockIdx.x) * 2 * H;
  const __nv_bfloat16* hrow = hidden_c + static_cast<size_t>(s0) * H + col;
  int64_t cur = lab[0];
  bool begun_before = (cur == lab_before);
  float a0 = 0.f, a1 = 0.f;
  for (int kb = 0; kb < n; kb += 8) {
    float2 hv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (kb + i < n)
        hv[i] = __bfloat1622float2(
            *reinterpret_cast<const __nv_bfloat162*>(hrow + static_cast<size_t>(kb + i) * H));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (kb + i >= n) break;
      const int64_t l = lab[kb + i];
      if (l != cur) {  // the run `cur` ends inside the segment
        if (begun_before) {
          part_seg[col] = a0;
          part_seg[col + 1] = a1;
        } else {
          dw_fix_add(d_weight, cur, V, H, col, g, a0, a1);
        }
        cur = l;
        begun_before = false;
        a0 = a1 = 0.f;
      }
      a0 = fmaf(es[kb + i], hv[i].x, a0);
      a1 = fmaf(es[kb + i], hv[i].y, a1);
    }
  }
  const bool goes_on = (cur == lab_after);
  if (begun_before) {
    part_seg[col] = a0;
    part_seg[col + 1] = a1;
  } else if (goes_on) {
    part_seg[H + col] = a0;
    part_seg[H + col + 1] = a1;
  } else {
    dw_fix_add(d_weight, cur, V, H, col, g, a0, a1);
  }
}

__global__ void __launch_bounds__(kFixThreads)
    dw_fix_runs_kernel(const int64_t* __restrict__ labels_c, const long long* __restrict__ rows_valid,
                       int H, int64_t V, float* __restrict__ d_weight,
                       const float* __restrict__ part, const float* grad_output, float grad_scale,
                       const long long* n_valid_for_mean, int mean) {
  const long long nv = *rows_valid;
  const long long s0 = static_cast<long long>(blockIdx.x) * kFixSeg;
  if (s0 >= nv) return;
  long long last = min(s0 + kFixSeg, nv) - 1;
  const int64_t L = labels_c[last];
  if (last + 1 >= nv || labels_c[last + 1] != L) return;  // the last run ends here
  if (s0 > 0 && labels_c[s0 - 1] == L) return;           // it began in an earlier segment
  const int col = blockIdx.y * kFixCols + 2 * threadIdx.x;
  if (col >= H) return;
  const float* p = part + static_cast<size_t>(blockIdx.x) * 2 * H;
  float a0 = p[H + col], a1 = p[H + col + 1];
  for (long long s = blockIdx.x + 1;; ++s) {
    p = part + static_cast<size_t>(s) * 2 * H;
    a0 += p[col];
    a1 += p[col + 1];
    last = min((s + 1) * kFixSeg, nv) - 1;
    if (last + 1 >= nv || labels_c[last + 1] != L) break;
  }
  const float g = backward_grad_factor(grad_output, grad_scale, n_valid_for_mean, mean);
  dw_fix_add(d_weight, L, V, H, col, g, a0, a1);
}

// Compact hidden: row j < n_valid is hidden[perm[j]]; rows past n_valid are
// zero.  Ignored rows of d_hidden are zeroed here (unless accumulating).
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint4* __restrict__ hidden, int H16, int N,
                       const int* __restrict__ perm, const long long* __restrict__ n_valid,
                       uint4* __restrict__ hidden_c, float4* __restrict__ d_hidden, int H4,
                       int zero_ignored_dh) {
  const int j = blockIdx.x;
  if (j >= N) return;
  const long long nv = *n_valid;
  uint4* dst = hidden_c + static_cast<size_t>(j) * H16;
  if (j < nv) {
    const uint4* src = hidden + static_cast<size_t>(perm[j]) * H16;
    for (int k = threadIdx.x; k < H16; k += blockDim.x) dst[k] = src[k];
  } else {
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int k = threadIdx.x; k < H16; k += blockDim.x) dst[k] = z;
    if (zero_ignored_dh) {
      float4* o = d_hidden + static_cast<size_t>(perm[j]) * H4;
      const float4 zf = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int k = threadIdx.x; k < H4; k += blockDim.x) o[k] = zf;
    }
  }
}

// dHidden of one token chunk back to token order.  The chunk's dHidden GEMMs
// accumulate g * dZ . W over the compact rows [t0, t0 + rows) into dh_c
// (fp32, chunk-local rows, TMA store then reduce-add); here compact row j
// adds the exact label term g * resid[j] * W[labels_c[j]] and lands on
// d_hidden row perm[j] (stored, or added with `accumulate`).  Rows past the
// valid count are not read: the GEMMs skip or leave them undefined.
__global__ void __launch_bounds__(256)
    dh_scatter_kernel(const float4* __restrict__ dh_c, int t0, int rows,
                      const int* __restrict__ perm, const long long* __restrict__ n_valid,
                      const int64_t* __restrict__ labels_c, const float* __restrict__ resid,
                      const __nv_bfloat16* __restrict__ weight, int64_t V, int H4,
                      float4* __restrict__ d_hidden, int accumulate, const float* grad_output,
                      float grad_scale, const long long* n_valid_for_mean, int mean) {
  const int jl = blockIdx.x;
  const long long j = static_cast<long long>(t0) + jl;
  if (jl >= rows || j >= *n_valid) return;
  const float4* src = dh_c + static_cast<size_t>(jl) * H4;
  float4* dst = d_hidden + static_cast<size_t>(perm[j]) * H4;
  const int64_t y = labels_c[j];
  const bool fix = resid != nullptr && y >= 0 && y < V;
  const float cfix =
      fix ? backward_grad_factor(grad_output, grad_scale, n_valid_for_mean, mean) * resid[j] : 0.f;
  const uint2* wrow = reinterpret_cast<const uint2*>(weight + static_cast<size_t>(fix ? y : 0) * H4 * 4);
  for (int k = threadIdx.x; k < H4; k += blockDim.x) {
    float4 o = src[k];
    if (fix) {
      const uint2 wv = wrow[k];
      const float2 w01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv.x));
      const float2 w23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv.y));
      o.x = fmaf(cfix, w01.x, o.x);
      o.y = fmaf(cfix, w01.y, o.y);
      o.z = fmaf(cfix, w23.x, o.z);
      o.w = fmaf(cfix, w23.y, o.w);
    }
    if (accumulate) {
      const float4 a = dst[k];
      o.x += a.x;
      o.y += a.y;
      o.z += a.z;
      o.w += a.w;
    }
    dst[k] = o;
  }
}

// Waits, bounded, on an mbarrier that nothing completes; records the timeout
// in the status word (the same wait and report as the GEMM pipelines).
__global__ void selftest_wait_kernel(unsigned int* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    if (!mbar_wait(smem_u32(&bar), 0, nullptr, timeout_ns)) atomicOr(status, kStatusTimeout);
  }
}

// ------------------------------------------------------------------ fp32 path
constexpr int kSimtThreads = 256;
constexpr int kSimtChunk = 1024;

__device__ __forceinline__ float capped(float z, float softcap) {
  return softcap > 0.f ? softcap * tanhf(z / softcap) : z;
}

// One block per token row: lse and the label logit, natural-log domain.
// Dynamic smem: H floats (the row of hidden).
__global__ void __launch_bounds__(kSimtThreads)
    simt_fwd_kernel(const float* __restrict__ hidden, const float* __restrict__ weight,
                    const int64_t* __restrict__ labels, int N, int H, int V, float softcap,
                    int64_t ignore_index, float* __restrict__ lse,
                    float* __restrict__ label_logit) {
  extern __shared__ float sh[];
  __shared__ float red_m[kSimtThreads], red_s[kSimtThreads];
  const int row = blockIdx.x;
  const int t = threadIdx.x;
  {  // a row outside the loss gets lse 0 and no work
    const int64_t y0 = labels[row];
    if (y0 == ignore_index || y0 < 0 || y0 >= V) {
      if (t == 0) lse[row] = 0.f;
      return;
    }
  }
  for (int k = t; k < H; k += kSimtThreads) sh[k] = hidden[static_cast<size_t>(row) * H + k];
  __syncthreads();
  const int64_t y = labels[row];
  float m = -CUDART_INF_F, s = 0.f;
  for (int v = t; v < V; v += kSimtThreads) {
    const float* w = weight + static_cast<size_t>(v) * H;
    float z = 0.f;
    for (int k = 0; k < H; ++k) z = fmaf(sh[k], w[k], z);
    const float L = capped(z, softcap);
    if (v == y) label_logit[row] = L;
    if (L > m) {
      s = (m == -CUDART_INF_F) ? 1.f : s * expf(m - L) + 1.f;
      m = L;
    } else {
      s += expf(L - m);
    }
  }
  red_m[t] = m;
  red_s[t] = s;
  __syncthreads();
  for (int w = kSimtThreads / 2; w > 0; w >>= 1) {
    if (t < w) {
      float M = red_m[t], S = red_s[t];
      const float m2 = red_m[t + w], s2 = red_s[t + w];
      if (m2 != -CUDART_INF_F) {
        if (m2 > M) {
          S = (M == -CUDART_INF_F) ? s2 : S * expf(M - m2) + s2;
          M = m2;
        } else {
          S += s2 * expf(m2 - M);
        }
      }
      red_m[t] = M;
      red_s[t] = S;
    }
    __syncthreads();
  }
  if (t == 0) lse[row] = red_m[0] + logf(red_s[0]);
}

__device__ __forceinline__ float simt_grad_scale(const float* grad_output, float grad_scale,
                                                 const long long* n_valid, int mean) {
  float g = (grad_output != nullptr ? grad_output[0] : 1.0f) * grad_scale;
  if (mean) {
    const long long n = *n_valid;
    g /= static_cast<float>(n > 0 ? n : 1);
  }
  return g;
}

// One block per token row: dHidden[row] = sum_v dZ[row, v] W[v].
// Dynamic smem: 2*H + kSimtChunk floats.
__global__ void __launch_bounds__(kSimtThreads)
    simt_dh_kernel(const float* __restrict__ hidden, const float* __restrict__ weight,
                   const int64_t* __restrict__ labels, const float* __restrict__ lse, int N,
                   int H, int V, int64_t ignore_index, float softcap, const float* grad_output,
                   float grad_scale, const long long* n_valid, int mean, int accumulate,
                   float* __restrict__ d_hidden) {
  extern __shared__ float sh[];
  float* h = sh;
  float* acc = sh + H;
  float* G = sh + 2 * H;
  const int row = blockIdx.x;
  const int t = threadIdx.x;
  const int64_t y = labels[row];
  const bool valid = (y != ignore_index) && y >= 0 && y < V;  // out of range: as ignored
  const float g = simt_grad_scale(grad_output, grad_scale, n_valid, mean);
  const float l = lse[row];
  for (int k = t; k < H; k += kSimtThreads) {
    h[k] = hidden[static_cast<size_t>(row) * H + k];
    acc[k] = 0.f;
  }
  __syncthreads();
  for (int v0 = 0; v0 < V; v0 += kSimtChunk) {
    const int nv = min(kSimtChunk, V - v0);
    for (int j = t; j < nv; j += kSimtThreads) {
      const int v = v0 + j;
      float gz = 0.f;
      if (valid) {
        const float* w = weight + static_cast<size_t>(v) * H;
        float z = 0.f;
        for (int k = 0; k < H; ++k) z = fmaf(h[k], w[k], z);
        const float L = capped(z, softcap);
        float d = expf(L - l) - (v == y ? 1.f : 0.f);
        if (softcap > 0.f) {
          const float u = L / softcap;
          d *= 1.f - u * u;
        }
        gz = g * d;
      }
      G[j] = gz;
    }
    __syncthreads();
    for (int k = t; k < H; k += kSimtThreads) {
      float a = acc[k];
      for (int j = 0; j < nv; ++j) a = fmaf(G[j], weight[static_cast<size_t>(v0 + j) * H + k], a);
      acc[k] = a;
    }
    __syncthreads();
  }
  for (int k = t; k < H; k += kSimtThreads) {
    float* o = d_hidden + static_cast<size_t>(row) * H + k;
    *o = accumulate ? *o + acc[k] : acc[k];
  }
}

// One block per vocab row: dWeight[v] = sum_i dZ[i, v] hidden[i].
// Dynamic smem: 2*H + kSimtThreads floats.
__global__ void __launch_bounds__(kSimtThreads)
    simt_dw_kernel(const float* __restrict__ hidden, const float* __restrict__ weight,
                   const int64_t* __restrict__ labels, const float* __restrict__ lse, int N,
                   int H, int V, int64_t ignore_index, float softcap, const float* grad_output,
                   float grad_scale, const long long* n_valid, int mean, int accumulate,
                   float* __restrict__ d_weight) {
  extern __shared__ float sh[];
  float* w = sh;
  float* acc = sh + H;
  float* G = sh + 2 * H;
  const int v = blockIdx.x;
  const int t = threadIdx.x;
  const float g = simt_grad_scale(grad_output, grad_scale, n_valid, mean);
  for (int k = t; k < H; k += kSimtThreads) {
    w[k] = weight[static_cast<size_t>(v) * H + k];
    acc[k] = 0.f;
  }
  __syncthreads();
  for (int i0 = 0; i0 < N; i0 += kSimtThreads) {
    const int ni = min(kSimtThreads, N - i0);
    if (t < ni) {
      const int i = i0 + t;
      const int64_t y = labels[i];
      float gz = 0.f;
      if (y != ignore_index && y >= 0 && y < V) {  // out of range: as ignored
        const float* hi = hidden + static_cast<size_t>(i) * H;
        float z = 0.f;
        for (int k = 0; k < H; ++k) z = fmaf(hi[k], w[k], z);
        const float L = capped(z, softcap);
        float d = expf(L - lse[i]) - (v == y ? 1.f : 0.f);
        if (softcap > 0.f) {
          const float u = L / softcap;
          d *= 1.f - u * u;
        }
        gz = g * d;
      }
      G[t] = gz;
    }
    __syncthreads();
    for (int k = t; k < H; k += kSimtThreads) {
      float a = acc[k];
      for (int j = 0; j < ni; ++j) a = fmaf(G[j], hidden[static_cast<size_t>(i0 + j) * H + k], a);
      acc[k] = a;
    }
    __syncthreads();
  }
  for (int k = t; k < H; k += kSimtThreads) {
    float* o = d_weight + static_cast<size_t>(v) * H + k;
    *o = accumulate ? *o + acc[k] : acc[k];
  }
}

}  // namespace flce
