"""Throughput of the SFU's exp2 (ex2.approx.ftz.f32) on one SM.

The tensor-core epilogues take one exp2 per logit (two more per logit with
softcap: the exp2 and the reciprocal of the tanh).  Whether an epilogue is
bound by the SFU or by its own instruction issue decides how its work is split
across warps, so the rate is measured here rather than assumed: one block of
1, 2, 4 or 8 warps, each thread running 8 independent exp2 chains, timed with
%clock64 on the SM.  The kernel is compiled with NVRTC.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ITERS = 4096
CHAINS = 8
SOURCE = rb"""
extern "C" __global__ void sfu_exp2(float* out, long long* cycles, int iters) {
  float a[8];
  for (int i = 0; i < 8; ++i) a[i] = threadIdx.x * 1e-3f + i * 1e-4f;
  __syncthreads();
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float y;
      asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(a[i]));
      a[i] = y * -0.5f;  /* stays in [-0.5, -0.35]: no overflow */
    }
  }
  const long long t1 = clock64();
  float s = 0.f;
  for (int i = 0; i < 8; ++i) s += a[i];
  out[threadIdx.x] = s;
  if (threadIdx.x == 0) cycles[0] = t1 - t0;
}
"""


def _rates(warp_counts):
    from cuda.bindings import driver as cu, nvrtc

    torch.zeros(1, device="cuda")  # the primary context is current
    err, prog = nvrtc.nvrtcCreateProgram(SOURCE, b"sfu_exp2.cu", 0, [], [])
    assert err == nvrtc.nvrtcResult.NVRTC_SUCCESS
    opts = [b"--gpu-architecture=sm_100a"]
    assert nvrtc.nvrtcCompileProgram(prog, len(opts), opts)[0] == nvrtc.nvrtcResult.NVRTC_SUCCESS
    err, size = nvrtc.nvrtcGetCUBINSize(prog)
    cubin = b" " * size
    assert nvrtc.nvrtcGetCUBIN(prog, cubin)[0] == nvrtc.nvrtcResult.NVRTC_SUCCESS
    err, mod = cu.cuModuleLoadData(cubin)
    assert err == cu.CUresult.CUDA_SUCCESS
    err, fn = cu.cuModuleGetFunction(mod, b"sfu_exp2")
    assert err == cu.CUresult.CUDA_SUCCESS
    out = torch.zeros(32 * max(warp_counts), device="cuda")
    cyc = torch.zeros(1, dtype=torch.int64, device="cuda")
    rates = {}
    for w in warp_counts:
        args = [ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(cyc.data_ptr()),
                ctypes.c_int(ITERS)]
        ptrs = (ctypes.c_void_p * len(args))(*[ctypes.addressof(a) for a in args])
        for _ in range(2):  # the second launch is timed (warm instruction cache)
            assert cu.cuLaunchKernel(fn, 1, 1, 1, 32 * w, 1, 1, 0, cu.CUstream(0),
                                     ctypes.addressof(ptrs), 0)[0] == cu.CUresult.CUDA_SUCCESS
        torch.cuda.synchronize()
        c = int(cyc.item())
        rates[w] = CHAINS * ITERS * 32 * w / c  # lane results per SM clock
        assert np.all(np.isfinite(out[:32 * w].cpu().numpy()))
    cu.cuModuleUnload(mod)
    return rates


def test_sfu_exp2_throughput():
    rates = _rates([1, 2, 4, 8])
    print("ex2.approx lane results per clock per SM:",
          {w: round(r, 2) for w, r in rates.items()})
    assert rates[1] >= 3.4     # one warp with 8 independent chains nearly fills its
                               # sub-partition's SFU (4 results per clock)
    assert rates[4] >= 13.5    # four sub-partitions: about 16 per clock per SM
    assert rates[8] <= 17.0    # and no more with more warps
