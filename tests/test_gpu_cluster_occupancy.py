"""How many thread-block clusters of each size fit on the GPU at once with the
shared memory and block size of this library's tensor-core GEMM kernel.

The design relies on it twice: CTA pairs (clusters of 2) must fill every SM,
and a flash-style fused forward + dHidden would need clusters of 8 or 16 CTAs
splitting the hidden dimension (its fp32 dHidden accumulator is 4*H bytes per
token row, 16 KiB at H = 4096, against 2 KiB per row of tensor memory), which
leave SMs idle.  The query runs on a trivial kernel compiled here with NVRTC;
cluster occupancy depends only on the launch shape (threads, shared memory,
cluster size), not on the kernel's code.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu

THREADS = 320          # threads of a GEMM CTA (producer, MMA and 8 epilogue warps)
SMEM = 230400          # dynamic shared memory of the largest GEMM CTA (ring + staging)
SOURCE = (b'extern "C" __global__ void occupancy_probe(int* p) {'
          b' extern __shared__ int s[]; if (p) p[threadIdx.x] = s[threadIdx.x]; }')


def _max_active_clusters(cluster_sizes):
    from cuda.bindings import driver as cu, nvrtc

    torch.zeros(1, device="cuda")  # the primary context is current
    err, prog = nvrtc.nvrtcCreateProgram(SOURCE, b"occupancy_probe.cu", 0, [], [])
    assert err == nvrtc.nvrtcResult.NVRTC_SUCCESS
    opts = [b"--gpu-architecture=sm_100a"]
    assert nvrtc.nvrtcCompileProgram(prog, len(opts), opts)[0] == nvrtc.nvrtcResult.NVRTC_SUCCESS
    err, size = nvrtc.nvrtcGetCUBINSize(prog)
    cubin = b" " * size
    assert nvrtc.nvrtcGetCUBIN(prog, cubin)[0] == nvrtc.nvrtcResult.NVRTC_SUCCESS
    err, mod = cu.cuModuleLoadData(cubin)
    assert err == cu.CUresult.CUDA_SUCCESS
    err, fn = cu.cuModuleGetFunction(mod, b"occupancy_probe")
    assert err == cu.CUresult.CUDA_SUCCESS
    attr = cu.CUfunction_attribute
    assert cu.cuFuncSetAttribute(fn, attr.CU_FUNC_ATTRIBUTE_MAX_DYNAMIC_SHARED_SIZE_BYTES,
                                 SMEM)[0] == cu.CUresult.CUDA_SUCCESS
    assert cu.cuFuncSetAttribute(fn, attr.CU_FUNC_ATTRIBUTE_NON_PORTABLE_CLUSTER_SIZE_ALLOWED,
                                 1)[0] == cu.CUresult.CUDA_SUCCESS
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    out = {}
    for cs in cluster_sizes:
        cfg = cu.CUlaunchConfig()
        cfg.gridDimX, cfg.gridDimY, cfg.gridDimZ = sms * cs, 1, 1
        cfg.blockDimX, cfg.blockDimY, cfg.blockDimZ = THREADS, 1, 1
        cfg.sharedMemBytes = SMEM
        a = cu.CUlaunchAttribute()
        a.id = cu.CUlaunchAttributeID.CU_LAUNCH_ATTRIBUTE_CLUSTER_DIMENSION
        a.value.clusterDim.x, a.value.clusterDim.y, a.value.clusterDim.z = cs, 1, 1
        cfg.attrs = [a]
        cfg.numAttrs = 1
        err, n = cu.cuOccupancyMaxActiveClusters(fn, cfg)
        assert err == cu.CUresult.CUDA_SUCCESS, (cs, err)
        out[cs] = n
    cu.cuModuleUnload(mod)
    return sms, out


def test_cluster_occupancy_at_the_gemm_shape():
    sms, clusters = _max_active_clusters([1, 2, 4, 8, 16])
    busy = {cs: n * cs for cs, n in clusters.items()}
    print(f"SMs {sms}; max active clusters {clusters}; SMs busy {busy}")
    assert busy[1] == sms            # one CTA per SM
    assert busy[2] == sms            # CTA pairs fill every SM
    assert busy[8] < 0.9 * sms       # an H-split over 8 CTAs leaves >10% of the SMs idle
    assert busy[16] < 0.9 * sms      # ... and over 16 CTAs too
