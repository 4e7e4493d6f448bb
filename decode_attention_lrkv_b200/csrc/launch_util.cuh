// Kernel launch with programmatic dependent launch enabled: the kernel may
// start while the preceding kernel of the stream finishes; it must execute
// griddepcontrol.wait before touching anything that kernel writes.
#pragma once

#include <cuda_runtime.h>

#include "lrkv.h"

namespace lrkv {

// Dynamic shared memory limit plus the largest shared-memory carveout: every
// kernel of the library runs with the same L1/shared split, so an SM never
// has to drain to reconfigure between consecutive kernels of a step.
template <typename Kernel>
inline bool set_smem(Kernel kern, size_t smem) {
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return true;
}

// An empty kernel, launched without programmatic dependent launch after a
// call that writes bases: the decode kernels read the bases before waiting on
// the preceding kernel of the stream, so that kernel must be one that writes
// none of them.
__global__ void stream_fence_kernel();
inline lrkv_status launch_stream_fence(cudaStream_t s) {
  stream_fence_kernel<<<1, 32, 0, s>>>();
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

template <typename Params>
inline lrkv_status launch_pdl(void (*kern)(Params), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, const Params& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) {
    cudaGetLastError();
    return LRKV_ERR_CUDA;
  }
  return LRKV_OK;
}

}  // namespace lrkv
