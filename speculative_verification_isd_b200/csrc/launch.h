// Kernel launches, optionally with programmatic dependent launch: a kernel
// may then be scheduled while its predecessor in the stream is finishing,
// runs its prologue (barriers, TMEM, tensor-map prefetch), and calls
// pdl_wait() before it touches anything the predecessor produces.  Without
// the attribute pdl_wait() returns at once and the launch is ordinary
// (isd_abi.cu says when the step uses it).
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace isd {

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace isd
