// launch.cuh -- programmatic dependent launch (PDL) between the kernels of one layer call.
//
// Every kernel of the library is launched with programmatic stream serialisation, so the next
// kernel's CTAs may start (and run their prologue: barrier set-up, TMEM allocation,
// tensor-map prefetch) while the previous kernel drains.  Each kernel calls
// griddep_launch_dependents() once all of its CTAs are running, and griddep_wait() before it
// reads anything an earlier kernel of the stream wrote; griddep_wait() returns only when the
// preceding grid has completed and its memory is visible.  Without the launch attribute both
// instructions are no-ops.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace moe {

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void griddep_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args &&...args)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace moe
