// pdl.cuh -- programmatic dependent launch between the layer's kernels.
//
// Every kernel of the layer is launched with the programmatic-stream-serialisation
// attribute, so it may be scheduled while the kernel before it in the stream still
// runs.  It calls pdl_wait() before it reads or writes anything an earlier kernel
// touches (griddepcontrol.wait returns once the earlier grids have completed and
// their memory is visible), and pdl_trigger() to let the next kernel start its own
// launch early.  Prologues that touch only the CTA's own resources (mbarrier init,
// TMEM allocation, tensor-map prefetch) run before the wait and so overlap the
// previous kernel's tail.  Launched without the attribute, both are no-ops.
#pragma once
#include <utility>

#include <cuda_runtime.h>

namespace moe {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace moe
