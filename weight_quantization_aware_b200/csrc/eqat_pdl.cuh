// Programmatic dependent launch (PDL).  A kernel launched with programmatic stream
// serialization may be scheduled before the kernel ahead of it in the stream has
// finished: once every CTA of that kernel has executed pdl_allow_dependents() (or
// exited), the dependent's CTAs are placed on SMs as resources free up and run
// their prologue (barrier set-up, tensor memory, descriptor prefetch).  pdl_wait()
// then blocks the calling thread until the preceding kernel has completed and its
// memory operations are visible, so a kernel touches global memory, for reading or
// writing, only after pdl_wait().  A kernel whose predecessor never signals starts
// when the predecessor ends, as without the attribute.
#pragma once

#include <cuda_runtime.h>

namespace eqat {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch with programmatic stream serialization; `extra` adds one more attribute
// (a cluster shape), when its id is not cudaLaunchAttributeIgnore.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          const cudaLaunchAttribute &extra, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int n = 1;
    if (extra.id != cudaLaunchAttributeIgnore) attr[n++] = extra;
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchAttribute none{};
    none.id = cudaLaunchAttributeIgnore;
    return launch_pdl_ex(kern, grid, block, smem, st, none, args...);
}

}  // namespace eqat
