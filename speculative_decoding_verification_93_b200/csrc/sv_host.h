// sv_host.h -- host-side helpers shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "sv.h"

namespace sv {

// Records `e` as the calling thread's last CUDA error; maps it to a status.
sv_status note_cuda(cudaError_t e);

// Launch `kernel` on `st` with programmatic stream serialisation: it may
// start while the previous kernel in the stream drains, and waits for it
// with griddepcontrol.wait before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// NVTX range over one library call, named after the entry point, so that a
// profiler timeline shows which call issued which kernels.  Header-only
// NVTX: without a profiler attached each push and pop returns at once.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// Optional CUDA events around the main verification kernel (benchmarks).
void profile_mark_begin(cudaStream_t st);
void profile_mark_end(cudaStream_t st);

}  // namespace sv
