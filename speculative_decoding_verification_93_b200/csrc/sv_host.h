// sv_host.h -- host-side helpers shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include "sv.h"

namespace sv {

// Records `e` as the calling thread's last CUDA error; maps it to a status.
sv_status note_cuda(cudaError_t e);

// Optional CUDA events around the main verification kernel (benchmarks).
void profile_mark_begin(cudaStream_t st);
void profile_mark_end(cudaStream_t st);

}  // namespace sv
