// sv_api.cu -- schedule kernel, Philox test exports, status strings and
// profiling hooks.
//
// Schedule (cited as page title + section): umans.ai, "DeepSeek V4 Pro DSpark:
// the model isn't ready, the architecture is", section "What DSpark adds",
// item "2. Verify smarter" -- per-position survival confidences multiplied
// along the block give the survival probability of every prefix; aiweekly.co
// alert -- verify length from prefix survival and system load; en.5iter.com
// article and techvisionai Ch. 7 "Confidence-Scheduled Verification" --
// verify longer when idle, only the confident prefix when busy.  The load
// enters as the threshold tau: L = max{i : S_i >= tau}.
#include <cstdint>
#include <vector>

#include "sv.h"
#include "sv_device.cuh"
#include "sv_host.h"

namespace sv {

static thread_local int g_last_cuda_error = 0;

sv_status note_cuda(cudaError_t e) {
    if (e == cudaSuccess) return SV_OK;
    g_last_cuda_error = static_cast<int>(e);
    return SV_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Schedule: one thread per row, the running product left to right in fp32.
// ---------------------------------------------------------------------------
__global__ void schedule_kernel(const float *__restrict__ conf, int B, int K, float tau,
                                int32_t *__restrict__ lengths) {
    griddep_wait();                 // the previous step may still read `lengths`
    griddep_launch_dependents();    // the verification prologue may launch now
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x)
        lengths[b] = schedule_length(conf + static_cast<long long>(b) * K, K, tau);
}

// ---------------------------------------------------------------------------
// Philox exports.
// ---------------------------------------------------------------------------
__global__ void philox_uniforms_kernel(uint64_t seed, const int64_t *row, const int32_t *pos,
                                       const int32_t *draw, int n, float *out) {
    for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += gridDim.x * blockDim.x)
        out[k] = uniform24(seed, static_cast<uint64_t>(row[k]), static_cast<uint32_t>(pos[k]),
                           static_cast<uint32_t>(draw[k]));
}

__global__ void philox_raw_kernel(const uint32_t *ctr, const uint32_t *key, int n, uint32_t *out) {
    for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += gridDim.x * blockDim.x) {
        const Philox4 o = philox4x32_10(ctr[4 * k], ctr[4 * k + 1], ctr[4 * k + 2], ctr[4 * k + 3],
                                        key[2 * k], key[2 * k + 1]);
        for (int q = 0; q < 4; ++q) out[4 * k + q] = o.w[q];
    }
}

// ---------------------------------------------------------------------------
// Profiling.
// ---------------------------------------------------------------------------
struct Profile {
    std::vector<cudaEvent_t> start, stop;
    int capacity = 0;
    int count = 0;
};
static Profile g_prof;

void profile_mark_begin(cudaStream_t st) {
    if (g_prof.count < g_prof.capacity) cudaEventRecord(g_prof.start[g_prof.count], st);
}

void profile_mark_end(cudaStream_t st) {
    if (g_prof.count < g_prof.capacity) {
        cudaEventRecord(g_prof.stop[g_prof.count], st);
        ++g_prof.count;
    }
}

static void profile_release() {
    for (auto e : g_prof.start) cudaEventDestroy(e);
    for (auto e : g_prof.stop) cudaEventDestroy(e);
    g_prof.start.clear();
    g_prof.stop.clear();
    g_prof.capacity = g_prof.count = 0;
}

}  // namespace sv

extern "C" sv_status sv_schedule(const float *conf, int B, int K, float load, int32_t *lengths,
                                 void *stream) {
    sv::NvtxRange nvtx_range("sv_schedule");
    if (!conf || !lengths) return SV_ERR_ARG;
    if (B < 1 || K < 1 || K > SV_MAX_K) return SV_ERR_SHAPE;
    const int threads = 256;
    int blocks = (B + threads - 1) / threads;
    if (blocks > 65535) blocks = 65535;
    return sv::note_cuda(sv::launch_pdl(sv::schedule_kernel, dim3(blocks), dim3(threads), 0,
                                        static_cast<cudaStream_t>(stream), conf, B, K, load,
                                        lengths));
}

extern "C" sv_status sv_philox_uniforms(uint64_t seed, const int64_t *row, const int32_t *pos,
                                        const int32_t *draw, int n, float *out, void *stream) {
    if (n < 0) return SV_ERR_SHAPE;
    if (n == 0) return SV_OK;
    if (!row || !pos || !draw || !out) return SV_ERR_ARG;
    int blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    sv::philox_uniforms_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        seed, row, pos, draw, n, out);
    return sv::note_cuda(cudaGetLastError());
}

extern "C" sv_status sv_philox4x32_10(const uint32_t *ctr, const uint32_t *key, int n,
                                      uint32_t *out, void *stream) {
    if (n < 0) return SV_ERR_SHAPE;
    if (n == 0) return SV_OK;
    if (!ctr || !key || !out) return SV_ERR_ARG;
    int blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    sv::philox_raw_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(ctr, key, n, out);
    return sv::note_cuda(cudaGetLastError());
}

extern "C" sv_status sv_profile_begin(int capacity) {
    sv::profile_release();
    if (capacity <= 0) return SV_OK;
    sv::g_prof.start.resize(capacity);
    sv::g_prof.stop.resize(capacity);
    for (int i = 0; i < capacity; ++i) {
        cudaError_t e1 = cudaEventCreate(&sv::g_prof.start[i]);
        cudaError_t e2 = cudaEventCreate(&sv::g_prof.stop[i]);
        if (e1 != cudaSuccess || e2 != cudaSuccess) {
            sv::g_prof.start.resize(i);
            sv::g_prof.stop.resize(i);
            sv::profile_release();
            return sv::note_cuda(e1 != cudaSuccess ? e1 : e2);
        }
    }
    sv::g_prof.capacity = capacity;
    sv::g_prof.count = 0;
    return SV_OK;
}

extern "C" int sv_profile_read(float *ms, int max) {
    int n = sv::g_prof.count < max ? sv::g_prof.count : max;
    for (int i = 0; i < n; ++i) {
        float t = -1.f;
        if (cudaEventSynchronize(sv::g_prof.stop[i]) == cudaSuccess)
            cudaEventElapsedTime(&t, sv::g_prof.start[i], sv::g_prof.stop[i]);
        ms[i] = t;
    }
    return n;
}

extern "C" const char *sv_status_string(sv_status s) {
    switch (s) {
    case SV_OK: return "SV_OK";
    case SV_ERR_ARG: return "SV_ERR_ARG";
    case SV_ERR_SHAPE: return "SV_ERR_SHAPE";
    case SV_ERR_DTYPE: return "SV_ERR_DTYPE";
    case SV_ERR_WORKSPACE: return "SV_ERR_WORKSPACE";
    case SV_ERR_CUDA: return "SV_ERR_CUDA";
    }
    return "SV_UNKNOWN";
}

extern "C" int sv_last_cuda_error(void) { return sv::g_last_cuda_error; }

extern "C" int sv_version(void) { return 1; }
