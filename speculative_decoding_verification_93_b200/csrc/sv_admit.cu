// sv_admit.cu -- hardware-aware admission of draft tokens (one CTA).
//
// Method (cited as page title + section): umans.ai, "DeepSeek V4 Pro DSpark:
// the model isn't ready, the architecture is", section "What DSpark adds",
// item "2. Verify smarter" -- the engine's speed is profiled once as a
// function of batch size; every step, expected system throughput is expected
// accepted tokens times the speed at that batch size; every candidate token
// of every active request is sorted by survival probability, admitted one at
// a time, and admission stops the moment the product stops rising.
// zhichai.net DSpark topic, "Under the hood" and techvisionai Ch. 7
// "Hardware-Aware Scheduling" describe the same scheduler.
//
// Reading: row b always verifies its final position, so after k admissions
// the batch holds n = B + k tokens and the expected emitted tokens are
// E(k) = B + (sum of the admitted S); f(k) = E(k) * speed[n]; candidate k+1
// is admitted iff n + 1 lies inside the speed table and f(k+1) > f(k).
// Candidates are ordered by S descending, ties by (row, position) ascending,
// so each row's admitted candidates form a prefix.  S is the fp64 running
// product of the clamped confidences (NaN counts as 0).
//
// Kernel: per-row products in fp64 in the same order as the definition,
// bitonic sort in shared memory, an fp64 block prefix scan for E(k), and a
// block-wide minimum for the first k at which f stops rising.
#include <cfloat>
#include <climits>
#include <cstdint>

#include "sv.h"
#include "sv_device.cuh"
#include "sv_host.h"

namespace sv {

constexpr int kAdmitThreads = 1024;
constexpr int kAdmitMax = SV_MAX_ADMIT;   // candidates (B * K) sorted in shared memory

// a precedes b in admission order
__device__ __forceinline__ bool admit_before(double ka, int ia, double kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}

__global__ void __launch_bounds__(kAdmitThreads) admit_kernel(const float *__restrict__ conf,
                                                              int B, int K,
                                                              const float *__restrict__ speed,
                                                              int n_speed, int32_t *lengths,
                                                              float *tau_out) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    griddep_wait();
    griddep_launch_dependents();
    const int n = B * K;
    int N = 1;
    while (N < n) N <<= 1;
    double *key = reinterpret_cast<double *>(smem_raw);        // [N]
    int *idx = reinterpret_cast<int *>(key + N);                // [N]
    __shared__ double s_wsum[kAdmitThreads / 32];
    __shared__ int s_stop;

    // 1. Prefix survival of every candidate.
    for (int b = tid; b < B; b += kAdmitThreads) {
        double S = 1.0;
        for (int i = 0; i < K; ++i) {
            double c = static_cast<double>(__ldg(conf + static_cast<long long>(b) * K + i));
            c = isnan(c) ? 0.0 : fmin(fmax(c, 0.0), 1.0);
            S = S * c;
            key[b * K + i] = S;
            idx[b * K + i] = b * K + i;
        }
    }
    for (int q = n + tid; q < N; q += kAdmitThreads) { key[q] = -1.0; idx[q] = INT_MAX; }
    __syncthreads();

    // 2. Bitonic sort into admission order.
    for (int k = 2; k <= N; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < N; i += kAdmitThreads) {
                const int p = i ^ j;
                if (p > i) {
                    const double ki = key[i], kp = key[p];
                    const int ii = idx[i], ip = idx[p];
                    const bool asc = (i & k) == 0;   // segment in admission order
                    const bool swap = asc ? admit_before(kp, ip, ki, ii) : admit_before(ki, ii, kp, ip);
                    if (swap) {
                        key[i] = kp; key[p] = ki;
                        idx[i] = ip; idx[p] = ii;
                    }
                }
            }
            __syncthreads();
        }
    }

    // 3. Exclusive prefix sums of the sorted survivals (per-thread runs of
    //    consecutive candidates, then a block scan of the run totals).
    const int per = N / kAdmitThreads > 0 ? N / kAdmitThreads : 1;
    const int r0 = tid * per;
    double run = 0.0;
    for (int q = 0; q < per; ++q)
        if (r0 + q < n) run += key[r0 + q];
    double x = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_wsum[warp] = x;
    if (tid == 0) s_stop = INT_MAX;
    __syncthreads();
    if (warp == 0) {
        double y = s_wsum[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double z = __shfl_up_sync(0xffffffffu, y, o);
            if (lane >= o) y += z;
        }
        s_wsum[lane] = y;
    }
    __syncthreads();
    const double xprev = __shfl_up_sync(0xffffffffu, x, 1);
    double pre = (lane ? xprev : 0.0) + (warp ? s_wsum[warp - 1] : 0.0);   // sum before this run

    // 4. First k whose admission does not raise f (or runs out of table).
    //    Each thread tests the candidates of its run: k = r0 + q.
    int stop = INT_MAX;
    for (int q = 0; q < per; ++q) {
        const int k = r0 + q;
        if (k > n || r0 + q >= N + 1) break;
        const double Ek = static_cast<double>(B) + pre;
        bool fail;
        if (k >= n || B + k + 1 >= n_speed) {
            fail = true;
        } else {
            const double fk = Ek * static_cast<double>(__ldg(speed + B + k));
            const double f1 = (Ek + key[k]) * static_cast<double>(__ldg(speed + B + k + 1));
            fail = !(f1 > fk);
        }
        if (fail) { stop = k; break; }
        pre += key[k];
    }
    if (stop != INT_MAX) atomicMin(&s_stop, stop);
    __syncthreads();
    int admitted = s_stop;
    if (admitted == INT_MAX) admitted = n;   // every candidate admitted (N == n case)
    if (B >= n_speed) admitted = 0;

    // 5. Per-row counts and the threshold.
    for (int b = tid; b < B; b += kAdmitThreads) lengths[b] = 0;
    __syncthreads();
    for (int q = tid; q < admitted; q += kAdmitThreads) atomicAdd(&lengths[idx[q] / K], 1);
    if (tid == 0 && tau_out)
        *tau_out = admitted > 0 ? static_cast<float>(key[admitted - 1])
                                : __int_as_float(0x7f800000);
}

}  // namespace sv

extern "C" sv_status sv_schedule_admit(const float *conf, int B, int K, const float *speed,
                                       int n_speed, int32_t *lengths, float *tau_out,
                                       void *stream) {
    if (!conf || !speed || !lengths) return SV_ERR_ARG;
    if (B < 1 || K < 1 || K > SV_MAX_K || static_cast<long long>(B) * K > sv::kAdmitMax ||
        n_speed < 1)
        return SV_ERR_SHAPE;
    int N = 1;
    while (N < B * K) N <<= 1;
    const size_t smem = static_cast<size_t>(N) * (sizeof(double) + sizeof(int));
    static bool attr_set[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return sv::note_cuda(e);
    if (!attr_set[dev & 63]) {
        e = cudaFuncSetAttribute(sv::admit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(sv::kAdmitMax * (sizeof(double) + sizeof(int))));
        if (e != cudaSuccess) return sv::note_cuda(e);
        attr_set[dev & 63] = true;
    }
    return sv::note_cuda(sv::launch_pdl(sv::admit_kernel, dim3(1), dim3(sv::kAdmitThreads), smem,
                                        static_cast<cudaStream_t>(stream), conf, B, K, speed,
                                        n_speed, lengths, tau_out));
}
