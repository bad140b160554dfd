// sv_admit.cu -- hardware-aware admission of draft tokens (one CTA).
//
// Method (cited as page title + section): umans.ai, "DeepSeek V4 Pro DSpark:
// the model isn't ready, the architecture is", section "What DSpark adds",
// item "2. Verify smarter" -- the engine's verification rate is measured
// once per batch size; at each step the candidates of all live requests are
// ranked by survival chance and taken one by one while the expected number
// of accepted tokens times the measured rate at the resulting batch size
// still grows.
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
// Kernel (one CTA): per-row products in fp64 in the same order as the
// definition; a stable block radix sort of (S, candidate index) pairs,
// descending in S (candidates enter in index order, so ties stay in index
// order); an fp64 block scan of the sorted S for E(k); and a block-wide
// minimum for the first k at which f stops rising.
#include <cfloat>
#include <climits>
#include <atomic>
#include <cstdint>

#include <cub/block/block_radix_sort.cuh>
#include <cub/block/block_scan.cuh>

#include "sv.h"
#include "sv_device.cuh"
#include "sv_host.h"

namespace sv {

constexpr int kAdmitMax = SV_MAX_ADMIT;     // B * K candidates in one CTA

template <int THREADS, int kAdmitItems>
struct AdmitSort {
    using Sort = cub::BlockRadixSort<double, THREADS, kAdmitItems, int, 5>;
    using Scan = cub::BlockScan<double, THREADS>;
    union Storage {
        typename Sort::TempStorage sort;
        typename Scan::TempStorage scan;
    };
};

template <int THREADS, int kAdmitItems>
__global__ void __launch_bounds__(THREADS) admit_kernel(const float *__restrict__ conf, int B,
                                                        int K, const float *__restrict__ speed,
                                                        int n_speed, int32_t *lengths,
                                                        float *tau_out) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto &tmp = *reinterpret_cast<typename AdmitSort<THREADS, kAdmitItems>::Storage *>(smem_raw);
    __shared__ int s_stop;
    __shared__ double s_last;
    const int tid = threadIdx.x;
    griddep_wait();
    griddep_launch_dependents();
    const int n = B * K;

    // 1. Prefix survival of every candidate; thread t holds candidates
    //    t * 8 .. t * 8 + 7 (index order).  Padding sorts last (key -1).
    double key[kAdmitItems];
    int idx[kAdmitItems];
#pragma unroll
    for (int q = 0; q < kAdmitItems; ++q) {
        key[q] = -1.0;
        idx[q] = INT_MAX;
    }
    {
        // survival products need the row's earlier positions: a thread walks
        // each row that its candidates touch from the row start.
        const int c0 = tid * kAdmitItems;
        if (c0 < n) {
            int b = c0 / K, i = c0 - b * K;
            double S = 1.0;
            for (int j = 0; j < i; ++j) {
                double c = static_cast<double>(__ldg(conf + static_cast<long long>(b) * K + j));
                c = isnan(c) ? 0.0 : fmin(fmax(c, 0.0), 1.0);
                S = S * c;
            }
#pragma unroll
            for (int q = 0; q < kAdmitItems; ++q) {
                const int cq = c0 + q;
                if (cq < n) {
                    if (i == K) { ++b; i = 0; S = 1.0; }
                    double c = static_cast<double>(__ldg(conf + cq));
                    c = isnan(c) ? 0.0 : fmin(fmax(c, 0.0), 1.0);
                    S = S * c;
                    key[q] = S;
                    idx[q] = cq;
                    ++i;
                }
            }
        }
    }
    if (tid == 0) s_stop = INT_MAX;

    // 2. Admission order: S descending, ties by index (stable sort).
    typename AdmitSort<THREADS, kAdmitItems>::Sort(tmp.sort).SortDescending(key, idx);
    __syncthreads();

    // 3. Exclusive prefix of the sorted survivals: thread totals, then a
    //    block scan.
    double run = 0.0;
#pragma unroll
    for (int q = 0; q < kAdmitItems; ++q)
        if (key[q] >= 0.0) run += key[q];
    double pre;
    typename AdmitSort<THREADS, kAdmitItems>::Scan(tmp.scan).ExclusiveSum(run, pre);

    // 4. First k whose admission does not raise f (or leaves the table).
    const int r0 = tid * kAdmitItems;
    int stop = INT_MAX;
#pragma unroll
    for (int q = 0; q < kAdmitItems; ++q) {
        const int k = r0 + q;
        if (stop == INT_MAX && k <= n) {
            bool fail;
            if (k >= n || B + k + 1 >= n_speed) {
                fail = true;
            } else {
                const double Ek = static_cast<double>(B) + pre;
                const double fk = Ek * static_cast<double>(__ldg(speed + B + k));
                const double f1 = (Ek + key[q]) * static_cast<double>(__ldg(speed + B + k + 1));
                fail = !(f1 > fk);
            }
            if (fail) stop = k;
            else pre += key[q];
        }
    }
    if (stop != INT_MAX) atomicMin(&s_stop, stop);
    __syncthreads();
    int admitted = s_stop;
    if (admitted == INT_MAX) admitted = n;   // every candidate admitted
    if (B >= n_speed) admitted = 0;

    // 5. Per-row counts and the threshold.
    for (int b = tid; b < B; b += THREADS) lengths[b] = 0;
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kAdmitItems; ++q) {
        const int k = r0 + q;
        if (k < admitted) atomicAdd(&lengths[idx[q] / K], 1);
        if (k == admitted - 1) s_last = key[q];
    }
    __syncthreads();
    if (tid == 0 && tau_out)
        *tau_out = admitted > 0 ? static_cast<float>(s_last) : __int_as_float(0x7f800000);
}

}  // namespace sv

template <int THREADS, int ITEMS>
static sv_status launch_admit(const float *conf, int B, int K, const float *speed, int n_speed,
                              int32_t *lengths, float *tau_out, cudaStream_t st) {
    constexpr size_t smem = sizeof(typename sv::AdmitSort<THREADS, ITEMS>::Storage);
    // Set once per device; threads that race on it set the same value.
    static std::atomic<bool> attr_set[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return sv::note_cuda(e);
    if (!attr_set[dev & 63].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(sv::admit_kernel<THREADS, ITEMS>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return sv::note_cuda(e);
        attr_set[dev & 63].store(true, std::memory_order_release);
    }
    return sv::note_cuda(sv::launch_pdl(sv::admit_kernel<THREADS, ITEMS>, dim3(1), dim3(THREADS), smem, st,
                                        conf, B, K, speed, n_speed, lengths, tau_out));
}

extern "C" sv_status sv_schedule_admit(const float *conf, int B, int K, const float *speed,
                                       int n_speed, int32_t *lengths, float *tau_out,
                                       void *stream) {
    sv::NvtxRange nvtx_range("sv_schedule_admit");
    if (!conf || !speed || !lengths) return SV_ERR_ARG;
    if (B < 1 || K < 1 || K > SV_MAX_K || static_cast<long long>(B) * K > sv::kAdmitMax ||
        n_speed < 1)
        return SV_ERR_SHAPE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (B * K <= 256 * 8)
        return launch_admit<256, 8>(conf, B, K, speed, n_speed, lengths, tau_out, st);
    return launch_admit<512, 16>(conf, B, K, speed, n_speed, lengths, tau_out, st);
}
