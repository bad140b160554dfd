// sv_sts.cu -- per-position temperature scaling of the confidence head.
//
// Method (cited as page title + section): umans.ai, "DeepSeek V4 Pro DSpark:
// the model isn't ready, the architecture is", section "What DSpark adds",
// item "2. Verify smarter" -- the head's raw confidences are overconfident
// (3-8% expected calibration error), and a temperature for each position,
// chosen on blocks kept aside, lowers that to about 1%; zhichai.net DSpark topic, "Under
// the hood": the head is calibrated by Sequential Temperature Scaling.
//
// Reading: the head predicts survival of position i given that every
// earlier position survived, so position i of a held-out block is observed
// iff i <= a (its accepted length) and survived iff i < a; each position is
// fitted on the blocks that reached it.  T_i = 1/beta_i minimises the binary
// negative log-likelihood NLL(beta) = sum log(1 + exp(-s beta l)), s = +1
// survived, -1 not, over beta in [1/tmax, 1/tmin].  NLL is convex in beta.
//
// Kernel: one persistent grid, launched cooperatively so that every CTA is
// resident, with a grid barrier between passes (bounded in wall time: on
// timeout the temperatures come out NaN instead of the kernel hanging).
// Every sum is in fp64 with a fixed order, so results do not depend on
// scheduling.
//   1. Init pass: per (position, chunk of 2048 blocks), the observed count
//      and NLL' at both ends of the interval; the CTA owning a position adds
//      the chunk partials in order and settles end points and degenerate
//      cases.
//   2. Newton passes: NLL'(beta) and NLL''(beta) of every unconverged
//      position; its owner takes a safeguarded Newton step inside the bracket
//      where NLL' changes sign (bisection whenever the step would leave it),
//      until the step is below 1e-10 of beta (the rounding noise of the sums
//      sets the floor; the output is fp32).
//   3. Final pass: T, and the 15-bin calibration error of sigmoid(l) and
//      sigmoid(l / T_i) over every observed (block, position).
#include <cmath>
#include <cstdint>

#include "sv.h"
#include "sv_device.cuh"
#include "sv_host.h"

namespace sv {

constexpr int kStsThreads = 256;
constexpr int kStsChunk = 2048;          // blocks per CTA
constexpr int kStsBins = 15;

struct StsState {
    double beta, lo, hi;
    int done;
    int pad;
};

struct StsArgs {
    const float *l;      // [N, K]
    const int32_t *a;    // [N]
    int N, K, nchunk;
    double lo0, hi0;     // 1/tmax, 1/tmin
    StsState *st;        // [K]
    double *part;        // [K, nchunk, 3]
    int *bar;            // [0] arrivals, [1] generation
    double *epart;       // [nchunk, 2 * kStsBins + 1]
    float *T;            // [K] out
    float *ece;          // [2] out, nullable
};

__device__ __forceinline__ double sts_sigmoid(double x) {
    if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
    const double e = exp(x);
    return e / (1.0 + e);
}

// Fixed-order block sum of three values (all threads get the result).
__device__ __forceinline__ void block_sum3(double &x, double &y, double &z) {
    __shared__ double s[3][kStsThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        x += __shfl_xor_sync(0xffffffffu, x, o);
        y += __shfl_xor_sync(0xffffffffu, y, o);
        z += __shfl_xor_sync(0xffffffffu, z, o);
    }
    if (lane == 0) { s[0][warp] = x; s[1][warp] = y; s[2][warp] = z; }
    __syncthreads();
    x = y = z = 0.0;
    for (int w = 0; w < kStsThreads / 32; ++w) { x += s[0][w]; y += s[1][w]; z += s[2][w]; }
    __syncthreads();
}

__device__ __forceinline__ int ld_acquire_i32(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Wall-time bound of a grid-barrier wait (1 s; no legitimate wait comes
// close) and the number of waits that ran out.  Both are set and read only
// through the test exports at the end of this file.
__device__ unsigned long long g_sts_wait_limit_ns = 1000000000ull;
__device__ unsigned int g_sts_timeouts;

// Grid barrier (sense by generation).  Every CTA of the cooperative launch
// is resident, so a wait ends as soon as the last CTA arrives; the wait is
// still bounded in wall time.  Returns false (in every thread) on timeout
// and counts the timeout.
__device__ bool grid_barrier(int *bar, int nblocks) {
    __shared__ int ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        const int gen = ld_acquire_i32(&bar[1]);
        __threadfence();
        int good = 1;
        if (atomicAdd(&bar[0], 1) + 1 == nblocks) {
            bar[0] = 0;
            __threadfence();
            atomicAdd(&bar[1], 1);
        } else {
            const uint64_t t0 = global_ns();
            const uint64_t limit = g_sts_wait_limit_ns;
            while (ld_acquire_i32(&bar[1]) == gen) {
                if (global_ns() - t0 > limit) {
                    good = 0;
                    atomicAdd(&g_sts_timeouts, 1u);
                    break;
                }
                __nanosleep(64);
            }
        }
        __threadfence();
        ok = good;
    }
    __syncthreads();
    return ok != 0;
}

// Partial sums of one (position, chunk) unit at `beta`; init: (count,
// NLL'(lo), NLL'(hi)), else (NLL'(beta), NLL''(beta), 0).
__device__ void sts_unit(const StsArgs &s, int i, int chunk, bool init, double beta) {
    double x = 0.0, y = 0.0, z = 0.0;
    const int n0 = chunk * kStsChunk, n1 = min(n0 + kStsChunk, s.N);
    for (int n = n0 + static_cast<int>(threadIdx.x); n < n1; n += kStsThreads) {
        const int an = __ldg(&s.a[n]);
        if (an < 0 || i > an) continue;
        const double sg = (i < an) ? 1.0 : -1.0;
        const double v = static_cast<double>(__ldg(&s.l[static_cast<long long>(n) * s.K + i]));
        if (init) {
            x += 1.0;
            y += -sg * v * sts_sigmoid(-sg * s.lo0 * v);
            z += -sg * v * sts_sigmoid(-sg * s.hi0 * v);
        } else {
            const double q = sts_sigmoid(-sg * beta * v);   // sigmoid(-s beta l)
            x += -sg * v * q;
            y += v * v * q * (1.0 - q);
        }
    }
    block_sum3(x, y, z);
    if (threadIdx.x == 0) {
        double *pp = s.part + (static_cast<long long>(i) * s.nchunk + chunk) * 3;
        pp[0] = x; pp[1] = y; pp[2] = z;
    }
}

// The owner of position i adds its chunk partials in order and updates it.
__device__ void sts_update(const StsArgs &s, int i, bool init) {
    double X = 0.0, Y = 0.0, Z = 0.0;
    for (int c = 0; c < s.nchunk; ++c) {
        const double *q = s.part + (static_cast<long long>(i) * s.nchunk + c) * 3;
        X += __ldcg(q); Y += __ldcg(q + 1); Z += __ldcg(q + 2);
    }
    StsState *ps = s.st + i;
    if (init) {
        StsState st;
        st.lo = s.lo0; st.hi = s.hi0; st.pad = 0; st.done = 1;
        if (X == 0.0) st.beta = 1.0;                     // no observed block
        else if (Y == 0.0 && Z == 0.0) st.beta = 1.0;    // every logit 0: flat
        else if (Y >= 0.0) st.beta = s.lo0;              // rising from the low end
        else if (Z <= 0.0) st.beta = s.hi0;              // falling to the high end
        else {
            st.beta = fmin(fmax(1.0, s.lo0), s.hi0);
            st.done = 0;
        }
        *ps = st;
        return;
    }
    StsState st;
    st.beta = __ldcg(&ps->beta); st.lo = __ldcg(&ps->lo); st.hi = __ldcg(&ps->hi);
    st.done = 0; st.pad = 0;
    const double g = X, h = Y;
    if (g == 0.0) { st.done = 1; *ps = st; return; }
    if (g < 0.0) st.lo = st.beta; else st.hi = st.beta;
    // A converged Newton step ends the search before the bracket test: at
    // the root the step lands on the bracket end just moved to beta.
    if (h > 0.0 && fabs(g / h) <= 1e-10 * st.beta) {
        st.beta = fmin(fmax(st.beta - g / h, st.lo), st.hi);
        st.done = 1;
        *ps = st;
        return;
    }
    double nb = st.beta - g / h;
    if (!(h > 0.0) || !(nb >= st.lo && nb <= st.hi)) nb = 0.5 * (st.lo + st.hi);
    if (fabs(nb - st.beta) <= 1e-10 * st.beta || st.hi - st.lo <= 1e-10 * st.hi) st.done = 1;
    st.beta = nb;
    *ps = st;
}

constexpr int kStsMaxIter = 64;    // safeguarded Newton; bisection alone needs < 40

__global__ void __launch_bounds__(kStsThreads) sts_fit_kernel(StsArgs s) {
    const int tid = threadIdx.x;
    const int G = gridDim.x, g = blockIdx.x;
    const int units = s.K * s.nchunk;
    bool ok = true;
    // 1. init pass
    for (int u = g; u < units; u += G) sts_unit(s, u / s.nchunk, u % s.nchunk, true, 0.0);
    ok = grid_barrier(s.bar, G);
    if (ok && tid == 0)
        for (int i = g; i < s.K; i += G) sts_update(s, i, true);
    if (ok) ok = grid_barrier(s.bar, G);
    // 2. Newton passes
    __shared__ int s_open;
    for (int it = 0; ok && it < kStsMaxIter; ++it) {
        if (tid == 0) {
            int open = 0;
            for (int i = 0; i < s.K; ++i) open |= !__ldcg(&s.st[i].done);
            s_open = open;
        }
        __syncthreads();
        if (!s_open) break;   // every CTA reads the same states after the barrier
        for (int u = g; u < units; u += G) {
            const int i = u / s.nchunk;
            if (__ldcg(&s.st[i].done)) continue;
            sts_unit(s, i, u % s.nchunk, false, __ldcg(&s.st[i].beta));
        }
        ok = grid_barrier(s.bar, G);
        if (ok && tid == 0)
            for (int i = g; i < s.K; i += G)
                if (!__ldcg(&s.st[i].done)) sts_update(s, i, false);
        if (ok) ok = grid_barrier(s.bar, G);
    }
    // 3. outputs
    __shared__ double invT[SV_MAX_K];
    for (int i = tid; i < s.K; i += kStsThreads) {
        invT[i] = ok ? __ldcg(&s.st[i].beta) : __longlong_as_double(0x7ff8000000000000ll);
        if (g == 0) s.T[i] = static_cast<float>(1.0 / invT[i]);
    }
    __syncthreads();
    if (!s.ece || !ok) return;
    double d0[kStsBins], d1[kStsBins];
    for (int chunk = g; chunk < s.nchunk; chunk += G) {
#pragma unroll
        for (int m = 0; m < kStsBins; ++m) d0[m] = d1[m] = 0.0;
        double cnt = 0.0;
        const int n0 = chunk * kStsChunk, n1 = min(n0 + kStsChunk, s.N);
        for (int n = n0 + tid; n < n1; n += kStsThreads) {
            const int an = __ldg(&s.a[n]);
            if (an < 0) continue;
            for (int i = 0; i < s.K && i <= an; ++i) {
                const double v =
                    static_cast<double>(__ldg(&s.l[static_cast<long long>(n) * s.K + i]));
                const double y = (i < an) ? 1.0 : 0.0;
                const double c0 = sts_sigmoid(v), c1 = sts_sigmoid(v * invT[i]);
                const int m0 = min(static_cast<int>(c0 * kStsBins), kStsBins - 1);
                const int m1 = min(static_cast<int>(c1 * kStsBins), kStsBins - 1);
#pragma unroll
                for (int m = 0; m < kStsBins; ++m) {
                    d0[m] += (m == m0) ? y - c0 : 0.0;
                    d1[m] += (m == m1) ? y - c1 : 0.0;
                }
                cnt += 1.0;
            }
        }
        double *pp = s.epart + static_cast<long long>(chunk) * (2 * kStsBins + 1);
#pragma unroll
        for (int m = 0; m < kStsBins; ++m) {
            double x = d0[m], y = d1[m], z = (m == 0) ? cnt : 0.0;
            block_sum3(x, y, z);
            if (tid == 0) {
                pp[m] = x;
                pp[kStsBins + m] = y;
                if (m == 0) pp[2 * kStsBins] = z;
            }
        }
    }
    if (!grid_barrier(s.bar, G)) return;
    if (g != 0 || tid != 0) return;
    double e0 = 0.0, e1 = 0.0, c = 0.0;
    for (int m = 0; m < kStsBins; ++m) {
        double x = 0.0, y = 0.0;
        for (int q = 0; q < s.nchunk; ++q) {
            const double *r = s.epart + static_cast<long long>(q) * (2 * kStsBins + 1);
            x += __ldcg(r + m);
            y += __ldcg(r + kStsBins + m);
        }
        e0 += fabs(x);
        e1 += fabs(y);
    }
    for (int q = 0; q < s.nchunk; ++q)
        c += __ldcg(s.epart + static_cast<long long>(q) * (2 * kStsBins + 1) + 2 * kStsBins);
    s.ece[0] = static_cast<float>(c > 0.0 ? e0 / c : 0.0);
    s.ece[1] = static_cast<float>(c > 0.0 ? e1 / c : 0.0);
}

__global__ void sts_apply_kernel(const float *__restrict__ l, const float *__restrict__ T,
                                 long long total, int K, float *__restrict__ conf) {
    griddep_wait();
    griddep_launch_dependents();
    for (long long q = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; q < total;
         q += static_cast<long long>(gridDim.x) * blockDim.x) {
        const float x = __ldg(&l[q]) / __ldg(&T[q % K]);
        conf[q] = 1.f / (1.f + expf(-x));
    }
}

struct StsPlan {
    int nchunk;
    size_t off_st, off_part, off_bar, off_epart, bytes;
};

static bool sts_plan(int N, int K, StsPlan *p) {
    if (N < 1 || K < 1 || K > SV_MAX_K) return false;
    p->nchunk = (N + kStsChunk - 1) / kStsChunk;
    auto align16 = [](size_t o) { return (o + 15) & ~static_cast<size_t>(15); };
    size_t off = 0;
    p->off_st = off;     off = align16(off + sizeof(StsState) * K);
    p->off_part = off;   off = align16(off + sizeof(double) * 3 * static_cast<size_t>(K) * p->nchunk);
    p->off_bar = off;    off = align16(off + sizeof(int) * 2);
    p->off_epart = off;  off = align16(off + sizeof(double) * (2 * kStsBins + 1) * p->nchunk);
    p->bytes = off;
    return true;
}

}  // namespace sv

extern "C" size_t sv_sts_workspace_bytes(int N, int K) {
    sv::StsPlan p;
    if (!sv::sts_plan(N, K, &p)) return 0;
    return p.bytes;
}

extern "C" sv_status sv_sts_fit(const float *logits, const int32_t *accept_len, int N, int K,
                                float tmin, float tmax, float *temperature, float *ece,
                                void *workspace, size_t workspace_bytes, void *stream) {
    sv::NvtxRange nvtx_range("sv_sts_fit");
    if (!logits || !accept_len || !temperature || !workspace) return SV_ERR_ARG;
    if (!(tmin > 0.f) || !(tmax > tmin) || !std::isfinite(tmax)) return SV_ERR_ARG;
    sv::StsPlan p;
    if (!sv::sts_plan(N, K, &p)) return SV_ERR_SHAPE;
    if (reinterpret_cast<uintptr_t>(workspace) & 15) return SV_ERR_ARG;
    if (workspace_bytes < p.bytes) return SV_ERR_WORKSPACE;
    char *w = static_cast<char *>(workspace);
    sv::StsArgs s;
    s.l = logits; s.a = accept_len; s.N = N; s.K = K; s.nchunk = p.nchunk;
    s.lo0 = 1.0 / static_cast<double>(tmax);
    s.hi0 = 1.0 / static_cast<double>(tmin);
    s.st = reinterpret_cast<sv::StsState *>(w + p.off_st);
    s.part = reinterpret_cast<double *>(w + p.off_part);
    s.bar = reinterpret_cast<int *>(w + p.off_bar);
    s.epart = reinterpret_cast<double *>(w + p.off_epart);
    s.T = temperature; s.ece = ece;
    int dev = 0, sms = 0, per = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, sv::sts_fit_kernel,
                                                          sv::kStsThreads, 0);
    if (e != cudaSuccess) return sv::note_cuda(e);
    const long long units = static_cast<long long>(K) * p.nchunk;
    const long long cap = static_cast<long long>(sms) * (per > 0 ? per : 1);
    const int grid = static_cast<int>(units < cap ? units : cap);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The barrier words start at zero; the kernel leaves them at zero again.
    e = cudaMemsetAsync(s.bar, 0, sizeof(int) * 2, st);
    if (e != cudaSuccess) return sv::note_cuda(e);
    // Cooperative launch: every CTA resident, which the grid barrier needs.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(sv::kStsThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, sv::sts_fit_kernel, s);
    if (e != cudaSuccess) return sv::note_cuda(e);
    return sv::note_cuda(cudaGetLastError());
}

extern "C" sv_status sv_sts_apply(const float *logits, const float *temperature, int N, int K,
                                  float *conf_out, void *stream) {
    sv::NvtxRange nvtx_range("sv_sts_apply");
    if (!logits || !temperature || !conf_out) return SV_ERR_ARG;
    if (N < 1 || K < 1 || K > SV_MAX_K) return SV_ERR_SHAPE;
    const long long total = static_cast<long long>(N) * K;
    const int blocks = static_cast<int>((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
    return sv::note_cuda(sv::launch_pdl(sv::sts_apply_kernel, dim3(blocks), dim3(256), 0,
                                        static_cast<cudaStream_t>(stream), logits, temperature,
                                        total, K, conf_out));
}

// Test exports for the bounded wait of the calibration's grid barrier: set
// the wall-time limit on the current device (0 restores the 1 s default),
// and read-and-clear the count of waits that ran out.  A limit near zero
// makes every CTA but the last to arrive give up at the first barrier, so
// the fit returns with T = NaN instead of waiting: the failure path runs
// without a fault or a hang.
extern "C" sv_status sv_debug_sts_wait_limit(uint64_t limit_ns) {
    const unsigned long long v = limit_ns ? limit_ns : 1000000000ull;
    return sv::note_cuda(cudaMemcpyToSymbol(sv::g_sts_wait_limit_ns, &v, sizeof(v)));
}

extern "C" int sv_debug_sts_timeouts(void) {
    unsigned int n = 0, z = 0;
    if (cudaMemcpyFromSymbol(&n, sv::g_sts_timeouts, sizeof(n)) != cudaSuccess) return -1;
    if (cudaMemcpyToSymbol(sv::g_sts_timeouts, &z, sizeof(z)) != cudaSuccess) return -1;
    return static_cast<int>(n);
}
