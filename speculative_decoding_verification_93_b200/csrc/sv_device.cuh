// sv_device.cuh -- device helpers for the verification kernels (sm_100a).
//
// Philox4x32-10 follows Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers:
// As Easy as 1, 2, 3" (SC'11): each round multiplies the two even words by the
// round multipliers, XORs the high halves with the odd words and the key,
// keeps the low halves, permutes the words, and bumps the key by the Weyl
// constants.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace sv {

// ---------------------------------------------------------------------------
// Philox4x32-10 and the verification uniforms.
// ---------------------------------------------------------------------------
struct Philox4 { uint32_t w[4]; };

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, uint32_t k0, uint32_t k1) {
    constexpr uint32_t kMulA = 0xD2511F53u, kMulB = 0xCD9E8D57u;
    constexpr uint32_t kWeylA = 0x9E3779B9u, kWeylB = 0xBB67AE85u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t hiA = __umulhi(kMulA, c0), loA = kMulA * c0;
        const uint32_t hiB = __umulhi(kMulB, c2), loB = kMulB * c2;
        const uint32_t n0 = hiB ^ c1 ^ k0;
        const uint32_t n2 = hiA ^ c3 ^ k1;
        c0 = n0; c1 = loB; c2 = n2; c3 = loA;
        k0 += kWeylA; k1 += kWeylB;
    }
    Philox4 o;
    o.w[0] = c0; o.w[1] = c1; o.w[2] = c2; o.w[3] = c3;
    return o;
}

// u(seed, row, pos, draw): top 24 bits of word 0 of the block for counter
// (row_lo, pos, draw, row_hi) under key (seed_lo, seed_hi); exact in fp32.
__device__ __forceinline__ float uniform24(uint64_t seed, uint64_t row, uint32_t pos,
                                           uint32_t draw) {
    const Philox4 o = philox4x32_10(static_cast<uint32_t>(row), pos, draw,
                                    static_cast<uint32_t>(row >> 32),
                                    static_cast<uint32_t>(seed),
                                    static_cast<uint32_t>(seed >> 32));
    return static_cast<float>(o.w[0] >> 8) * (1.0f / 16777216.0f);
}

// ---------------------------------------------------------------------------
// Arithmetic.
// ---------------------------------------------------------------------------
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kNegInf = -__builtin_huge_valf();

// 2^x on the special-function unit (ex2.approx, flush-to-zero); 2^-inf = 0.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Widen the two bf16 halves of a 32-bit word to fp32 (exact).  The element
// at the lower address is the low half.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162 *>(&a);
    __nv_bfloat162 y = *reinterpret_cast<__nv_bfloat162 *>(&b);
    __nv_bfloat162 r = __hmax2(x, y);
    return *reinterpret_cast<uint32_t *>(&r);
}

// Combine two (max, sum) online-softmax partials taken at scale k = log2e/T:
// sum is relative to its own max.  A partial with max -inf has sum 0.
__device__ __forceinline__ void lse_merge(float &m, float &s, float m2, float s2, float k) {
    const float mn = fmaxf(m, m2);
    if (mn == kNegInf) { m = mn; s = 0.f; return; }
    s = s * ex2((m - mn) * k) + s2 * ex2((m2 - mn) * k);
    m = mn;
}

// ---------------------------------------------------------------------------
// Memory.
// ---------------------------------------------------------------------------
// Streaming 16-byte load: read-only, not kept in L1 (the pass touches every
// byte once).
__device__ __forceinline__ uint4 ld_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16-byte load that may be cached (re-reads of recently streamed rows).
__device__ __forceinline__ uint4 ld_reuse(const void *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// Geometry of one logit vector of V elements split into a head (elements
// before the first 16-byte boundary), n16 full 16-byte units, and a tail.
struct VecGeom {
    const char *base;   // element 0
    const char *body;   // first 16-byte aligned byte (base + head * esize)
    int head;
    int n16;
    int tail;
};

template <int ESIZE>
__device__ __forceinline__ VecGeom vec_geom(const void *base, int V) {
    constexpr int kPer = 16 / ESIZE;
    VecGeom g;
    g.base = static_cast<const char *>(base);
    const uint32_t mis = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(base) & 15u);
    int h = mis ? static_cast<int>((16u - mis) / ESIZE) : 0;
    if (h > V) h = V;
    g.head = h;
    g.body = g.base + h * ESIZE;
    g.n16 = (V - h) / kPer;
    g.tail = V - h - g.n16 * kPer;
    return g;
}

// Scalar element load widened to fp32.
template <int ESIZE>
__device__ __forceinline__ float ld_elem(const char *base, long long v) {
    if (ESIZE == 4) return __ldg(reinterpret_cast<const float *>(base) + v);
    const unsigned short h = __ldg(reinterpret_cast<const unsigned short *>(base) + v);
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// Element value pattern for padding: -inf in both dtypes.
template <int ESIZE> __device__ __forceinline__ uint32_t neg_inf_word();
template <> __device__ __forceinline__ uint32_t neg_inf_word<4>() { return 0xff800000u; }
template <> __device__ __forceinline__ uint32_t neg_inf_word<2>() { return 0xff80ff80u; }

// A partial unit (head or tail): up to 16/ESIZE elements starting at element
// `first`, padded with -inf, packed like a body unit.
template <int ESIZE>
__device__ __forceinline__ uint4 ld_partial_unit(const char *base, int first, int count) {
    uint32_t w[4];
    const uint32_t pad = neg_inf_word<ESIZE>();
    w[0] = w[1] = w[2] = w[3] = pad;
    if (ESIZE == 4) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (e < count) w[e] = __float_as_uint(ld_elem<4>(base, first + e));
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (e < count) {
                const uint32_t h = __float_as_uint(ld_elem<2>(base, first + e)) >> 16;
                w[e >> 1] = (e & 1) ? ((w[e >> 1] & 0x0000ffffu) | (h << 16))
                                    : ((w[e >> 1] & 0xffff0000u) | h);
            }
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Element e (0 .. 16/ESIZE-1) of a packed unit, widened to fp32.
template <int ESIZE>
__device__ __forceinline__ float unit_elem(const uint4 &u, int e) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    if (ESIZE == 4) return __uint_as_float(w[e]);
    return (e & 1) ? bf16_hi(w[e >> 1]) : bf16_lo(w[e >> 1]);
}

// Element pair q (elements 2q, 2q+1) of a packed unit, widened to fp32.
template <int ESIZE>
__device__ __forceinline__ float2 unit_pair(const uint4 &u, int q) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    if (ESIZE == 2) return make_float2(bf16_lo(w[q]), bf16_hi(w[q]));
    return make_float2(__uint_as_float(w[2 * q]), __uint_as_float(w[2 * q + 1]));
}

// Online (max, sum) update with a batch of units.  The batch max is a
// balanced tree of packed bf16x2 (or f32) max operations; the running sum is
// rescaled once if the max grew; then one exp2 per element with the
// argument formed by one packed FMA, z * k + c with c = RN(-m * k).  The
// rounding of c is exact to recover, -m * k = c + e with e = fma(-m, k, -c),
// and common to the batch, so the batch sum is multiplied by 2^e
// (= 1 + e ln 2 to far below fp32 resolution, |e| < 1e-6).  Two packed
// accumulators halve the add chain.
template <int ESIZE, int N>
__device__ __forceinline__ void lse_update(const uint4 (&v)[N], float k, float &m, float &s) {
    float bm;
    if (ESIZE == 2) {
        uint32_t t[N];
#pragma unroll
        for (int j = 0; j < N; ++j) t[j] = bmax2(bmax2(v[j].x, v[j].y), bmax2(v[j].z, v[j].w));
#pragma unroll
        for (int w = 1; w < N; w <<= 1)
#pragma unroll
            for (int j = 0; j + w < N; j += 2 * w) t[j] = bmax2(t[j], t[j + w]);
        bm = fmaxf(bf16_lo(t[0]), bf16_hi(t[0]));
    } else {
        float t[N];
#pragma unroll
        for (int j = 0; j < N; ++j)
            t[j] = fmaxf(fmaxf(__uint_as_float(v[j].x), __uint_as_float(v[j].y)),
                         fmaxf(__uint_as_float(v[j].z), __uint_as_float(v[j].w)));
#pragma unroll
        for (int w = 1; w < N; w <<= 1)
#pragma unroll
            for (int j = 0; j + w < N; j += 2 * w) t[j] = fmaxf(t[j], t[j + w]);
        bm = t[0];
    }
    if (bm == kNegInf) return;              // nothing but padding / -inf
    if (bm > m) {
        s = (m == kNegInf) ? 0.f : s * ex2((m - bm) * k);
        m = bm;
    }
    const float c = -m * k;
    const float e = fmaf(-m, k, -c);
    const float2 cc = make_float2(c, c), kk = make_float2(k, k);
    float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < N; ++j) {
        const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
        if (ESIZE == 2) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 z = make_float2(bf16_lo(w[q]), bf16_hi(w[q]));
                const float2 d = __ffma2_rn(z, kk, cc);
                const float2 e = make_float2(ex2(d.x), ex2(d.y));
                if (q & 1) acc1 = __fadd2_rn(acc1, e); else acc0 = __fadd2_rn(acc0, e);
            }
        } else {
#pragma unroll
            for (int q = 0; q < 4; q += 2) {
                const float2 z = make_float2(__uint_as_float(w[q]), __uint_as_float(w[q + 1]));
                const float2 d = __ffma2_rn(z, kk, cc);
                const float2 e = make_float2(ex2(d.x), ex2(d.y));
                if (q & 2) acc1 = __fadd2_rn(acc1, e); else acc0 = __fadd2_rn(acc0, e);
            }
        }
    }
    s = fmaf((acc0.x + acc0.y) + (acc1.x + acc1.y), fmaf(e, 0.69314718055994531f, 1.f), s);
}

template <int ESIZE>
__device__ __forceinline__ void consider_unit(const uint4 &u, int first, float &best, int &bidx) {
    constexpr int kPer = 16 / ESIZE;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
        const float x = unit_elem<ESIZE>(u, e);
        if (x > best) { best = x; bidx = first + e; }
    }
}

}  // namespace sv

// ---------------------------------------------------------------------------
// mbarrier and bulk-copy (TMA) primitives, sm_90+ PTX.  Every wait is bounded
// by wall time read from %globaltimer.
// ---------------------------------------------------------------------------
namespace sv {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or the hint (ns) elapses, instead of spinning on issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase with the given parity to complete; false after
// `limit_ns` of wall time (the caller then reports a timeout and unwinds).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

// Bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completion counted on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst_smem)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Named barrier 1 over a group of N threads (the consumer warps); barrier 0
// stays reserved for __syncthreads.
template <int N>
__device__ __forceinline__ void group_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory");
}

// Programmatic dependent launch (sm_90+): a kernel launched with
// programmatic stream serialisation may start before the previous kernel in
// the stream has finished; griddep_wait() blocks until that kernel has
// completed and its writes are visible, and must precede every global
// access that could conflict with it.  griddep_launch_dependents() lets the
// next kernel start launching early.
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace sv

namespace sv {
// atomicAdd with acquire-release semantics at GPU scope: the caller's earlier
// writes are visible to whoever observes the new value, and the caller's
// later reads see every write released before earlier increments of the
// same counter.
__device__ __forceinline__ int atom_add_acq_rel(int *p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;"
                 : "=r"(old)
                 : "l"(p), "r"(v)
                 : "memory");
    return old;
}

// Verify length of one row from its K confidences: S_i = prod_{j<=i}
// clamp(c_{j-1}, 0, 1) (NaN counts as 0), left to right in fp32, and
// L = max{i in 0..K : S_i >= tau} with S_0 = 1.  The schedule kernel and the
// fused schedule-and-verify prologue both call this, so their lengths agree
// bit for bit.
__device__ __forceinline__ int schedule_length(const float *__restrict__ c, int K, float tau) {
    float S = 1.f;
    int L = 0;
    for (int i = 1; i <= K; ++i) {
        float ci = __ldg(c + (i - 1));
        ci = isnan(ci) ? 0.f : fminf(fmaxf(ci, 0.f), 1.f);
        S = S * ci;
        if (S >= tau) L = i;
    }
    return L;
}

// Relaxed load of a flag that other CTAs update (a stale value only makes
// the caller do redundant work).
__device__ __forceinline__ int ld_relaxed(const int *p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Acquire load at GPU scope: later reads see every write released before
// the value read was written.
__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Relaxed OR into a 64-bit flag word at GPU scope, no result.
__device__ __forceinline__ void red_or_relaxed(unsigned long long *p, unsigned long long v) {
    asm volatile("red.relaxed.gpu.global.or.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
}  // namespace sv
