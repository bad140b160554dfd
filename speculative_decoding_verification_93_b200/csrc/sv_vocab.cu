// sv_vocab.cu -- verification with the vocabulary split across ranks (sm_100a).
//
// Method: the rule of sv_verify -- umans.ai, "DeepSeek V4 Pro DSpark: the
// model isn't ready, the architecture is", section "Speculative decoding,
// briefly"; zhichai.net DSpark topic, section "Why LLMs speak so slowly" --
// evaluated where each rank holds only a contiguous slice [v0, v0 + Vs) of
// both models' logits, as a multi-GPU serving engine whose output heads are
// split by vocabulary produces them (zhichai.net topic, "From paper to
// running service in two weeks": the method runs inside vLLM and SGLang on
// 8-GPU nodes; techvisionai "DeepSeek-V4: Breaking the Efficiency Barrier",
// Ch. 7 "Deployment with vLLM").
//
// Three local steps; the caller runs an exchange after each of the first two
// and one at the end:
//   1. vp_stats_kernel, one CTA per (row, slot, chunk) of the slice: the
//      online (max, sum of exp2) of the chunk (greedy rows: max and first
//      argmax), plus -- in chunk 0 -- the logit of the row's draft token when
//      the token falls in the slice.  Exchange: all-gather, rank order.
//   2. vp_decide_kernel, one CTA per row: merges every rank's partials in a
//      fixed order, so every rank holds the same normalisers and takes the
//      same decisions; runs the accept tests; writes the accepted prefix and
//      the accept length.  vp_mass_kernel, several CTAs per row: sums the
//      draw weights of this slice at the final position by segments of
//      16-byte units, the segments by parts, the parts into the slice total
//      (the row's last CTA, found by an atomic count).
//      Exchange: all-gather of the per-row slice totals, rank order.
//   3. vp_draw_kernel, one warp per row: every rank scans the slice totals in
//      rank order and finds the slice that holds the CDF target; only that
//      rank locates the token, from its segment table and then inside one
//      segment.  Other ranks leave -1 there.  Exchange: all-reduce (max) of
//      out_tokens, after which every rank holds the same result.
// Every sum runs in a fixed order; nothing waits on another CTA.
#include <climits>
#include <cstdint>

#include "sv.h"
#include "sv_device.cuh"
#include "sv_host.h"

namespace sv {
namespace vp {

constexpr int kStatsThreads = 256;
constexpr int kStatsWarps = kStatsThreads / 32;
constexpr int kChunkBytes = 64 * 1024;         // target bytes per stats chunk
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s: no legitimate copy comes close
constexpr int kMaxChunks = 64;
constexpr int kDecideThreads = 256;
constexpr int kDecideWarps = kDecideThreads / 32;
constexpr int kMaxSlots = 2 * SV_MAX_K + 1;
constexpr int kMaxSeg = 512;                   // segments per slice vector
constexpr int kSegPerPart = 32;                // segments per mass CTA (a part)
constexpr int kMassThreads = 256;
constexpr int kMassWarps = kMassThreads / 32;
static_assert(kSegPerPart == 32, "the draw loads one part's segment sums, one per lane");
static_assert(kMaxSeg / kSegPerPart <= 32, "the draw loads the part sums, one per lane");
constexpr int kModeDone = -1, kModeP = 0, kModeResidual = 1, kModeOneHot = 2;

struct __align__(16) Record {
    int j;        // draw position
    int mode;     // kModeDone (outputs complete), kModeP, kModeResidual, kModeOneHot
    int xl;       // one-hot mode: slice-local index of x_j, or -1 if outside the slice
    int pad0;
    float u, k;   // draw uniform; log2(e) / T
    float mt, ist, md, isd; // maxima and reciprocal sums: p = 2^((z - mt) k) * ist
    int pad1[2];
};

struct Args {
    const char *zt, *zd;    // slices [B, K+1, Vs], [B, K, Vs]
    int B, K, V, v0, Vs, S, C, nshards, shard;
    int SU, G, P;           // units per segment, segments per table, parts per table
    const int32_t *tokens, *lengths;
    const float *temp;
    uint64_t seed;
    int64_t row_base;
    float4 *stats_local;        // [B, S, C]
    const float4 *stats_all;    // [nshards, B, S, C]
    float2 *mass_local;         // [B]: (mode mass, p mass)
    const float2 *mass_all;     // [nshards, B]
    int32_t *out_tokens, *out_accept, *status;
    float *norm;                // nullable [B, S, 2]
    Record *rec;                // [B]
    float *seg;                 // [B, 2, G] segment sums (draw weight, p weight)
    float *part;                // [B, 2, P] part sums: kSegPerPart segments each, in order
    int *cnt;                   // [B] mass CTAs of the row finished
};

__device__ __forceinline__ bool bad_temperature(float T) {
    return !(T >= 0.f) || isinf(T) || (T > 0.f && T < 1e-6f);
}

template <int ESIZE>
__device__ __forceinline__ const char *tgt_vec(const Args &a, int b, int i) {
    return a.zt + ((static_cast<long long>(b) * (a.K + 1) + i) * a.Vs) * ESIZE;
}
template <int ESIZE>
__device__ __forceinline__ const char *dft_vec(const Args &a, int b, int i) {
    return a.zd + ((static_cast<long long>(b) * a.K + i) * a.Vs) * ESIZE;
}

// ---------------------------------------------------------------------------
// 1. Slice statistics.  One CTA per (row, slot, chunk): the chunk's body is
//    brought into shared memory by one bulk copy per piece of up to 32 KB
//    (cp.async.bulk, mbarrier completion, no multicast), so a CTA holds no
//    load registers and six CTAs fit on an SM: their copies stay in flight
//    while other CTAs reduce.  Each thread reduces its units of the piece in
//    two batches of four (packed bf16x2 max tree, one exp2 per element).
// ---------------------------------------------------------------------------
constexpr int kPieceUnits = 2048;                       // 16-byte units per bulk copy (32 KB)
constexpr int kPieceBytes = kPieceUnits * 16;
constexpr int kUnitsPerThread = kPieceUnits / kStatsThreads;   // 8
static_assert(kUnitsPerThread == 8, "two batches of four units per thread");

template <int ESIZE>
__global__ void __launch_bounds__(kStatsThreads, 6) vp_stats_kernel(Args a) {
    constexpr int kPer = 16 / ESIZE;
    extern __shared__ __align__(128) uint4 piece[];
    __shared__ uint64_t full;
    __shared__ float4 wp[kStatsWarps];
    griddep_wait();
    griddep_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = static_cast<int>(blockIdx.x % a.C);
    const int bs = static_cast<int>(blockIdx.x / a.C);
    const int slot = bs % a.S, b = bs / a.S;
    const int L = __ldg(&a.lengths[b]);
    const float T = __ldg(&a.temp[b]);
    if (L < 0 || L > a.K || bad_temperature(T)) return;   // the decide step marks the row
    const bool greedy = !(T > 0.f);
    const float k = greedy ? 0.f : kLog2e / T;
    int i;
    const char *base;
    if (slot <= a.K) {
        i = slot;
        if (i > L) return;
        base = tgt_vec<ESIZE>(a, b, i);
    } else {
        i = slot - a.K - 1;
        if (greedy || a.zd == nullptr || i >= L) return;
        base = dft_vec<ESIZE>(a, b, i);
    }
    const VecGeom g = vec_geom<ESIZE>(base, a.Vs);
    const int U = (g.n16 + a.C - 1) / a.C;
    const int u0 = min(c * U, g.n16), u1 = min(u0 + U, g.n16);
    const uint32_t pw = neg_inf_word<ESIZE>();
    const uint4 pad = make_uint4(pw, pw, pw, pw);
    if (tid == 0) {
        mbar_init(&full, 1);
        fence_mbar_init();
    }
    __syncthreads();

    float m = kNegInf, s = 0.f;
    int idx = INT_MAX;
    // Head elements (chunk 0, thread 0) precede every body element.
    if (c == 0 && tid == 0 && g.head > 0) {
        const uint4 hu = ld_partial_unit<ESIZE>(g.base, 0, g.head);
        if (greedy) {
            consider_unit<ESIZE>(hu, 0, m, idx);
        } else {
            const uint4 h1[1] = {hu};
            lse_update<ESIZE, 1>(h1, k, m, s);
        }
    }
    bool ok = true;
    uint32_t phase = 0;
    for (int pb = u0; pb < u1 && ok; pb += kPieceUnits, phase ^= 1u) {
        const int n = min(kPieceUnits, u1 - pb);
        if (tid == 0) {
            mbar_arrive_expect_tx(&full, static_cast<uint32_t>(n) * 16u);
            bulk_g2s(piece, g.body + static_cast<long long>(pb) * 16, static_cast<uint32_t>(n) * 16u,
                     &full);
        }
        ok = mbar_wait(&full, phase, kWaitLimitNs);
        if (ok) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint4 v[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int u = (4 * h + q) * kStatsThreads + tid;
                    v[q] = u < n ? piece[u] : pad;
                }
                if (greedy) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        consider_unit<ESIZE>(v[q], g.head + (pb + (4 * h + q) * kStatsThreads + tid) * kPer,
                                             m, idx);
                } else {
                    lse_update<ESIZE, 4>(v, k, m, s);
                }
            }
        }
        __syncthreads();   // the piece is consumed before the next copy overwrites it
    }
    if (!ok) {
        // A copy that did not complete in time: wait (bounded) for it once
        // more so that nothing lands after the block exits, and leave a NaN
        // record, which the decide step turns into NaN normalisers.
        if (tid == 0) {
            mbar_wait(&full, phase, kWaitLimitNs / 4);
            const float nan = __int_as_float(0x7fc00000);
            a.stats_local[(static_cast<long long>(b) * a.S + slot) * a.C + c] =
                make_float4(nan, nan, nan, 0.f);
        }
        __syncthreads();
        return;
    }
    // Tail elements (last chunk, thread 1) follow every body element.
    if (c == a.C - 1 && tid == 1 && g.tail > 0) {
        const int first = g.head + g.n16 * kPer;
        const uint4 tu = ld_partial_unit<ESIZE>(g.base, first, g.tail);
        if (greedy) {
            consider_unit<ESIZE>(tu, first, m, idx);
        } else {
            const uint4 t1[1] = {tu};
            lse_update<ESIZE, 1>(t1, k, m, s);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, idx, o);
        if (greedy) {
            if (m2 > m || (m2 == m && i2 < idx)) { m = m2; idx = i2; }
        } else {
            lse_merge(m, s, m2, s2, k);
        }
    }
    if (lane == 0) wp[warp] = make_float4(m, s, 0.f, __int_as_float(idx));
    __syncthreads();
    if (tid != 0) return;
    float rm = wp[0].x, rs = wp[0].y;
    int ri = __float_as_int(wp[0].w);
    for (int w = 1; w < kStatsWarps; ++w) {
        const float4 p = wp[w];
        const int i2 = __float_as_int(p.w);
        if (greedy) {
            if (p.x > rm || (p.x == rm && i2 < ri)) { rm = p.x; ri = i2; }
        } else {
            lse_merge(rm, rs, p.x, p.y, k);
        }
    }
    float4 out;
    if (greedy) {
        // Slice-local argmax made global.
        out = make_float4(rm, 0.f, 0.f, __int_as_float(ri == INT_MAX ? INT_MAX : a.v0 + ri));
    } else {
        // Chunk 0 carries the draft token's logit when the slice holds it.
        float zx = 0.f;
        int own = 0;
        if (c == 0 && i < L) {
            const int xl = __ldg(&a.tokens[static_cast<long long>(b) * a.K + i]) - a.v0;
            if (xl >= 0 && xl < a.Vs) { zx = ld_elem<ESIZE>(g.base, xl); own = 1; }
        }
        out = make_float4(rm, rs, zx, __int_as_float(own));
    }
    a.stats_local[(static_cast<long long>(b) * a.S + slot) * a.C + c] = out;
}

// ---------------------------------------------------------------------------
// Draw weights of one 16-byte unit of the slice at the draw position.
// Local unit lu: 0 = head, 1..n16 = body units, n16+1 = tail.
// ---------------------------------------------------------------------------
struct DrawCtx {
    VecGeom gt, gd;
    bool aligned;     // target and draft slices share their 16-byte phase
    int mode, xl, NU;
    float k, mt, ist, md, isd;
};

template <int ESIZE>
__device__ __forceinline__ void load_unit(const DrawCtx &c, int lu, bool want_draft, uint4 &t,
                                          uint4 &d, int &first, int &count) {
    constexpr int kPer = 16 / ESIZE;
    const uint32_t pw = neg_inf_word<ESIZE>();
    d = make_uint4(pw, pw, pw, pw);
    if (lu == 0) {
        first = 0; count = c.gt.head;
        t = ld_partial_unit<ESIZE>(c.gt.base, 0, count);
    } else if (lu <= c.gt.n16) {
        first = c.gt.head + (lu - 1) * kPer; count = kPer;
        t = ld_reuse(c.gt.body + static_cast<long long>(lu - 1) * 16);
    } else {
        first = c.gt.head + c.gt.n16 * kPer; count = c.gt.tail;
        t = ld_partial_unit<ESIZE>(c.gt.base, first, count);
    }
    if (want_draft && c.aligned) {
        if (lu >= 1 && lu <= c.gt.n16) d = ld_reuse(c.gd.body + static_cast<long long>(lu - 1) * 16);
        else d = ld_partial_unit<ESIZE>(c.gd.base, first, count);
    }
}

// Weights of the elements of a loaded unit: table 0 is the draw's own
// weight (p, p without x_j, or max(0, p - q) with p and q normalised),
// table 1 the unnormalised p that a zero residual falls back to.  Elements
// past `count` weigh 0.  One exp2 per element and model: the normalised p
// is the unnormalised one times 1 / Sigma.
template <int ESIZE>
__device__ __forceinline__ float2 elem_weights(const DrawCtx &c, const uint4 &t, const uint4 &d,
                                               int first, int count, int e) {
    if (e >= count) return make_float2(0.f, 0.f);
    const float pu = ex2((unit_elem<ESIZE>(t, e) - c.mt) * c.k);
    if (c.mode == kModeP) return make_float2(pu, pu);
    if (c.mode == kModeOneHot) return make_float2(first + e == c.xl ? 0.f : pu, pu);
    const float zd = c.aligned ? unit_elem<ESIZE>(d, e) : ld_elem<ESIZE>(c.gd.base, first + e);
    const float q = ex2((zd - c.md) * c.k) * c.isd;
    return make_float2(fmaxf(fmaf(pu, c.ist, -q), 0.f), pu);
}

template <int ESIZE>
__device__ __forceinline__ float elem_weight(const DrawCtx &c, int table, const uint4 &t,
                                             const uint4 &d, int first, int count, int e) {
    const float2 w = elem_weights<ESIZE>(c, t, d, first, count, e);
    return table ? w.y : w.x;
}

// Both tables' weight of a unit.  A full body unit (not holding a
// one-hot x_j, draft in phase) takes a packed path: per element pair one
// packed add and one packed multiply form (z - m) k, then two exp2, and for
// the residual the same for q, a packed multiply by 1/Sigma, a packed FMA
// and the clamp; the element values equal elem_weights', summed in two
// interleaved chains.  Other units sum elem_weights in element order.  The
// mass and draw kernels both call this, so a unit weighs the same in both.
template <int ESIZE>
__device__ __forceinline__ float2 unit_weights(const DrawCtx &c, const uint4 &t, const uint4 &d,
                                               int first, int count) {
    constexpr int kPer = 16 / ESIZE;
    const bool fast = count == kPer && (c.mode != kModeResidual || c.aligned) &&
                      (c.mode != kModeOneHot || c.xl < first || c.xl >= first + kPer);
    if (fast) {
        const float2 kk = make_float2(c.k, c.k), nmt = make_float2(-c.mt, -c.mt);
        float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
        if (c.mode == kModeResidual) {
            const float2 nmd = make_float2(-c.md, -c.md);
            const float2 ist = make_float2(c.ist, c.ist), isd = make_float2(c.isd, c.isd);
#pragma unroll
            for (int q = 0; q < kPer / 2; ++q) {
                const float2 x = __fmul2_rn(__fadd2_rn(unit_pair<ESIZE>(t, q), nmt), kk);
                const float2 pu = make_float2(ex2(x.x), ex2(x.y));
                const float2 y = __fmul2_rn(__fadd2_rn(unit_pair<ESIZE>(d, q), nmd), kk);
                const float2 qn = __fmul2_rn(make_float2(ex2(y.x), ex2(y.y)), isd);
                const float2 r = __ffma2_rn(pu, ist, make_float2(-qn.x, -qn.y));
                a0 = __fadd2_rn(a0, make_float2(fmaxf(r.x, 0.f), fmaxf(r.y, 0.f)));
                a1 = __fadd2_rn(a1, pu);
            }
            return make_float2(a0.x + a0.y, a1.x + a1.y);
        }
#pragma unroll
        for (int q = 0; q < kPer / 2; ++q) {
            const float2 x = __fmul2_rn(__fadd2_rn(unit_pair<ESIZE>(t, q), nmt), kk);
            a1 = __fadd2_rn(a1, make_float2(ex2(x.x), ex2(x.y)));
        }
        const float s1 = a1.x + a1.y;
        return make_float2(s1, s1);
    }
    float w0 = 0.f, w1 = 0.f;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
        const float2 w = elem_weights<ESIZE>(c, t, d, first, count, e);
        w0 += w.x;
        w1 += w.y;
    }
    return make_float2(w0, w1);
}

template <int ESIZE>
__device__ __forceinline__ float unit_weight(const DrawCtx &c, int table, const uint4 &t,
                                             const uint4 &d, int first, int count) {
    const float2 w = unit_weights<ESIZE>(c, t, d, first, count);
    return table ? w.y : w.x;
}

template <int ESIZE>
__device__ __forceinline__ DrawCtx draw_ctx(const Args &a, int b, const Record &r) {
    DrawCtx c;
    c.gt = vec_geom<ESIZE>(tgt_vec<ESIZE>(a, b, r.j), a.Vs);
    const bool resid = r.mode == kModeResidual;
    c.gd = resid ? vec_geom<ESIZE>(dft_vec<ESIZE>(a, b, r.j), a.Vs) : c.gt;
    c.aligned = !resid || c.gd.head == c.gt.head;
    c.mode = r.mode;
    c.xl = r.xl;
    c.NU = c.gt.n16 + 2;
    c.k = r.k; c.mt = r.mt; c.ist = r.ist; c.md = r.md; c.isd = r.isd;
    return c;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ---------------------------------------------------------------------------
// 2. Decide: merge, accept tests, outputs, slice draw masses.
// ---------------------------------------------------------------------------
struct DecideSmem {
    float m[kMaxSlots], s[kMaxSlots], zx[kMaxSlots];
    int arg[kMaxSlots];
    int tok[SV_MAX_K];
    int j;
    Record rec;
};

template <int ESIZE>
__global__ void __launch_bounds__(kDecideThreads) vp_decide_kernel(Args a) {
    __shared__ DecideSmem sm;
    griddep_wait();
    griddep_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x, K = a.K, S = a.S;
    // Row checks, with the row's draft tokens loaded in parallel.
    const int L = __ldg(&a.lengths[b]);
    const float T = __ldg(&a.temp[b]);
    int bits = 0;
    if (L < 0 || L > K) bits |= SV_ROW_BAD_LENGTH;
    if (bad_temperature(T)) bits |= SV_ROW_BAD_TEMPERATURE;
    int x = 0;
    if (tid < K) {
        x = __ldg(&a.tokens[static_cast<long long>(b) * K + tid]);
        sm.tok[tid] = x;
    }
    const bool bad_tok = !(bits & SV_ROW_BAD_LENGTH) && tid < L && (x < 0 || x >= a.V);
    if (__syncthreads_or(bad_tok)) bits |= SV_ROW_BAD_TOKEN;
    if (tid == 0) a.cnt[b] = 0;   // the mass kernel of this step counts its CTAs here
    if (bits) {
        for (int t = tid; t <= K; t += kDecideThreads)
            a.out_tokens[static_cast<long long>(b) * (K + 1) + t] = -1;
        if (tid == 0) {
            a.out_accept[b] = -1;
            if (a.status) atomicOr(a.status, bits);
            a.rec[b].mode = kModeDone;
            a.mass_local[b] = make_float2(0.f, 0.f);
        }
        return;
    }
    const bool greedy = !(T > 0.f);
    const bool has_draft = a.zd != nullptr && !greedy;
    const float k = greedy ? 0.f : kLog2e / T;

    // Normalisers: target slots 0..L and draft slots 0..L-1, each merged
    // over (rank, chunk) in a fixed order by one warp.
    const int nslot = L + 1 + (has_draft ? L : 0);
    const int nparts = a.nshards * a.C;
    for (int q = warp; q < nslot; q += kDecideWarps) {
        const int slot = q <= L ? q : K + 1 + (q - L - 1);
        float m = kNegInf, s = 0.f, zx = 0.f;
        int idx = INT_MAX, own = 0;
        for (int p = lane; p < nparts; p += 32) {
            const int r = p / a.C, c = p - r * a.C;
            const float4 v =
                __ldg(&a.stats_all[((static_cast<long long>(r) * a.B + b) * S + slot) * a.C + c]);
            const int w = __float_as_int(v.w);
            if (greedy) {
                if (v.x > m || (v.x == m && w < idx)) { m = v.x; idx = w; }
            } else {
                lse_merge(m, s, v.x, v.y, k);
                if (w && !own) { zx = v.z; own = 1; }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
            const int i2 = __shfl_xor_sync(0xffffffffu, idx, o);
            const float z2 = __shfl_xor_sync(0xffffffffu, zx, o);
            const int o2 = __shfl_xor_sync(0xffffffffu, own, o);
            if (greedy) {
                if (m2 > m || (m2 == m && i2 < idx)) { m = m2; idx = i2; }
            } else {
                lse_merge(m, s, m2, s2, k);
                if (o2 && !own) { zx = z2; own = 1; }
            }
        }
        if (lane == 0) {
            sm.m[slot] = m;
            sm.s[slot] = greedy ? 1.f : s;
            sm.zx[slot] = own ? zx : kNegInf;
            sm.arg[slot] = idx == INT_MAX ? 0 : idx;
            if (a.norm) {
                a.norm[(static_cast<long long>(b) * S + slot) * 2 + 0] = m;
                a.norm[(static_cast<long long>(b) * S + slot) * 2 + 1] = greedy ? 1.f : s;
            }
        }
    }
    __syncthreads();

    // Accept tests (the rule of sv_verify), one position per lane of warp
    // 0: each depends only on its own position's normalisers and uniform, so
    // the first rejection is the lowest lane that rejects.
    const uint64_t row = static_cast<uint64_t>(a.row_base) + static_cast<uint64_t>(b);
    if (warp == 0) {
        int j = L;
        for (int i0 = 0; i0 < L; i0 += 32) {
            const int i = i0 + lane;
            bool rej = false;
            if (i < L) {
                const int xi = sm.tok[i];
                if (greedy) {
                    rej = xi != sm.arg[i];
                } else {
                    const float lp = fmaf(sm.zx[i] - sm.m[i], k, -log2f(sm.s[i]));
                    float lq = 0.f;
                    if (has_draft)
                        lq = fmaf(sm.zx[K + 1 + i] - sm.m[K + 1 + i], k,
                                  -log2f(sm.s[K + 1 + i]));
                    const float u = uniform24(a.seed, row, static_cast<uint32_t>(i), 0u);
                    bool acc;
                    if (lp == kNegInf) acc = false;
                    else if (lq == kNegInf) acc = true;
                    else acc = (lp >= lq) || (u < exp2f(lp - lq));
                    rej = !acc;
                }
            }
            const unsigned bal = __ballot_sync(0xffffffffu, rej);
            if (bal) { j = i0 + __ffs(bal) - 1; break; }
        }
        if (lane == 0) {
            sm.j = j;
            Record r;
            r.j = j;
            r.pad0 = 0; r.pad1[0] = r.pad1[1] = 0;
            r.k = k;
            r.u = greedy ? 0.f : uniform24(a.seed, row, static_cast<uint32_t>(j), 1u);
            r.mt = sm.m[j];
            const bool resid = has_draft && j < L;
            r.mode = greedy ? kModeDone : (j == L ? kModeP : (resid ? kModeResidual : kModeOneHot));
            r.ist = resid ? 1.f / sm.s[j] : 1.f;
            r.md = resid ? sm.m[K + 1 + j] : 0.f;
            r.isd = resid ? 1.f / sm.s[K + 1 + j] : 1.f;
            r.xl = -1;
            if (r.mode == kModeOneHot) {
                const int xl = sm.tok[j] - a.v0;
                r.xl = (xl >= 0 && xl < a.Vs) ? xl : -1;
            }
            sm.rec = r;
            a.rec[b] = r;
            a.out_accept[b] = j;
        }
    }
    __syncthreads();
    const int j = sm.j;
    for (int t = tid; t <= K; t += kDecideThreads) {
        int v = -1;
        if (t < j) v = sm.tok[t];
        else if (t == j && greedy) v = sm.arg[j];
        a.out_tokens[static_cast<long long>(b) * (K + 1) + t] = v;
    }
    if (greedy && tid == 0) a.mass_local[b] = make_float2(0.f, 0.f);
}

// ---------------------------------------------------------------------------
// 2b. Slice draw masses at the draw position: kSegPerPart segments of SU
//     units per CTA (two per warp), each segment summed in rounds of 32
//     units with the round's warp sum added in round order; the CTA adds its
//     segments in order into its part sum; the last CTA of the row (atomic
//     count, no waiting) adds the parts in order into the slice total.
// ---------------------------------------------------------------------------
template <int ESIZE>
__global__ void __launch_bounds__(kMassThreads, 4) vp_mass_kernel(Args a) {
    __shared__ float s0v[kSegPerPart], s1v[kSegPerPart];
    __shared__ int is_last;
    griddep_wait();
    griddep_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = static_cast<int>(blockIdx.x / a.P), p = static_cast<int>(blockIdx.x % a.P);
    const Record r = a.rec[b];
    if (r.mode == kModeDone) return;   // greedy or invalid row: no draw
    const DrawCtx c = draw_ctx<ESIZE>(a, b, r);
    const bool want_draft = c.mode == kModeResidual;
    float *tb = a.seg + static_cast<long long>(b) * 2 * a.G;
    // Warp w holds segments w + 8q, q = 0..3; per round of 32 units the
    // loads of all four segments are issued before any weight is computed.
    constexpr int kQ = kSegPerPart / kMassWarps;
    const int g0 = p * kSegPerPart + warp;
    float s0[kQ], s1[kQ];
#pragma unroll
    for (int q = 0; q < kQ; ++q) { s0[q] = 0.f; s1[q] = 0.f; }
    for (int r0 = 0; r0 < a.SU; r0 += 32) {
        uint4 t[kQ], d[kQ];
        int first[kQ], count[kQ];
        bool in[kQ];
#pragma unroll
        for (int q = 0; q < kQ; ++q) {
            const int g = g0 + q * kMassWarps;
            const int e0 = min(g * a.SU, c.NU), e1 = min(e0 + a.SU, c.NU);
            const int lu = e0 + r0 + lane;
            in[q] = g < a.G && lu < e1;
            count[q] = 0;
            first[q] = 0;
            if (in[q]) load_unit<ESIZE>(c, lu, want_draft, t[q], d[q], first[q], count[q]);
        }
#pragma unroll
        for (int q = 0; q < kQ; ++q) {
            float2 w = make_float2(0.f, 0.f);
            if (in[q]) w = unit_weights<ESIZE>(c, t[q], d[q], first[q], count[q]);
            s0[q] += warp_sum(w.x);
            s1[q] += warp_sum(w.y);
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int q = 0; q < kQ; ++q) {
            const int gg = warp + q * kMassWarps, g = g0 + q * kMassWarps;
            s0v[gg] = s0[q];
            s1v[gg] = s1[q];
            if (g < a.G) { tb[g] = s0[q]; tb[a.G + g] = s1[q]; }
        }
    }
    __syncthreads();
    float *pt = a.part + static_cast<long long>(b) * 2 * a.P;
    if (tid == 0) {
        float q0 = 0.f, q1 = 0.f;
        for (int gg = 0; gg < kSegPerPart; ++gg) { q0 += s0v[gg]; q1 += s1v[gg]; }
        pt[p] = q0;
        pt[a.P + p] = q1;
        __threadfence();
        is_last = atomicAdd(&a.cnt[b], 1) == a.P - 1;
    }
    __syncthreads();
    if (is_last && tid == 0) {
        __threadfence();
        float W0 = 0.f, W1 = 0.f;
        for (int q = 0; q < a.P; ++q) { W0 += __ldcg(&pt[q]); W1 += __ldcg(&pt[a.P + q]); }
        a.mass_local[b] = make_float2(W0, W1);
    }
}

// ---------------------------------------------------------------------------
// 3. Draw: owner slice by the slice totals in rank order; the owner locates
//    the token.
// ---------------------------------------------------------------------------
template <int ESIZE>
__global__ void __launch_bounds__(32) vp_draw_kernel(Args a) {
    constexpr int kPer = 16 / ESIZE;
    griddep_wait();
    griddep_launch_dependents();
    const int lane = threadIdx.x, b = blockIdx.x;
    // Everything that depends only on the row is loaded at once: the record,
    // this row's slice masses of every rank (32 at a time) and this rank's
    // part sums of both tables.  The scans below run in the order the totals
    // were formed, every lane in step, values passed by shuffles.
    const float *pt = a.part + static_cast<long long>(b) * 2 * a.P;
    const float pw0 = lane < a.P ? pt[lane] : 0.f;
    const float pw1 = lane < a.P ? pt[a.P + lane] : 0.f;
    float2 mw = make_float2(0.f, 0.f);
    if (lane < a.nshards) mw = a.mass_all[static_cast<long long>(lane) * a.B + b];
    const Record r = a.rec[b];
    if (r.mode == kModeDone) return;
    int table = 0, note = 0;
    float R = 0.f;
    for (int q0 = 0; q0 < a.nshards; q0 += 32) {
        const float2 m = (q0 == 0) ? mw
                         : (q0 + lane < a.nshards
                                ? a.mass_all[static_cast<long long>(q0 + lane) * a.B + b]
                                : make_float2(0.f, 0.f));
        for (int q = 0; q < 32 && q0 + q < a.nshards; ++q) R += __shfl_sync(0xffffffffu, m.x, q);
    }
    if (!(R > 0.f)) {
        // A rejection that left no residual mass: draw from p_j.
        if (r.mode != kModeP) note |= SV_NOTE_ZERO_RESIDUAL;
        table = 1;
        R = 0.f;
        for (int q0 = 0; q0 < a.nshards; q0 += 32) {
            const float2 m = (q0 == 0) ? mw
                             : (q0 + lane < a.nshards
                                    ? a.mass_all[static_cast<long long>(q0 + lane) * a.B + b]
                                    : make_float2(0.f, 0.f));
            for (int q = 0; q < 32 && q0 + q < a.nshards; ++q)
                R += __shfl_sync(0xffffffffu, m.y, q);
        }
    }
    const float tgt = r.u * R;
    float cum = 0.f, tl = 0.f;
    int owner = -1, last = 0;
    for (int q0 = 0; q0 < a.nshards; q0 += 32) {
        const float2 m = (q0 == 0) ? mw
                         : (q0 + lane < a.nshards
                                ? a.mass_all[static_cast<long long>(q0 + lane) * a.B + b]
                                : make_float2(0.f, 0.f));
        for (int q = 0; q < 32 && q0 + q < a.nshards; ++q) {
            const float w = __shfl_sync(0xffffffffu, table ? m.y : m.x, q);
            if (w > 0.f) last = q0 + q;
            if (owner < 0 && cum + w > tgt) { owner = q0 + q; tl = tgt - cum; }
            if (owner < 0) cum += w;
        }
    }
    if (owner < 0) {
        // Rounding left the target at or past the total: the last slice with
        // positive weight, and inside it the last positive element.
        owner = last;
        tl = __int_as_float(0x7f800000);   // +inf: falls through every scan
        note |= SV_NOTE_CDF_FALLBACK;
    }
    if (lane == 0 && note && a.status) atomicOr(a.status, note);
    if (owner != a.shard) return;

    // Part, then segment inside it.
    const float *tb = a.seg + static_cast<long long>(b) * 2 * a.G + (table ? a.G : 0);
    const float pw = table ? pw1 : pw0;
    float tp = 0.f;
    int psel = -1;
    bool fb = false;
    cum = 0.f;
    last = 0;
    for (int q = 0; q < a.P; ++q) {
        const float w = __shfl_sync(0xffffffffu, pw, q);
        if (w > 0.f) last = q;
        if (psel < 0 && cum + w > tl) { psel = q; tp = tl - cum; }
        if (psel < 0) cum += w;
    }
    if (psel < 0) { psel = last; fb = true; tp = __int_as_float(0x7f800000); }
    const int g0 = psel * kSegPerPart, g1 = min(g0 + kSegPerPart, a.G);
    const float sw = g0 + lane < g1 ? tb[g0 + lane] : 0.f;
    int gsel = -1;
    float tg = 0.f;
    cum = 0.f;
    last = g0;
    for (int g = g0; g < g1; ++g) {
        const float w = __shfl_sync(0xffffffffu, sw, g - g0);
        if (w > 0.f) last = g;
        if (gsel < 0 && cum + w > tp) { gsel = g; tg = tp - cum; }
        if (gsel < 0) cum += w;
    }
    if (gsel < 0) { gsel = last; fb = true; }

    // Inside the segment: rounds of 32 units, running sum of the round warp
    // sums exactly as the segment total was formed; the lane whose inclusive
    // prefix first passes the target scans its unit's elements.
    const DrawCtx c = draw_ctx<ESIZE>(a, b, r);
    const bool want_draft = c.mode == kModeResidual && table == 0;
    const int e0 = min(gsel * a.SU, c.NU), e1 = min(e0 + a.SU, c.NU);
    float running = 0.f;
    int y = -1, ylast = -1;
    for (int r0 = e0; r0 < e1 && y < 0; r0 += 32) {
        const int lu = r0 + lane;
        uint4 t = make_uint4(0, 0, 0, 0), d = make_uint4(0, 0, 0, 0);
        int first = 0, count = 0;
        float w = 0.f;
        if (lu < e1) {
            load_unit<ESIZE>(c, lu, want_draft, t, d, first, count);
            w = unit_weight<ESIZE>(c, table, t, d, first, count);
        }
        // Last positive element of this round (fallback).
        const unsigned pos = __ballot_sync(0xffffffffu, w > 0.f);
        if (pos) {
            const int hl = 31 - __clz(pos);
            int le = -1;
            if (lane == hl)
                for (int e = 0; e < kPer; ++e)
                    if (elem_weight<ESIZE>(c, table, t, d, first, count, e) > 0.f) le = first + e;
            ylast = __shfl_sync(0xffffffffu, le, hl);
        }
        const float tot = warp_sum(w);
        if (!fb && running + tot > tg) {
            float incl = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const unsigned hit = __ballot_sync(0xffffffffu, running + incl > tg);
            if (hit) {
                const int hl = __ffs(hit) - 1;
                int ye = -1;
                if (lane == hl) {
                    float cc = running + (incl - w);
                    int lp = -1;
                    for (int e = 0; e < kPer && ye < 0; ++e) {
                        const float we = elem_weight<ESIZE>(c, table, t, d, first, count, e);
                        if (we > 0.f) lp = first + e;
                        cc += we;
                        if (cc > tg && we > 0.f) ye = first + e;
                    }
                    if (ye < 0) ye = lp;   // rounding inside the unit
                }
                y = __shfl_sync(0xffffffffu, ye, hl);
                if (y < 0) y = ylast;
            } else {
                y = ylast;            // rounding inside the round
            }
            if (y >= 0) break;
        }
        running += tot;
    }
    if (y < 0) y = ylast >= 0 ? ylast : 0;
    if (lane == 0) a.out_tokens[static_cast<long long>(b) * (a.K + 1) + r.j] = a.v0 + y;
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
struct Plan {
    int es, S, C, SU, G, P;
    size_t stats_bytes, off_seg, off_part, off_cnt, ws_bytes;
};

static bool make_plan(const sv_vp_slice *s, Plan *p) {
    if (s->B < 1 || s->K < 1 || s->K > SV_MAX_K || s->V < 1 || s->V > SV_MAX_V) return false;
    if (s->nshards < 1 || s->nshards > s->V || s->shard < 0 || s->shard >= s->nshards) return false;
    const int vmax = (s->V + s->nshards - 1) / s->nshards;
    if (s->Vs < 1 || s->Vs > vmax || s->v0 < 0 || s->v0 > s->V - s->Vs) return false;
    if (s->dtype != SV_F32 && s->dtype != SV_BF16) return false;
    p->es = s->dtype == SV_F32 ? 4 : 2;
    p->S = 2 * s->K + 1;
    // Chunks from the largest slice, so that every rank uses the same count.
    const long long vbytes = static_cast<long long>(vmax) * p->es;
    p->C = static_cast<int>((vbytes + kChunkBytes - 1) / kChunkBytes);
    if (p->C < 1) p->C = 1;
    if (p->C > kMaxChunks) p->C = kMaxChunks;
    const long long blocks = static_cast<long long>(s->B) * p->S * p->C;
    if (blocks >= INT_MAX) return false;
    const long long nu = static_cast<long long>(s->Vs) * p->es / 16 + 2;   // >= any vector's n16 + 2
    const long long per = (nu + kMaxSeg - 1) / kMaxSeg;
    p->SU = static_cast<int>((per + 31) / 32 * 32);
    p->G = static_cast<int>((nu + p->SU - 1) / p->SU);
    p->P = (p->G + kSegPerPart - 1) / kSegPerPart;
    p->stats_bytes = sizeof(float4) * static_cast<size_t>(blocks);
    auto align16 = [](size_t o) { return (o + 15) & ~static_cast<size_t>(15); };
    p->off_seg = align16(sizeof(Record) * static_cast<size_t>(s->B));
    p->off_part = align16(p->off_seg + sizeof(float) * 2 * static_cast<size_t>(p->G) * s->B);
    p->off_cnt = align16(p->off_part + sizeof(float) * 2 * static_cast<size_t>(p->P) * s->B);
    p->ws_bytes = align16(p->off_cnt + sizeof(int) * static_cast<size_t>(s->B));
    return true;
}

static sv_status check_slice(const sv_vp_slice *s, Plan *p) {
    if (!s || !s->target_logits) return SV_ERR_ARG;
    if (s->dtype != SV_F32 && s->dtype != SV_BF16) return SV_ERR_DTYPE;
    if (!make_plan(s, p)) return SV_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(s->target_logits) % p->es) ||
        (s->draft_logits && (reinterpret_cast<uintptr_t>(s->draft_logits) % p->es)))
        return SV_ERR_ARG;
    return SV_OK;
}

static Args base_args(const sv_vp_slice *s, const Plan &p) {
    Args a = {};
    a.zt = static_cast<const char *>(s->target_logits);
    a.zd = static_cast<const char *>(s->draft_logits);
    a.B = s->B; a.K = s->K; a.V = s->V; a.v0 = s->v0; a.Vs = s->Vs;
    a.S = p.S; a.C = p.C; a.nshards = s->nshards; a.shard = s->shard;
    a.SU = p.SU; a.G = p.G; a.P = p.P;
    return a;
}

static bool aligned16(const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; }

}  // namespace vp
}  // namespace sv

using sv::vp::Plan;

extern "C" size_t sv_vp_stats_bytes(const sv_vp_slice *s) {
    Plan p;
    if (!s || !sv::vp::make_plan(s, &p)) return 0;
    return p.stats_bytes;
}

extern "C" size_t sv_vp_workspace_bytes(const sv_vp_slice *s) {
    Plan p;
    if (!s || !sv::vp::make_plan(s, &p)) return 0;
    return p.ws_bytes;
}

extern "C" sv_status sv_vp_stats(const sv_vp_slice *s, const int32_t *draft_tokens,
                                 const int32_t *lengths, const float *temperature,
                                 void *stats_local, void *stream) {
    sv::NvtxRange nvtx_range("sv_vp_stats");
    Plan p;
    const sv_status st0 = sv::vp::check_slice(s, &p);
    if (st0 != SV_OK) return st0;
    if (!draft_tokens || !lengths || !temperature || !stats_local) return SV_ERR_ARG;
    if (!sv::vp::aligned16(stats_local)) return SV_ERR_ARG;
    sv::vp::Args a = sv::vp::base_args(s, p);
    a.tokens = draft_tokens; a.lengths = lengths; a.temp = temperature;
    a.stats_local = static_cast<float4 *>(stats_local);
    const unsigned grid = static_cast<unsigned>(s->B) * static_cast<unsigned>(p.S * p.C);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    sv::profile_mark_begin(st);
    const cudaError_t e =
        p.es == 4 ? sv::launch_pdl(sv::vp::vp_stats_kernel<4>, dim3(grid),
                                   dim3(sv::vp::kStatsThreads), sv::vp::kPieceBytes, st, a)
                  : sv::launch_pdl(sv::vp::vp_stats_kernel<2>, dim3(grid),
                                   dim3(sv::vp::kStatsThreads), sv::vp::kPieceBytes, st, a);
    if (e != cudaSuccess) return sv::note_cuda(e);
    sv::profile_mark_end(st);
    return sv::note_cuda(cudaGetLastError());
}

extern "C" sv_status sv_vp_decide(const sv_vp_slice *s, const void *stats_all,
                                  const int32_t *draft_tokens, const int32_t *lengths,
                                  const float *temperature, uint64_t seed, int64_t row_base,
                                  int32_t *out_tokens, int32_t *out_accept_len, float *mass_local,
                                  float *norm_out, void *workspace, size_t workspace_bytes,
                                  int32_t *status, void *stream) {
    sv::NvtxRange nvtx_range("sv_vp_decide");
    Plan p;
    const sv_status st0 = sv::vp::check_slice(s, &p);
    if (st0 != SV_OK) return st0;
    if (!stats_all || !draft_tokens || !lengths || !temperature || !out_tokens ||
        !out_accept_len || !mass_local || !workspace)
        return SV_ERR_ARG;
    if (row_base < 0 || !sv::vp::aligned16(stats_all) || !sv::vp::aligned16(workspace) ||
        (reinterpret_cast<uintptr_t>(mass_local) & 7))
        return SV_ERR_ARG;
    if (workspace_bytes < p.ws_bytes) return SV_ERR_WORKSPACE;
    sv::vp::Args a = sv::vp::base_args(s, p);
    a.tokens = draft_tokens; a.lengths = lengths; a.temp = temperature;
    a.seed = seed; a.row_base = row_base;
    a.stats_all = static_cast<const float4 *>(stats_all);
    a.mass_local = reinterpret_cast<float2 *>(mass_local);
    a.out_tokens = out_tokens; a.out_accept = out_accept_len; a.status = status;
    a.norm = norm_out;
    char *w = static_cast<char *>(workspace);
    a.rec = reinterpret_cast<sv::vp::Record *>(w);
    a.seg = reinterpret_cast<float *>(w + p.off_seg);
    a.part = reinterpret_cast<float *>(w + p.off_part);
    a.cnt = reinterpret_cast<int *>(w + p.off_cnt);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e =
        p.es == 4 ? sv::launch_pdl(sv::vp::vp_decide_kernel<4>, dim3(s->B),
                                   dim3(sv::vp::kDecideThreads), 0, st, a)
                  : sv::launch_pdl(sv::vp::vp_decide_kernel<2>, dim3(s->B),
                                   dim3(sv::vp::kDecideThreads), 0, st, a);
    if (e != cudaSuccess) return sv::note_cuda(e);
    const unsigned mgrid = static_cast<unsigned>(s->B) * static_cast<unsigned>(p.P);
    e = p.es == 4 ? sv::launch_pdl(sv::vp::vp_mass_kernel<4>, dim3(mgrid),
                                   dim3(sv::vp::kMassThreads), 0, st, a)
                  : sv::launch_pdl(sv::vp::vp_mass_kernel<2>, dim3(mgrid),
                                   dim3(sv::vp::kMassThreads), 0, st, a);
    if (e != cudaSuccess) return sv::note_cuda(e);
    return sv::note_cuda(cudaGetLastError());
}

extern "C" sv_status sv_vp_draw(const sv_vp_slice *s, const float *mass_all, int32_t *out_tokens,
                                void *workspace, size_t workspace_bytes, int32_t *status,
                                void *stream) {
    sv::NvtxRange nvtx_range("sv_vp_draw");
    Plan p;
    const sv_status st0 = sv::vp::check_slice(s, &p);
    if (st0 != SV_OK) return st0;
    if (!mass_all || !out_tokens || !workspace) return SV_ERR_ARG;
    if (!sv::vp::aligned16(workspace) || (reinterpret_cast<uintptr_t>(mass_all) & 7))
        return SV_ERR_ARG;
    if (workspace_bytes < p.ws_bytes) return SV_ERR_WORKSPACE;
    sv::vp::Args a = sv::vp::base_args(s, p);
    a.mass_all = reinterpret_cast<const float2 *>(mass_all);
    a.out_tokens = out_tokens; a.status = status;
    char *w = static_cast<char *>(workspace);
    a.rec = reinterpret_cast<sv::vp::Record *>(w);
    a.seg = reinterpret_cast<float *>(w + p.off_seg);
    a.part = reinterpret_cast<float *>(w + p.off_part);
    a.cnt = reinterpret_cast<int *>(w + p.off_cnt);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const cudaError_t e =
        p.es == 4 ? sv::launch_pdl(sv::vp::vp_draw_kernel<4>, dim3(s->B), dim3(32), 0, st, a)
                  : sv::launch_pdl(sv::vp::vp_draw_kernel<2>, dim3(s->B), dim3(32), 0, st, a);
    if (e != cudaSuccess) return sv::note_cuda(e);
    return sv::note_cuda(cudaGetLastError());
}
