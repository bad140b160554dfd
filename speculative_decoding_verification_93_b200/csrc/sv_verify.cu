// sv_verify.cu -- batched speculative verification on B200 (sm_100a).
//
// Method (cited as page title + section):
//  - umans.ai, "DeepSeek V4 Pro DSpark: the model isn't ready, the
//    architecture is", section "Speculative decoding, briefly": the target
//    scores the whole draft block in one pass, keeps the prefix it agrees
//    with plus one token of its own; the acceptance rule is rejection
//    sampling under which accepted tokens follow the target distribution
//    exactly, and a rejected token is replaced by one the target would emit.
//  - zhichai.net DSpark topic, section "Why LLMs speak so slowly": the test
//    is on the target/draft probability ratio; generation restarts from the
//    first error.
//  - techvisionai "DeepSeek-V4: Breaking the Efficiency Barrier", Ch. 7
//    "Deployment with vLLM": greedy drafting (q one-hot at the draft token).
// In symbols: accept x_i iff u_i < min(1, p_i(x_i)/q_i(x_i)); at the first
// rejection j draw from norm(max(0, p_j - q_j)); if all L drafts survive
// draw the bonus from p_L.  Draws are by inverse CDF in token order.
//
// Design.  Everything a row needs is a set of logit vectors (target
// positions 0..L, draft positions 0..L-1 for sampled rows).  Every vector is
// cut into C equal chunks of 16-byte units, and one *item* is one chunk.
//   1. prologue_kernel (1 CTA): validates rows, counts items per row, writes
//      the exclusive prefix of item counts (the work list is implicit in
//      it) and resets the counters.
//   2. verify_kernel (persistent, 2 CTAs/SM): CTAs take items from a global
//      atomic counter in row-major order.  An item is one HBM pass over its
//      chunk: 16-byte streaming loads, 8 per thread in flight, packed bf16x2
//      max, then one exp2 per element against the thread's max, then a
//      block (max, sum) merge; greedy rows keep (max, first argmax) instead.
//      The partial is published and a per-row atomic counter is bumped.  The
//      CTA that completes a row's last item (no waiting: the atomic tells it)
//      merges the row's partials, runs the accept test with Philox uniforms,
//      and draws the final token, re-reading only position j while the row's
//      bytes are still resident in L2.  No CTA ever waits on another.
#include <climits>
#include <cstdint>
#include <cstdio>

#include "sv.h"
#include "sv_device.cuh"
#include "sv_host.h"

namespace sv {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 8;                     // 16-byte units per thread per item
constexpr int kMaxUnitsPerItem = kThreads * kUnroll;
constexpr int kMaxSlots = 2 * SV_MAX_K + 1;
constexpr int kPrologueThreads = 1024;

struct VerifyArgs {
    const char *zt;            // [B, K+1, V]
    const char *zd;            // [B, K, V] or nullptr (greedy drafter)
    int B, K, V, S, C, U;      // S = 2K+1 slots per row, C chunks per vector, U units per chunk
    const int32_t *tokens;     // [B, K]
    const int32_t *lengths;    // [B]
    const float *temp;         // [B]
    uint64_t seed;
    int64_t row_base;
    int32_t *out_tokens;       // [B, K+1]
    int32_t *out_accept;       // [B]
    int32_t *status;           // nullable
    float *dbg;                // nullable [B, S, 2]
    int *ctr;                  // [0] next item, [1] total items
    int *row_cnt;              // [B]
    int *row_off;              // [B+1]
    float4 *part;              // [B, S, C]: (m, s, argmax bits, 0)
};

template <int ESIZE>
__device__ __forceinline__ const char *vec_ptr(const VerifyArgs &a, int b, int slot) {
    if (slot <= a.K)
        return a.zt + ((static_cast<long long>(b) * (a.K + 1) + slot) * a.V) * ESIZE;
    return a.zd + ((static_cast<long long>(b) * a.K + (slot - a.K - 1)) * a.V) * ESIZE;
}

// Row data checks: status bits, 0 if the row is valid.
__device__ __forceinline__ int row_errors(const VerifyArgs &a, int b) {
    const int L = a.lengths[b];
    const float T = a.temp[b];
    int bits = 0;
    if (L < 0 || L > a.K) bits |= SV_ROW_BAD_LENGTH;
    if (!(T >= 0.f) || isinf(T) || (T > 0.f && T < 1e-6f)) bits |= SV_ROW_BAD_TEMPERATURE;
    if (!(bits & SV_ROW_BAD_LENGTH)) {
        for (int i = 0; i < L; ++i) {
            const int x = a.tokens[static_cast<long long>(b) * a.K + i];
            if (x < 0 || x >= a.V) { bits |= SV_ROW_BAD_TOKEN; break; }
        }
    }
    return bits;
}

__device__ __forceinline__ int row_slots(const VerifyArgs &a, int L, float T) {
    return L + 1 + ((T > 0.f && a.zd != nullptr) ? L : 0);
}

// ---------------------------------------------------------------------------
// 1. Prologue: validation, item counts, exclusive prefix, counter reset.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPrologueThreads) prologue_kernel(VerifyArgs a) {
    __shared__ int s_warp[kPrologueThreads / 32];
    __shared__ int s_carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) s_carry = 0;
    __syncthreads();
    for (int base = 0; base < a.B; base += kPrologueThreads) {
        const int b = base + tid;
        int n = 0;
        if (b < a.B) {
            const int bits = row_errors(a, b);
            if (bits) {
                a.out_accept[b] = -1;
                for (int i = 0; i <= a.K; ++i)
                    a.out_tokens[static_cast<long long>(b) * (a.K + 1) + i] = -1;
                if (a.status) atomicOr(a.status, bits);
            } else {
                n = row_slots(a, a.lengths[b], a.temp[b]) * a.C;
            }
            a.row_cnt[b] = 0;
        }
        int x = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int y = s_warp[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int z = __shfl_up_sync(0xffffffffu, y, o);
                if (lane >= o) y += z;
            }
            s_warp[lane] = y;
        }
        __syncthreads();
        const int incl = x + (warp ? s_warp[warp - 1] : 0) + s_carry;
        if (b < a.B) a.row_off[b] = incl - n;
        __syncthreads();
        if (tid == kPrologueThreads - 1) s_carry = incl;
        __syncthreads();
    }
    if (tid == 0) {
        a.row_off[a.B] = s_carry;
        a.ctr[0] = 0;
        a.ctr[1] = s_carry;
    }
}

// ---------------------------------------------------------------------------
// 2a. One item: a chunk of one vector.
// ---------------------------------------------------------------------------
struct ItemResult { float m, s; int idx; };

// Per-thread (max, sum exp2((z - max) k)) over the thread's units.
template <int ESIZE>
__device__ __forceinline__ void thread_lse(const uint4 (&v)[kUnroll + 1], float k, float &m_out,
                                           float &s_out) {
    float m;
    if (ESIZE == 2) {
        uint32_t mx = v[0].x;
#pragma unroll
        for (int j = 0; j <= kUnroll; ++j) {
            mx = bmax2(mx, v[j].x); mx = bmax2(mx, v[j].y);
            mx = bmax2(mx, v[j].z); mx = bmax2(mx, v[j].w);
        }
        m = fmaxf(bf16_lo(mx), bf16_hi(mx));
    } else {
        m = kNegInf;
#pragma unroll
        for (int j = 0; j <= kUnroll; ++j)
            m = fmaxf(fmaxf(fmaxf(m, __uint_as_float(v[j].x)), __uint_as_float(v[j].y)),
                      fmaxf(__uint_as_float(v[j].z), __uint_as_float(v[j].w)));
    }
    float s = 0.f;
    if (m != kNegInf) {
        const float2 nm = make_float2(-m, -m), kk = make_float2(k, k);
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j <= kUnroll; ++j) {
            const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
            if (ESIZE == 2) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 z = make_float2(bf16_lo(w[q]), bf16_hi(w[q]));
                    const float2 d = __fmul2_rn(__fadd2_rn(z, nm), kk);
                    acc = __fadd2_rn(acc, make_float2(ex2(d.x), ex2(d.y)));
                }
            } else {
#pragma unroll
                for (int q = 0; q < 4; q += 2) {
                    const float2 z = make_float2(__uint_as_float(w[q]), __uint_as_float(w[q + 1]));
                    const float2 d = __fmul2_rn(__fadd2_rn(z, nm), kk);
                    acc = __fadd2_rn(acc, make_float2(ex2(d.x), ex2(d.y)));
                }
            }
        }
        s = acc.x + acc.y;
    }
    m_out = m;
    s_out = s;
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

template <int ESIZE>
__device__ ItemResult process_item(const VerifyArgs &a, const char *vbase, int chunk, bool greedy,
                                   float k, float *s_red_m, float *s_red_s, int *s_red_i) {
    constexpr int kPer = 16 / ESIZE;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const VecGeom g = vec_geom<ESIZE>(vbase, a.V);
    const int u0 = chunk * a.U;
    const int u1 = min(u0 + a.U, g.n16);
    const uint32_t pw = neg_inf_word<ESIZE>();
    const uint4 pad = make_uint4(pw, pw, pw, pw);

    uint4 v[kUnroll + 1];
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
        const int u = u0 + tid + j * kThreads;
        v[j] = (u < u1) ? ld_stream(g.body + static_cast<long long>(u) * 16) : pad;
    }
    // Head (chunk 0, thread 0) and tail (last chunk, thread 1) elements.
    v[kUnroll] = pad;
    int extra_first = 0;
    bool extra_is_head = false;
    if (chunk == 0 && tid == 0 && g.head > 0) {
        v[kUnroll] = ld_partial_unit<ESIZE>(g.base, 0, g.head);
        extra_is_head = true;
    }
    if (chunk == a.C - 1 && tid == 1 && g.tail > 0) {
        extra_first = g.head + g.n16 * kPer;
        v[kUnroll] = ld_partial_unit<ESIZE>(g.base, extra_first, g.tail);
    }

    ItemResult r;
    if (!greedy) {
        float m, s;
        thread_lse<ESIZE>(v, k, m, s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
            lse_merge(m, s, m2, s2, k);
        }
        if (lane == 0) { s_red_m[warp] = m; s_red_s[warp] = s; }
        __syncthreads();
        if (warp == 0) {
            m = lane < kWarps ? s_red_m[lane] : kNegInf;
            s = lane < kWarps ? s_red_s[lane] : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
                const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
                lse_merge(m, s, m2, s2, k);
            }
        }
        r.m = m; r.s = s; r.idx = 0;
    } else {
        // (max, first index of max); each thread scans its units in index order.
        float best = kNegInf;
        int bidx = INT_MAX;
        if (extra_is_head) consider_unit<ESIZE>(v[kUnroll], 0, best, bidx);
#pragma unroll
        for (int j = 0; j < kUnroll; ++j)
            consider_unit<ESIZE>(v[j], g.head + (u0 + tid + j * kThreads) * kPer, best, bidx);
        if (!extra_is_head) consider_unit<ESIZE>(v[kUnroll], extra_first, best, bidx);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float b2 = __shfl_xor_sync(0xffffffffu, best, o);
            const int i2 = __shfl_xor_sync(0xffffffffu, bidx, o);
            if (b2 > best || (b2 == best && i2 < bidx)) { best = b2; bidx = i2; }
        }
        if (lane == 0) { s_red_m[warp] = best; s_red_i[warp] = bidx; }
        __syncthreads();
        if (warp == 0) {
            best = lane < kWarps ? s_red_m[lane] : kNegInf;
            bidx = lane < kWarps ? s_red_i[lane] : INT_MAX;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float b2 = __shfl_xor_sync(0xffffffffu, best, o);
                const int i2 = __shfl_xor_sync(0xffffffffu, bidx, o);
                if (b2 > best || (b2 == best && i2 < bidx)) { best = b2; bidx = i2; }
            }
        }
        r.m = best; r.s = 0.f; r.idx = bidx;
    }
    return r;   // valid in thread 0
}

// ---------------------------------------------------------------------------
// 2b. Row finisher: merge partials, accept test, final draw.
// ---------------------------------------------------------------------------
struct FinSmem {
    float m[kMaxSlots];
    float s[kMaxSlots];
    int arg[kMaxSlots];
    float wsum[kWarps];
    float tsum_warp[kWarps];
    int j;
    int gsel;
    float dsel;
    int tsel;
    int lastpos;
    int ysel;
    int mode;
};

enum DrawMode { kDrawP = 0, kDrawResidual = 1, kDrawResidualOneHot = 2 };

struct DrawCtx {
    VecGeom gt, gd;
    bool aligned;      // target and draft vectors share their 16-byte phase
    int mode;
    float k, ct, cd;   // p(v) = 2^((zt_v - mt) k - ct), q(v) = 2^((zd_v - md) k - cd)
    float mt, md;
    int xj;
};

// Weights of the elements of unit u (0 = head, 1..n16 = body, n16+1 = tail)
// of the draw at position j; returns the element count and first index.
template <int ESIZE>
__device__ __forceinline__ int unit_weights(const DrawCtx &c, int u, float (&w)[8], int &first) {
    constexpr int kPer = 16 / ESIZE;
    int count;
    uint4 ut, ud = make_uint4(0, 0, 0, 0);
    const bool resid = c.mode == kDrawResidual;
    if (u == 0) {
        count = c.gt.head; first = 0;
        ut = ld_partial_unit<ESIZE>(c.gt.base, 0, count);
        if (resid && c.aligned) ud = ld_partial_unit<ESIZE>(c.gd.base, 0, count);
    } else if (u <= c.gt.n16) {
        count = kPer; first = c.gt.head + (u - 1) * kPer;
        ut = ld_reuse(c.gt.body + static_cast<long long>(u - 1) * 16);
        if (resid && c.aligned) ud = ld_reuse(c.gd.body + static_cast<long long>(u - 1) * 16);
    } else {
        count = c.gt.tail; first = c.gt.head + c.gt.n16 * kPer;
        ut = ld_partial_unit<ESIZE>(c.gt.base, first, count);
        if (resid && c.aligned) ud = ld_partial_unit<ESIZE>(c.gd.base, first, count);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        float x = 0.f;
        if (e < kPer && e < count) {
            const float p = ex2(fmaf(unit_elem<ESIZE>(ut, e) - c.mt, c.k, -c.ct));
            if (c.mode == kDrawP) {
                x = p;
            } else if (c.mode == kDrawResidual) {
                const float zd = c.aligned ? unit_elem<ESIZE>(ud, e)
                                           : ld_elem<ESIZE>(c.gd.base, first + e);
                const float q = ex2(fmaf(zd - c.md, c.k, -c.cd));
                x = fmaxf(p - q, 0.f);
            } else {
                x = (first + e == c.xj) ? 0.f : p;
            }
        }
        w[e] = x;
    }
    return count;
}

// Inverse-CDF draw over one vector with the whole block: warp segments give
// the coarse CDF, one block pass over the selected segment gives the thread,
// and that thread walks its elements.  Returns the token, -1 if the total
// weight is zero (then *zero_mass is set).
template <int ESIZE>
__device__ int block_draw(const DrawCtx &c, float u, FinSmem &fs, bool *zero_mass, bool *fallback) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int NU = c.gt.n16 + 2;
    const int SU = (NU + kWarps - 1) / kWarps;
    const int seg0 = warp * SU, seg1 = min(seg0 + SU, NU);
    // Pass A: per-warp segment totals.
    float acc = 0.f;
#pragma unroll 4
    for (int uu = seg0 + lane; uu < seg1; uu += 32) {
        float w[8];
        int first;
        unit_weights<ESIZE>(c, uu, w, first);
        acc += ((w[0] + w[1]) + (w[2] + w[3])) + ((w[4] + w[5]) + (w[6] + w[7]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) fs.wsum[warp] = acc;
    __syncthreads();
    if (tid == 0) {
        float P = 0.f;
        for (int g = 0; g < kWarps; ++g) P += fs.wsum[g];
        const float R = P;
        int gsel = -1;
        float dsel = 0.f;
        if (R > 0.f) {
            const float t = u * R;
            float pre = 0.f;
            int lastg = -1;
            for (int g = 0; g < kWarps; ++g) {
                const float d = t - pre;
                if (fs.wsum[g] > 0.f) lastg = g;
                if (gsel < 0 && fs.wsum[g] > d) { gsel = g; dsel = d; }
                pre += fs.wsum[g];
            }
            if (gsel < 0) { gsel = lastg; dsel = __int_as_float(0x7f800000); }
        }
        fs.gsel = gsel;
        fs.dsel = dsel;
        fs.tsel = INT_MAX;
        fs.lastpos = -1;
        fs.ysel = -1;
    }
    __syncthreads();
    const int gsel = fs.gsel;
    if (gsel < 0) { *zero_mass = true; return -1; }
    const float dsel = fs.dsel;
    // Pass B: the block splits segment gsel into contiguous runs per thread.
    const int s0 = gsel * SU, s1 = min(s0 + SU, NU);
    const int per = (s1 - s0 + kThreads - 1) / kThreads;
    const int r0 = min(s0 + tid * per, s1), r1 = min(r0 + per, s1);
    float mine = 0.f;
    int lastpos = -1;
    for (int uu = r0; uu < r1; ++uu) {
        float w[8];
        int first;
        const int cnt = unit_weights<ESIZE>(c, uu, w, first);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (e < cnt && w[e] > 0.f) lastpos = first + e;
            mine += w[e];
        }
    }
    // Block inclusive scan of the per-thread sums.
    float x = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) fs.tsum_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        float y = lane < kWarps ? fs.tsum_warp[lane] : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float z = __shfl_up_sync(0xffffffffu, y, o);
            if (lane >= o) y += z;
        }
        if (lane < kWarps) fs.tsum_warp[lane] = y;
    }
    __syncthreads();
    const float wpre = warp ? fs.tsum_warp[warp - 1] : 0.f;
    const float xprev = __shfl_up_sync(0xffffffffu, x, 1);
    const float incl = x + wpre;
    const float excl = (lane ? xprev : 0.f) + wpre;
    if (incl > dsel) atomicMin(&fs.tsel, tid);
    if (lastpos >= 0) atomicMax(&fs.lastpos, lastpos);
    __syncthreads();
    if (tid == fs.tsel) {
        // Walk this thread's elements from the exclusive prefix.
        float cum = excl;
        int y = -1;
        for (int uu = r0; uu < r1 && y < 0; ++uu) {
            float w[8];
            int first;
            const int cnt = unit_weights<ESIZE>(c, uu, w, first);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (y < 0 && e < cnt) {
                    cum += w[e];
                    if (cum > dsel) y = first + e;
                }
            }
        }
        if (y < 0) { y = lastpos; *fallback = true; }
        fs.ysel = y;
    }
    __syncthreads();
    int y = fs.ysel;
    if (y < 0) { y = fs.lastpos; if (tid == 0) *fallback = true; }
    return y;
}

template <int ESIZE>
__device__ void finish_row(const VerifyArgs &a, int b, FinSmem &fs) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = a.K, S = a.S, C = a.C;
    const int L = a.lengths[b];
    const float T = a.temp[b];
    const bool greedy = !(T > 0.f);
    const bool has_draft = (a.zd != nullptr) && !greedy;
    const float k = greedy ? 0.f : kLog2e / T;
    const uint64_t row = static_cast<uint64_t>(a.row_base) + static_cast<uint64_t>(b);
    const int nslots = L + 1 + (has_draft ? L : 0);

    // Merge the C chunk partials of every vector of the row.
    for (int q = warp; q < nslots; q += kWarps) {
        const int slot = q <= L ? q : (K + 1 + (q - L - 1));
        float m = kNegInf, s = 0.f;
        int idx = INT_MAX;
        for (int cc = lane; cc < C; cc += 32) {
            const float4 p = __ldcg(&a.part[(static_cast<long long>(b) * S + slot) * C + cc]);
            if (greedy) {
                const int i2 = __float_as_int(p.z);
                if (p.x > m || (p.x == m && i2 < idx)) { m = p.x; idx = i2; }
            } else {
                lse_merge(m, s, p.x, p.y, k);
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
        if (lane == 0) {
            if (idx == INT_MAX) idx = 0;   // every logit -inf: documented as invalid input
            fs.m[slot] = m;
            fs.s[slot] = greedy ? 1.f : s;
            fs.arg[slot] = idx;
            if (a.dbg) {
                a.dbg[(static_cast<long long>(b) * S + slot) * 2 + 0] = m;
                a.dbg[(static_cast<long long>(b) * S + slot) * 2 + 1] = greedy ? 1.f : s;
            }
        }
    }
    if (tid == 0) fs.j = L;
    __syncthreads();

    // Accept test, one thread per verified position; first rejection wins.
    if (tid < L) {
        const int i = tid;
        const int x = a.tokens[static_cast<long long>(b) * K + i];
        bool acc;
        if (greedy) {
            acc = (x == fs.arg[i]);
        } else {
            const float zt_x = ld_elem<ESIZE>(vec_ptr<ESIZE>(a, b, i), x);
            const float lp = fmaf(zt_x - fs.m[i], k, -log2f(fs.s[i]));
            float lq = 0.f;
            if (has_draft) {
                const float zd_x = ld_elem<ESIZE>(vec_ptr<ESIZE>(a, b, K + 1 + i), x);
                lq = fmaf(zd_x - fs.m[K + 1 + i], k, -log2f(fs.s[K + 1 + i]));
            }
            const float u = uniform24(a.seed, row, static_cast<uint32_t>(i), 0u);
            if (lp == kNegInf) acc = false;
            else if (lq == kNegInf) acc = true;
            else acc = (lp >= lq) || (u < exp2f(lp - lq));
        }
        if (!acc) atomicMin(&fs.j, i);
    }
    __syncthreads();
    const int j = fs.j;

    int y;
    if (greedy) {
        y = fs.arg[j];
    } else {
        DrawCtx c;
        c.k = k;
        c.gt = vec_geom<ESIZE>(vec_ptr<ESIZE>(a, b, j), a.V);
        c.mt = fs.m[j];
        c.ct = log2f(fs.s[j]);
        c.xj = (j < L) ? a.tokens[static_cast<long long>(b) * K + j] : -1;
        if (j == L) {
            c.mode = kDrawP;
        } else if (has_draft) {
            c.mode = kDrawResidual;
            c.gd = vec_geom<ESIZE>(vec_ptr<ESIZE>(a, b, K + 1 + j), a.V);
            c.md = fs.m[K + 1 + j];
            c.cd = log2f(fs.s[K + 1 + j]);
        } else {
            c.mode = kDrawResidualOneHot;
        }
        if (c.mode != kDrawResidual) { c.gd = c.gt; c.md = 0.f; c.cd = 0.f; }
        c.aligned = (c.gd.head == c.gt.head);
        const float u = uniform24(a.seed, row, static_cast<uint32_t>(j), 1u);
        bool zero = false, fb = false;
        y = block_draw<ESIZE>(c, u, fs, &zero, &fb);
        if (zero) {
            // Rejection with no residual mass (p_j == q_j to rounding).
            c.mode = kDrawP;
            y = block_draw<ESIZE>(c, u, fs, &zero, &fb);
            if (a.status && tid == 0) atomicOr(a.status, SV_NOTE_ZERO_RESIDUAL);
            if (y < 0) y = fs.arg[j];
        }
        if (fb && a.status) atomicOr(a.status, SV_NOTE_CDF_FALLBACK);
    }
    for (int t = tid; t <= K; t += kThreads) {
        int v = -1;
        if (t < j) v = a.tokens[static_cast<long long>(b) * K + t];
        else if (t == j) v = y;
        a.out_tokens[static_cast<long long>(b) * (K + 1) + t] = v;
    }
    if (tid == 0) a.out_accept[b] = j;
}

// ---------------------------------------------------------------------------
// 2c. Persistent kernel.
// ---------------------------------------------------------------------------
template <int ESIZE>
__global__ void __launch_bounds__(kThreads, 2) verify_kernel(VerifyArgs a) {
    __shared__ float s_red_m[kWarps];
    __shared__ float s_red_s[kWarps];
    __shared__ int s_red_i[kWarps];
    __shared__ int s_w, s_b, s_last;
    __shared__ FinSmem fs;
    const int tid = threadIdx.x;
    const int total = __ldcg(&a.ctr[1]);

    if (tid == 0) {
        const int w = atomicAdd(&a.ctr[0], 1);
        s_w = w;
        if (w < total) {
            int lo = 0, hi = a.B - 1;   // largest b with row_off[b] <= w
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (__ldcg(&a.row_off[mid]) <= w) lo = mid; else hi = mid - 1;
            }
            s_b = lo;
        }
    }
    __syncthreads();
    while (true) {
        const int w = s_w;
        if (w >= total) break;
        const int b = s_b;
        const int off = __ldcg(&a.row_off[b]);
        const int nitems = __ldcg(&a.row_off[b + 1]) - off;
        const int r = w - off;
        const int L = a.lengths[b];
        const float T = a.temp[b];
        const bool greedy = !(T > 0.f);
        const int q = r / a.C, chunk = r - q * a.C;
        const int slot = q <= L ? q : (a.K + 1 + (q - L - 1));
        const float k = greedy ? 0.f : kLog2e / T;
        int wnext = 0;
        if (tid == 0) wnext = atomicAdd(&a.ctr[0], 1);   // consumed after the item

        const ItemResult res = process_item<ESIZE>(a, vec_ptr<ESIZE>(a, b, slot), chunk, greedy, k,
                                                   s_red_m, s_red_s, s_red_i);
        if (tid == 0) {
            a.part[(static_cast<long long>(b) * a.S + slot) * a.C + chunk] =
                make_float4(res.m, res.s, __int_as_float(res.idx), 0.f);
            __threadfence();
            const int done = atomicAdd(&a.row_cnt[b], 1) + 1;
            __threadfence();
            s_last = (done == nitems);
            s_w = wnext;
            if (wnext < total) {
                int lo = 0, hi = a.B - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (__ldcg(&a.row_off[mid]) <= wnext) lo = mid; else hi = mid - 1;
                }
                s_b = lo;
            }
        }
        __syncthreads();
        if (s_last) finish_row<ESIZE>(a, b, fs);
        __syncthreads();
    }
}

// Kernel launched per call, used for occupancy queries.
template <int ESIZE> static const void *verify_kernel_ptr() {
    return reinterpret_cast<const void *>(&verify_kernel<ESIZE>);
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
struct Plan {
    int C, U, S;
    size_t off_rowcnt, off_rowoff, off_part, bytes;
};

static bool make_plan(int B, int K, int V, sv_dtype dtype, Plan *p) {
    if (B < 1 || K < 1 || K > SV_MAX_K || V < 1 || V > SV_MAX_V) return false;
    if (dtype != SV_F32 && dtype != SV_BF16) return false;
    const int es = dtype == SV_F32 ? 4 : 2;
    const int per = 16 / es;
    const long long n16 = (V + per - 1) / per;
    int C = static_cast<int>((n16 + kMaxUnitsPerItem - 1) / kMaxUnitsPerItem);
    if (C < 1) C = 1;
    const int U = static_cast<int>((n16 + C - 1) / C);
    const int S = 2 * K + 1;
    const long long items = static_cast<long long>(B) * S * C;
    if (items >= INT_MAX / 2) return false;
    p->C = C; p->U = U; p->S = S;
    size_t off = 16;
    p->off_rowcnt = off;
    off += sizeof(int) * static_cast<size_t>(B);
    p->off_rowoff = off;
    off += sizeof(int) * static_cast<size_t>(B + 1);
    off = (off + 15) & ~static_cast<size_t>(15);
    p->off_part = off;
    off += sizeof(float4) * static_cast<size_t>(items);
    p->bytes = off;
    return true;
}

static int grid_for(int esize, long long max_items) {
    static int cache[2][64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    int &slot = cache[esize == 4 ? 1 : 0][dev & 63];
    if (slot == 0) {
        int sms = 0, per = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return -1;
        const void *fn = esize == 4 ? verify_kernel_ptr<4>() : verify_kernel_ptr<2>();
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fn, kThreads, 0) != cudaSuccess)
            return -1;
        slot = sms * (per > 0 ? per : 1);
    }
    return static_cast<int>(max_items < slot ? max_items : slot);
}

static sv_status verify_impl(const void *zt, const void *zd, sv_dtype dtype, int B, int K, int V,
                             const int32_t *tokens, const int32_t *lengths, const float *temp,
                             uint64_t seed, int64_t row_base, int32_t *out_tokens,
                             int32_t *out_accept, void *ws, size_t ws_bytes, int32_t *status,
                             float *dbg, void *stream) {
    if (!zt || !tokens || !lengths || !temp || !out_tokens || !out_accept || !ws)
        return SV_ERR_ARG;
    if (dtype != SV_F32 && dtype != SV_BF16) return SV_ERR_DTYPE;
    Plan p;
    if (!make_plan(B, K, V, dtype, &p)) return SV_ERR_SHAPE;
    if (row_base < 0) return SV_ERR_ARG;
    const int es = dtype == SV_F32 ? 4 : 2;
    if ((reinterpret_cast<uintptr_t>(zt) % es) || (zd && (reinterpret_cast<uintptr_t>(zd) % es)))
        return SV_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(ws) & 15) return SV_ERR_ARG;
    if (ws_bytes < p.bytes) return SV_ERR_WORKSPACE;

    VerifyArgs a;
    a.zt = static_cast<const char *>(zt);
    a.zd = static_cast<const char *>(zd);
    a.B = B; a.K = K; a.V = V; a.S = p.S; a.C = p.C; a.U = p.U;
    a.tokens = tokens; a.lengths = lengths; a.temp = temp;
    a.seed = seed; a.row_base = row_base;
    a.out_tokens = out_tokens; a.out_accept = out_accept; a.status = status; a.dbg = dbg;
    char *w = static_cast<char *>(ws);
    a.ctr = reinterpret_cast<int *>(w);
    a.row_cnt = reinterpret_cast<int *>(w + p.off_rowcnt);
    a.row_off = reinterpret_cast<int *>(w + p.off_rowoff);
    a.part = reinterpret_cast<float4 *>(w + p.off_part);

    const int grid = grid_for(es, static_cast<long long>(B) * p.S * p.C);
    if (grid <= 0) return note_cuda(cudaGetLastError());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    prologue_kernel<<<1, kPrologueThreads, 0, st>>>(a);
    profile_mark_begin(st);
    if (es == 4) verify_kernel<4><<<grid, kThreads, 0, st>>>(a);
    else verify_kernel<2><<<grid, kThreads, 0, st>>>(a);
    profile_mark_end(st);
    return note_cuda(cudaGetLastError());
}

}  // namespace sv

extern "C" size_t sv_verify_workspace_bytes(int B, int K, int V, sv_dtype dtype) {
    sv::Plan p;
    if (!sv::make_plan(B, K, V, dtype, &p)) return 0;
    return p.bytes;
}

extern "C" sv_status sv_verify(const void *target_logits, const void *draft_logits, sv_dtype dtype,
                               int B, int K, int V, const int32_t *draft_tokens,
                               const int32_t *lengths, const float *temperature, uint64_t seed,
                               int64_t row_base, int32_t *out_tokens, int32_t *out_accept_len,
                               void *workspace, size_t workspace_bytes, int32_t *status,
                               void *stream) {
    return sv::verify_impl(target_logits, draft_logits, dtype, B, K, V, draft_tokens, lengths,
                           temperature, seed, row_base, out_tokens, out_accept_len, workspace,
                           workspace_bytes, status, nullptr, stream);
}

extern "C" sv_status sv_verify_debug(const void *target_logits, const void *draft_logits,
                                     sv_dtype dtype, int B, int K, int V,
                                     const int32_t *draft_tokens, const int32_t *lengths,
                                     const float *temperature, uint64_t seed, int64_t row_base,
                                     int32_t *out_tokens, int32_t *out_accept_len,
                                     void *workspace, size_t workspace_bytes, int32_t *status,
                                     float *stats_out, void *stream) {
    if (!stats_out) return SV_ERR_ARG;
    return sv::verify_impl(target_logits, draft_logits, dtype, B, K, V, draft_tokens, lengths,
                           temperature, seed, row_base, out_tokens, out_accept_len, workspace,
                           workspace_bytes, status, stats_out, stream);
}

extern "C" int sv_verify_launches(void) { return 2; }
