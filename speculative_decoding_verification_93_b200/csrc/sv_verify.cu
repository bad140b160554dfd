// sv_verify.cu -- batched speculative verification on B200 (sm_100a).
//
// Method (cited as page title + section):
//  - umans.ai, "DeepSeek V4 Pro DSpark: the model isn't ready, the
//    architecture is", section "Speculative decoding, briefly": one target
//    pass checks the whole draft block; the drafts it agrees with stay and
//    one token of its own follows; the test is rejection sampling, which
//    leaves the emitted tokens distributed exactly as the target's, and a
//    rejected draft gives way to a token of the target's choosing.
//  - zhichai.net DSpark topic, section "Why LLMs speak so slowly": the test
//    compares the target and draft probabilities by their ratio; decoding
//    goes on from the first rejected position.
//  - techvisionai "DeepSeek-V4: Breaking the Efficiency Barrier", Ch. 7
//    "Deployment with vLLM": greedy drafting (q one-hot at the draft token).
// In symbols: accept x_i iff u_i < min(1, p_i(x_i)/q_i(x_i)); at the first
// rejection j draw from norm(max(0, p_j - q_j)); if all L drafts survive
// draw the bonus from p_L.  Draws are by inverse CDF in token order.
//
// Design.  Everything a row needs is a set of logit vectors (target
// positions 0..L, draft positions 0..L-1 for sampled rows).  Every vector is
// cut into C chunks of 16-byte units, and one *item* is one chunk.
//   1. prologue_kernel (1 CTA): validates rows, resets the per-row state
//      and writes the position-major work list, implicit in per-level row
//      prefixes: every row's position 0 comes before any row's position 1.
//   2. stream_kernel (persistent, 3 CTAs/SM, warp-specialised): a producer
//      thread claims items from a global counter, skips an item whose row
//      has already rejected an earlier position, and streams the others
//      into a 4-stage shared-memory ring with bulk copies (cp.async.bulk,
//      mbarrier completion), abandoning an item between stages once it is
//      known to be unneeded.  Eight consumer warps reduce each stage --
//      packed bf16x2 max, one exp2 per element against the running max --
//      into (max, sum) partials (greedy rows: max and first argmax).  A
//      publisher warp merges each item's warp partials, publishes one
//      partial per item, counts finished items per (row, position), and
//      runs the accept test of a position as soon as it is complete,
//      lowering the row's first-rejection marker on a rejection.  Every
//      mbarrier wait is bounded in wall time and reports SV_NOTE_TIMEOUT.
//   3. draw_kernel (one CTA per row and chunk), launched while the stream
//      kernel runs: each CTA waits until its row is settled (the publisher
//      sets a bit per accepted position; a rejection lowers the marker),
//      then merges the normalisers of position j from the stream partials.
//      Greedy rows: the argmax.  p-mass draws: the row's lead CTA picks the
//      chunk from the partials' masses and locates the token inside it.
//      Residual draws: every chunk CTA sums max(0, p_j - q_j) over its
//      chunk by 64-unit sub-ranges; the last chunk CTA of the row (atomic
//      count, no waiting) stages the row's sub-range table, forms the chunk
//      totals in the order its scan walks them, and picks the chunk, the
//      sub-range and the token inside it.  Only position j of a rejecting
//      row is read a second time.
#include <climits>
#include <cstdint>
#include <cstdio>
#include <atomic>

#include "sv.h"
#include "sv_device.cuh"
#include "sv_host.h"

namespace sv {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;   // consumer group (warps 0..7)
constexpr int kBlock = kConsumers + 64;           // + one producer and one publisher warp
constexpr int kStages = 4;                        // shared-memory ring depth
constexpr int kStageUnits = 1024;                 // 16-byte units per stage (16 KB)
constexpr int kRingBytes = kStages * kStageUnits * 16;
constexpr int kMaxUnitsPerItem = 8 * kStageUnits; // an item spans up to 8 stages (128 KB)
constexpr int kMaxSlots = 2 * SV_MAX_K + 1;
constexpr int kMaxChunks = 64;                    // V <= SV_MAX_V keeps C within this
constexpr int kPrologueThreads = 1024;

struct VerifyArgs {
    const char *zt;            // [B, K+1, V]
    const char *zd;            // [B, K, V] or nullptr (greedy drafter)
    int B, K, V, S, C, U;      // S = 2K+1 slots per row, C chunks per vector, U units per chunk
    int P;                     // draw CTAs per chunk of a residual draw (1 or 2)
    const int32_t *tokens;     // [B, K]
    const int32_t *lengths;    // [B]
    const float *temp;         // [B]
    uint64_t seed;
    int64_t row_base;
    int32_t *out_tokens;       // [B, K+1]
    int32_t *out_accept;       // [B]
    int32_t *status;           // nullable
    float *dbg;                // nullable [B, S, 2]
    const float *conf;         // [B, K] confidences, or null: lengths given
    float tau;                 // schedule threshold when conf is set
    int32_t *lengths_out;      // [B] scheduled lengths, written when conf is set
    int *ctr;                  // [0] next item, [1] total items, [2] a wait ran out
    int *rcnt;                 // [B]  chunks of the residual draw done
    int *leff;                 // [B]  verify length of a valid row, -1 for an invalid one
    int *row_j;                // [B]  first rejection found so far (starts at L)
    int *pcnt;                 // [B, K+1] item partials published per (row, position)
    unsigned long long *dec;   // [B]  positions accepted (bit i)
    int *lvl_off;              // [K+2] first item of each position level
    int *lvl_row;              // [K+1, B+1] per-level exclusive prefix of row item counts
    float4 *part;              // [B, S, C]: (m, s, argmax bits, 0)
    float *rtbl;               // [B, nsub] residual mass per sub-range
    int nsub;                  // sub-ranges per row
};

template <int ESIZE>
__device__ __forceinline__ const char *vec_ptr(const VerifyArgs &a, int b, int slot) {
    if (slot <= a.K)
        return a.zt + ((static_cast<long long>(b) * (a.K + 1) + slot) * a.V) * ESIZE;
    return a.zd + ((static_cast<long long>(b) * a.K + (slot - a.K - 1)) * a.V) * ESIZE;
}

// Row data checks: status bits, 0 if the row is valid.
__device__ __forceinline__ int row_errors(const VerifyArgs &a, int b, int L) {
    const float T = a.temp[b];
    int bits = 0;
    if (L < 0 || L > a.K) bits |= SV_ROW_BAD_LENGTH;
    if (!(T >= 0.f) || isinf(T) || (T > 0.f && T < 1e-6f)) bits |= SV_ROW_BAD_TEMPERATURE;
    if (!(bits & SV_ROW_BAD_LENGTH)) {
        // Eight loads in flight at a time, no early exit.
        const int32_t *x = a.tokens + static_cast<long long>(b) * a.K;
        bool bad = false;
        for (int i0 = 0; i0 < L; i0 += 8) {
            int v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = (i0 + q < L) ? __ldg(x + i0 + q) : 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) bad |= (v[q] < 0 || v[q] >= a.V);
        }
        if (bad) bits |= SV_ROW_BAD_TOKEN;
    }
    return bits;
}

__device__ __forceinline__ int row_slots(const VerifyArgs &a, int L, float T) {
    return L + 1 + ((T > 0.f && a.zd != nullptr) ? L : 0);
}

// ---------------------------------------------------------------------------
// 1. Prologue: validation, the position-major work list, counter reset.
//    Items are ordered by position level i = 0..K, then by row: level i holds
//    the C chunks of target position i of every row with L >= i, followed in
//    each row by the C chunks of draft position i when i < L and the row
//    samples with draft logits.  The list is implicit in per-level row
//    prefixes (one warp scans each level).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int level_items(const VerifyArgs &a, int Lb, bool sampled, int i) {
    if (Lb < 0 || i > Lb) return 0;
    return a.C * (1 + ((i < Lb && sampled) ? 1 : 0));
}

constexpr int kPrologueSmemRows = 8192;   // rows whose (L, sampled) the scans read from shared memory

__global__ void __launch_bounds__(kPrologueThreads) prologue_kernel(VerifyArgs a) {
    __shared__ int s_row[kPrologueSmemRows];   // L | sampled << 30, -1 for an invalid row
    __shared__ int s_lvl[SV_MAX_K + 1];         // items per level
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    griddep_wait();
    griddep_launch_dependents();   // the stream kernel may take its SMs now
    const int K1 = a.K + 1;
    const bool draft = a.zd != nullptr;
    // Rows: validity, effective length, first-rejection marker, counters.
    for (int b = tid; b < a.B; b += kPrologueThreads) {
        // The row's length: given, or scheduled here from its confidences
        // (the schedule kernel's own function, so the lengths agree).
        const int L0 = a.conf ? schedule_length(a.conf + static_cast<long long>(b) * a.K, a.K, a.tau)
                              : a.lengths[b];
        if (a.conf) a.lengths_out[b] = L0;
        const int bits = row_errors(a, b, L0);
        int Lb = -1;
        if (bits) {
            a.out_accept[b] = -1;
            for (int i = 0; i <= a.K; ++i)
                a.out_tokens[static_cast<long long>(b) * K1 + i] = -1;
            if (a.status) atomicOr(a.status, bits);
        } else {
            Lb = L0;
        }
        a.leff[b] = Lb;
        a.row_j[b] = Lb;
        a.rcnt[b] = 0;
        a.dec[b] = 0ull;
        if (b < kPrologueSmemRows)
            s_row[b] = Lb < 0 ? -1 : (Lb | ((draft && a.temp[b] > 0.f) ? (1 << 30) : 0));
    }
    // Completion counts of every (row, position), zeroed with coalesced stores.
    for (long long q = tid; q < static_cast<long long>(a.B) * K1; q += kPrologueThreads) a.pcnt[q] = 0;
    __syncthreads();
    // Levels: warp w scans levels w, w + 32, ... over the rows.
    for (int i = warp; i < K1; i += kPrologueThreads / 32) {
        int carry = 0;
        int *off = a.lvl_row + static_cast<long long>(i) * (a.B + 1);
        for (int b0 = 0; b0 < a.B; b0 += 32) {
            const int b = b0 + lane;
            int n = 0;
            if (b < a.B) {
                if (b < kPrologueSmemRows) {
                    const int r = s_row[b];
                    n = r < 0 ? 0 : level_items(a, r & 0xffff, (r >> 30) & 1, i);
                } else {
                    n = level_items(a, a.leff[b], draft && a.temp[b] > 0.f, i);
                }
            }
            int x = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (b < a.B) off[b] = carry + x - n;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0) { off[a.B] = carry; s_lvl[i] = carry; }
    }
    __syncthreads();
    if (tid == 0) {
        int acc = 0;
        for (int i = 0; i < K1; ++i) {
            const int c = s_lvl[i];
            a.lvl_off[i] = acc;
            acc += c;
        }
        a.lvl_off[K1] = acc;
        a.ctr[0] = 0;
        a.ctr[1] = acc;
        a.ctr[2] = 0;
    }
}

// ---------------------------------------------------------------------------
// 2. Stream kernel: softmax statistics of every scheduled vector.
// ---------------------------------------------------------------------------
constexpr int kGroup = kConsumers;   // threads of the consumer group

struct __align__(16) StageDesc {
    int b;        // row; -1 = no more work
    int slot;
    int chunk;
    int unit0;    // first body unit of the stage, relative to the vector
    int nunits;   // body units in the stage
    int flags;    // kFirst | kLast
    float k;      // log2(e)/T; 0 for greedy rows
    int level;    // position i of the item
};
constexpr int kFirst = 1, kLast = 2;
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s: no legitimate wait comes close

__device__ __forceinline__ int vload(const int &x) {
    return *reinterpret_cast<const volatile int *>(&x);
}
__device__ __forceinline__ void vstore(int &x, int v) {
    *reinterpret_cast<volatile int *>(&x) = v;
}

constexpr int kItemSlots = 8;   // > kStages: consumer warps are never more than kStages items apart

struct ItemMeta {
    int b;        // row; -1 = no more items
    int slot;
    int chunk;
    int level;
    float k;
    int pad[3];
};

struct StreamSmem {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    StageDesc desc[kStages];
    // Mailbox from the consumer warps to the publisher warp, one slot per
    // recent item: each consumer warp leaves its partial and arrives on
    // ifull; the publisher merges, arrives on ifree, and publishes.
    float4 ipart[kItemSlots][kConsumerWarps];
    ItemMeta imeta[kItemSlots];
    uint64_t ifull[kItemSlots];
    uint64_t ifree[kItemSlots];
    int abort;
};

// Accept test of position i of row b, once every chunk partial of that
// position is published (one warp; lane 0 decides).  Same rule as the
// oracle: accept x_i iff u(seed, row, i, 0) < min(1, p_i(x_i) / q_i(x_i)),
// greedy rows iff x_i is the target argmax.  A rejection lowers row_j[b].
template <int ESIZE>
__device__ void decide_position(const VerifyArgs &a, int b, int i, int x, float zt_x,
                                float zd_x) {
    const int lane = threadIdx.x & 31;
    const int K = a.K, S = a.S, C = a.C;
    const float T = __ldg(&a.temp[b]);
    const bool greedy = !(T > 0.f);
    const bool has_draft = (a.zd != nullptr) && !greedy;
    const float k = greedy ? 0.f : kLog2e / T;
    float mt = kNegInf, st = 0.f, md = kNegInf, sd = 0.f;
    int at = INT_MAX;
    const long long bt = (static_cast<long long>(b) * S + i) * C;
    const long long bd = (static_cast<long long>(b) * S + K + 1 + i) * C;
    for (int cc = lane; cc < C; cc += 32) {
        const float4 p = __ldcg(&a.part[bt + cc]);
        if (greedy) {
            const int i2 = __float_as_int(p.z);
            if (p.x > mt || (p.x == mt && i2 < at)) { mt = p.x; at = i2; }
        } else {
            lse_merge(mt, st, p.x, p.y, k);
        }
        if (has_draft) {
            const float4 q = __ldcg(&a.part[bd + cc]);
            lse_merge(md, sd, q.x, q.y, k);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, mt, o);
        const float s2 = __shfl_xor_sync(0xffffffffu, st, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, at, o);
        const float n2 = __shfl_xor_sync(0xffffffffu, md, o);
        const float d2 = __shfl_xor_sync(0xffffffffu, sd, o);
        if (greedy) {
            if (m2 > mt || (m2 == mt && i2 < at)) { mt = m2; at = i2; }
        } else {
            lse_merge(mt, st, m2, s2, k);
            lse_merge(md, sd, n2, d2, k);
        }
    }
    if (lane == 0) {
        bool acc;
        if (greedy) {
            acc = (x == (at == INT_MAX ? 0 : at));
        } else {
            const float lp = fmaf(zt_x - mt, k, -log2f(st));
            float lq = 0.f;
            if (has_draft) lq = fmaf(zd_x - md, k, -log2f(sd));
            const uint64_t row = static_cast<uint64_t>(a.row_base) + static_cast<uint64_t>(b);
            const float u = uniform24(a.seed, row, static_cast<uint32_t>(i), 0u);
            if (lp == kNegInf) acc = false;
            else if (lq == kNegInf) acc = true;
            else acc = (lp >= lq) || (u < exp2f(lp - lq));
        }
        // A rejection lowers the row's marker, an acceptance sets the
        // position's bit: the draw kernel settles a row from the two.
        if (!acc) atomicMin(&a.row_j[b], i);
        else red_or_relaxed(&a.dec[b], 1ull << i);
    }
}

// A wait that ran out: raise the status note, and tell the draw CTAs that
// rows may never settle.
__device__ __forceinline__ void report_timeout(const VerifyArgs &a) {
    if (a.status) atomicOr(a.status, SV_NOTE_TIMEOUT);
    atomicExch(&a.ctr[2], 1);
}

// Producer: fetch items (global atomic counter, prefetched one item ahead),
// decode them, stream their 16-byte body units into the ring.
// Position-major item w decoded: level i, row b, slot and chunk.
struct ItemRef {
    int i, b, slot, chunk;
};

__device__ __forceinline__ ItemRef decode_item(const VerifyArgs &a, int w) {
    int lo = 0, hi = a.K;   // largest level with lvl_off[i] <= w
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(&a.lvl_off[mid]) <= w) lo = mid; else hi = mid - 1;
    }
    ItemRef it;
    it.i = lo;
    const int r = w - __ldg(&a.lvl_off[lo]);
    const int *off = a.lvl_row + static_cast<long long>(lo) * (a.B + 1);
    lo = 0; hi = a.B - 1;   // largest row with off[b] <= r (a row with items)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(&off[mid]) <= r) lo = mid; else hi = mid - 1;
    }
    it.b = lo;
    const int q = r - __ldg(&off[lo]);
    it.chunk = q < a.C ? q : q - a.C;
    it.slot = q < a.C ? it.i : a.K + 1 + it.i;
    return it;
}

template <int ESIZE>
__device__ void producer(const VerifyArgs &a, StreamSmem &sm, uint4 *ring, int total) {
    uint32_t it = 0;
    bool ok = true;
    // The next claim is taken as the current item starts, so that the
    // counter's round trip overlaps the item.  The row's status is read when
    // the item's turn comes and again before each later stage: a rejection
    // only ever lowers it, so a stale value costs redundant bytes, never a
    // wrong result.
    int w = atomicAdd(&a.ctr[0], 1);
    while (ok) {
        if (w >= total) {
            const int st = it % kStages;
            const uint32_t ph = (it / kStages) & 1u;
            if (!mbar_wait(&sm.empty[st], ph ^ 1u, kWaitLimitNs)) { ok = false; break; }
            sm.desc[st].b = -1;
            mbar_arrive(&sm.full[st]);
            ++it;
            break;
        }
        const ItemRef cur = decode_item(a, w);
        const int rj = ld_relaxed(&a.row_j[cur.b]);
        const int wnext = atomicAdd(&a.ctr[0], 1);
        // A row that has already rejected an earlier position never needs
        // this one: skip it without reading a byte.
        if (rj >= cur.i) {
            const int b = cur.b, i = cur.i, slot = cur.slot, chunk = cur.chunk;
            const float T = __ldg(&a.temp[b]);
            const float k = (T > 0.f) ? kLog2e / T : 0.f;
            const VecGeom g = vec_geom<ESIZE>(vec_ptr<ESIZE>(a, b, slot), a.V);
            const int u0 = chunk * a.U;
            const int u1 = max(u0, min(u0 + a.U, g.n16));
            const int npieces = max(1, (u1 - u0 + kStageUnits - 1) / kStageUnits);
            for (int p = 0; p < npieces; ++p) {
                // Abandon the rest of the item once the row has rejected an
                // earlier position: the consumers reset at the next item's
                // first stage, and no partial of this item is ever read.
                if (p > 0 && ld_relaxed(&a.row_j[b]) < i) break;
                const int st = it % kStages;
                const uint32_t ph = (it / kStages) & 1u;
                if (!mbar_wait(&sm.empty[st], ph ^ 1u, kWaitLimitNs) || vload(sm.abort)) {
                    ok = false;
                    break;
                }
                const int pu0 = u0 + p * kStageUnits;
                const int pn = max(0, min(u1 - pu0, kStageUnits));
                StageDesc &d = sm.desc[st];
                d.b = b; d.slot = slot; d.chunk = chunk; d.unit0 = pu0; d.nunits = pn;
                d.flags = (p == 0 ? kFirst : 0) | (p == npieces - 1 ? kLast : 0);
                d.k = k;
                d.level = i;
                if (pn > 0) {
                    mbar_arrive_expect_tx(&sm.full[st], static_cast<uint32_t>(pn) * 16u);
                    bulk_g2s(ring + static_cast<size_t>(st) * kStageUnits,
                             g.body + static_cast<long long>(pu0) * 16,
                             static_cast<uint32_t>(pn) * 16u, &sm.full[st]);
                } else {
                    mbar_arrive(&sm.full[st]);
                }
                ++it;
            }
        }
        w = wnext;
    }
    if (!ok) {
        // Unwind: report, then wait (bounded) for the copies still in flight
        // so that none lands in shared memory after the block exits.
        vstore(sm.abort, 1);
        report_timeout(a);
        const uint32_t n = it < kStages ? it : kStages;
        for (uint32_t i = 0; i < n; ++i) {
            const uint32_t t = it - 1 - i;
            mbar_wait(&sm.full[t % kStages], (t / kStages) & 1u, kWaitLimitNs / 4);
        }
    }
}

// Consumers: reduce each stage into the running (max, sum) -- or (max,
// first argmax) for greedy rows -- and publish one partial per item.
template <int ESIZE>
__device__ void consumers(const VerifyArgs &a, StreamSmem &sm, const uint4 *ring) {
    constexpr int kPer = 16 / ESIZE;
    constexpr int kPerThread = kStageUnits / kGroup;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t pw = neg_inf_word<ESIZE>();
    const uint4 pad = make_uint4(pw, pw, pw, pw);
    uint32_t it = 0;
    uint32_t iseq = 0;   // items finished by this warp (same sequence in every warp)
    float m = kNegInf, s = 0.f;
    int bidx = INT_MAX;
    while (true) {
        const int st = it % kStages;
        const uint32_t ph = (it / kStages) & 1u;
        if (!mbar_wait(&sm.full[st], ph, kWaitLimitNs) || vload(sm.abort)) {
            vstore(sm.abort, 1);
            if (tid == 0) report_timeout(a);
            break;
        }
        const StageDesc d = sm.desc[st];
        if (d.b < 0) break;
        const bool greedy = d.k == 0.f;
        if (d.flags & kFirst) { m = kNegInf; s = 0.f; bidx = INT_MAX; }
        const uint4 *src = ring + static_cast<size_t>(st) * kStageUnits;
        uint4 v[kPerThread];
#pragma unroll
        for (int j = 0; j < kPerThread; ++j) {
            const int u = tid + j * kGroup;
            v[j] = u < d.nunits ? src[u] : pad;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[st]);
        ++it;

        // Head (first stage of chunk 0, thread 0) and tail (last stage of the
        // last chunk, thread 1) elements, loaded directly.
        uint4 extra = pad;
        int extra_first = 0;
        bool have_head = false, have_tail = false;
        const bool head_here = (d.flags & kFirst) && d.chunk == 0 && tid == 0;
        const bool tail_here = (d.flags & kLast) && d.chunk == a.C - 1 && tid == 1;
        int vhead = 0;
        if (head_here || tail_here || greedy) {
            const VecGeom g = vec_geom<ESIZE>(vec_ptr<ESIZE>(a, d.b, d.slot), a.V);
            vhead = g.head;
            if (head_here && g.head > 0) {
                extra = ld_partial_unit<ESIZE>(g.base, 0, g.head);
                have_head = true;
            }
            if (tail_here && g.tail > 0) {
                extra_first = g.head + g.n16 * kPer;
                extra = ld_partial_unit<ESIZE>(g.base, extra_first, g.tail);
                have_tail = true;
            }
        }
        if (!greedy) {
            lse_update<ESIZE, kPerThread>(v, d.k, m, s);
            if (have_head || have_tail) {
                uint4 e1[1] = {extra};
                lse_update<ESIZE, 1>(e1, d.k, m, s);
            }
        } else {
            // Index order within the thread: head, then body, then tail.
            if (have_head) consider_unit<ESIZE>(extra, 0, m, bidx);
#pragma unroll
            for (int j = 0; j < kPerThread; ++j)
                consider_unit<ESIZE>(v[j], vhead + (d.unit0 + tid + j * kGroup) * kPer, m, bidx);
            if (have_tail) consider_unit<ESIZE>(extra, extra_first, m, bidx);
        }

        if (!(d.flags & kLast)) continue;
        // End of item: warp reduction; the CTA-level merge, the publication
        // and the accept test belong to the publisher warp.
        float rm = m, rs = s;
        int ri = bidx;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, rm, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, rs, o);
            const int i2 = __shfl_xor_sync(0xffffffffu, ri, o);
            if (greedy) {
                if (m2 > rm || (m2 == rm && i2 < ri)) { rm = m2; ri = i2; }
            } else {
                lse_merge(rm, rs, m2, s2, d.k);
            }
        }
        // Hand the warp partial to the publisher warp and go on streaming.
        const uint32_t slot_i = iseq % kItemSlots, use = iseq / kItemSlots;
        ++iseq;
        int ok = 1;
        if (lane == 0) {
            ok = mbar_wait(&sm.ifree[slot_i], (use & 1u) ^ 1u, kWaitLimitNs);
            if (ok) {
                sm.ipart[slot_i][warp] = make_float4(rm, rs, __int_as_float(ri), 0.f);
                if (warp == 0) {
                    ItemMeta &im = sm.imeta[slot_i];
                    im.b = d.b; im.slot = d.slot; im.chunk = d.chunk; im.level = d.level;
                    im.k = d.k;
                }
                mbar_arrive(&sm.ifull[slot_i]);
            }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
            vstore(sm.abort, 1);
            if (lane == 0) report_timeout(a);
            break;
        }
    }
    // No more items: tell the publisher through the next mailbox slot.
    if (lane == 0 && !vload(sm.abort)) {
        const uint32_t slot_i = iseq % kItemSlots, use = iseq / kItemSlots;
        if (mbar_wait(&sm.ifree[slot_i], (use & 1u) ^ 1u, kWaitLimitNs)) {
            if (warp == 0) sm.imeta[slot_i].b = -1;
            mbar_arrive(&sm.ifull[slot_i]);
        } else {
            vstore(sm.abort, 1);
        }
    }
}

// Publisher warp: merges each item's eight warp partials in fixed order
// (the result does not depend on timing), publishes one partial per item,
// counts completed chunks per (row, position), and runs the accept test of a
// position the moment its last chunk lands.
template <int ESIZE>
__device__ void publisher(const VerifyArgs &a, StreamSmem &sm) {
    const int lane = threadIdx.x & 31;
    uint32_t iseq = 0;
    while (true) {
        const uint32_t slot_i = iseq % kItemSlots, use = iseq / kItemSlots;
        if (!mbar_wait(&sm.ifull[slot_i], use & 1u, kWaitLimitNs) || vload(sm.abort)) {
            vstore(sm.abort, 1);
            if (lane == 0) report_timeout(a);
            break;
        }
        const ItemMeta im = sm.imeta[slot_i];
        if (im.b < 0) break;
        const bool greedy = im.k == 0.f;
        float4 pv = make_float4(kNegInf, 0.f, __int_as_float(INT_MAX), 0.f);
        if (lane < kConsumerWarps) pv = sm.ipart[slot_i][lane];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.ifree[slot_i]);
        ++iseq;
        float rm = pv.x, rs = pv.y;
        int ri = __float_as_int(pv.z);
#pragma unroll
        for (int o = 1; o < kConsumerWarps; o <<= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, rm, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, rs, o);
            const int i2 = __shfl_xor_sync(0xffffffffu, ri, o);
            if (greedy) {
                if (m2 > rm || (m2 == rm && i2 < ri)) { rm = m2; ri = i2; }
            } else {
                lse_merge(rm, rs, m2, s2, im.k);
            }
        }
        int complete = 0, x = 0;
        float zt_x = 0.f, zd_x = 0.f;
        if (lane == 0) {
            const int Lb = __ldg(&a.leff[im.b]);
            const bool tested = im.level < Lb;   // positions 0..L-1 take an accept test
            const bool draft_here = (a.zd != nullptr) && !greedy && tested;
            const int need = a.C * (draft_here ? 2 : 1);
            // The draft token is requested before the count's round trip, and
            // both models' logits at it right after, so that the item that
            // completes the position can test it at once.
            if (tested) x = __ldg(&a.tokens[static_cast<long long>(im.b) * a.K + im.level]);
            a.part[(static_cast<long long>(im.b) * a.S + im.slot) * a.C + im.chunk] =
                make_float4(rm, greedy ? 0.f : rs, __int_as_float(greedy ? ri : 0), 0.f);
            // Release: this partial is visible before the count; acquire: the
            // completing item sees every partial counted before it.
            const int done =
                atom_add_acq_rel(&a.pcnt[static_cast<long long>(im.b) * (a.K + 1) + im.level], 1) + 1;
            if (tested && !greedy) {
                zt_x = ld_elem<ESIZE>(vec_ptr<ESIZE>(a, im.b, im.level), x);
                if (draft_here) zd_x = ld_elem<ESIZE>(vec_ptr<ESIZE>(a, im.b, a.K + 1 + im.level), x);
            }
            complete = (done == need) && tested;
        }
        complete = __shfl_sync(0xffffffffu, complete, 0);
        if (complete) {
            x = __shfl_sync(0xffffffffu, x, 0);
            zt_x = __shfl_sync(0xffffffffu, zt_x, 0);
            zd_x = __shfl_sync(0xffffffffu, zd_x, 0);
            decide_position<ESIZE>(a, im.b, im.level, x, zt_x, zd_x);
        }
    }
}

// Persistent warp-specialised kernel: warps 0..7 consume stages, warp 8 is
// the producer (work fetch + bulk copies into the shared-memory ring), warp
// 9 is the publisher (item partials, completion counts, accept tests).
template <int ESIZE>
__global__ void __launch_bounds__(kBlock, 3) stream_kernel(VerifyArgs a) {
    extern __shared__ __align__(128) uint4 ring[];
    __shared__ StreamSmem sm;
    const int tid = threadIdx.x;
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], kConsumerWarps);
        }
        for (int i = 0; i < kItemSlots; ++i) {
            mbar_init(&sm.ifull[i], kConsumerWarps);
            mbar_init(&sm.ifree[i], 1);
        }
        sm.abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    griddep_wait();
    // The draw kernel may launch at once: its CTAs take SMs as this grid's
    // CTAs leave, and each waits for its own row to settle.
    griddep_launch_dependents();
    const int total = __ldcg(&a.ctr[1]);
    if (tid >= kConsumers + 32) {
        publisher<ESIZE>(a, sm);
        return;
    }
    if (tid >= kConsumers) {
        if (tid == kConsumers) producer<ESIZE>(a, sm, ring, total);
        return;
    }
    consumers<ESIZE>(a, sm, ring);
}

// ---------------------------------------------------------------------------
// 3. Draw kernel helpers: the final token by inverse CDF over chunks, then
//    within a chunk (p-mass draws) or by sub-ranges (residual draws).
// ---------------------------------------------------------------------------
constexpr int kDrawThreads = 256;
constexpr int kDrawWarps = kDrawThreads / 32;

constexpr int kTblSmem = 1024;   // sub-range entries the last residual CTA stages in shared memory

struct DrawSmem {
    float tbl[kTblSmem];
    float m[kMaxSlots];
    float s[kMaxSlots];
    int arg[kMaxSlots];
    float cm[kMaxChunks];
    float wsum[kDrawWarps];
    float tsum_warp[kDrawWarps];
    int j;
    int gsel;
    float dsel;
    int tsel;
    int lastpos;
    int ysel;
    int last;
    int note;
};

enum DrawMode { kDrawP = 0, kDrawResidual = 1, kDrawOneHot = 2 };

struct DrawCtx {
    VecGeom gt, gd;
    bool aligned;      // target and draft vectors share their 16-byte phase
    int mode;
    float k;
    float ct, cd;      // weight offsets: p(v) = 2^((zt_v - mt) k - ct), q likewise
    float mt, md;
    int xj;
    // chunk range in local units: 0 = head (if any), 1..nbody = body units
    // [ubody0, ubody0 + nbody), nbody+1 = tail (if any)
    int ubody0, nbody;
    bool has_head, has_tail;
};

// Raw data of one local unit of the chunk: 0 = head (if any), 1..nbody =
// body units, nbody+1 = tail (if any).  `d` is the draft unit, loaded only
// for residual draws of aligned vectors.
struct UnitData {
    uint4 t, d;
    int count, first;
};

template <int ESIZE, int MODE>
__device__ __forceinline__ UnitData load_unit(const DrawCtx &c, int lu) {
    constexpr int kPer = 16 / ESIZE;
    constexpr bool kResid = MODE == kDrawResidual;
    UnitData r;
    r.d = make_uint4(0, 0, 0, 0);
    if (lu == 0) {
        r.count = c.has_head ? c.gt.head : 0; r.first = 0;
        r.t = ld_partial_unit<ESIZE>(c.gt.base, 0, r.count);
        if (kResid && c.aligned) r.d = ld_partial_unit<ESIZE>(c.gd.base, 0, r.count);
    } else if (lu <= c.nbody) {
        const int u = c.ubody0 + lu - 1;
        r.count = kPer; r.first = c.gt.head + u * kPer;
        r.t = ld_reuse(c.gt.body + static_cast<long long>(u) * 16);
        if (kResid && c.aligned) r.d = ld_reuse(c.gd.body + static_cast<long long>(u) * 16);
    } else {
        r.count = c.has_tail ? c.gt.tail : 0; r.first = c.gt.head + c.gt.n16 * kPer;
        r.t = ld_partial_unit<ESIZE>(c.gt.base, r.first, r.count);
        if (kResid && c.aligned) r.d = ld_partial_unit<ESIZE>(c.gd.base, r.first, r.count);
    }
    return r;
}

__device__ __forceinline__ UnitData empty_unit() {
    UnitData r;
    r.t = r.d = make_uint4(0, 0, 0, 0);
    r.count = 0;
    r.first = 0;
    return r;
}

// Draw weight of element e of a loaded unit (0 past its count).
template <int ESIZE, int MODE>
__device__ __forceinline__ float elem_weight(const DrawCtx &c, const UnitData &u, int e) {
    if (e >= u.count) return 0.f;
    const float p = ex2(fmaf(unit_elem<ESIZE>(u.t, e) - c.mt, c.k, -c.ct));
    if (MODE == kDrawP) return p;
    if (MODE == kDrawOneHot) return (u.first + e == c.xj) ? 0.f : p;
    const float zd = c.aligned ? unit_elem<ESIZE>(u.d, e) : ld_elem<ESIZE>(c.gd.base, u.first + e);
    const float q = ex2(fmaf(zd - c.md, c.k, -c.cd));
    return fmaxf(p - q, 0.f);
}

// Sum of the draw weights of a unit.  Full body units take a packed path:
// per element pair, (z - m) by one packed add, (z - m) k - c by one packed
// FMA, two exp2, and for the residual the same for q, a packed p - q, and
// the clamp at 0.  Partial units, the one-hot unit that holds x_j, and
// draft vectors out of phase with the target take the scalar path.
template <int ESIZE, int MODE>
__device__ __forceinline__ float unit_sum(const DrawCtx &c, const UnitData &u) {
    constexpr int kPer = 16 / ESIZE;
    const bool fast = u.count == kPer && (MODE != kDrawResidual || c.aligned) &&
                      (MODE != kDrawOneHot || c.xj < u.first || c.xj >= u.first + kPer);
    if (fast) {
        const float2 kk = make_float2(c.k, c.k);
        const float2 nmt = make_float2(-c.mt, -c.mt), nct = make_float2(-c.ct, -c.ct);
        const float2 nmd = make_float2(-c.md, -c.md), ncd = make_float2(-c.cd, -c.cd);
        const float2 neg1 = make_float2(-1.f, -1.f);
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < kPer / 2; ++q) {
            const float2 at = __ffma2_rn(__fadd2_rn(unit_pair<ESIZE>(u.t, q), nmt), kk, nct);
            float2 w = make_float2(ex2(at.x), ex2(at.y));
            if (MODE == kDrawResidual) {
                const float2 ad = __ffma2_rn(__fadd2_rn(unit_pair<ESIZE>(u.d, q), nmd), kk, ncd);
                const float2 qv = make_float2(ex2(ad.x), ex2(ad.y));
                const float2 r = __ffma2_rn(qv, neg1, w);
                w = make_float2(fmaxf(r.x, 0.f), fmaxf(r.y, 0.f));
            }
            acc = __fadd2_rn(acc, w);
        }
        return acc.x + acc.y;
    }
    float t = 0.f;
#pragma unroll
    for (int e = 0; e < kPer; ++e) t += elem_weight<ESIZE, MODE>(c, u, e);
    return t;
}

// Units per thread in the located segment of a chunk: a chunk of at most
// kMaxUnitsPerItem body units plus head and tail, split into kDrawWarps
// segments, each spread over the kDrawThreads threads of the CTA.
constexpr int kRunMax =
    (((kMaxUnitsPerItem + 2 + kDrawWarps - 1) / kDrawWarps) + kDrawThreads - 1) / kDrawThreads;
static_assert(kRunMax == 5, "128 KB items: five units per thread in the located segment");

// Segment g of the chunk (for warp g of the draw CTA): local units
// [g * SU, min((g+1) * SU, NU)), SU = ceil(NU / kDrawWarps).
__device__ __forceinline__ void segment_range(const DrawCtx &c, int g, int &s0, int &s1) {
    const int NU = c.nbody + 2;
    const int SU = (NU + kDrawWarps - 1) / kDrawWarps;
    s0 = min(g * SU, NU);
    s1 = min(s0 + SU, NU);
}

// Sum of the draw weights of a full body unit given as raw 16-byte words
// (packed path; -inf padding contributes 0).  One-hot exclusion is not
// applied here.
template <int ESIZE, int MODE>
__device__ __forceinline__ float body_sum(const DrawCtx &c, const uint4 &t, const uint4 &d) {
    constexpr int kPer = 16 / ESIZE;
    const float2 kk = make_float2(c.k, c.k);
    const float2 nmt = make_float2(-c.mt, -c.mt), nct = make_float2(-c.ct, -c.ct);
    const float2 nmd = make_float2(-c.md, -c.md), ncd = make_float2(-c.cd, -c.cd);
    const float2 neg1 = make_float2(-1.f, -1.f);
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < kPer / 2; ++q) {
        const float2 at = __ffma2_rn(__fadd2_rn(unit_pair<ESIZE>(t, q), nmt), kk, nct);
        float2 w = make_float2(ex2(at.x), ex2(at.y));
        if (MODE == kDrawResidual) {
            const float2 ad = __ffma2_rn(__fadd2_rn(unit_pair<ESIZE>(d, q), nmd), kk, ncd);
            const float2 r = __ffma2_rn(make_float2(ex2(ad.x), ex2(ad.y)), neg1, w);
            w = make_float2(fmaxf(r.x, 0.f), fmaxf(r.y, 0.f));
        }
        acc = __fadd2_rn(acc, w);
    }
    return acc.x + acc.y;
}

// Total draw weight of segment `warp` of the chunk.  Body units go through a
// tight loop -- lanes stride through the segment (coalesced), 8 units per
// lane in flight, raw 16-byte loads padded with -inf -- and the head, the
// tail and the one-hot exclusion are applied once by lane 0.  A draft
// vector out of 16-byte phase with the target takes the generic path.  All
// lanes get the total.
template <int ESIZE, int MODE>
__device__ float warp_segment_total(const DrawCtx &c) {
    constexpr int kPer = 16 / ESIZE;
    constexpr int kB = 8;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int s0, s1;
    segment_range(c, warp, s0, s1);
    float acc = 0.f;
    if (MODE == kDrawResidual && !c.aligned) {
        for (int lu = s0 + lane; lu < s1; lu += 32)
            acc += unit_sum<ESIZE, MODE>(c, load_unit<ESIZE, MODE>(c, lu));
    } else {
        const int b0 = max(s0, 1), b1 = min(s1, c.nbody + 1);   // body local units
        const uint32_t pw = neg_inf_word<ESIZE>();
        const uint4 pad = make_uint4(pw, pw, pw, pw);
        for (int base = b0; base < b1; base += 32 * kB) {
            uint4 t[kB], d[kB];
#pragma unroll
            for (int i = 0; i < kB; ++i) {
                const int lu = base + lane + 32 * i;
                const long long off = static_cast<long long>(c.ubody0 + lu - 1) * 16;
                t[i] = lu < b1 ? ld_reuse(c.gt.body + off) : pad;
                if (MODE == kDrawResidual) d[i] = lu < b1 ? ld_reuse(c.gd.body + off) : pad;
                else d[i] = pad;
            }
#pragma unroll
            for (int i = 0; i < kB; ++i) acc += body_sum<ESIZE, MODE>(c, t[i], d[i]);
        }
        if (lane == 0) {
            if (s0 == 0) acc += unit_sum<ESIZE, MODE>(c, load_unit<ESIZE, MODE>(c, 0));
            const int lt = c.nbody + 1;
            if (s0 <= lt && lt < s1) acc += unit_sum<ESIZE, MODE>(c, load_unit<ESIZE, MODE>(c, lt));
            if (MODE == kDrawOneHot) {
                // the body loop counted p(x_j); take it out if x_j is ours
                const int ux = c.xj - c.gt.head;
                if (c.xj >= c.gt.head && ux / kPer < c.gt.n16) {
                    const int lx = ux / kPer - c.ubody0 + 1;
                    if (lx >= b0 && lx < b1) {
                        const float zx = ld_elem<ESIZE>(c.gt.base, c.xj);
                        acc -= ex2(fmaf(zx - c.mt, c.k, -c.ct));
                    }
                }
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc;
}

// Smallest element of the chunk whose cumulative weight exceeds d, given
// the chunk's segment totals in ds.wsum.  The block splits the selected
// segment into contiguous runs (one per thread), scans the run totals, and
// the owning thread walks its elements (weights recomputed from the units
// it holds).  If rounding leaves d at or past the total, the last element
// with positive weight is returned and *fallback is set; -1 if the chunk
// has none.
template <int ESIZE, int MODE>
__device__ int chunk_locate(const DrawCtx &c, float d, DrawSmem &ds, bool *fallback) {
    constexpr int kPer = 16 / ESIZE;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        int gsel = -1, lastg = -1;
        float dsel = 0.f, pre = 0.f;
        for (int g = 0; g < kDrawWarps; ++g) {
            const float dd = d - pre;
            if (ds.wsum[g] > 0.f) lastg = g;
            if (gsel < 0 && ds.wsum[g] > dd) { gsel = g; dsel = dd; }
            pre += ds.wsum[g];
        }
        if (gsel < 0) { gsel = lastg; dsel = __int_as_float(0x7f800000); }
        ds.gsel = gsel;
        ds.dsel = dsel;
        ds.tsel = INT_MAX;
        ds.lastpos = -1;
        ds.ysel = -1;
    }
    __syncthreads();
    const int gsel = ds.gsel;
    if (gsel < 0) return -1;
    const float dsel = ds.dsel;
    int s0, s1;
    segment_range(c, gsel, s0, s1);
    const int per = (s1 - s0 + kDrawThreads - 1) / kDrawThreads;   // <= kRunMax
    const int r0 = min(s0 + tid * per, s1);
    UnitData ud[kRunMax];
#pragma unroll
    for (int i = 0; i < kRunMax; ++i)
        ud[i] = (i < per && r0 + i < s1) ? load_unit<ESIZE, MODE>(c, r0 + i) : empty_unit();
    float mine = 0.f;
    int lastpos = -1;
#pragma unroll
    for (int i = 0; i < kRunMax; ++i) {
#pragma unroll
        for (int e = 0; e < kPer; ++e) {
            const float w = elem_weight<ESIZE, MODE>(c, ud[i], e);
            if (w > 0.f) lastpos = ud[i].first + e;
            mine += w;
        }
    }
    float x = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) ds.tsum_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        float y = lane < kDrawWarps ? ds.tsum_warp[lane] : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float z = __shfl_up_sync(0xffffffffu, y, o);
            if (lane >= o) y += z;
        }
        if (lane < kDrawWarps) ds.tsum_warp[lane] = y;
    }
    __syncthreads();
    const float wpre = warp ? ds.tsum_warp[warp - 1] : 0.f;
    const float xprev = __shfl_up_sync(0xffffffffu, x, 1);
    const float incl = x + wpre;
    const float excl = (lane ? xprev : 0.f) + wpre;
    if (incl > dsel) atomicMin(&ds.tsel, tid);
    if (lastpos >= 0) atomicMax(&ds.lastpos, lastpos);
    __syncthreads();
    if (tid == ds.tsel) {
        float cum = excl;
        int y = -1;
#pragma unroll
        for (int i = 0; i < kRunMax; ++i) {
#pragma unroll
            for (int e = 0; e < kPer; ++e) {
                if (y < 0) {
                    cum += elem_weight<ESIZE, MODE>(c, ud[i], e);
                    if (cum > dsel && e < ud[i].count) y = ud[i].first + e;
                }
            }
        }
        if (y < 0) { y = lastpos; *fallback = true; }
        ds.ysel = y;
    }
    __syncthreads();
    int y = ds.ysel;
    if (y < 0) { y = ds.lastpos; if (tid == 0) *fallback = true; }
    return y;
}

// Mode dispatch (the mode is uniform across the block).
template <int ESIZE>
__device__ float segment_total_any(const DrawCtx &c) {
    if (c.mode == kDrawResidual) return warp_segment_total<ESIZE, kDrawResidual>(c);
    if (c.mode == kDrawOneHot) return warp_segment_total<ESIZE, kDrawOneHot>(c);
    return warp_segment_total<ESIZE, kDrawP>(c);
}

template <int ESIZE>
__device__ int chunk_locate_any(const DrawCtx &c, float d, DrawSmem &ds, bool *fallback) {
    if (c.mode == kDrawResidual) return chunk_locate<ESIZE, kDrawResidual>(c, d, ds, fallback);
    if (c.mode == kDrawOneHot) return chunk_locate<ESIZE, kDrawOneHot>(c, d, ds, fallback);
    return chunk_locate<ESIZE, kDrawP>(c, d, ds, fallback);
}

template <int ESIZE>
__device__ __forceinline__ int chunk_of_element(const VecGeom &g, int x, int U, int C) {
    constexpr int kPer = 16 / ESIZE;
    if (x < g.head) return 0;
    const int u = (x - g.head) / kPer;
    if (u >= g.n16) return C - 1;
    return min(u / U, C - 1);
}

// First chunk whose cumulative mass exceeds t = u * R (R = total mass);
// *d receives t minus the mass before it.  If rounding leaves t at or past
// the total, the last chunk with mass is chosen and *d = +inf.  -1 if R == 0.
__device__ __forceinline__ int select_chunk(const float *cm, int C, float u, float *d) {
    float R = 0.f;
    for (int cc = 0; cc < C; ++cc) R += cm[cc];
    if (!(R > 0.f)) { *d = 0.f; return -1; }
    const float t = u * R;
    float pre = 0.f;
    int lastc = -1;
    for (int cc = 0; cc < C; ++cc) {
        if (cm[cc] > 0.f) lastc = cc;
        if (cm[cc] > t - pre) { *d = t - pre; return cc; }
        pre += cm[cc];
    }
    *d = __int_as_float(0x7f800000);
    return lastc;
}

// Same masses, computed by a single thread (rare fallback paths).
__device__ __forceinline__ void chunk_masses_serial(const VerifyArgs &a, int b, int j, float mj,
                                                    float k, float *cm) {
    const long long base = (static_cast<long long>(b) * a.S + j) * a.C;
    for (int cc = 0; cc < a.C; ++cc) {
        const float4 p = __ldcg(&a.part[base + cc]);
        cm[cc] = (p.x != kNegInf) ? p.y * ex2((p.x - mj) * k) : 0.f;
    }
}

// Mass of p_j per chunk, in units of 2^((z - m_j) k), from the stream
// partials (one per chunk).  Thread-parallel; the result lands in cm[0..C).
__device__ __forceinline__ void chunk_masses(const VerifyArgs &a, int b, int j, float mj, float k,
                                             float *cm) {
    const long long base = (static_cast<long long>(b) * a.S + j) * a.C;
    for (int q = threadIdx.x; q < a.C; q += blockDim.x) {
        const float4 p = __ldcg(&a.part[base + q]);
        cm[q] = (p.x != kNegInf) ? p.y * ex2((p.x - mj) * k) : 0.f;
    }
}

// ---------------------------------------------------------------------------
// Residual draw by sub-ranges of kSubUnits units.
// ---------------------------------------------------------------------------
constexpr int kSubUnits = 64;   // units per sub-range; chunk sizes are multiples of it
constexpr int kRunUnits = 3;    // local units per lane in a located sub-range (66 / 32)
constexpr int kResidLaneUnits = 8;   // units per lane per block of the residual sums (even)
static_assert(kResidLaneUnits % 2 == 0, "a sub-range is two units per lane");

// Draw weight of `count` (< one unit) elements from element `first`,
// loaded directly (vector head or tail).
template <int ESIZE, int MODE>
__device__ __forceinline__ float partial_sum(const DrawCtx &c, int first, int count) {
    constexpr int kPer = 16 / ESIZE;
    UnitData u;
    u.first = first;
    u.count = count;
    u.t = ld_partial_unit<ESIZE>(c.gt.base, first, count);
    u.d = (MODE == kDrawResidual && c.aligned) ? ld_partial_unit<ESIZE>(c.gd.base, first, count)
                                               : make_uint4(0u, 0u, 0u, 0u);
    float t = 0.f;
#pragma unroll
    for (int e = 0; e < kPer; ++e) t += elem_weight<ESIZE, MODE>(c, u, e);
    return t;
}

// Residual weight of every sub-range of part `part` of chunk `ch` into tbl.
// Warp w takes the blocks w, w + 8, ... of 32 NQ units (NQ units per lane
// in flight, loaded without L1 allocation: the pass touches them once) of
// the part; unit base + lane + 32 q lies in sub-range base / 64 + q / 2.
// The head joins sub-range 0 and the tail the last one.  Each sum has a
// fixed order.
template <int ESIZE>
__device__ void residual_subranges(const DrawCtx &c, int ch, int part, int P, int U, float *tbl) {
    constexpr int kPer = 16 / ESIZE;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int PU = (U / P + kSubUnits - 1) / kSubUnits * kSubUnits;   // units per part
    const int u0 = ch * U + part * PU;
    const int u1 = max(u0, min(min(u0 + PU, (ch + 1) * U), c.gt.n16));
    const int slast = c.gt.n16 > 0 ? (c.gt.n16 - 1) / kSubUnits : 0;
    const uint32_t pw = neg_inf_word<ESIZE>();
    const uint4 pad = make_uint4(pw, pw, pw, pw);
    constexpr int NQ = kResidLaneUnits, NS = NQ / 2;   // units per lane, sub-ranges per block
    int nblk = (u1 - u0 + 32 * NQ - 1) / (32 * NQ);
    if (c.gt.n16 == 0 && ch == 0 && part == 0) nblk = 1;   // head and tail only
    for (int blk = warp; blk < nblk; blk += kDrawWarps) {
        const int base = u0 + blk * 32 * NQ;
        float acc[NS];
#pragma unroll
        for (int r = 0; r < NS; ++r) acc[r] = 0.f;
        if (c.aligned) {
            uint4 t[NQ], d[NQ];
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const int u = base + lane + 32 * q;
                const long long off = static_cast<long long>(u) * 16;
                t[q] = u < u1 ? ld_stream(c.gt.body + off) : pad;
                d[q] = u < u1 ? ld_stream(c.gd.body + off) : pad;
            }
#pragma unroll
            for (int q = 0; q < NQ; ++q) acc[q >> 1] += body_sum<ESIZE, kDrawResidual>(c, t[q], d[q]);
        } else {
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const int u = base + lane + 32 * q;
                if (u < u1) {
                    UnitData ud;
                    ud.t = ld_reuse(c.gt.body + static_cast<long long>(u) * 16);
                    ud.d = make_uint4(0u, 0u, 0u, 0u);
                    ud.count = kPer;
                    ud.first = c.gt.head + u * kPer;
#pragma unroll
                    for (int e = 0; e < kPer; ++e)
                        acc[q >> 1] += elem_weight<ESIZE, kDrawResidual>(c, ud, e);
                }
            }
        }
        const int s0 = base / kSubUnits;
        if (lane == 0) {
            if (s0 == 0 && c.gt.head > 0) acc[0] += partial_sum<ESIZE, kDrawResidual>(c, 0, c.gt.head);
            if (c.gt.tail > 0 && slast >= s0 && slast < s0 + NS)
                acc[slast - s0] += partial_sum<ESIZE, kDrawResidual>(
                    c, c.gt.head + c.gt.n16 * kPer, c.gt.tail);
        }
#pragma unroll
        for (int r = 0; r < NS; ++r)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], o);
        if (lane == 0) {
#pragma unroll
            for (int r = 0; r < NS; ++r) {
                const int s = s0 + r;
                if (s * kSubUnits < u1 || (c.gt.n16 == 0 && s == 0)) tbl[s] = acc[r];
            }
        }
    }
}

// Sum of n table entries by one warp: rounds of 32 entries in order, a
// fixed tree inside each round.  table_find walks the entries in the same
// rounds, so a target below this total always finds its entry.
template <bool SMEM>
__device__ __forceinline__ float tbl_ld(const float *tb, int s) {
    return SMEM ? tb[s] : __ldcg(tb + s);
}

template <bool SMEM>
__device__ float table_total(const float *tb, int n) {
    constexpr int kRounds = 8;
    const int lane = threadIdx.x & 31;
    float R = 0.f;
    if constexpr (SMEM) {
        // The same rounds in the same order, one at a time: a staged table
        // needs no loads in flight, and the loop keeps this once-per-row
        // code small.
#pragma unroll 1
        for (int r0 = 0; r0 < n; r0 += 32) {
            float r = r0 + lane < n ? tb[r0 + lane] : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
            R += r;
        }
    } else {
        float v[kRounds];
        for (int base = 0; base < n; base += 32 * kRounds) {
#pragma unroll
            for (int q = 0; q < kRounds; ++q) {
                const int s = base + q * 32 + lane;
                v[q] = s < n ? tbl_ld<SMEM>(tb, s) : 0.f;
            }
#pragma unroll
            for (int q = 0; q < kRounds; ++q) {
                float r = v[q];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
                R += r;
            }
        }
    }
    return R;
}

// First entry with positive weight whose running sum exceeds t (one warp);
// *d_out is t minus the sum before it.  If rounding leaves t at or past the
// end, the last entry with weight is returned with *fb set and an infinite
// target.
template <bool SMEM>
__device__ int table_find(const float *tb, int n, float t, float *d_out, bool *fb) {
    constexpr int kRounds = 8;
    const int lane = threadIdx.x & 31;
    int sel = -1, lastpos = -1;
    float dsel = 0.f, cum = 0.f;
    auto round = [&](int r0, float v) {   // one round of 32 entries from r0
        if (v > 0.f) lastpos = r0 + lane;
        float incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, v > 0.f && cum + incl > t);
        if (hit) {
            const int l = __ffs(hit) - 1;
            sel = r0 + l;
            dsel = t - (cum + __shfl_sync(0xffffffffu, incl - v, l));
        } else {
            float r = v;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
            cum += r;
        }
    };
    if constexpr (SMEM) {
        // Staged table: the rounds one at a time (same order), small code.
#pragma unroll 1
        for (int r0 = 0; r0 < n && sel < 0; r0 += 32) round(r0, r0 + lane < n ? tb[r0 + lane] : 0.f);
    } else {
        float v[kRounds];
        for (int base = 0; base < n && sel < 0; base += 32 * kRounds) {
#pragma unroll
            for (int q = 0; q < kRounds; ++q) {
                const int s = base + q * 32 + lane;
                v[q] = s < n ? tbl_ld<SMEM>(tb, s) : 0.f;
            }
#pragma unroll
            for (int q = 0; q < kRounds; ++q) {
                if (sel >= 0) break;
                round(base + q * 32, v[q]);
            }
        }
    }
    if (sel < 0) {
        sel = __reduce_max_sync(0xffffffffu, lastpos);
        dsel = __int_as_float(0x7f800000);
        *fb = true;
    }
    *d_out = dsel;
    return sel;
}

// Sub-ranges [*s0, *s1) of chunk ch (the head joins sub-range 0 of chunk 0,
// the tail the last sub-range).
__device__ __forceinline__ void chunk_subranges(const VecGeom &g, int ch, int U, int *s0, int *s1) {
    const int u0 = min(ch * U, g.n16), u1 = min((ch + 1) * U, g.n16);
    *s0 = u0 / kSubUnits;
    *s1 = (u1 + kSubUnits - 1) / kSubUnits;
    if (g.n16 == 0 && ch == 0) *s1 = 1;   // head and tail only
}

// Smallest element of the sub-range described by c (ubody0, nbody, head,
// tail) whose cumulative weight exceeds d (one warp; lane l owns local units
// 3l .. 3l+2: 0 = head, 1..nbody = body units, nbody+1 = tail).  If
// rounding leaves d at or past the total, the last element with positive
// weight is returned and *fb is set; -1 if there is none.
template <int ESIZE, int MODE>
__device__ int locate_in_subrange(const DrawCtx &c, float d, bool *fb, float *wbuf) {
    constexpr int kPer = 16 / ESIZE;
    static_assert(kRunUnits == 3, "three units per lane");
    const int lane = threadIdx.x & 31;
    const int NU = c.nbody + 2;
    const int l0 = min(lane * kRunUnits, NU);
    const int l1 = min(l0 + kRunUnits, NU);
    // The three loads go out together; the weights are then formed by a loop
    // over the units that is not unrolled.  This code runs once per row, as
    // the last step of the draw, when its instructions are no longer cached:
    // its size, not its arithmetic, sets how long it takes.
    const UnitData v0 = (l0 < l1) ? load_unit<ESIZE, MODE>(c, l0) : empty_unit();
    const UnitData v1 = (l0 + 1 < l1) ? load_unit<ESIZE, MODE>(c, l0 + 1) : empty_unit();
    const UnitData v2 = (l0 + 2 < l1) ? load_unit<ESIZE, MODE>(c, l0 + 2) : empty_unit();
    float mine = 0.f;
    int lastpos = -1;
#pragma unroll 1
    for (int q = 0; q < kRunUnits; ++q) {
        const UnitData u = q == 0 ? v0 : (q == 1 ? v1 : v2);
#pragma unroll
        for (int e = 0; e < kPer; ++e) {
            const float w = elem_weight<ESIZE, MODE>(c, u, e);
            if (w > 0.f) lastpos = u.first + e;
            mine += w;
            wbuf[(q * kPer + e) * 32 + lane] = w;   // for the second pass below
        }
    }
    float incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    float excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.f;
    int y = -1;
    const unsigned hit = __ballot_sync(0xffffffffu, incl > d);
    if (hit && lane == __ffs(hit) - 1) {
        // The same weights, in the same order, from shared memory.
        float cum = excl;
#pragma unroll 1
        for (int k = 0; k < kRunUnits * kPer; ++k) {
            const float w = wbuf[k * 32 + lane];
            if (y < 0 && w > 0.f && cum + w > d) {
                const int q = k / kPer;
                y = (q == 0 ? v0.first : (q == 1 ? v1.first : v2.first)) + (k - q * kPer);
            }
            cum += w;
        }
    }
    y = __reduce_max_sync(0xffffffffu, y);
    if (y < 0) {
        *fb = true;
        y = __reduce_max_sync(0xffffffffu, lastpos);
    }
    return y;
}

// Wait (bounded, with back-off) until row b is settled, and return its j:
// positions 0..j-1 accepted (their bits set) and position j rejected
// (row_j == j), or all L positions accepted and the bonus position's
// partials complete.  A position is accepted or rejected, never both, and
// bits and marker only move one way, so the two reads need no order.  The
// acquire of position j's completion count makes its partials visible.
// -1 if the wait ran out or a stream wait did.
__device__ int wait_row_settled(const VerifyArgs &a, int b, int L, bool draft) {
    const uint64_t t0 = global_ns();
    uint32_t backoff = 32;
    while (true) {
        const unsigned long long M = ld_relaxed(&a.dec[b]);
        const int j = min(ld_relaxed(&a.row_j[b]), L);
        const unsigned long long want = j >= 64 ? ~0ull : ((1ull << j) - 1ull);
        if ((M & want) == want) {
            const int need = a.C * ((draft && j < L) ? 2 : 1);
            if (ld_acquire(&a.pcnt[static_cast<long long>(b) * (a.K + 1) + j]) >= need) return j;
        }
        if (ld_relaxed(&a.ctr[2]) != 0 || global_ns() - t0 > kWaitLimitNs) return -1;
        __nanosleep(backoff);
        if (backoff < 1024) backoff <<= 1;
    }
}

// ---------------------------------------------------------------------------
// 3. Draw kernel: one CTA per (row, chunk, part), rows fastest.  It
//    launches while the stream kernel runs; a CTA starts once its row is
//    settled (positions 0..j-1 accepted, j rejected, or all accepted and the
//    bonus position complete) and merges the normalisers of position j from
//    the stream partials: the same values, in the same order, in every CTA
//    of the row.  Greedy rows: the row's lead CTA writes the argmax.  p-mass
//    draws (the bonus position, or p_j without x_j for a greedy drafter):
//    the lead CTA picks the chunk from the partials' masses and locates the
//    token inside it.  Residual draws: every chunk CTA sums max(0, p_j -
//    q_j) over its chunk by 64-unit sub-ranges; the last one (atomic count,
//    no waiting) stages the row's sub-range table, forms the chunk totals in
//    the order its scan walks them, and picks the chunk, the sub-range and
//    the token.  Only position j of a rejecting row is read a second time.
// ---------------------------------------------------------------------------
template <int ESIZE>
__global__ void __launch_bounds__(kDrawThreads, 3) draw_kernel(VerifyArgs a) {
    __shared__ DrawSmem ds;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // This grid launches while the stream kernel still runs (its CTAs take
    // SMs as the stream kernel's leave), and each CTA waits for its own row
    // instead of the whole stream.  The last CTA waits for the stream grid,
    // so that this grid never completes before it.  The prologue's writes
    // are visible: every stream CTA passed its own wait for the prologue
    // before letting this grid launch.
    if (blockIdx.x == gridDim.x - 1) griddep_wait();
    const int K = a.K, C = a.C;
    const int b = static_cast<int>(blockIdx.x % static_cast<unsigned>(a.B));
    const int cp = static_cast<int>(blockIdx.x / static_cast<unsigned>(a.B));
    const int chunk = cp / a.P, part = cp - chunk * a.P;
    const int L = __ldcg(&a.leff[b]);
    const float T = __ldg(&a.temp[b]);
    if (L < 0) return;   // invalid row: the prologue wrote its outputs
    const bool greedy = !(T > 0.f);
    const bool has_draft = (a.zd != nullptr) && !greedy;
    const float k = greedy ? 0.f : kLog2e / T;
    const uint64_t row = static_cast<uint64_t>(a.row_base) + static_cast<uint64_t>(b);
    // The row's lead CTA (spread over the grid by row) takes greedy rows and
    // p-mass draws alone; only a row with a draft can need the others.
    const bool lead = cp == b % (C * a.P);
    if (!lead && !has_draft) return;
    if (tid == 0) {
        const int jw = wait_row_settled(a, b, L, has_draft);
        if (jw < 0 && a.status) atomicOr(a.status, SV_NOTE_TIMEOUT);
        // The normaliser output reads positions 0..j-1 as well: acquire
        // their completion counts (complete, since they were accepted).
        if (lead && a.dbg != nullptr)
            for (int i = 0; i < jw; ++i) (void)ld_acquire(&a.pcnt[static_cast<long long>(b) * (K + 1) + i]);
        ds.j = jw;
    }
    __syncthreads();
    const int j = ds.j;   // first rejection, or L
    if (j < 0) return;    // a wait ran out: outputs undefined, status raised
    const bool resid = (j < L) && has_draft;
    if (!resid && !lead) return;

    // Normalisers of position j (target; draft too for a residual draw).
    // The row's lead CTA, when normalisers are requested, takes every
    // position that was read in full: target 0..j, draft 0..min(j, L-1).
    // Warp w takes slots w, w + 8, ...
    const bool all = lead && a.dbg != nullptr;
    const int ntgt = all ? j + 1 : 1;
    const int ndft = !has_draft ? 0 : (all ? min(j + 1, L) : (resid ? 1 : 0));
    const int first = all ? 0 : j;
    for (int q = warp; q < ntgt + ndft; q += kDrawWarps) {
        const int slot = q < ntgt ? first + q : K + 1 + first + (q - ntgt);
        const long long pb = (static_cast<long long>(b) * a.S + slot) * C;
        float m = kNegInf, sm = 0.f;
        int idx = INT_MAX;
        float4 pv[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {   // C <= kMaxChunks = 64: two chunks per lane
            const int cc = lane + 32 * h;
            pv[h] = make_float4(kNegInf, 0.f, 0.f, 0.f);
            if (cc < C) {
                const float4 p = __ldcg(&a.part[pb + cc]);
                pv[h] = p;
                if (greedy) {
                    const int i2 = __float_as_int(p.z);
                    if (p.x > m || (p.x == m && i2 < idx)) { m = p.x; idx = i2; }
                } else {
                    lse_merge(m, sm, p.x, p.y, k);
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, sm, o);
            const int i2 = __shfl_xor_sync(0xffffffffu, idx, o);
            if (greedy) {
                if (m2 > m || (m2 == m && i2 < idx)) { m = m2; idx = i2; }
            } else {
                lse_merge(m, sm, m2, s2, k);
            }
        }
        if (slot == j && !greedy && !resid) {
            // p-mass draws: the mass of p_j per chunk, in units of
            // 2^((z - m_j) k), straight from the partials.
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int cc = lane + 32 * h;
                if (cc < C) ds.cm[cc] = (pv[h].x != kNegInf) ? pv[h].y * ex2((pv[h].x - m) * k) : 0.f;
            }
        }
        if (lane == 0) {
            if (idx == INT_MAX) idx = 0;   // every logit -inf: documented as invalid input
            ds.m[slot] = m;
            ds.s[slot] = greedy ? 1.f : sm;
            ds.arg[slot] = idx;
            if (all) {
                a.dbg[(static_cast<long long>(b) * a.S + slot) * 2 + 0] = m;
                a.dbg[(static_cast<long long>(b) * a.S + slot) * 2 + 1] = greedy ? 1.f : sm;
            }
        }
    }
    __syncthreads();

    if (greedy) {
        const int y = ds.arg[j];
        for (int t = tid; t <= K; t += kDrawThreads) {
            int v = -1;
            if (t < j) v = a.tokens[static_cast<long long>(b) * K + t];
            else if (t == j) v = y;
            a.out_tokens[static_cast<long long>(b) * (K + 1) + t] = v;
        }
        if (tid == 0) a.out_accept[b] = j;
        return;
    }

    // Sampled row: the final draw at position j.
    const float mt = ds.m[j];
    const float u = uniform24(a.seed, row, static_cast<uint32_t>(j), 1u);
    const int xj = (j < L) ? a.tokens[static_cast<long long>(b) * K + j] : -1;
    int mode = (j == L) ? kDrawP : (resid ? kDrawResidual : kDrawOneHot);
    int note = 0;
    int csel = -1;
    float d = 0.f;
    if (!resid) {
        // p_j (bonus) or p_j without x_j (greedy drafter): pick the chunk
        // from the partials' masses, then locate the token inside it.
        if (tid == 0) {
            if (mode == kDrawOneHot) {
                const VecGeom g = vec_geom<ESIZE>(vec_ptr<ESIZE>(a, b, j), a.V);
                const int cx = chunk_of_element<ESIZE>(g, xj, a.U, C);
                const float wx = ex2((ld_elem<ESIZE>(g.base, xj) - mt) * k);
                ds.cm[cx] = fmaxf(ds.cm[cx] - wx, 0.f);
            }
            float dd = 0.f;
            int cs = select_chunk(ds.cm, C, u, &dd);
            if (cs < 0) {
                // p_j one-hot at the rejected x_j (rounding): draw from p_j.
                mode = kDrawP;
                note = SV_NOTE_ZERO_RESIDUAL;
                chunk_masses_serial(a, b, j, mt, k, ds.cm);
                cs = select_chunk(ds.cm, C, u, &dd);
            }
            ds.gsel = cs;
            ds.dsel = dd;
            ds.lastpos = mode;
            ds.note = note;
        }
        __syncthreads();
        csel = ds.gsel;
        d = ds.dsel;
        mode = ds.lastpos;
        note = ds.note;
    }

    DrawCtx c;
    c.k = k;
    c.mode = mode;
    c.gt = vec_geom<ESIZE>(vec_ptr<ESIZE>(a, b, j), a.V);
    c.mt = mt;
    c.ct = resid ? log2f(ds.s[j]) : 0.f;
    c.xj = xj;
    if (resid) {
        c.gd = vec_geom<ESIZE>(vec_ptr<ESIZE>(a, b, K + 1 + j), a.V);
        c.md = ds.m[K + 1 + j];
        c.cd = log2f(ds.s[K + 1 + j]);
    } else {
        c.gd = c.gt; c.md = 0.f; c.cd = 0.f;
    }
    c.aligned = (c.gd.head == c.gt.head);
    auto set_chunk = [&](int cc) {
        c.ubody0 = cc * a.U;
        c.nbody = max(0, min(c.ubody0 + a.U, c.gt.n16) - c.ubody0);
        c.has_head = (cc == 0);
        c.has_tail = (cc == C - 1);
    };
    int y = -1;
    bool fb = false;
    if (resid) {
        // Residual weight of this chunk by sub-ranges; the last chunk CTA of
        // the row (atomic counter, no waiting) picks the sub-range from the
        // row's table and the token inside it.
        set_chunk(chunk);
        float *tb = a.rtbl + static_cast<long long>(b) * a.nsub;
        residual_subranges<ESIZE>(c, chunk, part, a.P, a.U, tb);
        __syncthreads();
        if (tid == 0) {
            // Release: this CTA's table entries (ordered before this thread
            // by the barrier) are visible before the count; acquire: the
            // last CTA sees every entry counted before it.
            const int done = atom_add_acq_rel(&a.rcnt[b], 1) + 1;
            ds.last = (done == C * a.P);
        }
        __syncthreads();
        if (!ds.last) return;
        // The row's whole table in one parallel round trip (shared memory
        // when it fits), then every step of the pick reads it from there.
        const int nsub = max(1, (c.gt.n16 + kSubUnits - 1) / kSubUnits);
        const bool staged = nsub <= kTblSmem;
        if (staged) {
            for (int q = tid; q < nsub; q += kDrawThreads) ds.tbl[q] = __ldcg(tb + q);
            __syncthreads();
        }
        if (warp == 0) {
            // Chunk totals, each formed as the scan below walks it, summed in
            // chunk order; then the sub-ranges of the chosen chunk.
            bool zero = false, fbw = false;
            float R = 0.f;
            for (int q = 0; q < C; ++q) {
                int s0, s1;
                chunk_subranges(c.gt, q, a.U, &s0, &s1);
                const float tot = staged ? table_total<true>(ds.tbl + s0, s1 - s0)
                                         : table_total<false>(tb + s0, s1 - s0);
                if (lane == 0) ds.cm[q] = tot;
                R += tot;
            }
            __syncwarp();
            int sel = -1;
            float dsel = 0.f;
            if (!(R > 0.f)) {
                zero = true;
            } else {
                const float t = u * R;
                float cum = 0.f, tc = 0.f;
                int cs = -1, clast = 0;
                for (int q = 0; q < C; ++q) {
                    const float w = ds.cm[q];
                    if (w > 0.f) clast = q;
                    if (cs < 0 && cum + w > t) { cs = q; tc = t - cum; }
                    if (cs < 0) cum += w;
                }
                if (cs < 0) { cs = clast; tc = __int_as_float(0x7f800000); fbw = true; }
                int s0, s1;
                chunk_subranges(c.gt, cs, a.U, &s0, &s1);
                sel = s0 + (staged ? table_find<true>(ds.tbl + s0, s1 - s0, tc, &dsel, &fbw)
                                   : table_find<false>(tb + s0, s1 - s0, tc, &dsel, &fbw));
            }
            int yw = -1;
            if (!zero && sel >= 0) {
                DrawCtx cs = c;
                cs.ubody0 = sel * kSubUnits;
                cs.nbody = max(0, min(kSubUnits, c.gt.n16 - cs.ubody0));
                cs.has_head = (sel == 0) && c.gt.head > 0;
                cs.has_tail = (sel == nsub - 1) && c.gt.tail > 0;
                yw = locate_in_subrange<ESIZE, kDrawResidual>(cs, dsel, &fbw, ds.tbl);
            }
            if (lane == 0) {
                ds.ysel = yw;
                ds.gsel = zero ? 1 : 0;
                ds.lastpos = fbw ? 1 : 0;
            }
        }
        __syncthreads();
        if (ds.gsel == 0) {
            y = ds.ysel;
            fb = ds.lastpos != 0;
            csel = -1;
        } else {
            // The residual vanished to rounding (p_j == q_j): draw from p_j.
            if (tid == 0) {
                float dd = 0.f;
                note |= SV_NOTE_ZERO_RESIDUAL;
                chunk_masses_serial(a, b, j, mt, k, ds.cm);
                ds.gsel = select_chunk(ds.cm, C, u, &dd);
                ds.dsel = dd;
            }
            __syncthreads();
            csel = ds.gsel;
            d = ds.dsel;
            c.mode = kDrawP;
            c.ct = 0.f;
        }
    }
    if (csel >= 0) {
        set_chunk(csel);
        const float segtot = segment_total_any<ESIZE>(c);
        if (lane == 0) ds.wsum[warp] = segtot;
        __syncthreads();
        y = chunk_locate_any<ESIZE>(c, d, ds, &fb);
    }
    if (y < 0) { y = 0; fb = true; }
    if (fb) note |= SV_NOTE_CDF_FALLBACK;
    if (tid == 0 && a.status && note) atomicOr(a.status, note);
    for (int t = tid; t <= K; t += kDrawThreads) {
        int v = -1;
        if (t < j) v = a.tokens[static_cast<long long>(b) * K + t];
        else if (t == j) v = y;
        a.out_tokens[static_cast<long long>(b) * (K + 1) + t] = v;
    }
    if (tid == 0) a.out_accept[b] = j;
}

template <int ESIZE> static const void *stream_kernel_ptr() {
    return reinterpret_cast<const void *>(&stream_kernel<ESIZE>);
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
struct Plan {
    int C, U, S;
    int nsub;
    size_t off_rcnt, off_leff, off_rowj, off_pcnt, off_dec, off_lvloff, off_lvlrow, off_part, off_rtbl, bytes;
};

static bool make_plan(int B, int K, int V, sv_dtype dtype, Plan *p) {
    if (B < 1 || K < 1 || K > SV_MAX_K || V < 1 || V > SV_MAX_V) return false;
    if (dtype != SV_F32 && dtype != SV_BF16) return false;
    const int es = dtype == SV_F32 ? 4 : 2;
    const int per = 16 / es;
    const long long n16 = (V + per - 1) / per;
    int C = static_cast<int>((n16 + kMaxUnitsPerItem - 1) / kMaxUnitsPerItem);
    if (C < 1) C = 1;
    if (C > kMaxChunks) return false;
    int U = static_cast<int>((n16 + C - 1) / C);
    U = (U + kSubUnits - 1) / kSubUnits * kSubUnits;   // chunks hold whole sub-ranges
    const int S = 2 * K + 1;
    const long long items = static_cast<long long>(B) * S * C;
    if (items >= INT_MAX / 2 || static_cast<long long>(B) * C >= INT_MAX / 2) return false;
    p->C = C; p->U = U; p->S = S;
    const size_t iB = sizeof(int) * static_cast<size_t>(B);
    auto align16 = [](size_t o) { return (o + 15) & ~static_cast<size_t>(15); };
    size_t off = 16;
    p->off_rcnt = off;   off = align16(off + iB);
    p->off_leff = off;   off = align16(off + iB);
    p->off_rowj = off;   off = align16(off + iB);
    p->off_pcnt = off;   off = align16(off + iB * (K + 1));
    p->off_dec = off;    off = align16(off + sizeof(unsigned long long) * static_cast<size_t>(B));
    p->off_lvloff = off; off = align16(off + sizeof(int) * static_cast<size_t>(K + 2));
    p->off_lvlrow = off; off = align16(off + sizeof(int) * static_cast<size_t>(K + 1) * (B + 1));
    p->off_part = off;   off = align16(off + sizeof(float4) * static_cast<size_t>(items));
    p->nsub = static_cast<int>((n16 + kSubUnits - 1) / kSubUnits);
    if (p->nsub < 1) p->nsub = 1;
    p->off_rtbl = off;   off = align16(off + sizeof(float) * static_cast<size_t>(B) * p->nsub);
    p->bytes = off;
    return true;
}

// Persistent grid of the stream kernel: resident CTAs per SM x SMs, cached
// per (dtype, device).  Threads that race on an empty entry compute the
// same value; the entry is an atomic so each reads a whole one.
static int stream_grid(int esize, long long max_items) {
    static std::atomic<int> cache[2][64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    std::atomic<int> &slot = cache[esize == 4 ? 1 : 0][dev & 63];
    int n = slot.load(std::memory_order_relaxed);
    if (n == 0) {
        int sms = 0, per = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return -1;
        const void *fn = esize == 4 ? stream_kernel_ptr<4>() : stream_kernel_ptr<2>();
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kRingBytes) !=
            cudaSuccess)
            return -1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fn, kBlock, kRingBytes) !=
            cudaSuccess)
            return -1;
        n = sms * (per > 0 ? per : 1);
        slot.store(n, std::memory_order_relaxed);
    }
    return static_cast<int>(max_items < n ? max_items : n);
}

static sv_status verify_impl(const void *zt, const void *zd, sv_dtype dtype, int B, int K, int V,
                             const int32_t *tokens, const int32_t *lengths, const float *temp,
                             uint64_t seed, int64_t row_base, int32_t *out_tokens,
                             int32_t *out_accept, void *ws, size_t ws_bytes, int32_t *status,
                             float *dbg, void *stream, const float *conf = nullptr,
                             float tau = 0.f, int32_t *lengths_out = nullptr) {
    if (!zt || !tokens || !temp || !out_tokens || !out_accept || !ws) return SV_ERR_ARG;
    if (conf ? !lengths_out : !lengths) return SV_ERR_ARG;
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
    a.conf = conf; a.tau = tau; a.lengths_out = lengths_out;
    a.seed = seed; a.row_base = row_base;
    a.out_tokens = out_tokens; a.out_accept = out_accept; a.status = status; a.dbg = dbg;
    char *w = static_cast<char *>(ws);
    a.ctr = reinterpret_cast<int *>(w);
    a.rcnt = reinterpret_cast<int *>(w + p.off_rcnt);
    a.leff = reinterpret_cast<int *>(w + p.off_leff);
    a.row_j = reinterpret_cast<int *>(w + p.off_rowj);
    a.pcnt = reinterpret_cast<int *>(w + p.off_pcnt);
    a.dec = reinterpret_cast<unsigned long long *>(w + p.off_dec);
    a.lvl_off = reinterpret_cast<int *>(w + p.off_lvloff);
    a.lvl_row = reinterpret_cast<int *>(w + p.off_lvlrow);
    a.part = reinterpret_cast<float4 *>(w + p.off_part);
    a.rtbl = reinterpret_cast<float *>(w + p.off_rtbl);
    a.nsub = p.nsub;

    const int grid = stream_grid(es, static_cast<long long>(B) * p.S * p.C);
    if (grid <= 0) return note_cuda(cudaGetLastError());
    // Residual chunks are split over two draw CTAs when the rows' chunk CTAs
    // would fill at most two rounds of the SMs' slots (three per SM, like
    // the stream kernel's); with more rows one CTA per chunk keeps the
    // per-row count round trips fewer.
    const int slots = stream_grid(es, LLONG_MAX);
    a.P = (static_cast<long long>(B) * p.C <= 2LL * slots) ? 2 : 1;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // Every launch below may overlap the tail of the one before it
    // (programmatic dependent launch); each kernel waits for its
    // predecessor before touching global memory.  Profiling events, when
    // enabled, sit between launches and serialise them as usual.
    cudaError_t e = launch_pdl(prologue_kernel, dim3(1), dim3(kPrologueThreads), 0, st, a);
    if (e != cudaSuccess) return note_cuda(e);
    profile_mark_begin(st);
    e = (es == 4) ? launch_pdl(stream_kernel<4>, dim3(grid), dim3(kBlock), kRingBytes, st, a)
                  : launch_pdl(stream_kernel<2>, dim3(grid), dim3(kBlock), kRingBytes, st, a);
    if (e != cudaSuccess) return note_cuda(e);
    profile_mark_end(st);
    const unsigned draw_grid = static_cast<unsigned>(B) * static_cast<unsigned>(p.C) * a.P;
    e = (es == 4) ? launch_pdl(draw_kernel<4>, dim3(draw_grid), dim3(kDrawThreads), 0, st, a)
                  : launch_pdl(draw_kernel<2>, dim3(draw_grid), dim3(kDrawThreads), 0, st, a);
    if (e != cudaSuccess) return note_cuda(e);
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
    sv::NvtxRange nvtx_range("sv_verify");
    return sv::verify_impl(target_logits, draft_logits, dtype, B, K, V, draft_tokens, lengths,
                           temperature, seed, row_base, out_tokens, out_accept_len, workspace,
                           workspace_bytes, status, nullptr, stream);
}

extern "C" sv_status sv_schedule_verify(const void *target_logits, const void *draft_logits,
                                        sv_dtype dtype, int B, int K, int V,
                                        const int32_t *draft_tokens, const float *conf, float load,
                                        int32_t *lengths, const float *temperature, uint64_t seed,
                                        int64_t row_base, int32_t *out_tokens,
                                        int32_t *out_accept_len, void *workspace,
                                        size_t workspace_bytes, int32_t *status, void *stream) {
    sv::NvtxRange nvtx_range("sv_schedule_verify");
    if (!conf || !lengths) return SV_ERR_ARG;
    return sv::verify_impl(target_logits, draft_logits, dtype, B, K, V, draft_tokens, nullptr,
                           temperature, seed, row_base, out_tokens, out_accept_len, workspace,
                           workspace_bytes, status, nullptr, stream, conf, load, lengths);
}

extern "C" sv_status sv_verify_debug(const void *target_logits, const void *draft_logits,
                                     sv_dtype dtype, int B, int K, int V,
                                     const int32_t *draft_tokens, const int32_t *lengths,
                                     const float *temperature, uint64_t seed, int64_t row_base,
                                     int32_t *out_tokens, int32_t *out_accept_len,
                                     void *workspace, size_t workspace_bytes, int32_t *status,
                                     float *stats_out, void *stream) {
    sv::NvtxRange nvtx_range("sv_verify_debug");
    if (!stats_out) return SV_ERR_ARG;
    return sv::verify_impl(target_logits, draft_logits, dtype, B, K, V, draft_tokens, lengths,
                           temperature, seed, row_base, out_tokens, out_accept_len, workspace,
                           workspace_bytes, status, stats_out, stream);
}

extern "C" int sv_verify_launches(void) { return 3; }

// ---------------------------------------------------------------------------
// Allocation-free variant: the scratch lives in a fixed device array that
// the library owns, so callers that must not allocate device memory can
// still verify.  The array is sized for moderate batches; larger ones must
// use sv_verify with their own workspace.
// ---------------------------------------------------------------------------
namespace sv {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB per device
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device.  In host code
// the symbol names only a host-side stand-in, so the address is looked up
// with the device current.  It is looked up on every call (a cheap table
// lookup in the runtime), so that it stays right when the device's context
// is torn down and created again (cudaDeviceReset reloads the module and
// may move the array).  The first lookup on a device may load the module.
static sv_status static_scratch_address(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return note_cuda(e);
    if (p == nullptr) return note_cuda(cudaErrorUnknown);
    *out = p;
    return SV_OK;
}

}  // namespace sv

extern "C" sv_status sv_verify_noalloc(const void *target_logits, const void *draft_logits,
                                       sv_dtype dtype, int B, int K, int V,
                                       const int32_t *draft_tokens, const int32_t *lengths,
                                       const float *temperature, uint64_t seed, int64_t row_base,
                                       int32_t *out_tokens, int32_t *out_accept_len,
                                       int32_t *status, void *stream) {
    sv::NvtxRange nvtx_range("sv_verify_noalloc");
    if (!target_logits || !draft_tokens || !lengths || !temperature || !out_tokens ||
        !out_accept_len)
        return SV_ERR_ARG;
    const size_t need = sv_verify_workspace_bytes(B, K, V, dtype);
    if (need == 0) return (dtype != SV_F32 && dtype != SV_BF16) ? SV_ERR_DTYPE : SV_ERR_SHAPE;
    if (need > sv::kStaticScratchBytes) return SV_ERR_WORKSPACE;
    void *ws = nullptr;
    const sv_status st = sv::static_scratch_address(&ws);
    if (st != SV_OK) return st;
    // The counters that must start at zero are reset by the first kernel of
    // every call; everything else in the scratch is written before it is read.
    return sv::verify_impl(target_logits, draft_logits, dtype, B, K, V, draft_tokens, lengths,
                           temperature, seed, row_base, out_tokens, out_accept_len, ws,
                           sv::kStaticScratchBytes, status, nullptr, stream);
}
