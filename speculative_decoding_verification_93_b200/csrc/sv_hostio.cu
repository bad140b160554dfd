// sv_hostio.cu -- verification of host-resident inputs: only the scheduled
// logit vectors cross the host link.
//
// Per row, verification reads the target positions 0..L and the draft
// positions 0..L-1 that the confidence schedule keeps, and nothing past
// them (umans.ai, "DeepSeek V4 Pro DSpark: the model isn't ready, the
// architecture is", section "What DSpark adds", item "2. Verify smarter":
// the confident prefix is what gets verified; aiweekly.co alert: the verify
// length follows prefix survival and load).  So with the logits in host
// memory the schedule runs first, its lengths come back (the one
// synchronisation; a caller that already has the lengths passes them
// instead), and only each row's scheduled runs are copied -- one
// cudaMemcpyAsync per contiguous run, adjacent runs merged -- before the
// device verification and the copy of its outputs back to the host.
//
// Level-wise mode copies less: level l copies position l of the rows still
// undecided (target if l <= L, draft if l < L; one strided 2-D copy per run
// of consecutive rows) and, from level 1 on, verifies with lengths
// min(L, l); a row is final once it rejects below l or l reaches L.  What
// crosses is the logits the outcome depends on (target 0..a, draft
// 0..min(a, L-1), a = accepted length) plus, for a row that rejects at
// a < L, position a+1, copied before the rejection is known.  The uniforms
// are keyed by (row, position, draw), so every decision and draw equals
// that of one verification with the full lengths, and no kernel reads a
// position that was not copied.
#include <cstdint>
#include <mutex>
#include <vector>

#include "sv.h"
#include "sv_host.h"

namespace sv {
namespace hostio {

struct Layout {
    size_t zt, zd, conf, tok, temp, len, lcur, otok, oacc, status, ver, ver_bytes, ver1,
        ver1_bytes, bytes;
    int half;   // rows of the first group in level-wise mode
};

static size_t align256(size_t o) { return (o + 255) & ~static_cast<size_t>(255); }

static bool make_layout(int B, int K, int V, sv_dtype dtype, Layout *L) {
    const size_t ver = sv_verify_workspace_bytes(B, K, V, dtype);
    if (ver == 0) return false;   // unsupported sizes or dtype
    const size_t es = dtype == SV_F32 ? 4 : 2;
    const size_t b = static_cast<size_t>(B), k = static_cast<size_t>(K), v = static_cast<size_t>(V);
    size_t o = 0;
    L->zt = o;     o = align256(o + b * (k + 1) * v * es);
    L->zd = o;     o = align256(o + b * k * v * es);
    L->conf = o;   o = align256(o + b * k * sizeof(float));
    L->tok = o;    o = align256(o + b * k * sizeof(int32_t));
    L->temp = o;   o = align256(o + b * sizeof(float));
    L->len = o;    o = align256(o + b * sizeof(int32_t));
    L->lcur = o;   o = align256(o + b * sizeof(int32_t));
    L->otok = o;   o = align256(o + b * (k + 1) * sizeof(int32_t));
    L->oacc = o;   o = align256(o + b * sizeof(int32_t));
    L->status = o; o = align256(o + sizeof(int32_t));
    L->ver = o;    o = align256(o + ver);
    L->ver_bytes = ver;
    // Level-wise mode runs the rows in two halves on two streams; the second
    // half needs its own sv_verify workspace (the first uses `ver`).
    L->half = B >= 2 ? B / 2 : B;
    const size_t ver1 = B - L->half > 0 ? sv_verify_workspace_bytes(B - L->half, K, V, dtype) : 0;
    L->ver1 = o;   o = align256(o + ver1);
    L->ver1_bytes = ver1;
    L->bytes = o;
    return true;
}

// Host-to-device copies of contiguous byte runs, merging a run that starts
// where the pending one ends.
struct RunCopier {
    const char *src = nullptr;
    char *dst = nullptr;
    size_t n = 0;
    size_t total = 0;
    cudaStream_t st;
    cudaError_t err = cudaSuccess;
    explicit RunCopier(cudaStream_t s) : st(s) {}
    void add(const char *s, char *d, size_t bytes) {
        if (bytes == 0) return;
        if (n && s == src + n && d == dst + n) { n += bytes; return; }
        flush();
        src = s; dst = d; n = bytes;
    }
    void flush() {
        if (n && err == cudaSuccess) err = cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, st);
        total += n;
        n = 0;
    }
};

// Level-wise copies: position l of a set of rows, one strided 2-D copy per
// run of consecutive rows (row pitch = one row of the logit array).
struct LevelCopier {
    const char *src;
    char *dst;
    size_t pitch, width;   // bytes between rows, bytes per vector
    cudaStream_t st;
    int b0 = -1, n = 0;
    size_t total = 0;
    cudaError_t err = cudaSuccess;
    LevelCopier(const char *s, char *d, size_t p, size_t w, cudaStream_t q)
        : src(s), dst(d), pitch(p), width(w), st(q) {}
    void add(int b) {
        if (n && b == b0 + n) { ++n; return; }
        flush();
        b0 = b;
        n = 1;
    }
    void flush() {
        if (n && err == cudaSuccess) {
            const size_t off = static_cast<size_t>(b0) * pitch;
            err = cudaMemcpy2DAsync(dst + off, pitch, src + off, pitch, width,
                                    static_cast<size_t>(n), cudaMemcpyHostToDevice, st);
        }
        total += static_cast<size_t>(n) * width;
        n = 0;
    }
};

// Lengths of level l (l >= 1) of level-wise mode, from each row's
// scheduled length L and its accepted length at level l - 1: a row that
// accepted every position tested so far (a == l - 1 < L) verifies min(L, l);
// every other valid row is final and re-runs with length 0 on its copied
// position 0; an invalid length is passed on so the row is marked again.
__global__ void level_lengths_kernel(const int32_t *__restrict__ L,
                                     const int32_t *__restrict__ acc_prev, int n, int K, int l,
                                     int32_t *__restrict__ lcur) {
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < n; b += gridDim.x * blockDim.x) {
        const int Lb = L[b];
        int v;
        if (Lb < 0 || Lb > K) v = Lb;
        else if (l == 1) v = Lb < 1 ? Lb : 1;
        else v = (acc_prev[b] == l - 1 && l - 1 < Lb) ? (Lb < l ? Lb : l) : 0;
        lcur[b] = v;
    }
}

// A second stream (and an event to order it after the caller's stream) per
// device, created on first use and kept for the life of the process: the
// level-wise mode copies one half of the rows while the other half verifies.
struct Aux {
    cudaStream_t st = nullptr;
    cudaEvent_t ev = nullptr;
};
static std::mutex g_aux_mu;
static Aux g_aux[64];

static sv_status aux_stream(Aux *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return note_cuda(e);
    if (dev < 0 || dev >= 64) return SV_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_aux_mu);
    Aux &a = g_aux[dev];
    if (!a.st) {
        e = cudaStreamCreateWithFlags(&a.st, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&a.ev, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            a.st = nullptr;
            return note_cuda(e);
        }
    }
    *out = a;
    return SV_OK;
}

}  // namespace hostio
}  // namespace sv

extern "C" size_t sv_verify_host_workspace_bytes(int B, int K, int V, sv_dtype dtype) {
    sv::hostio::Layout L;
    if (!sv::hostio::make_layout(B, K, V, dtype, &L)) return 0;
    return L.bytes;
}

extern "C" sv_status sv_verify_host(const void *target_logits, const void *draft_logits,
                                    sv_dtype dtype, int B, int K, int V, const float *conf,
                                    float load, const int32_t *draft_tokens,
                                    const float *temperature, uint64_t seed, int64_t row_base,
                                    int32_t *out_tokens, int32_t *out_accept_len,
                                    int32_t *lengths, int32_t *status, int levelwise,
                                    void *workspace, size_t workspace_bytes, size_t *h2d_bytes,
                                    void *stream) {
    sv::NvtxRange nvtx_range("sv_verify_host");
    using sv::hostio::Layout;
    if (!target_logits || !draft_tokens || !temperature || !out_tokens ||
        !out_accept_len || !lengths || !workspace)
        return SV_ERR_ARG;
    if (dtype != SV_F32 && dtype != SV_BF16) return SV_ERR_DTYPE;
    Layout L;
    if (!sv::hostio::make_layout(B, K, V, dtype, &L)) return SV_ERR_SHAPE;
    if (row_base < 0 || (reinterpret_cast<uintptr_t>(workspace) & 255)) return SV_ERR_ARG;
    if (workspace_bytes < L.bytes) return SV_ERR_WORKSPACE;
    const size_t es = dtype == SV_F32 ? 4 : 2;
    const size_t vb = static_cast<size_t>(V) * es;   // bytes per logit vector
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *w = static_cast<char *>(workspace);
    float *conf_d = reinterpret_cast<float *>(w + L.conf);
    int32_t *tok_d = reinterpret_cast<int32_t *>(w + L.tok);
    float *temp_d = reinterpret_cast<float *>(w + L.temp);
    int32_t *len_d = reinterpret_cast<int32_t *>(w + L.len);
    int32_t *otok_d = reinterpret_cast<int32_t *>(w + L.otok);
    int32_t *oacc_d = reinterpret_cast<int32_t *>(w + L.oacc);
    int32_t *status_d = reinterpret_cast<int32_t *>(w + L.status);
    const size_t nb = static_cast<size_t>(B);
    const size_t nk = static_cast<size_t>(K);

    // 1. Small inputs in; with confidences, schedule and bring the lengths
    //    back (the one synchronisation), else take the caller's lengths.
    cudaError_t e =
        cudaMemcpyAsync(tok_d, draft_tokens, nb * nk * sizeof(int32_t), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(temp_d, temperature, nb * sizeof(float), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(status_d, 0, sizeof(int32_t), st);
    sv_status s = SV_OK;
    size_t small = nb * nk * sizeof(int32_t) + nb * sizeof(float);
    if (conf) {
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(conf_d, conf, nb * nk * sizeof(float), cudaMemcpyHostToDevice, st);
        if (e != cudaSuccess) return sv::note_cuda(e);
        s = sv_schedule(conf_d, B, K, load, len_d, stream);
        if (s != SV_OK) return s;
        e = cudaMemcpyAsync(lengths, len_d, nb * sizeof(int32_t), cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        small += nb * nk * sizeof(float);
    } else if (e == cudaSuccess) {
        e = cudaMemcpyAsync(len_d, lengths, nb * sizeof(int32_t), cudaMemcpyHostToDevice, st);
        small += nb * sizeof(int32_t);
    }
    if (e != cudaSuccess) return sv::note_cuda(e);

    const char *zt_h = static_cast<const char *>(target_logits);
    const char *zd_h = static_cast<const char *>(draft_logits);
    char *zt_d = w + L.zt;
    char *zd_d = w + L.zd;
    if (levelwise) {
        // Level l: position l of every undecided row in; from level 1 on,
        // verify with lengths min(L, l) (finished rows re-run with length 0
        // on data already present, their outputs ignored), decisions out.
        // The rows run in two halves, each on its own stream, ping-pong:
        // while the host waits for one half's decisions, the other half's
        // copies keep the host link busy.  The lengths of each level are
        // computed on the device from the previous level's accept lengths.
        const size_t K1 = nk + 1;
        sv::hostio::Aux aux;
        const int h = L.half;
        const bool two = B - h > 0;
        if (two) {
            s = sv::hostio::aux_stream(&aux);
            if (s != SV_OK) return s;
            // the second stream starts after the small inputs and the schedule
            e = cudaEventRecord(aux.ev, st);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(aux.st, aux.ev, 0);
            if (e != cudaSuccess) return sv::note_cuda(e);
        }
        struct Group {
            int b0, n;
            cudaStream_t st;
            char *ver;
            size_t ver_bytes;
            bool active;
        };
        Group grp[2] = {{0, h, st, w + L.ver, L.ver_bytes, true},
                        {h, B - h, two ? aux.st : st, w + L.ver1, L.ver1_bytes, two}};
        int32_t *lcur_d = reinterpret_cast<int32_t *>(w + L.lcur);
        std::vector<int32_t> acc(nb), tok(nb * K1);
        std::vector<char> alive(nb);
        for (int b = 0; b < B; ++b) {
            alive[b] = 1;
            for (size_t i = 0; i < K1; ++i) out_tokens[b * K1 + i] = -1;
            out_accept_len[b] = -1;
        }
        size_t copied = 0;
        // Copies of level l for the live rows of group g (target position l
        // if l <= L, draft position l if l < L and the row samples).
        auto copy_level = [&](const Group &g, int l) -> cudaError_t {
            const size_t lo = static_cast<size_t>(l) * vb;
            sv::hostio::LevelCopier ct(zt_h + lo, zt_d + lo, K1 * vb, vb, g.st);
            for (int b = g.b0; b < g.b0 + g.n; ++b) {
                const int Lb = lengths[b];
                if (!alive[b] || Lb < 0 || Lb > K || l > Lb) continue;
                ct.add(b);
            }
            ct.flush();
            copied += ct.total;
            if (ct.err != cudaSuccess) return ct.err;
            if (zd_h && l < K) {
                sv::hostio::LevelCopier cd(zd_h + lo, zd_d + lo, nk * vb, vb, g.st);
                for (int b = g.b0; b < g.b0 + g.n; ++b) {
                    const int Lb = lengths[b];
                    if (!alive[b] || Lb < 0 || Lb > K || l >= Lb || !(temperature[b] > 0.f))
                        continue;
                    cd.add(b);
                }
                cd.flush();
                copied += cd.total;
                if (cd.err != cudaSuccess) return cd.err;
            }
            return cudaSuccess;
        };
        // Lengths of level l and the verification of group g's rows.
        auto verify_level = [&](const Group &g, int l) -> sv_status {
            const int threads = 256;
            const int blocks = (g.n + threads - 1) / threads;
            sv::hostio::level_lengths_kernel<<<blocks, threads, 0, g.st>>>(
                len_d + g.b0, oacc_d + g.b0, g.n, K, l, lcur_d + g.b0);
            cudaError_t le = cudaGetLastError();
            if (le != cudaSuccess) return sv::note_cuda(le);
            return sv_verify(zt_d + static_cast<size_t>(g.b0) * K1 * vb,
                             zd_h ? zd_d + static_cast<size_t>(g.b0) * nk * vb : nullptr, dtype,
                             g.n, K, V, tok_d + static_cast<size_t>(g.b0) * nk, lcur_d + g.b0,
                             temp_d + g.b0, seed, row_base + g.b0,
                             otok_d + static_cast<size_t>(g.b0) * K1, oacc_d + g.b0, g.ver,
                             g.ver_bytes, status_d, g.st);
        };
        // Decisions of level l of group g back (the copy into pageable host
        // memory returns once the group's stream has reached it); rows that
        // rejected below l, reached their length, or are invalid are final.
        auto read_level = [&](Group &g, int l) -> cudaError_t {
            cudaError_t re = cudaMemcpyAsync(acc.data() + g.b0, oacc_d + g.b0,
                                             static_cast<size_t>(g.n) * sizeof(int32_t),
                                             cudaMemcpyDeviceToHost, g.st);
            if (re == cudaSuccess)
                re = cudaMemcpyAsync(tok.data() + static_cast<size_t>(g.b0) * K1,
                                     otok_d + static_cast<size_t>(g.b0) * K1,
                                     static_cast<size_t>(g.n) * K1 * sizeof(int32_t),
                                     cudaMemcpyDeviceToHost, g.st);
            if (re == cudaSuccess) re = cudaStreamSynchronize(g.st);
            if (re != cudaSuccess) return re;
            int n_alive = 0;
            for (int b = g.b0; b < g.b0 + g.n; ++b) {
                if (!alive[b]) continue;
                const int Lb = lengths[b];
                const bool bad = Lb < 0 || Lb > K;
                if (bad || acc[b] < 0 || acc[b] < l || l >= Lb) {
                    alive[b] = 0;
                    out_accept_len[b] = acc[b];
                    for (size_t i = 0; i < K1; ++i) out_tokens[b * K1 + i] = tok[b * K1 + i];
                } else {
                    ++n_alive;
                }
            }
            g.active = n_alive > 0;
            return cudaSuccess;
        };
        for (Group &g : grp) {
            if (!g.active) continue;
            e = copy_level(g, 0);
            if (e != cudaSuccess) return sv::note_cuda(e);
        }
        int last = 0;
        for (int l = 1; l <= K && (grp[0].active || grp[1].active); ++l) {
            for (Group &g : grp) {
                if (!g.active) continue;
                if (l >= 2) {
                    e = read_level(g, l - 1);
                    if (e != cudaSuccess) return sv::note_cuda(e);
                    if (!g.active) continue;
                }
                e = copy_level(g, l);
                if (e != cudaSuccess) return sv::note_cuda(e);
                s = verify_level(g, l);
                if (s != SV_OK) return s;
            }
            last = l;
        }
        for (Group &g : grp) {
            if (!g.active || last == 0) continue;
            e = read_level(g, last);
            if (e != cudaSuccess) return sv::note_cuda(e);
        }
        if (h2d_bytes) *h2d_bytes = copied + small;
        if (status) {
            e = cudaMemcpyAsync(status, status_d, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
            if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        }
        return sv::note_cuda(e);
    }

    // 2. The scheduled runs of every row: target positions 0..L, and draft
    //    positions 0..L-1 of rows that sample with draft logits.
    sv::hostio::RunCopier cp(st);
    for (int b = 0; b < B; ++b) {
        const int Lb = lengths[b];
        if (Lb < 0 || Lb > K) continue;   // verification marks the row invalid
        const size_t off_t = static_cast<size_t>(b) * (nk + 1) * vb;
        cp.add(zt_h + off_t, zt_d + off_t, static_cast<size_t>(Lb + 1) * vb);
    }
    cp.flush();
    if (zd_h) {
        for (int b = 0; b < B; ++b) {
            const int Lb = lengths[b];
            if (Lb < 1 || Lb > K || !(temperature[b] > 0.f)) continue;
            const size_t off_d = static_cast<size_t>(b) * nk * vb;
            cp.add(zd_h + off_d, zd_d + off_d, static_cast<size_t>(Lb) * vb);
        }
        cp.flush();
    }
    if (cp.err != cudaSuccess) return sv::note_cuda(cp.err);
    if (h2d_bytes) *h2d_bytes = cp.total + small;

    // 3. Verification on the device, outputs back to the host.
    s = sv_verify(zt_d, zd_h ? zd_d : nullptr, dtype, B, K, V, tok_d, len_d, temp_d, seed,
                  row_base, otok_d, oacc_d, w + L.ver, L.ver_bytes, status_d, stream);
    if (s != SV_OK) return s;
    e = cudaMemcpyAsync(out_tokens, otok_d, nb * (nk + 1) * sizeof(int32_t),
                        cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(out_accept_len, oacc_d, nb * sizeof(int32_t), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess && status)
        e = cudaMemcpyAsync(status, status_d, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
    return sv::note_cuda(e);
}
