/*
 * sv.h -- C ABI of the B200 (sm_100a) speculative-verification library.
 *
 * The library implements the data-parallel hot path of confidence-scheduled
 * speculative decoding: the per-row verify length from the drafter's
 * survival confidences (sv_schedule, sv_schedule_admit), batched draft
 * verification by speculative rejection sampling (sv_verify), the same
 * verification with the vocabulary split across ranks (sv_vp_*), and the
 * confidence head's per-position temperature (sv_sts_*).
 *
 * Conventions for every entry point:
 *  - Pointers named as device pointers must be CUDA device memory (or
 *    managed memory) owned by the caller.  The library never allocates
 *    device memory, never frees caller memory and never synchronises the
 *    stream; all work is enqueued on `stream` (a cudaStream_t passed as
 *    void*, NULL = legacy default stream) and completes asynchronously.
 *  - Argument errors are detected on the host before anything is launched
 *    and returned synchronously; nothing is written in that case.
 *  - Data errors that can only be seen on the device never fault or trap:
 *    the affected row is marked in the outputs and a bit is OR-ed into the
 *    optional device status word.
 *  - Row-major layouts; the vocabulary index is the contiguous one.
 *
 * Sources are cited as page title + section.  The pages describe the method
 * in words; the symbolic rule implemented here is the standard
 * speculative-sampling rule that their words describe.
 */
#ifndef SV_H
#define SV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SV_OK = 0,
    SV_ERR_ARG = 1,        /* null pointer, negative size, bad seed/row base, misaligned pointer */
    SV_ERR_SHAPE = 2,      /* B, K or V out of the supported range */
    SV_ERR_DTYPE = 3,      /* unknown logit dtype */
    SV_ERR_WORKSPACE = 4,  /* workspace smaller than sv_verify_workspace_bytes() */
    SV_ERR_CUDA = 5        /* a CUDA launch or query failed (see sv_last_cuda_error) */
} sv_status;

typedef enum { SV_F32 = 0, SV_BF16 = 1 } sv_dtype;

/* Bits OR-ed into the optional device status word by sv_verify. */
#define SV_ROW_BAD_TOKEN        1   /* a verified draft token lies outside [0, V) */
#define SV_ROW_BAD_LENGTH       2   /* lengths[b] outside [0, K] */
#define SV_ROW_BAD_TEMPERATURE  4   /* T < 0, NaN, inf, or 0 < T < 1e-6 */
#define SV_NOTE_ZERO_RESIDUAL   8   /* informational: a rejection left zero residual mass (drew from p_j) */
#define SV_NOTE_CDF_FALLBACK   16   /* informational: rounding put the CDF target past the total */
#define SV_NOTE_TIMEOUT        32   /* an internal wait exceeded its 1 s bound; outputs are undefined */

/* Supported sizes. */
#define SV_MAX_K  64
#define SV_MAX_V  (1 << 20)
#define SV_MAX_ADMIT 8192   /* B * K candidates for sv_schedule_admit */

/*
 * sv_schedule -- per-row verify length from prefix survival.
 *
 * Defined by: umans.ai, "DeepSeek V4 Pro DSpark: the model isn't ready, the
 * architecture is", section "What DSpark adds", item "2. Verify smarter"
 * (for each draft position a confidence head estimates the chance that the
 * token is kept once every token before it was kept; the running product
 * along the block is then the chance that each prefix is kept); aiweekly.co
 * alert (the verify length follows the estimated survival of each prefix
 * and the current load); en.5iter.com article, section "What DSpark changed is how to generate a
 * draft", and techvisionai "DeepSeek-V4: Breaking the Efficiency Barrier",
 * Ch. 7 "Confidence-Scheduled Verification" (verify longer when idle, only
 * the confident prefix when busy).
 *
 * Computes, per row b, S_i = prod_{j<=i} clamp(conf[b, j-1], 0, 1) (NaN
 * counts as 0) for i = 1..K, left to right in fp32, and
 * lengths[b] = max{ i in 0..K : S_i >= load } with S_0 = 1.  `load` is the
 * load-dependent threshold tau (larger under heavier load).
 *
 *   conf     device, float32 [B, K], read only.
 *   B, K     rows and drafts per row; B >= 1, 1 <= K <= SV_MAX_K.
 *   load     threshold tau; any float (tau <= 0 keeps every draft, tau > 1
 *            keeps none, NaN keeps none).
 *   lengths  device, int32 [B], written.
 * Returns SV_OK, SV_ERR_ARG (null pointer), SV_ERR_SHAPE, or SV_ERR_CUDA.
 *
 * The confidences must be causal with respect to this step's sampling (the
 * umans.ai page sizes the truncation from confidences measured two steps
 * earlier); that is the caller's contract, not checked here.
 */
sv_status sv_schedule(const float *conf, int B, int K, float load,
                      int32_t *lengths, void *stream);

/*
 * sv_schedule_admit -- per-row verify lengths by hardware-aware admission.
 *
 * Defined by: umans.ai, "DeepSeek V4 Pro DSpark: the model isn't ready, the
 * architecture is", section "What DSpark adds", item "2. Verify smarter"
 * (the engine's verification rate is measured once for each batch size;
 * at each step the candidates of all requests are ranked by their survival
 * chance and taken in that order for as long as the expected number of
 * accepted tokens, multiplied by the measured rate at the resulting batch
 * size, keeps growing);
 * techvisionai "DeepSeek-V4: Breaking the Efficiency Barrier", Ch. 7
 * "Hardware-Aware Scheduling"; zhichai.net DSpark topic, "Under the hood".
 *
 * Per row, S_i = prod_{j<=i} clamp(conf[b, j-1], 0, 1) (NaN counts as 0),
 * computed in fp64.  Candidates (b, i) are taken in order of S descending,
 * ties by (b, i) ascending.  After k admissions the verify batch holds
 * n = B + k tokens (every row verifies its final position) and the expected
 * emitted tokens are E(k) = B + (sum of the admitted S).  Candidate k+1 is
 * admitted iff n + 1 < n_speed and E(k+1) * speed[n+1] > E(k) * speed[n];
 * admission stops at the first candidate that fails.
 *
 *   conf     device float32 [B, K], read only.
 *   B, K     1 <= B, 1 <= K <= SV_MAX_K, B * K <= SV_MAX_ADMIT.
 *   speed    device float32 [n_speed]: the profiled verification steps per
 *            second at a batch of n tokens, n = 0 .. n_speed-1 (the load
 *            enters through this table).  n_speed >= 1.
 *   lengths  device int32 [B], written: admitted candidates of each row (a
 *            prefix of its draft block).
 *   tau_out  device float32 [1], nullable: S of the last admitted candidate,
 *            rounded to fp32 (+inf if none), the threshold that sv_schedule
 *            would need to keep the same prefixes.
 * Returns SV_OK, SV_ERR_ARG, SV_ERR_SHAPE or SV_ERR_CUDA.  One CTA; no
 * workspace.  The partial sums run in a parallel order, so a candidate whose
 * throughput gain is zero to ~1e-15 relative may be decided differently from
 * a strictly sequential sum.
 */
sv_status sv_schedule_admit(const float *conf, int B, int K, const float *speed, int n_speed,
                            int32_t *lengths, float *tau_out, void *stream);

/*
 * sv_sts_fit -- per-position temperature of the confidence head, fitted on
 * held-out blocks (the calibration that feeds sv_schedule / sv_schedule_admit).
 *
 * Defined by: umans.ai, "DeepSeek V4 Pro DSpark: the model isn't ready, the
 * architecture is", section "What DSpark adds", item "2. Verify smarter"
 * (the head's raw confidence is overconfident by 3-8% expected calibration
 * error; a temperature for each position, chosen on blocks kept aside,
 * lowers that to about 1%); zhichai.net DSpark topic, "Under the hood" (Sequential
 * Temperature Scaling).
 *
 * The head predicts survival of position i given that every earlier
 * position survived, so position i of block n is observed iff
 * i <= accept_len[n] and survived iff i < accept_len[n] (blocks with
 * accept_len < 0 are skipped).  T_i = 1/beta_i minimises
 * sum over observed n of log(1 + exp(-s beta logits[n, i])), s = +1 survived,
 * -1 not, over beta in [1/tmax, 1/tmin] (convex in beta; fp64 sums).  A
 * position that no block reached, or whose observed logits are all 0, gets
 * T = 1.  The expected calibration error uses 15 equal-width bins over every
 * observed (n, i): sum over bins |sum (y - conf)| / count.
 *
 *   logits       device float32 [N, K], read only: the head's logits
 *                (confidence = sigmoid(logit)).
 *   accept_len   device int32 [N], read only: accepted length of each
 *                held-out block (e.g. out_accept_len of sv_verify).
 *   N, K         1 <= N, 1 <= K <= SV_MAX_K.
 *   tmin, tmax   0 < tmin < tmax, finite: the temperature range.
 *   temperature  device float32 [K], written.
 *   ece          device float32 [2], nullable: calibration error before
 *                (T = 1) and after the fit.
 *   workspace    device scratch of sv_sts_workspace_bytes(N, K) bytes,
 *                16-byte aligned, owned by the caller.
 * Returns SV_OK, SV_ERR_ARG, SV_ERR_SHAPE, SV_ERR_WORKSPACE or SV_ERR_CUDA.
 * Enqueues one memset and one cooperative launch (all CTAs resident, a
 * bounded grid barrier between passes) on `stream`; never synchronises.
 */
size_t sv_sts_workspace_bytes(int N, int K);
sv_status sv_sts_fit(const float *logits, const int32_t *accept_len, int N, int K, float tmin,
                     float tmax, float *temperature, float *ece, void *workspace,
                     size_t workspace_bytes, void *stream);

/*
 * sv_sts_apply -- calibrated confidences conf[n, i] = sigmoid(logits[n, i] /
 * temperature[i]) (same passages as sv_sts_fit), ready for sv_schedule.
 *   logits [N, K], temperature [K] read only; conf_out [N, K] written; all
 *   device float32.  Returns SV_OK, SV_ERR_ARG, SV_ERR_SHAPE or SV_ERR_CUDA.
 */
sv_status sv_sts_apply(const float *logits, const float *temperature, int N, int K,
                       float *conf_out, void *stream);

/*
 * Test exports for the bounded wait of sv_sts_fit's grid barrier (no
 * counterpart on the pages: they exist so that the failure path of a wait
 * can be exercised without hanging or faulting a GPU).
 *
 * sv_debug_sts_wait_limit -- wall-time limit, in ns, of one barrier wait of
 *   the calibration kernel on the current device; 0 restores the default
 *   (1 s).  With a limit near zero the fit gives up at its first barrier:
 *   sv_sts_fit still returns SV_OK, the temperatures come out NaN and ECE is
 *   left unwritten.  Affects later launches only; not thread-safe against
 *   fits in flight.  Returns SV_OK or SV_ERR_CUDA.
 * sv_debug_sts_timeouts -- the number of barrier waits on the current device
 *   that ran out since the previous call (then cleared); -1 on a CUDA error.
 *   Synchronous (it copies from device memory).
 */
sv_status sv_debug_sts_wait_limit(uint64_t limit_ns);
int sv_debug_sts_timeouts(void);

/*
 * sv_verify_workspace_bytes -- device scratch that sv_verify needs for
 * (B, K, V, dtype): work counters, per-row state (length, first rejection
 * found so far, per-position completion counts), the position-major work
 * list, the per-chunk softmax partials and the residual draw table: about
 * B * V * elt / 256 + B * (2K+1) * V * elt / 8192 bytes (0.42 MB at
 * B = 256, K = 8, V = 129280 bf16).  Returns 0 for
 * unsupported sizes.
 */
size_t sv_verify_workspace_bytes(int B, int K, int V, sv_dtype dtype);

/*
 * sv_verify -- batched speculative verification.
 *
 * Defined by: umans.ai page above, section "Speculative decoding, briefly"
 * (one target pass scores the whole draft block; the drafts the target
 * agrees with are kept, followed by one token of the target's own, and the
 * rest are dropped; the test is rejection sampling, which leaves the emitted
 * tokens distributed exactly as the target's, and a rejected draft gives way
 * to a token of the target's choosing); zhichai.net DSpark topic, section
 * "Why LLMs speak so slowly" (rejection sampling on the ratio of target to
 * draft probability; decoding goes on from the first rejected position).
 * In symbols, per row b
 * with verify length L = lengths[b] and temperature T = temperature[b]:
 *
 *   p_i = softmax(zt[b, i, :] / T),  q_i = softmax(zd[b, i, :] / T);
 *   for i = 0..L-1: accept x_i = draft_tokens[b, i] iff
 *       u(seed, row, i, 0) < min(1, p_i(x_i) / q_i(x_i));
 *   j = first rejected i, or L if all survive;
 *   y drawn by inverse CDF, in token order, with u(seed, row, j, 1) from
 *       max(0, p_j - q_j) (j < L) or p_L (j == L): the smallest v whose
 *       cumulative weight exceeds u * (total weight);
 *   out_tokens[b] = x_0 .. x_{j-1}, y, then -1;  out_accept_len[b] = j.
 *   T == 0 is greedy verification: accept while x_i equals the target argmax
 *   (lowest index on ties), y = target argmax at j; no uniforms are drawn and
 *   the draft logits are not read.
 *   draft_logits == NULL selects a greedy drafter (q_i one-hot at x_i, the
 *   techvisionai page, Ch. 7 "Deployment with vLLM", draft_sample_method
 *   greedy): accept with probability p_i(x_i), resample from p_j with x_j
 *   removed.
 *
 * u(seed, row, pos, draw) = (w0 >> 8) * 2^-24 where w0 is word 0 of
 * Philox4x32-10 (Salmon et al., SC'11) with key (seed_lo, seed_hi) and
 * counter (row_lo, pos, draw, row_hi); row = row_base + b, so that shards of
 * one batch verified separately with their row offsets reproduce the
 * unsharded result.  Change `seed` every decoding step.
 *
 *   target_logits  device [B, K+1, V] of `dtype`; read only.  Positions
 *                  i > L of row b are never read.
 *   draft_logits   device [B, K, V] of `dtype`, or NULL (greedy drafter);
 *                  read only; positions i >= L and rows with T == 0 are
 *                  never read.
 *   dtype          SV_F32 or SV_BF16; both logit arrays share it.  Logits
 *                  must be finite or -inf, with at least one finite logit
 *                  per vector that is read.
 *   B, K, V        1 <= B, 1 <= K <= SV_MAX_K, 1 <= V <= SV_MAX_V.
 *   draft_tokens   device int32 [B, K]; entries i >= L are ignored.
 *   lengths        device int32 [B] (e.g. the output of sv_schedule).
 *   temperature    device float32 [B].
 *   seed           Philox key.
 *   row_base       Philox row id of local row 0 (>= 0).
 *   out_tokens     device int32 [B, K+1], written.
 *   out_accept_len device int32 [B], written; -1 for an invalid row.
 *   workspace      device, >= sv_verify_workspace_bytes(B, K, V, dtype)
 *                  bytes, 16-byte aligned; scratch owned by the caller,
 *                  contents need not be initialised and are undefined
 *                  afterwards.  Calls that share a workspace must be
 *                  stream-ordered.
 *   status         device int32, nullable; SV_ROW_* and SV_NOTE_* bits are
 *                  OR-ed in (the library never clears it).
 * Logit pointers must be aligned to their element size; any 16-byte
 * misalignment of individual vectors is handled.
 * Returns SV_OK, SV_ERR_ARG, SV_ERR_SHAPE, SV_ERR_DTYPE, SV_ERR_WORKSPACE or
 * SV_ERR_CUDA.  An invalid row (bad length, temperature or token) gets
 * out_accept_len = -1 and a row of -1 in out_tokens; other rows are
 * unaffected.
 */
sv_status sv_verify(const void *target_logits, const void *draft_logits, sv_dtype dtype,
                    int B, int K, int V,
                    const int32_t *draft_tokens, const int32_t *lengths,
                    const float *temperature, uint64_t seed, int64_t row_base,
                    int32_t *out_tokens, int32_t *out_accept_len,
                    void *workspace, size_t workspace_bytes, int32_t *status,
                    void *stream);

/*
 * sv_schedule_verify -- sv_schedule followed by sv_verify, in one call and
 * without the schedule launch: the verification prologue computes each
 * row's length from its confidences with the same function as sv_schedule
 * (same formula, same fp32 order), writes it to `lengths`, and verifies
 * with it.  Lengths and outputs are identical, bit for bit, to calling
 * sv_schedule(conf, B, K, load, lengths) and then sv_verify with `lengths`.
 *
 * Defined by: the passages cited at sv_schedule and sv_verify.
 *
 *   conf      device, float32 [B, K], read only (as sv_schedule).
 *   load      threshold tau (as sv_schedule).
 *   lengths   device, int32 [B], written: the scheduled verify lengths.
 *   Every other argument is that of sv_verify.
 * Returns SV_OK, SV_ERR_ARG (a null pointer, including conf or lengths),
 * SV_ERR_DTYPE, SV_ERR_SHAPE, SV_ERR_WORKSPACE or SV_ERR_CUDA; the workspace
 * is sv_verify_workspace_bytes(B, K, V, dtype).
 */
sv_status sv_schedule_verify(const void *target_logits, const void *draft_logits, sv_dtype dtype,
                             int B, int K, int V, const int32_t *draft_tokens,
                             const float *conf, float load, int32_t *lengths,
                             const float *temperature, uint64_t seed, int64_t row_base,
                             int32_t *out_tokens, int32_t *out_accept_len,
                             void *workspace, size_t workspace_bytes, int32_t *status,
                             void *stream);

/*
 * sv_verify_debug -- sv_verify plus an export of the softmax normalisers it
 * computed: stats_out (device float32 [B, 2K+1, 2]) receives, for every
 * vector the call read, (m, Sigma) with m = max_v z_v and
 * Sigma = sum_v exp((z_v - m) / T) (Sigma = 1 at T == 0).  Slot i <= K is
 * target position i, slot K+1+i is draft position i.  Slots that were not
 * read are left untouched.  For tests and diagnostics.
 */
sv_status sv_verify_debug(const void *target_logits, const void *draft_logits, sv_dtype dtype,
                          int B, int K, int V,
                          const int32_t *draft_tokens, const int32_t *lengths,
                          const float *temperature, uint64_t seed, int64_t row_base,
                          int32_t *out_tokens, int32_t *out_accept_len,
                          void *workspace, size_t workspace_bytes, int32_t *status,
                          float *stats_out, void *stream);

/*
 * sv_verify_noalloc -- sv_verify without a caller-provided workspace.
 *
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory when they verify: a serving loop that
 * plans all of its memory up front and forbids allocation afterwards, a
 * plain C host program with no device allocator of its own, or code that
 * must not touch the allocator while other work is in flight.  The scratch
 * that sv_verify takes as `workspace` lives instead in one fixed device
 * array inside this library, 16 MiB per GPU, which every GPU that loads the
 * library holds until the process exits.
 *
 *   Arguments and results are those of sv_verify, minus workspace and
 *   workspace_bytes.  Batches whose sv_verify_workspace_bytes(B, K, V, dtype)
 *   exceeds 16 MiB (16777216 bytes) are rejected with SV_ERR_WORKSPACE
 *   before anything is launched; use sv_verify with a workspace for those.
 *   The library calls no cudaMalloc, cudaFree or other allocating routine.
 *   Each call looks up the array's device address on the current device
 *   (cudaGetSymbolAddress), so the address stays right after the device's
 *   context is reset; the first call on a device may load the library's
 *   device code, so make it before any stream capture.  Every call shares the one array and leaves its contents
 *   behind: counters that must start at zero are reset by each call's
 *   first kernel, everything else is written before it is read.  Calls
 *   whose work overlaps on the GPU (other streams, other host threads on the
 *   same device) race on the array; order them on one stream.
 */
sv_status sv_verify_noalloc(const void *target_logits, const void *draft_logits, sv_dtype dtype,
                            int B, int K, int V,
                            const int32_t *draft_tokens, const int32_t *lengths,
                            const float *temperature, uint64_t seed, int64_t row_base,
                            int32_t *out_tokens, int32_t *out_accept_len, int32_t *status,
                            void *stream);

/*
 * Vocabulary-parallel verification: sv_vp_stats, sv_vp_decide, sv_vp_draw.
 *
 * The rule is that of sv_verify (the umans.ai and zhichai.net passages cited
 * there), for a target and drafter whose output heads are split across
 * ranks by vocabulary, so that each rank holds only a contiguous slice of
 * both models' logits (zhichai.net DSpark topic, "From paper to running
 * service in two weeks": the method is served by vLLM and SGLang on 8-GPU
 * nodes; techvisionai "DeepSeek-V4: Breaking the Efficiency Barrier",
 * Ch. 7 "Deployment with vLLM").  The pages do not say how the heads are
 * split; slices ordered by rank that partition [0, V) are the reading taken.
 *
 * One verification step on every rank, with the caller's exchanges between:
 *   sv_vp_stats     partials of this slice           -> stats_local
 *   all-gather      stats_local of every rank, in rank order -> stats_all
 *   sv_vp_decide    accept tests, accepted prefix    -> out_tokens, out_accept_len,
 *                   this slice's draw masses          -> mass_local
 *   all-gather      mass_local of every rank, in rank order -> mass_all
 *   sv_vp_draw      the rank whose slice holds the draw writes the drawn token
 *   all-reduce(max) out_tokens over the ranks
 * Every rank computes the same normalisers, decisions and uniforms from the
 * same gathered data, so out_accept_len and the accepted prefix agree on
 * all ranks without an exchange; before the final all-reduce the drawn
 * position holds -1 on every rank but one.  Results equal those of
 * sv_verify on the whole vocabulary up to the rounding of the sums (fp32,
 * a different summation order); decisions inside the tie windows of
 * sv_verify may differ.  SV_NOTE_CDF_FALLBACK can be raised on one rank
 * only (the one that drew); every other bit is raised on every rank.
 *
 * sv_vp_slice describes this rank's slice; every call of a step takes the
 * same description.
 */
typedef struct {
    const void *target_logits;  /* device [B, K+1, Vs] of dtype: this slice of zt */
    const void *draft_logits;   /* device [B, K, Vs] of dtype, or NULL (greedy drafter) */
    sv_dtype dtype;
    int B, K;                   /* 1 <= B, 1 <= K <= SV_MAX_K */
    int V;                      /* whole vocabulary, 1 <= V <= SV_MAX_V */
    int v0, Vs;                 /* this slice holds tokens v0 .. v0+Vs-1; 1 <= Vs <= ceil(V / nshards) */
    int nshards;                /* ranks the vocabulary is split over, 1 <= nshards <= V */
    int shard;                  /* this rank's place in slice order, 0 .. nshards-1 */
} sv_vp_slice;

/*
 * sv_vp_stats_bytes -- bytes of stats_local: B * (2K+1) * C records of 16
 * bytes, C = ceil(ceil(V / nshards) * elt / 65536) clamped to [1, 64] (the
 * same on every rank).  stats_all is nshards times that.  0 for an invalid
 * slice.
 * sv_vp_workspace_bytes -- per-rank scratch of sv_vp_decide and sv_vp_draw:
 * a 48-byte draw record, two segment tables of the slice (at most 2 * 512
 * floats), their part sums (at most 2 * 32 floats) and a counter per row.
 * 0 for an invalid slice.
 */
size_t sv_vp_stats_bytes(const sv_vp_slice *slice);
size_t sv_vp_workspace_bytes(const sv_vp_slice *slice);

/*
 * sv_vp_stats -- per (row, slot, chunk) of the slice: (m, Sigma, z_x, w) with
 * m = max z, Sigma = sum exp((z - m) / T) over the chunk; in chunk 0, z_x is
 * the logit of the row's draft token at that position and w = 1 when the
 * slice holds the token (else z_x = 0, w = 0).  Greedy rows (T == 0): (max,
 * 0, 0, global index of the first argmax).  Slot i <= K is target position
 * i, slot K+1+i draft position i; only the slots sv_vp_decide reads
 * (target 0..L, draft 0..L-1 of sampled rows with draft logits) are written;
 * rows with a bad length or temperature are skipped.
 *   draft_tokens, lengths, temperature  as for sv_verify.
 *   stats_local  device, sv_vp_stats_bytes() bytes, 16-byte aligned, written.
 * Returns SV_OK, SV_ERR_ARG, SV_ERR_SHAPE, SV_ERR_DTYPE or SV_ERR_CUDA.
 */
sv_status sv_vp_stats(const sv_vp_slice *slice, const int32_t *draft_tokens,
                      const int32_t *lengths, const float *temperature, void *stats_local,
                      void *stream);

/*
 * sv_vp_decide -- per row: validates it (as sv_verify: an invalid row gets
 * -1 everywhere and its SV_ROW_* bit), merges the partials of every rank in
 * a fixed order, runs the accept tests with u(seed, row, i, 0), writes
 * out_accept_len[b] = j and out_tokens[b] = x_0 .. x_{j-1}, y, -1 ... where
 * y is the target argmax for greedy rows and -1 (to be drawn) otherwise,
 * and sums this slice's draw weights at position j.
 *   stats_all      device [nshards] x stats_local, rank order, 16-byte aligned.
 *   seed, row_base as for sv_verify.
 *   out_tokens     device int32 [B, K+1]; out_accept_len device int32 [B].
 *   mass_local     device float32 [B, 2], 8-byte aligned, written: the
 *                  slice's total draw weight and its total unnormalised
 *                  target weight (the zero-residual fallback); 0 for rows
 *                  with no draw.
 *   norm_out       device float32 [B, 2K+1, 2], nullable: the merged
 *                  (m, Sigma) of every slot read (as sv_verify_debug).
 *   workspace      device, >= sv_vp_workspace_bytes(), 16-byte aligned,
 *                  kept for sv_vp_draw of the same step.
 *   status         device int32, nullable; bits OR-ed in.
 * Returns SV_OK, SV_ERR_ARG, SV_ERR_SHAPE, SV_ERR_DTYPE, SV_ERR_WORKSPACE or
 * SV_ERR_CUDA.  Two launches: the decisions (one CTA per row), then the
 * slice masses (up to 32 CTAs per row).
 */
sv_status sv_vp_decide(const sv_vp_slice *slice, const void *stats_all,
                       const int32_t *draft_tokens, const int32_t *lengths,
                       const float *temperature, uint64_t seed, int64_t row_base,
                       int32_t *out_tokens, int32_t *out_accept_len, float *mass_local,
                       float *norm_out, void *workspace, size_t workspace_bytes,
                       int32_t *status, void *stream);

/*
 * sv_vp_draw -- per row with a draw: R = sum of the slices' masses in rank
 * order (the unnormalised target weight if the draw's own mass is zero,
 * raising SV_NOTE_ZERO_RESIDUAL), t = u(seed, row, j, 1) * R; the slice
 * whose exclusive prefix is <= t < prefix + mass holds the token, and only
 * that rank writes out_tokens[b, j] = the smallest token of its slice whose
 * cumulative weight passes t (the last positive one, with
 * SV_NOTE_CDF_FALLBACK, if rounding leaves t at or past the total).
 *   mass_all   device float32 [nshards, B, 2], rank order, 8-byte aligned.
 *   out_tokens as written by sv_vp_decide of this step.
 *   workspace  the one sv_vp_decide of this step used.
 * Returns SV_OK, SV_ERR_ARG, SV_ERR_SHAPE, SV_ERR_DTYPE, SV_ERR_WORKSPACE or
 * SV_ERR_CUDA.
 */
sv_status sv_vp_draw(const sv_vp_slice *slice, const float *mass_all, int32_t *out_tokens,
                     void *workspace, size_t workspace_bytes, int32_t *status, void *stream);

/*
 * sv_verify_host -- schedule and verify a batch whose inputs live in host
 * memory, moving only the logits the method reads across the host link.
 *
 * Verification reads, per row, the target positions 0..L and the draft
 * positions 0..L-1 that the schedule keeps and nothing past them (umans.ai
 * page, section "What DSpark adds", item "2. Verify smarter": only the
 * confident prefix is verified).  This call copies the confidences, tokens
 * and temperatures in, runs sv_schedule with threshold `load`, copies the
 * lengths out and waits for them (its one synchronisation of `stream`),
 * then copies only each row's scheduled runs of both logit arrays (one
 * cudaMemcpyAsync per contiguous run, adjacent runs merged), runs
 * sv_verify, and copies out_tokens, out_accept_len and status back.  The
 * results equal sv_schedule followed by sv_verify on device copies of the
 * same inputs.
 *
 *   target_logits, draft_logits  HOST [B, K+1, V] and [B, K, V] of dtype
 *                  (draft NULL: greedy drafter); pinned memory lets the copies
 *                  run asynchronously.
 *   conf           HOST float32 [B, K], and load: the schedule threshold tau.
 *                  conf NULL: no schedule and no synchronisation; `lengths`
 *                  is then a HOST input (e.g. lengths fixed by the caller).
 *   draft_tokens   HOST int32 [B, K]; temperature: HOST float32 [B].
 *   out_tokens, out_accept_len   HOST, written once `stream` has drained.
 *   lengths        HOST int32 [B]: written (by the time the call returns)
 *                  when conf is given, read when conf is NULL.
 *   status         HOST int32, nullable: the SV_ROW_* / SV_NOTE_* bits of
 *                  this call (written once `stream` has drained).
 *   levelwise      0: copy every scheduled run at once (one synchronisation).
 *                  1: level by level: level l copies position l of the rows
 *                  still undecided and, from l = 1, verifies with lengths
 *                  min(L, l); a row is final once it rejects below l or l
 *                  reaches L.  What crosses is what the outcome depends on
 *                  (target 0..a, draft 0..min(a, L-1), a = accepted length)
 *                  plus, for a row rejecting at a < L, position a+1, copied
 *                  before the rejection is known.  Same results (the
 *                  uniforms are keyed by row, position and draw), up to K
 *                  synchronisations per half; SV_NOTE_* bits may also come
 *                  from draws whose rows were still undecided.  The rows
 *                  run in two halves on `stream` and on a second stream the
 *                  library creates once per device (kept until exit), so
 *                  one half's copies overlap the other half's verification;
 *                  each level's lengths are computed on the device.
 *   workspace      DEVICE, >= sv_verify_host_workspace_bytes(), 256-byte
 *                  aligned: device copies of both logit arrays (only the
 *                  scheduled runs are written), the small arrays and the
 *                  sv_verify workspaces (one per half in level-wise mode).
 *   h2d_bytes      nullable: bytes copied host-to-device by this call.
 * Returns SV_OK, SV_ERR_ARG, SV_ERR_SHAPE, SV_ERR_DTYPE, SV_ERR_WORKSPACE or
 * SV_ERR_CUDA.  Argument errors are returned before anything is enqueued.
 */
size_t sv_verify_host_workspace_bytes(int B, int K, int V, sv_dtype dtype);
sv_status sv_verify_host(const void *target_logits, const void *draft_logits, sv_dtype dtype,
                         int B, int K, int V, const float *conf, float load,
                         const int32_t *draft_tokens, const float *temperature, uint64_t seed,
                         int64_t row_base, int32_t *out_tokens, int32_t *out_accept_len,
                         int32_t *lengths, int32_t *status, int levelwise, void *workspace,
                         size_t workspace_bytes, size_t *h2d_bytes, void *stream);

/*
 * sv_philox_uniforms -- the uniforms sv_verify draws, for tests:
 * out[k] = u(seed, row[k], pos[k], draw[k]) as defined above.
 * row: device int64 [n] (>= 0); pos, draw: device int32 [n]; out: device
 * float32 [n].  n >= 0.
 */
sv_status sv_philox_uniforms(uint64_t seed, const int64_t *row, const int32_t *pos,
                             const int32_t *draw, int n, float *out, void *stream);

/*
 * sv_philox4x32_10 -- raw Philox4x32-10 blocks (Salmon et al., SC'11), for
 * tests: out[4k..4k+3] = Philox(ctr[4k..4k+3], key[2k..2k+1]).
 * ctr, out: device uint32 [n, 4]; key: device uint32 [n, 2].
 */
sv_status sv_philox4x32_10(const uint32_t *ctr, const uint32_t *key, int n, uint32_t *out,
                           void *stream);

/*
 * Profiling hooks (benchmark use).  sv_profile_begin(capacity) makes the
 * next `capacity` sv_verify calls on this process record CUDA events around
 * their main verification kernel (capacity <= 0 disables recording).
 * sv_profile_read(ms, max) waits for those events and writes up to `max`
 * per-launch durations in milliseconds; returns how many were recorded.
 * Not thread-safe.
 */
sv_status sv_profile_begin(int capacity);
int sv_profile_read(float *ms, int max);

/* Number of CUDA kernels one sv_verify call launches. */
int sv_verify_launches(void);

/* Human-readable status name; never NULL. */
const char *sv_status_string(sv_status s);

/* The last CUDA error code seen by the calling thread (0 if none). */
int sv_last_cuda_error(void);

/* Library ABI version. */
int sv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SV_H */
