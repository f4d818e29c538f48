/*
 * dspark.h — C ABI of the B200 (sm_100a) hot path of one DSpark-style
 * confidence-scheduled speculative-decoding round:
 *
 *   dspark_draft_sample    semi-autoregressive draft: parallel base logits plus
 *                          a low-rank Markov-head bias, sampled position by position
 *                          (dspark_draft_logits / dspark_draft_pick: one position's
 *                          two halves; dspark_draft_sample_recurrent: the recurrent
 *                          head in place of the Markov head; dspark_draft_sample_beside:
 *                          either head, leaving SMs to other streams)
 *   dspark_prefix_schedule calibrated confidence, survival products and the
 *                          early-stopping prefix cut against a cost-per-token table
 *   dspark_sts_fit         Sequential Temperature Scaling of the confidences, ECE
 *   dspark_verify          lossless rejection-sampling verification, residual or
 *                          bonus token, accepted lengths and emitted tokens
 *                          (dspark_verify_target_stats / dspark_verify_from_stats:
 *                          its two halves, so the first can run beside the draft)
 *
 * Sources, cited by page title and section:
 *   [P1] "DSpark turns speculation into a scheduler" (benebsworth.pages.dev)
 *   [P2] "notes/dspark-deepseek" (skandtandon.pages.dev)
 *   [P3] "DSpark LLM inference speedup" (probackend.com)
 *
 * Conventions shared by every entry point
 *   - Tensors are caller-owned DEVICE pointers, row-major with the vocabulary
 *     innermost, 16-byte aligned. V must be a multiple of 8.
 *   - dtype is DSPARK_F32 or DSPARK_BF16 and applies to every logit tensor and
 *     to the Markov factors U, W. Temperatures, probabilities, confidences and
 *     costs are always fp32; token ids are int32.
 *   - The library never allocates or frees device memory. Each call takes a
 *     caller-owned device workspace of at least dspark_workspace_bytes() bytes;
 *     its first 256 bytes are a status block that must be zero before first use
 *     (dspark_clear_status) and that the calls only ever OR bits into.
 *   - Every call is asynchronous on the given stream (a cudaStream_t; NULL is
 *     the legacy default stream): no host synchronisation, no device trap.
 *   - Return value: DSPARK_OK or a negative DSPARK_ERR_* code. Argument errors
 *     are detected on the host before anything is launched.
 *   - Data errors found on the device (a token id outside [0, V), a row whose
 *     logits are NaN, +inf or all -inf, a cut outside [0, K], a negative or NaN
 *     temperature, a bounded device wait that gave up) set DSPARK_STATUS_* bits
 *     and the lowest offending request index in the status block; the kernel
 *     then writes a defined value (token 0, accepted length 0) and carries on.
 *     dspark_read_status() returns them.
 *   - Random numbers: Philox4x32-10 (Salmon et al., SC'11), key = seed,
 *     counter = (request, purpose << 24 | position, lo32(round_id),
 *     hi32(round_id)), u = (word0 >> 8) * 2^-24; purposes 0 draft, 1 accept,
 *     2 residual, 3 bonus. A round is fully reproducible from (seed, round_id).
 */
#ifndef DSPARK_H
#define DSPARK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same underlying type as cudaStream_t, so that C callers need no CUDA header. */
typedef struct CUstream_st* dspark_stream_t;

enum { DSPARK_F32 = 0, DSPARK_BF16 = 1 };

enum {
  DSPARK_OK = 0,
  DSPARK_ERR_INVALID_ARG = -1,  /* null pointer, bad size, misalignment      */
  DSPARK_ERR_UNSUPPORTED = -2,  /* dtype, shape or device not supported      */
  DSPARK_ERR_CUDA = -3,         /* a CUDA launch or runtime call failed      */
  DSPARK_ERR_WORKSPACE = -4,    /* workspace smaller than the query's answer */
  DSPARK_ERR_TIMEOUT = -5       /* reported by dspark_read_status only       */
};

enum { DSPARK_OP_DRAFT = 0, DSPARK_OP_SCHEDULE = 1, DSPARK_OP_VERIFY = 2, DSPARK_OP_CALIB = 3 };

/* Prefix-cut modes of dspark_prefix_schedule. */
enum { DSPARK_CUT_COST = 0, DSPARK_CUT_THRESHOLD = 1, DSPARK_CUT_NONE = 2 };

/* Bits of the device status word. */
#define DSPARK_STATUS_BAD_TOKEN 0x1u /* token id outside [0, V)                 */
#define DSPARK_STATUS_BAD_ROW 0x2u   /* NaN / +inf / all -inf logits in a row    */
#define DSPARK_STATUS_BAD_CUT 0x4u   /* cut outside [0, K]                       */
#define DSPARK_STATUS_BAD_TEMP 0x8u  /* temperature negative or NaN             */
#define DSPARK_STATUS_TIMEOUT 0x10u  /* a bounded device wait gave up           */
#define DSPARK_STATUS_INTERNAL 0x20u /* a kernel precondition failed (alignment) */

/*
 * Workspace bytes needed by operation `op` (DSPARK_OP_*) for these sizes
 * (r is ignored except by DSPARK_OP_DRAFT). Pure host function. Returns 0 for
 * unsupported arguments. One workspace of the largest size may serve all the
 * operations of a round: the draft's chunk partials and verification's target
 * statistics occupy different regions of it, so dspark_verify_target_stats may
 * run beside dspark_draft_sample; otherwise the calls must not overlap.
 */
size_t dspark_workspace_bytes(int op, int B, int K, int V, int r, int dtype);

/*
 * Draft sampling with the Markov head, K positions in turn.
 * [P1] "DSpark's semi-autoregressive compromise" (parallel base logits plus a
 * prefix-dependent transition bias from the previous sampled token);
 * [P3] "The Semi-Autoregressive Trick" (low-rank Markov head, rank 256).
 *
 * For k = 1..K and every request b:
 *   bias     = bias_scale[b] * U[x_{b,k-1}, :] @ W          (fp32 accumulation)
 *   d[b,k-1] = round_dtype(base[b,k-1] + bias)              (stored logits)
 *   x[b,k-1] ~ softmax(d[b,k-1] / temp[b]) by inverse CDF in index order with
 *              u = Philox(seed, b, k, purpose 0, round_id); argmax (lowest index
 *              on ties) when temp[b] == 0
 *   q_lse    = log-sum-exp of d/temp; q_tok = q(x). For greedy requests
 *              q_tok = 1 and q_lse = max d.
 * with x_{b,0} = last_tok[b] (the last committed token).
 *
 *   base       [B, K, V] dtype   parallel drafter's base logits
 *   U          [V, r]    dtype   Markov factor, row per previous token
 *   W          [r, V]    dtype   Markov factor
 *   bias_scale [B] f32 or NULL   per-request multiplier of the bias (NULL: 1)
 *   last_tok   [B] i32           last committed token of each request
 *   temp       [B] f32           sampling temperature, 0 = greedy
 *   x          [B, K] i32  out   drafted tokens
 *   d          [B, K, V] dtype out  stored draft logits (verification uses them)
 *   q_lse      [B, K] f32  out   log normaliser of d/temp
 *   q_tok      [B, K] f32  out   draft probability of each drafted token
 *   q_norm     [B, K, 2] f32 out or NULL: the draw's normaliser as (m, s) with
 *                                z = d log2(e) / temp, m = max z, s = sum 2^(z - m)
 *                                ((max d, 1) for greedy rows); dspark_verify
 *                                takes it to skip recomputing it
 * Limits: 1 <= B <= 65535, 1 <= K <= 64, 8 <= V < 2^24, 1 <= r <= 1024;
 * bf16 additionally needs r % 16 == 0.
 */
int dspark_draft_sample(const void* base, const void* U, const void* W,
                        const float* bias_scale, const int32_t* last_tok,
                        const float* temp, int B, int K, int V, int r, int dtype,
                        uint64_t seed, uint64_t round_id, int32_t* x, void* d,
                        float* q_lse, float* q_tok, float* q_norm, void* ws,
                        size_t ws_bytes, dspark_stream_t stream);

/*
 * dspark_draft_sample with the recurrent sequential head in place of the
 * Markov head. [P1] "DSpark's semi-autoregressive compromise" (recurrent head
 * machinery beside the Markov head); [P3] "The Semi-Autoregressive Trick" (an
 * optional head that tracks the full block prefix, with marginal gains). The
 * pages give no equations; this library's reading is a state h_k in R^r with
 *   h_1 = U[x_0],  h_k = round_dtype(U[x_{k-1}] + tanh(h_{k-1} @ R))  (k >= 2)
 *   bias_k = bias_scale[b] * h_k @ W
 * (fp32 accumulation in ascending order of the rank index, tanh in fp32), so
 * that R = 0 gives dspark_draft_sample's results bit for bit, while a non-zero
 * R lets position k depend on every earlier token of the block.
 *
 *   R   [r, r] dtype   the state matrix (row j multiplies h_j)
 *   h   [B, K, r] dtype out   the states h_1..h_K of every request
 * Every other argument, output and limit as for dspark_draft_sample; r must
 * also be a multiple of 8, and R and h 16-byte aligned. The draw of position k
 * forms h_{k+1} in the same launch (one warp per request: about r^2 multiply-
 * adds and r tanh evaluations).
 */
int dspark_draft_sample_recurrent(const void* base, const void* U, const void* W,
                                  const void* R, const float* bias_scale,
                                  const int32_t* last_tok, const float* temp, int B,
                                  int K, int V, int r, int dtype, uint64_t seed,
                                  uint64_t round_id, int32_t* x, void* d, float* q_lse,
                                  float* q_tok, float* q_norm, void* h, void* ws,
                                  size_t ws_bytes, dspark_stream_t stream);

/*
 * dspark_draft_sample (R == NULL) or dspark_draft_sample_recurrent (R and h
 * given) for a caller that runs other work on another stream at the same time.
 * [P1] "DSpark turns speculation into a scheduler", intro and "Caveats" (the
 * verifier's pass over the target rows is the other large cost of a round; it
 * needs only the target logits and the cut, so it can run beside the draft).
 *
 * The whole-block launch of dspark_draft_sample (tensor-core path: bf16,
 * r % 16 == 0, r <= 256, ceil(B / 128) + 2 <= SMs) takes one CTA per SM and
 * leaves 2 SMs free; this call leaves free_sms SMs free instead (clamped so
 * that each group of 128 requests keeps at least one SM), for kernels of other
 * streams such as dspark_verify_target_stats. Fewer CTAs means more vocabulary
 * tiles per CTA, so the draft itself takes longer; the results are identical
 * bit for bit to dspark_draft_sample's (or the recurrent call's) for every
 * free_sms. On the other paths (two launches per position) free_sms has no
 * effect.
 *
 *   R        [r, r] dtype or NULL   the recurrent head's state matrix; NULL
 *                                   selects the Markov head
 *   h        [B, K, r] dtype out    the recurrent states (only with R; may be
 *                                   NULL otherwise)
 *   free_sms >= 0                   SMs to leave free
 * Every other argument, output and limit as for dspark_draft_sample; with R
 * as for dspark_draft_sample_recurrent. DSPARK_ERR_INVALID_ARG for a negative
 * free_sms.
 */
int dspark_draft_sample_beside(const void* base, const void* U, const void* W, const void* R,
                               const float* bias_scale, const int32_t* last_tok,
                               const float* temp, int B, int K, int V, int r, int dtype,
                               uint64_t seed, uint64_t round_id, int32_t* x, void* d,
                               float* q_lse, float* q_tok, float* q_norm, void* h,
                               int free_sms, void* ws, size_t ws_bytes,
                               dspark_stream_t stream);

/*
 * The two halves of one draft position of dspark_draft_sample, for callers
 * that interleave other work between positions or time the halves apart.
 * Calling, for k = 1..K in turn, dspark_draft_logits(k) then
 * dspark_draft_pick(k) on one stream with one workspace gives results
 * identical to dspark_draft_sample (the same kernels run in the same order).
 * [P1] "DSpark's semi-autoregressive compromise"; [P3] "The Semi-Autoregressive
 * Trick".
 *
 * dspark_draft_logits(k): d[:, k-1, :] = round_dtype(base[:, k-1, :] +
 *   bias_scale * U[x_{k-1}] @ W), with x_{b,0} = last_tok[b] and x_{b,k-1} =
 *   x[b, k-2] for k >= 2 (so x[:, k-2] must hold position k-1's tokens), and
 *   the per-(request, 256-entry chunk) softmax partials of d/temp, kept in the
 *   workspace for the pick that follows. Arguments as for dspark_draft_sample.
 * dspark_draft_pick(k): x[:, k-1], q_lse[:, k-1], q_tok[:, k-1] (and q_norm
 *   when not NULL) from
 *   d[:, k-1, :] and the workspace partials that dspark_draft_logits(k) left
 *   (the workspace must not be used by another call in between). last_tok is
 *   read only to report a bad token at k = 1.
 * Both need 1 <= k <= K and a workspace of
 * dspark_workspace_bytes(DSPARK_OP_DRAFT, B, K, V, r, dtype) bytes (pick takes
 * no r; the size does not depend on it). Errors as for dspark_draft_sample.
 */
int dspark_draft_logits(const void* base, const void* U, const void* W,
                        const float* bias_scale, const int32_t* last_tok,
                        const int32_t* x, const float* temp, int B, int K, int V,
                        int r, int dtype, int k, void* d, void* ws, size_t ws_bytes,
                        dspark_stream_t stream);

int dspark_draft_pick(const void* d, const int32_t* last_tok, const float* temp,
                      int B, int K, int V, int dtype, uint64_t seed,
                      uint64_t round_id, int k, int32_t* x, float* q_lse,
                      float* q_tok, float* q_norm, void* ws, size_t ws_bytes,
                      dspark_stream_t stream);

/*
 * Calibrated confidence, survival and the prefix cut.
 * [P1] "Confidence is a serving primitive" (c_k, survival product
 * P(prefix 1:k survives) = prod_{i<=k} c_i, Sequential Temperature Scaling,
 * hardware-aware prefix scheduler, static threshold as the rule it departs
 * from); [P1] "The speculative loop" (latency equation, the objective);
 * [P3] "The Real Innovation: Confidence-Scheduled Verification" (early stop).
 *
 *   c[b,k] = sigmoid(conf_logit[b,k] / pos_temp[k]),  S[b,k] = prod_{i<=k} c[b,i]
 * mode DSPARK_CUT_COST: every request verifies one slot for its correction or
 *   bonus token; verifying n tokens costs fixed_cost + step_cost[0] + ... +
 *   step_cost[n-1]. Drafts are visited by descending S (ties: smaller k, then
 *   smaller b) and admitted while S_j * C_{j-1} >= A_{j-1} * step_cost[B+j-1]
 *   (A = B + admitted S, C = current cost, j 1-based); the first failure stops
 *   the walk. cut[b] = admitted drafts of request b (a prefix of its block).
 * mode DSPARK_CUT_THRESHOLD: cut[b] = #{k : S[b,k] >= threshold}.
 * mode DSPARK_CUT_NONE: cut[b] = K.
 * Computed in fp64 on the device; survival is returned rounded to fp32.
 *
 *   conf_logit [B, K] f32, pos_temp [K] f32 (> 0), step_cost [B*(K+1)] f32
 *   cut [B] i32 out, survival [B, K] f32 out
 * Limits: 1 <= K <= 64; the cost rule needs B*K <= 16384 (one CTA sorts all
 * drafts, so that the call fits beside the draft kernel on the SMs it leaves
 * free), the other modes take any B >= 1.
 */
int dspark_prefix_schedule(const float* conf_logit, const float* pos_temp,
                           const float* step_cost, float fixed_cost, int B, int K,
                           int mode, float threshold, int32_t* cut,
                           float* survival, void* ws, size_t ws_bytes,
                           dspark_stream_t stream);

/*
 * Lossless verification of the first cut[b] drafts of every request.
 * [P1] intro and "Caveats" (accept the longest valid prefix, correct at the
 * first rejection; lossless only with the proper acceptance rule); [P2]
 * "Sources" (the rule of "Fast Inference from Transformers via Speculative
 * Decoding"); [P3] "Speculative Decoding in Two Sentences" (plus one bonus
 * token; the target distribution is preserved exactly).
 *
 * Target row j (0-based) scores draft token j+1; row cut[b] gives the bonus.
 * For k = 1..cut[b]: p = softmax(target[b,k-1] / temp[b]); accept x[b,k-1]
 * iff Philox(seed, b, k, purpose 1, round_id) < p(x) / q_tok[b,k-1]; stop at
 * the first rejection. accepted[b] = a. If a < cut[b]: y ~ norm(max(0, p - q))
 * over target row a and q = softmax(d[b,a] / temp[b]) (purpose 2, position
 * a+1; p itself if the residual is exactly zero). Else y ~ p of target row
 * cut[b] (purpose 3, position a+1). Greedy requests (temp 0) accept iff
 * x == argmax of the target row and emit argmax of target row a.
 * out[b] = x[b,0..a-1], y, then -1 up to K+1 entries; n_emit[b] = a + 1.
 *
 * Two launches on `stream`: dspark_verify_target_stats (one streaming pass over
 * target rows 0..cut[b] of every request, which leaves each row's softmax
 * partials in the workspace), then dspark_verify_from_stats (the acceptance
 * tests from those normalisers, one pass over target row a and draft row a of
 * every rejected request for the residual, a one-chunk rescan for the bonus).
 * Target rows past cut[b] and draft rows other than a are never read.
 *
 *   target [B, K+1, V] dtype, d [B, K, V] dtype, x [B, K] i32,
 *   q_tok [B, K] f32, cut [B] i32 or NULL (all K), temp [B] f32
 *   q_norm [B, K, 2] f32 or NULL: the draft rows' normalisers as written by
 *     dspark_draft_sample; with it a rejected request's residual starts at
 *     once, without it the draft row's normaliser is recomputed (one more pass
 *     over draft row a). The two agree up to fp32 summation order.
 *   accepted [B] i32 out, out [B, K+1] i32 out, n_emit [B] i32 out
 * Limits: 1 <= B <= 65535, 1 <= K <= 64, 8 <= V < 2^24.
 */
int dspark_verify(const void* target, const void* d, const int32_t* x,
                  const float* q_tok, const float* q_norm, const int32_t* cut,
                  const float* temp,
                  int B, int K, int V, int dtype, uint64_t seed,
                  uint64_t round_id, int32_t* accepted, int32_t* out,
                  int32_t* n_emit, void* ws, size_t ws_bytes,
                  dspark_stream_t stream);

/*
 * The two halves of dspark_verify, for callers that start the first one as
 * soon as the cut is known, beside the draft (it needs neither d, x nor the
 * draft's probabilities). Calling dspark_verify_target_stats and then
 * dspark_verify_from_stats with the same target, cut, temp and workspace gives
 * results identical to dspark_verify (the same kernels run).
 * [P1] intro and "Caveats"; [P2] "Sources"; [P3] "Speculative Decoding in Two
 * Sentences".
 *
 * dspark_verify_target_stats: for every request b and target row j <= cut[b]
 *   (all K + 1 rows when cut is NULL), the softmax partials of every 2 KB
 *   chunk of the row, (max z, sum 2^(z - max z)) of z = target * log2(e) /
 *   temp[b], or (max, lowest argmax) for temp[b] == 0, written to the
 *   workspace's statistics region, and (with a cut) the order in which the
 *   final kernel takes the requests (cut descending, index ascending) after
 *   it. The statistics region lies past the draft's partials
 *   of a workspace of the same size, so this call may run on another stream
 *   concurrently with dspark_draft_sample on that workspace; it must complete
 *   before dspark_verify_from_stats starts (an event or the same stream).
 * dspark_verify_from_stats: everything else dspark_verify does, reading the
 *   statistics instead of the target rows' normalisers. Its arguments are
 *   dspark_verify's; cut and temp must be the ones the statistics were made
 *   with.
 * Both take a workspace of dspark_workspace_bytes(DSPARK_OP_VERIFY, ...) bytes.
 */
int dspark_verify_target_stats(const void* target, const int32_t* cut,
                               const float* temp, int B, int K, int V, int dtype,
                               void* ws, size_t ws_bytes, dspark_stream_t stream);

int dspark_verify_from_stats(const void* target, const void* d, const int32_t* x,
                             const float* q_tok, const float* q_norm,
                             const int32_t* cut, const float* temp, int B, int K,
                             int V, int dtype, uint64_t seed, uint64_t round_id,
                             int32_t* accepted, int32_t* out, int32_t* n_emit,
                             void* ws, size_t ws_bytes, dspark_stream_t stream);

/*
 * Sequential Temperature Scaling of the per-position confidences, and their
 * expected calibration error before and after.
 * [P1] "Confidence is a serving primitive" (one temperature per draft
 * position, fitted left to right, because the scheduler multiplies the
 * calibrated confidences into survival probabilities); [P3] "The Real
 * Innovation" (calibration error from 3-8% to about 1%).
 *
 * For k = 0..K-1 in turn, with T_0..T_{k-1} fixed:
 *   S_n(T) = prod_{i<k} sigmoid(z[n,i] / T_i) * sigmoid(z[n,k] / T)
 *   T_k = the temperature of a fixed grid (256 values log-spaced on
 *         [0.05, 20], index i -> exp(ln 0.05 + i (ln 400) / 255)) minimising
 *         -sum_n [y log S + (1 - y) log(1 - S)] with y = survived[n,k] and S
 *         clamped to [1e-12, 1 - 1e-12]; the lowest index wins a tie.
 * ECE of position k: 15 equal-width bins of S_n on [0, 1] (S = 1 in the last),
 * sum over bins of (count / N) * |mean S - mean y|; before = every T_i = 1.
 * Losses and bin sums are fp64.
 *
 *   conf_logit [N, K] f32, survived [N, K] u8 (1: drafts 1..k+1 all accepted)
 *   T_out [K] f32 out, index_out [K] i32 out or NULL (grid index of T_k)
 *   ece_before, ece_after [K] f32 out or NULL
 * Workspace: dspark_workspace_bytes(DSPARK_OP_CALIB, N, K, 0, 0, 0) (N in the
 * B argument). Limits: N >= 1, 1 <= K <= 64. 2K + 4 launches on `stream`.
 */
int dspark_sts_fit(const float* conf_logit, const uint8_t* survived, int N, int K,
                   float* T_out, int32_t* index_out, float* ece_before,
                   float* ece_after, void* ws, size_t ws_bytes,
                   dspark_stream_t stream);

/*
 * dspark_draft_sample for callers that cannot allocate device memory. The pages
 * have no counterpart to this entry point: it only changes where the scratch
 * lives. dspark_draft_sample needs a caller-owned workspace; callers that run
 * inside another runtime's memory manager (an inference server or framework
 * whose caching allocator has reserved the device memory, so that an extra
 * cudaMalloc can fail or upset its accounting), plug-in hosts that hand over
 * only input and output buffers, and latency-critical paths that cannot accept
 * cudaMalloc's implicit synchronisation have no way to provide one.
 *
 * Same arguments, computation, launches and results as dspark_draft_sample, without
 * ws/ws_bytes and without the optional q_norm output (dspark_verify then
 * recomputes the draft rows' normalisers). The scratch is a fixed 8 MiB array inside the library's device
 * image, held on every GPU that loads the library until the process exits; the
 * call allocates and frees nothing. Its device address is looked up once per
 * device, by the first call made while that device is current, so that first
 * call should come before any stream capture. The address is kept for the
 * life of the process: calls after a cudaDeviceReset (or from another CUDA
 * context on the same device) are not supported. Every call uses the same array
 * and clears its status part first: calls that overlap on the GPU (other
 * streams, other threads) race and must not be issued. A call needs
 * 256 + 8 * B * ceil(V / 256) bytes of the 8 MiB (B = 1024 at V = 151936 takes
 * 4.9 MB); larger sizes return DSPARK_ERR_WORKSPACE.
 *
 *   status_out  [2] i32 device, out, or NULL: {OR of DSPARK_STATUS_* bits,
 *               lowest offending request or -1} of this call
 */
int dspark_draft_sample_static(const void* base, const void* U, const void* W,
                               const float* bias_scale, const int32_t* last_tok,
                               const float* temp, int B, int K, int V, int r,
                               int dtype, uint64_t seed, uint64_t round_id,
                               int32_t* x, void* d, float* q_lse, float* q_tok,
                               int32_t* status_out, dspark_stream_t stream);

/*
 * Synchronises `stream`, reads the status block of `ws` into *code (OR of
 * DSPARK_STATUS_* bits) and *first_bad_request (-1 if none), then clears it.
 * Either output pointer may be NULL.
 */
int dspark_read_status(void* ws, dspark_stream_t stream, uint32_t* code,
                       int32_t* first_bad_request);

/* Zeroes the status block of `ws` asynchronously on `stream`. */
int dspark_clear_status(void* ws, dspark_stream_t stream);

/* Static description of a DSPARK_OK / DSPARK_ERR_* return code. */
const char* dspark_status_string(int code);

/* ABI version of this header: (major << 16) | minor. */
int dspark_version(void);

/*
 * dspark_selftest_waits — makes the library's bounded device waits run out.
 * One thread waits on an mbarrier phase that no arrival completes, then at a
 * grid barrier that it reaches alone. Each wait gives up after the limit every
 * kernel of the library uses (2 s of the GPU's global timer), reports
 * DSPARK_STATUS_TIMEOUT in the status block (wait site 30) and lets the kernel
 * return, so the context stays usable; the call takes about 4 s of GPU time.
 * For tests of failure detection; nothing else calls it.
 *   result    [2] i32 device, out: 1 where the mbarrier wait / the grid-barrier
 *             wait gave up, 0 where it completed
 *   ws        workspace of at least 256 bytes (its status block is used,
 *             including the grid-barrier counter at byte 64)
 * Errors: DSPARK_ERR_INVALID_ARG (null pointer, workspace too small or
 * misaligned), DSPARK_ERR_UNSUPPORTED (no sm_100 device), DSPARK_ERR_CUDA.
 */
int dspark_selftest_waits(int32_t* result, void* ws, size_t ws_bytes, dspark_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* DSPARK_H */
