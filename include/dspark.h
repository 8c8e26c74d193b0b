/*
 * dspark.h — C ABI of the DSpark confidence-scheduled verify step (libdspark.so, sm_100a).
 *
 * One verify round of confidence-scheduled speculative decoding, as the DSpark write-ups
 * describe it, split into the steps that run on the GPU:
 *
 *   dspark_schedule        survival scan + greedy marginal-gain prefix scheduler + flattening
 *   dspark_verify_attn_plan / dspark_verify_attn
 *                          flattened ragged GQA attention of every verify token over its
 *                          request's paged KV cache and its own earlier verify tokens
 *   dspark_accept          exact acceptance rule, longest accepted prefix, residual / bonus
 *                          resampling (or greedy verification)
 *   dspark_kv_commit       the kept tokens' K/V into the paged cache (after acceptance)
 *   dspark_calibrate_confidence / dspark_fit_temperature
 *                          temporal temperature scaling of the confidence head
 *   dspark_markov_draft    synthetic Markov-head draft step (cost of the drafter's sequential part)
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument is DEVICE memory owned by the caller, unless stated otherwise.
 *     The library allocates nothing; scratch comes from caller-provided workspaces whose
 *     size the *_workspace_bytes queries return.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and performs no host synchronisation, except dspark_read_error.
 *   - Launch shapes depend only on capacity arguments (R, K, T_cap, V, ...), never on
 *     device-resident results such as the scheduled token count, so one verify step can be
 *     enqueued without reading anything back.
 *   - Host-side argument validation returns a negative dspark_status before anything is
 *     enqueued.  Bad device-resident data (a marker that does not match its request, a page
 *     index outside the cache, a draft token outside the vocabulary, ...) sets bits in a
 *     sticky per-device error word and the affected unit of work is skipped; kernels never
 *     trap.  dspark_read_error returns and clears that word.
 *   - Integer tensors are int32, row-major, densely packed.
 *
 * Sources (news write-ups of the DSpark paper; they describe the method, not an interface):
 *   [P1] "刚融完500亿创始人亲自下场写代码DeepSeek不卷参数专治AI“嘴慢”" (mooersco.com),
 *        section "2. 置信度调度验证" and the engineering table.
 *   [P2] "DSpark 的 661% 提速，是真突破还是数字游戏？" (new-universe.cn), §一, §3.2.
 *   [P3] "DeepSeek服务器不再卡顿！DSpark加速60% - 80%，推理成本降40%" (qwbw.cn),
 *        sections "DSpark的神奇之处", "成本与质量的考量".
 *   [P4] "DeepSeek DSpark speculative decoding 85 percent faster LLM inference"
 *        (aibuzzwire.news), section "置信度计划、负载感知验证".
 */
#ifndef DSPARK_H
#define DSPARK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *dspark_stream_t; /* identical to cudaStream_t */

/* Return codes. */
enum dspark_status {
  DSPARK_OK = 0,
  DSPARK_EINVAL = -1,        /* an argument is out of range or a required pointer is NULL */
  DSPARK_ECUDA = -2,         /* a CUDA runtime call failed (launch, attribute, copy) */
  DSPARK_EWORKSPACE = -3,    /* workspace NULL or smaller than the size query returned */
  DSPARK_EDEVICE_DATA = -4,  /* dspark_read_error: device-resident data was invalid */
  DSPARK_ETIMEOUT = -5,      /* not returned by any entry point: an in-kernel wait that runs
                                out (the tensor-core attention kernel bounds every wait at
                                about 2 s) is reported as DSPARK_DERR_TIMEOUT in the device
                                error word instead, because kernels return no status */
  DSPARK_EUNSUPPORTED = -6   /* valid arguments outside what this build implements */
};

/* Element types of floating-point tensors. */
enum dspark_dtype { DSPARK_F32 = 0, DSPARK_BF16 = 1 };

/* Bits of the device error word (see dspark_read_error). */
enum dspark_device_error {
  DSPARK_DERR_CONF = 1 << 0,        /* a confidence outside [0, 1] or NaN (treated as 0) */
  DSPARK_DERR_TABLE = 1 << 1,       /* a step-time entry <= 0 or NaN (scan stops there) */
  DSPARK_DERR_KV_LEN = 1 << 2,      /* kv_len < 0 or beyond the block table */
  DSPARK_DERR_PAGE = 1 << 3,        /* a block-table entry outside [0, num_pages) */
  DSPARK_DERR_MARKER = 1 << 4,      /* markers[t] != (r, kv_len[r] + j) for token t = q_offsets[r]+j */
  DSPARK_DERR_OFFSETS = 1 << 5,     /* q_offsets not a scan of 1 + verify_len within T_cap */
  DSPARK_DERR_VERIFY_LEN = 1 << 6,  /* verify_len outside [0, K] */
  DSPARK_DERR_TOKEN = 1 << 7,       /* a draft token outside [0, V) */
  DSPARK_DERR_LOGITS = 1 << 8,      /* a logit row whose maximum is not finite */
  DSPARK_DERR_TIMEOUT = 1 << 9,     /* a bounded in-kernel wait expired; results undefined */
  DSPARK_DERR_ACCEPTED = 1 << 10    /* an accepted length outside [0, verify_len] (or a
                                       verify length outside [0, K] in a temperature fit) */
};

#define DSPARK_CONF_LAG 2             /* rounds between producing and consuming confidences */
#define DSPARK_MAX_K 16               /* largest supported max-draft length K */
#define DSPARK_MAX_CANDIDATES 16384   /* largest R*K the scheduler sorts in one CTA */

/* Human-readable name of a dspark_status value (static storage, never NULL). */
const char *dspark_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int dspark_version(void);

/*
 * dspark_schedule — pick every request's verify length for one round.
 *
 * Defined by [P2 §3.2] (inputs: load, per-position confidence, the engine's throughput curve),
 * [P3 "DSpark的神奇之处"] (measure speed per batch size in advance; queue all requests' draft
 * tokens by score, high to low; keep adding the next ones while the extra correct tokens pay
 * for the extra time), [P4] (survival probabilities, global throughput maximisation) and
 * [P1 engineering table] (the asynchronous scheduler reads confidences from two rounds
 * earlier; all verify tokens are flattened and tagged with markers).  Computes:
 *   S[r][k]   = c[r][0] * ... * c[r][k]       (float64, left to right), c = conf of round
 *                                              max(round_idx - DSPARK_CONF_LAG, 0)
 *   order     = all (r, k) by S descending, ties by k ascending then r ascending
 *   f(n)      = (R + sum of the first n S in that order) / t_ms[R + n]
 *   n*        = first n with f(n + 1) <= f(n), else min(R*K, T_cap - R)
 *   verify_len[r] = number of r's candidates among the first n*  (a prefix of r's block)
 *   q_offsets = exclusive scan of 1 + verify_len (length R + 1); *T_out = q_offsets[R]
 *   markers[q_offsets[r] + j] = (r, kv_len[r] + j), j = 0..verify_len[r]
 *
 * conf_ring   float32 [ring_depth][R][K]; slot (i % ring_depth) holds the confidences
 *             produced in round i.  ring_depth >= DSPARK_CONF_LAG + 1.
 * round_idx   current round (>= 0); slot max(round_idx - 2, 0) % ring_depth is read.
 * kv_len      int32 [R] cached tokens per request (positions of the verify tokens follow).
 * t_ms        float64 [T_cap + 1], t_ms[T] = engine step time for T verify tokens (> 0).
 * T_cap       capacity of the flattened batch, R <= T_cap.
 * verify_len  out int32 [R]; q_offsets out int32 [R + 1]; markers out int32 [T_cap][2]
 *             (entries past *T_out untouched); T_out out int32 [1]; objective out
 *             float64 [1] = f(n*).
 * kv_len and markers may both be NULL: the call then decides the lengths and offsets only,
 * which need nothing but the lagged confidences, so that a pipeline can schedule round i + 1
 * while round i still runs; dspark_flatten_markers writes the markers once round i has
 * committed the cache lengths.
 * Limits: 1 <= K <= DSPARK_MAX_K, R*K <= DSPARK_MAX_CANDIDATES.
 */
int dspark_schedule(const float *conf_ring, int ring_depth, int round_idx, int R, int K,
                    const int32_t *kv_len, const double *t_ms, int T_cap,
                    int32_t *verify_len, int32_t *q_offsets, int32_t *markers,
                    int32_t *T_out, double *objective, dspark_stream_t stream);

/*
 * dspark_flatten_markers — the flattening step of dspark_schedule on its own.
 *
 * Defined by [P1 engineering table, row "内核利用率暴跌"] (verify tokens flattened, a marker
 * tensor carries sequence membership and position) and row "GPU流水线停滞" (the scheduler
 * runs ahead of the round it feeds).  markers[q_offsets[r] + j] = (r, kv_len[r] + j) for
 * j = 0 .. q_offsets[r+1] - q_offsets[r] - 1, from the offsets of an earlier lengths-only
 * dspark_schedule and the cache lengths current now.  kv_len int32 [R], q_offsets int32
 * [R + 1], markers int32 [T_cap][2] (device).  A request whose offsets are not a flattening of
 * 1..K+1 tokens inside [0, T_cap) sets DSPARK_DERR_OFFSETS and gets no markers.
 */
int dspark_flatten_markers(const int32_t *kv_len, const int32_t *q_offsets, int R, int K,
                           int T_cap, int32_t *markers, dspark_stream_t stream);

/*
 * Workspace of the attention pair (plan + calls).  rows = (Hq / Hkv) * (K + 1) query rows
 * per (request, KV head).  The workspace holds the work partition, per-segment arrival
 * counters and split-KV partial results; it is reused by every attention call of a step.
 */
size_t dspark_verify_attn_workspace_bytes(int R, int Hq, int Hkv, int D, int K);

/*
 * dspark_verify_attn_plan — partition one step's attention work across the GPU and check the
 * flattened batch once.
 *
 * Work is the sequence of (request r, KV head g, unit) in request-major order, each request
 * contributing Hkv * (ceil(kv_len[r] / 64) + 8) units (its 64-key cache tiles, then eight
 * units standing for its own verify tokens and the segment's epilogue).  The plan splits it
 * into contiguous ranges, one per persistent CTA of the tensor-core kernel, chosen to minimise
 * the largest modelled cost of a range: one per 64-key page, four for a segment's verify
 * tokens and query rows, seven per piece (a segment cut by range boundaries is computed in
 * pieces) and six for merging a cut segment's partials; boundaries fall on even page counts and never inside a
 * segment's verify-token units.  It runs the greedy fill for 1024 candidate bounds at once.
 * It also records, per request, the flattened offset, the token count and whether the
 * flattening is well formed (1 <= Q_r <= K + 1 tokens inside [0, T_cap), token j carrying the
 * marker (r, kv_len[r] + j)); a malformed request sets DSPARK_DERR_OFFSETS / _MARKER here and
 * every dspark_verify_attn that uses this plan skips it.  Call once per step after the
 * schedule and before any dspark_verify_attn of that step, and again whenever kv_len,
 * q_offsets or markers change; it also zeroes the workspace's arrival counters.
 * kv_len int32 [R], q_offsets int32 [R + 1], markers int32 [T_cap][2] (device); ws/ws_bytes as
 * returned by the query above.
 */
int dspark_verify_attn_plan(const int32_t *kv_len, const int32_t *q_offsets,
                            const int32_t *markers, int R, int T_cap, int Hq, int Hkv, int D,
                            int K, void *ws, size_t ws_bytes, dspark_stream_t stream);

/*
 * dspark_verify_attn — flattened ragged GQA attention of every verify token.
 *
 * Defined by [P1 engineering table, row "内核利用率暴跌"]: variable-length verification pads
 * and unbalances standard decode kernels, so every verify token is an independent element
 * and a marker tensor carries its sequence and position; [P2 §一] the target checks all draft
 * tokens in one batched pass.  For verify token t = q_offsets[r] + j with markers[t] =
 * (r, pos) and every query head h (KV head g = h / (Hq/Hkv)):
 *   keys   = r's cached positions 0..kv_len[r]-1, then r's verify tokens i with
 *            kv_len[r] + i <= pos (causal)
 *   out[t][h] = softmax(scale * q[t][h] . keys) . values   (fp32 accumulation)
 *
 * q          [T_cap][Hq][D], k_new / v_new [T_cap][Hkv][D] — the verify tokens' own query,
 *            key and value rows (post positional encoding), in flattened token order.
 * kv_pages   [num_pages][2][Hkv][page_size][D] paged cache: index 0 = K, 1 = V; one
 *            page holds page_size consecutive positions of one request.
 * block_table int32 [R][max_pages]: physical page of each request's i-th page.
 * kv_len     int32 [R]; markers int32 [T_cap][2]; q_offsets int32 [R + 1] (from the schedule;
 *            only rows t < q_offsets[R] are read or written).
 * out        [T_cap][Hq][D], same dtype as the inputs.
 * dtype      DSPARK_BF16 or DSPARK_F32; scale is usually 1/sqrt(D).  bf16 with D == 128,
 *            page_size % 64 == 0, K + 1 <= 16, (Hq/Hkv)*(K+1) <= 64 and the cache below 2^31
 *            rows of D elements runs on the tensor cores (tcgen05 + TMA); every other shape
 *            runs on CUDA cores.  The tensor-core path takes each request's offset, token count
 *            and validity from the records of the last dspark_verify_attn_plan (which checked
 *            the markers); the CUDA-core path checks the markers itself.  The tensor-core kernel
 *            splits its register pool across warp roles; a build whose compiled register count
 *            cannot hold that split is refused with DSPARK_EUNSUPPORTED before any launch.
 *            A bounded in-kernel wait that expires (a stalled copy or tensor-core pipe, after
 *            about 2 s) sets DSPARK_DERR_TIMEOUT and leaves the output undefined.
 * Limits: 1 <= D <= 256 with D % 8 == 0, Hq % Hkv == 0, (Hq/Hkv)*(K+1) <= 128.
 */
int dspark_verify_attn(const void *q, const void *k_new, const void *v_new,
                       const void *kv_pages, int64_t num_pages, const int32_t *block_table,
                       int max_pages, const int32_t *kv_len, const int32_t *markers,
                       const int32_t *q_offsets, int R, int T_cap, int Hq, int Hkv, int D,
                       int K, int page_size, int dtype, float scale, void *out,
                       void *ws, size_t ws_bytes, dspark_stream_t stream);

/* Workspace of dspark_accept: per-row softmax statistics. */
size_t dspark_accept_workspace_bytes(int R, int K, int T_cap);

/*
 * dspark_accept — exact acceptance, longest accepted prefix, correction / bonus token.
 *
 * Defined by [P2 §一] (verify the N draft tokens in one pass, keep the verified ones,
 * resample after the first divergence; the output distribution equals the target's),
 * [P3 "DSpark的神奇之处"] (from the first wrong guess the large model writes a correct token
 * itself) and [P3 "成本与质量的考量"] (the acceptance rule preserves the target distribution
 * exactly).  With p_j = softmax(target row q_offsets[r]+j / temperature) and
 * q_j = softmax(draft_logits[r][j] / temperature):
 *   draft token k (k = 0..L-1, L = verify_len[r]) is accepted iff
 *       u_acc[r][k] < min(1, p_k(x_k) / q_k(x_k));
 *   a = accepted count before the first rejection;
 *   a < L : correction drawn from max(0, p_a - q_a) (normalised), a == L: bonus from p_L;
 *   draw = smallest v with C(v) > u_res[r][a] * C(V-1), C the running sum in index order;
 *   a residual that is empty in floating point (p_a <= q_a everywhere, e.g. a draft row equal
 *   to its target row) falls back to a draw from p_a.
 * temperature <= 0 selects greedy verification: accept iff x_k == argmax of target row k
 * (lowest index on ties); the correction / bonus is the argmax of target row a.
 * u_acc = 1 rejects at any ratio.
 *
 * Launches: one CTA per scheduled logit row for the statistics, then the finalize kernel.
 * In sampled mode the finalize kernel runs a thread-block cluster of up to 8 CTAs per request,
 * which share the draw through distributed shared memory; in greedy mode it runs one CTA per
 * request.  The result does not depend on the cluster size.
 *
 * target_logits [T_cap][V] (row q_offsets[r] + j = position j+1 of request r),
 * draft_logits [R][K][V], dtype DSPARK_BF16 or DSPARK_F32; draft_tokens int32 [R][K];
 * verify_len int32 [R]; q_offsets int32 [R + 1]; u_acc float32 [R][K]; u_res float32
 * [R][K + 1] (uniforms in [0, 1)).  Outputs: accepted_len int32 [R]; out_tokens int32
 * [R][K + 1] (accepted drafts, then the correction / bonus, then -1); n_out int32 [R] = a + 1.
 * In greedy mode draft_logits, u_acc and u_res may be NULL.
 */
int dspark_accept(const void *target_logits, const void *draft_logits, int dtype, int V,
                  int R, int K, int T_cap, const int32_t *draft_tokens,
                  const int32_t *verify_len, const int32_t *q_offsets, const float *u_acc,
                  const float *u_res, float temperature, int32_t *accepted_len,
                  int32_t *out_tokens, int32_t *n_out, void *ws, size_t ws_bytes,
                  dspark_stream_t stream);

/*
 * dspark_accept_noalloc — dspark_accept for callers that cannot allocate device memory.
 *
 * The paper has no counterpart to this entry point; it exists for library users.  Some hosts
 * of this library may not call cudaMalloc: an inference engine whose memory pool has already
 * reserved the GPU's free memory at start-up, a plugin running inside a runtime that forbids
 * allocation after initialisation, or a latency-critical loop where an allocation (which can
 * synchronise the device) is not acceptable.  They still pass their own inputs and outputs,
 * but get the acceptance kernels' scratch (per-row softmax statistics) from a fixed array
 * compiled into the library instead of a workspace argument.
 *
 * Arguments and results are those of dspark_accept without ws / ws_bytes.
 * Limit: T_cap + R*K <= DSPARK_ACCEPT_NOALLOC_MAX_ROWS; larger calls return
 * DSPARK_EUNSUPPORTED before anything is enqueued.  The array (16 bytes per row, 1 MiB) is held
 * by every GPU that loads the library until the process exits.
 * The first call on each device looks up the array's device address (cudaGetSymbolAddress)
 * with that device current, and so does the first call after the device's context was
 * recreated (cudaDeviceReset moves the array); make such a first call before any stream
 * capture.
 * All calls on a device share the one array and it keeps the previous call's contents (every
 * row a call reads is written by that call first).  Calls whose executions overlap on the GPU
 * — on different streams, or from different host threads — race on the array: serialise them.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
#define DSPARK_ACCEPT_NOALLOC_MAX_ROWS 65536
int dspark_accept_noalloc(const void *target_logits, const void *draft_logits, int dtype, int V,
                          int R, int K, int T_cap, const int32_t *draft_tokens,
                          const int32_t *verify_len, const int32_t *q_offsets,
                          const float *u_acc, const float *u_res, float temperature,
                          int32_t *accepted_len, int32_t *out_tokens, int32_t *n_out,
                          dspark_stream_t stream);

/*
 * dspark_kv_commit — the kept verify rows of every request join its paged KV cache.
 *
 * Defined by [P1 opening section: drafts the target confirms are adopted, "猜对了就采纳"] and
 * [P2 §一: the verified tokens are kept].  After dspark_accept, request r keeps its verify tokens
 * j = 0 .. accepted_len[r]: token 0 sits at position kv_len[r] (the previous round's last
 * emitted token, whose K/V this verify pass computed), tokens 1.. are its accepted drafts.  For
 * every layer l, KV head g and kept j, the rows k_new / v_new [l][q_offsets[r] + j][g] are
 * copied into the cache slot of position p = kv_len[r] + j (page block_table[r][p / page_size],
 * row p % page_size), and kv_len_out[r] = kv_len[r] + accepted_len[r] + 1.  Rejected drafts are
 * never written, so nothing is rolled back.  (The pages describe no cache layout or interface:
 * this reading is listed in the design notes.)
 *
 * k_new, v_new: `layers` blocks [T_cap][Hkv][D] of `dtype`, new_layer_stride ELEMENTS apart;
 * kv_pages: `layers` caches [num_pages][2][Hkv][page_size][D], cache_layer_stride ELEMENTS apart
 * (callers whose per-layer caches are separate allocations call once per layer, layers = 1);
 * block_table int32 [R][max_pages] must already hold pages for positions up to
 * kv_len[r] + accepted_len[r]; kv_len, q_offsets, accepted_len int32 (read); kv_len_out int32
 * [R] (written; must not alias kv_len).  D * element size must be a multiple of 16 bytes and
 * every tensor 16-byte aligned.
 * Bad device data (q_offsets malformed, accepted_len outside [0, verify_len], a kept position
 * beyond the block table, a page outside [0, num_pages)) sets DSPARK_DERR_OFFSETS / _ACCEPTED /
 * _KV_LEN / _PAGE; that request is left untouched and kv_len_out[r] = kv_len[r].
 */
int dspark_kv_commit(const void *k_new, const void *v_new, int64_t new_layer_stride,
                     void *kv_pages, int64_t num_pages, int64_t cache_layer_stride, int layers,
                     const int32_t *block_table, int max_pages, const int32_t *kv_len,
                     const int32_t *q_offsets, const int32_t *accepted_len, int R, int T_cap,
                     int Hkv, int D, int K, int page_size, int dtype, int32_t *kv_len_out,
                     dspark_stream_t stream);

/*
 * dspark_calibrate_confidence — temporal temperature scaling of raw confidence logits.
 *
 * Defined by [P1 "2. 置信度调度验证": a post-hoc calibration, "temporal temperature scaling",
 * corrects the raw confidence head's over-confidence] with [P2 §3.2: the confidence of block
 * position k is the acceptance probability given an accepted prefix].  Reading (the pages give
 * only the name): conf[r][k] = sigmoid(logits[r][k] / tau[k]), one temperature per block
 * position.  Evaluated in float64 and rounded to float32; write the result into the slot of the
 * confidence ring that dspark_schedule reads two rounds later.
 * logits float32 [R][K], tau float32 [K], conf float32 [R][K] (device).  A temperature that is
 * not a positive finite number, or a NaN logit, gives 0 and sets DSPARK_DERR_CONF.
 */
int dspark_calibrate_confidence(const float *logits, const float *tau, int R, int K, float *conf,
                                dspark_stream_t stream);

/*
 * dspark_fit_temperature — maximum-likelihood temperatures from observed accept outcomes.
 *
 * Same passages and reading as above.  Sample i (one verified request) verified verify_len[i]
 * drafts and accepted accepted_len[i] of them; its block position k (0-based column) is
 * observed iff k + 1 <= min(accepted_len[i] + 1, verify_len[i]), accepted iff
 * k + 1 <= accepted_len[i].  tau[k] = 1 / beta minimises
 * sum_observed log(1 + exp(-s * beta * logits[i][k])) (s = +1 accepted, -1 rejected) over
 * beta in [1/64, 64]; a position without observations or with all-zero observed logits gets 1.
 * logits float32 [N][K] (the raw logits the head produced for those requests), verify_len and
 * accepted_len int32 [N], tau float32 [K] out (device).  Samples with lengths outside
 * 0 <= accepted_len <= verify_len <= K are ignored and set DSPARK_DERR_ACCEPTED.
 */
int dspark_fit_temperature(const float *logits, const int32_t *verify_len,
                           const int32_t *accepted_len, int N, int K, float *tau,
                           dspark_stream_t stream);

/*
 * dspark_markov_draft — synthetic Markov-head draft step (the drafter's sequential part).
 *
 * Defined by [P1 "1. 半自回归生成": a parallel backbone drafts the whole block and a light
 * sequential module injects the prefix token by token; one form is a Markov head that depends
 * only on the previous token].  Reading (no formulas or trained weights are published): block
 * position k = 1..K of request r has draft logits z_k = bf16(B[r][k-1] + E[x_{k-1}] . U) — the
 * backbone's block logits plus a rank-d transition term of the previous token — and
 * x_k = argmax_v z_k[v] / temperature + g_v, g = -log(-log(u)), u from Philox4x32-10 with
 * counter (round_idx, r, v / 4, 3 + 256 (k - 1)), key (seed, 0), word v % 4,
 * u = ((word >> 8) + 1/2) 2^-24; temperature <= 0 takes the lowest index of the maximum of z_k.
 * x_0 = x0[r], the request's last emitted token.  Its purpose is the cost of this sequential
 * part next to a verify step (the backbone's block logits are an input).
 * block_logits bf16 [R][K][V]; E bf16 [V][d]; U bf16 [d][V]; d a multiple of 8 up to 64;
 * V a multiple of 8; block_logits, E, U and draft_logits 16-byte aligned; x0 int32 [R]; outputs
 * draft_logits bf16
 * [R][K][V] (the q distributions the verifier reads) and draft_tokens int32 [R][K]; ws from
 * dspark_markov_draft_workspace_bytes(R, V).  2K + 1 launches.  An x0 outside [0, V) sets
 * DSPARK_DERR_TOKEN and is read as token 0.
 */
size_t dspark_markov_draft_workspace_bytes(int R, int V);
int dspark_markov_draft(const void *block_logits, const void *E, const void *U, int d,
                        const int32_t *x0, int R, int K, int V, float temperature,
                        uint32_t round_idx, uint32_t seed, void *draft_logits,
                        int32_t *draft_tokens, void *ws, size_t ws_bytes,
                        dspark_stream_t stream);

/*
 * dspark_selftest_wait_timeout — exercise the bounded in-kernel wait (no counterpart on the
 * pages: it tests this library's failure handling).  One GPU thread waits, through the same
 * bounded mbarrier wait the tensor-core attention kernel uses, on a barrier nothing arrives at,
 * for limit_cycles SM cycles (1 .. about 4e9); it then records DSPARK_DERR_TIMEOUT in the error
 * word and returns.  result int32 [2] (device): result[0] = 1 if the wait completed (it never
 * should), result[1] = 1 if the abort flag was raised.  The context stays usable afterwards.
 */
int dspark_selftest_wait_timeout(long long limit_cycles, int32_t *result, dspark_stream_t stream);

/*
 * dspark_read_error — synchronise `stream`, return the current device's sticky error word
 * in *host_code (HOST pointer; 0 = no error, else DSPARK_DERR_* bits) and clear it.
 * Returns DSPARK_OK, or DSPARK_ECUDA if the synchronisation or copy failed.
 */
int dspark_read_error(int32_t *host_code, dspark_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DSPARK_H */
