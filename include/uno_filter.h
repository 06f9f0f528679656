/*
 * uno_filter.h -- C ABI of libuno_filter.so: UNO's per-cycle sampling and
 * verification step over vocabulary-wide logits, on one NVIDIA B200 (sm_100a).
 *
 * Method sources (web pages):
 *   [UNO PR]     "sgl-project/sglang pull request 37667: UNO" -- "Motivation"
 *                (lossless; linear sampler draws each of B tokens from its own
 *                marginal; tree sampler keeps the top K candidates of each
 *                marginal and considers V candidate sequences), "Modifications"
 *                (sparse and dense proposal and rejection sampling for linear
 *                UNO; tree UNO reuses EAGLE tree verification with compact-
 *                support target sampling), review thread (top-k is applied and
 *                renormalised before top-p).
 *   [eval guide] "用 SGLang benchmark/uno 复现 UNO 全量数学评测：run_math_eval
 *                实战与源码解析" -- "run_math_eval 全参数详解" (top_k > 0,
 *                top_p in (0, 1], temperature >= 0), "B/K/V 参数映射" (B draft
 *                width, K candidates per depth, V verification width) and
 *                "启动期硬性约束" (V >= B, V <= 128, V*K <= 2048, acceptance
 *                thresholds 1.0).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers.  Every tensor argument is a DEVICE pointer owned by the caller;
 *   the library keeps no pointer after a call returns and allocates no memory.
 *   Logits may be binary32 (UNO_F32) or bfloat16 (UNO_BF16, the top half of a
 *   binary32) and must be aligned to their element size; 16-byte-aligned rows
 *   are read fastest.
 * Stream.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Calls are asynchronous: results are ready when the stream
 *   reaches them.  A call enqueues one or two kernels and nothing else.
 * Workspace.  Entry points that need scratch take (workspace, workspace_bytes),
 *   caller-owned device memory of at least the size the matching
 *   uno_*_workspace_bytes() returns (256-byte aligned).  Its first
 *   UNO_WORKSPACE_COUNTER_BYTES hold arrival counters: zero-fill them once,
 *   before the first use (zero-filling the whole buffer is simplest).  Every
 *   call leaves them at zero again and writes nothing else there, so one
 *   workspace serves any later call of any entry point and size.  The next
 *   UNO_WORKSPACE_HINT_BYTES hold threshold hints that a call leaves for the
 *   next call of the same entry point (see uno_filter_softmax): a speed aid
 *   only, whatever they hold (zero included) the results are the same.  The
 *   rest is scratch the library overwrites.  Calls that run at the same time on the
 *   GPU must not share a workspace.  Verifiers take at most
 *   UNO_WORKSPACE_COUNTER_BYTES / 8 requests per call.
 * Compact distributions.  A filtered row is stored as `count` pairs
 *   (id, prob) in ascending id order, probabilities binary32, in slots
 *   [0, count) of a row of `cap` slots; unused slots hold id -1 and prob 0.
 * Randomness.  Each decision draws u in [0, 1) from Philox4x32-10 (Salmon et
 *   al., SC'11) with key = seed (low word first) and counter
 *   (request, position, draw, cycle); u = (x0 * 2^21 + (x1 >> 11)) * 2^-53.
 *   draw = 0 proposal/sample, 1 accept test, 2 residual, 3 target/bonus.
 * Filter.  Per row: keep the top_k finite logits ordered by (logit desc,
 *   id asc); temperature 0 keeps the first alone (greedy); otherwise
 *   w_j = exp((l_j - l_0) / T) and P_j = w_j / sum(w); keep j while the mass
 *   before j is < top_p (always the first; top_p = 1 keeps all); the result
 *   is w_j / sum of kept w_j.  The softmax over the kept support runs in
 *   double precision; the scan over the vocabulary reads every logit once.
 * Errors.  Arguments are checked on the host before anything is enqueued:
 *   UNO_ERR_INVALID_ARG for null pointers, non-positive sizes, top_k < 1,
 *   top_p outside (0, 1], temperature negative or non-finite, a bad tree
 *   shape; UNO_ERR_UNSUPPORTED for cap < min(top_k, vocab) or
 *   top_k > UNO_MAX_TOP_K; UNO_ERR_WORKSPACE for a null or short workspace;
 *   UNO_ERR_CUDA when a launch fails (cudaGetLastError).  Data errors never
 *   trap: they set per-row or per-request flag bits (UNO_FLAG_*).
 */
#ifndef UNO_FILTER_H
#define UNO_FILTER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    UNO_OK = 0,
    UNO_ERR_INVALID_ARG = 1,
    UNO_ERR_UNSUPPORTED = 2,
    UNO_ERR_CUDA = 3,
    UNO_ERR_WORKSPACE = 4
} uno_status;

typedef enum { UNO_F32 = 0, UNO_BF16 = 1 } uno_dtype;

/* Request sampling parameters ([eval guide, run_math_eval 全参数详解]). */
typedef struct {
    float temperature; /* >= 0; 0 = greedy                  */
    int32_t top_k;     /* >= 1; clamped to the vocabulary     */
    float top_p;       /* in (0, 1]                           */
} uno_sampling_params;

/* Counter-based RNG state of one decode cycle.  first_request is the global
 * index of the call's first request: the counter's request word is
 * first_request + local request index, so a batch split across calls or GPUs
 * draws the same uniforms as one call over the whole batch.
 *
 * cycle_word is NULL or a 4-byte aligned device address of a uint32_t.  When
 * it is set, the kernels read the cycle word there when they run and ignore
 * `cycle`.  A CUDA graph captured around a call replays the call's arguments
 * unchanged; with cycle_word set, writing the next cycle's number to that
 * word (on the graph's stream, before the replay) makes each replay draw that
 * cycle's uniforms.  The word must stay valid, and unchanged while a call
 * that reads it runs, until the call (or graph replay) completes.  A
 * misaligned address returns UNO_ERR_INVALID_ARG. */
typedef struct {
    uint64_t seed;
    uint32_t cycle;
    uint32_t first_request;
    const uint32_t* cycle_word;
} uno_rng;

#define UNO_MAX_TOP_K 1024
#define UNO_WORKSPACE_COUNTER_BYTES (1 << 20)
#define UNO_WORKSPACE_HINT_BYTES 16384
#define UNO_MAX_TREE_NODES 128   /* V <= 128   ([eval guide, 启动期硬性约束]) */
#define UNO_MAX_TREE_FRONTIER 2048 /* V*K <= 2048 (same section) */

/* Flag bits (per row of uno_filter_softmax, per request of the verifiers). */
#define UNO_FLAG_NONFINITE_ROW 1u        /* NaN or +inf logit, or no finite logit */
#define UNO_FLAG_DRAFT_NOT_IN_SUPPORT 2u /* draft token has q = 0: rejected      */
#define UNO_FLAG_RESIDUAL_EMPTY 4u       /* max(0, p - q) summed to 0: drew p    */
#define UNO_FLAG_TIMEOUT 8u              /* a bounded wait for the row's own     */
                                         /* asynchronous copies gave up; the row */
                                         /* result is not valid                  */
#define UNO_FLAG_BAD_PARAMS 32u          /* *_params entry points: the request's */
                                         /* parameter entries are out of range;  */
                                         /* the row has no support               */

/* ------------------------------------------------------------------------
 * uno_filter_softmax -- filter each row and optionally draw from it.
 * [UNO PR, review thread]: top-k first, renormalise, then top-p; [UNO PR,
 * Motivation]: the linear sampler draws each draft token independently from
 * its marginal.
 *
 * logits      [rows][row_stride] elements of dtype `dt` (row_stride >= vocab).
 * rows_per_request  maps row -> (request = rng->first_request + row / rpr,
 *             position = row % rpr) for the RNG counter (e.g. B for draft
 *             marginals).
 * cap         slots per compact row, >= min(top_k, vocab).
 * out_ids     [rows][cap] int32, out_probs [rows][cap] float, out_count [rows].
 * out_dense   nullable [rows][vocab] float: the filtered distribution.
 * rng         nullable; when given, out_sample [rows] receives one token drawn
 *             by inverse CDF (ascending id) with draw 0; -1 for a row with no
 *             support.
 * out_flags   [rows] UNO_FLAG_NONFINITE_ROW for rows with NaN/+inf/no finite.
 * workspace   see uno_filter_softmax_workspace_bytes.
 * ---------------------------------------------------------------------- */
size_t uno_filter_softmax_workspace_bytes(int64_t rows, int64_t vocab, int32_t top_k);
uno_status uno_filter_softmax(const void* logits, uno_dtype dt, int64_t rows, int64_t vocab, int64_t row_stride,
                              int32_t rows_per_request, uno_sampling_params sp, int32_t cap, int32_t* out_ids,
                              float* out_probs, int32_t* out_count, float* out_dense, const uno_rng* rng,
                              int32_t* out_sample, uint32_t* out_flags, void* workspace, size_t workspace_bytes,
                              void* stream);

/* ------------------------------------------------------------------------
 * uno_linear_verify -- linear-mode rejection sampling for R requests.
 * [UNO PR, Motivation]: lossless like speculative decoding; [UNO PR,
 * Modifications]: proposal and rejection sampling for linear UNO.  Rule (the
 * standard speculative-sampling rule; the pages print no formula): for draft
 * position i = 0..B-1 accept x_i iff u_accept * q_i(x_i) < p_i(x_i); at the
 * first rejection draw from normalise(max(0, p_i - q_i)) over supp p_i with
 * the residual draw (from p_i, flagged, if that sums to 0) and stop; if all B
 * are accepted draw a bonus token from p_B with the target draw.  p_i is
 * target row i filtered as in uno_filter_softmax.
 *
 * target_logits [R][B+1][vocab] (dtype dt), contiguous.
 * draft_ids     [R][B] int32 (ids outside supp q_i are rejected and flagged).
 * q_ids/q_probs [R*B][q_cap], q_count [R*B]: the draft marginals as written by
 *               uno_filter_softmax (ascending ids).
 * out_tokens    [R][B+1]: accepted drafts then the correction/bonus token;
 *               unused slots -1.  out_accept_len [R] in [0, B];
 *               out_num_tokens [R] = accept_len + 1 (accept_len when a
 *               non-finite target row is reached; its slot holds -1).
 * out_flags     [R] OR of the request's flag bits.
 * ---------------------------------------------------------------------- */
size_t uno_linear_verify_workspace_bytes(int32_t R, int32_t B, int64_t vocab, int32_t top_k);
uno_status uno_linear_verify(const void* target_logits, uno_dtype dt, int32_t R, int32_t B, int64_t vocab,
                             uno_sampling_params sp, const int32_t* draft_ids, const int32_t* q_ids,
                             const float* q_probs, const int32_t* q_count, int32_t q_cap, uno_rng rng,
                             int32_t* out_tokens, int32_t* out_accept_len, int32_t* out_num_tokens,
                             uint32_t* out_flags, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * uno_linear_cycle -- one whole linear cycle: filter the draft marginals and
 * draw the proposals, filter the target rows, and verify, in one launch over
 * all the cycle's rows (then one short launch for the request decisions).
 * [UNO PR, Motivation]: one model, two forward passes per cycle; the
 * diffusion pass drafts B tokens and produces the first output token, the
 * autoregressive pass verifies; [UNO PR, Modifications]: the B + 1 output
 * layout and the counters (num_correct_drafts = accept_len - 2).
 *
 * layout UNO_LAYOUT_GENERIC: B draft rows and B + 1 target rows per request;
 *   every proposal x_i is tested against target row i, target row B gives
 *   the bonus (uno_filter_softmax with a draw, then uno_linear_verify).
 * layout UNO_LAYOUT_TWO_PASS: B draft rows and B target rows per request, the
 *   pages' layout: draft row 0 comes from the base weights and its draw x_0
 *   is emitted untested; target row i - 1 (the distribution of output token
 *   i) tests proposal x_i (i = 1 .. B-1); if all are accepted target row
 *   B - 1 gives the bonus with the target draw at position B.
 * Draws: proposal i with (request, i, PROPOSAL), its test with (request, i,
 *   ACCEPT), the correction with (request, i, RESIDUAL), the bonus with
 *   (request, B, TARGET), as in the separate calls.
 *
 * draft_logits  [R][B][vocab]; target_logits [R][B+1][vocab] (generic) or
 *               [R][B][vocab] (two-pass); dtype dt, contiguous.
 * out_tokens    [R][B+1] emitted tokens, unused slots -1.
 * out_num_accepted [R]: proposals accepted by the test (generic: the
 *               accept length in [0, B]; two-pass: num_correct_drafts in
 *               [0, B-1], x_0 not counted).
 * out_num_tokens [R]: tokens emitted (two-pass: the pages' accept_len).
 * out_flags     [R]: OR of the flags of the request's draft rows, target rows
 *               and decisions.
 * out_draft_ids [R][B] the proposals (nullable).
 * workspace     see uno_linear_cycle_workspace_bytes (same rules as above).
 * ---------------------------------------------------------------------- */
#define UNO_LAYOUT_GENERIC 0
#define UNO_LAYOUT_TWO_PASS 1
size_t uno_linear_cycle_workspace_bytes(int32_t R, int32_t B, int64_t vocab, int32_t top_k, int32_t layout);
uno_status uno_linear_cycle(const void* draft_logits, const void* target_logits, uno_dtype dt, int32_t R, int32_t B,
                            int64_t vocab, int32_t layout, uno_sampling_params sp, uno_rng rng, int32_t* out_tokens,
                            int32_t* out_num_accepted, int32_t* out_num_tokens, uint32_t* out_flags,
                            int32_t* out_draft_ids, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * uno_tree_topk_expand -- top-K candidates per marginal and a V-node tree.
 * [UNO PR, Motivation]: the tree sampler considers V candidate sequences by
 * selecting the top K candidates from each marginal, hyperparameters
 * (B, K, V); [eval guide, 启动期硬性约束]: V >= B, V <= 128, V*K <= 2048.  The
 * pages fix no construction rule.  This library's rule: candidates of depth
 * d+1 are the first min(K, count_d) tokens of q_d by (prob desc, id asc);
 * node 0 is the root; a child's score is its parent's score times q_d(token)
 * (double); the frontier node with the highest score joins next, ties to the
 * lower depth, then lower parent index, then lower candidate rank; stop at V
 * nodes (root included) or an empty frontier.  Parents precede children.
 *
 * q_ids/q_probs [R*B][q_cap], q_count [R*B] (ascending ids, as written by
 *               uno_filter_softmax).
 * node_token, node_parent, node_depth [R][V] int32, node_score [R][V] float;
 *               root: token -1, parent -1, depth 0, score 1; unused slots
 *               token -1, parent -1, depth -1, score 0.  num_nodes [R].
 * No workspace.
 * ---------------------------------------------------------------------- */
uno_status uno_tree_topk_expand(const int32_t* q_ids, const float* q_probs, const int32_t* q_count, int32_t q_cap,
                                int32_t R, int32_t B, int32_t K, int32_t V, int32_t* node_token,
                                int32_t* node_parent, int32_t* node_depth, float* node_score, int32_t* num_nodes,
                                void* stream);

/* ------------------------------------------------------------------------
 * uno_tree_verify -- target-only verification of the candidate trees.
 * [UNO PR, Modifications]: tree UNO reuses EAGLE tree verification with
 * compact-support target sampling; [eval guide, 启动期硬性约束]: acceptance
 * thresholds 1.0 (pure target sampling).  From the root: draw y from node j's
 * filtered target row with the target draw at position j; if a child of j
 * (lowest index first) carries y, emit y and continue from it; otherwise emit
 * y and stop.  Stops after B+1 tokens at most.
 *
 * target_logits [R][V][vocab] (dtype dt), one row per node; rows at or past
 *               num_nodes[r] are not read.
 * node_token, node_parent [R][V], num_nodes [R]: as written by
 *               uno_tree_topk_expand.
 * out_tokens, out_path_nodes [R][B+1] (path_nodes[t] = node whose row drew
 *               token t; unused -1); out_accept_len [R] = tokens - 1;
 *               out_num_tokens [R]; out_flags [R].
 * ---------------------------------------------------------------------- */
size_t uno_tree_verify_workspace_bytes(int32_t R, int32_t V, int64_t vocab, int32_t top_k);
uno_status uno_tree_verify(const void* target_logits, uno_dtype dt, int32_t R, int32_t B, int32_t V, int64_t vocab,
                           uno_sampling_params sp, const int32_t* node_token, const int32_t* node_parent,
                           const int32_t* num_nodes, uno_rng rng, int32_t* out_tokens, int32_t* out_accept_len,
                           int32_t* out_num_tokens, int32_t* out_path_nodes, uint32_t* out_flags, void* workspace,
                           size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Per-request sampling parameters and the filter order.
 * [eval guide, run_math_eval 全参数详解]: temperature, top_p and top_k are
 * set per run (temperature >= 0, 0 greedy; top_p in (0, 1]; top_k > 0); a
 * serving batch mixes requests that carry different ones.  [UNO PR, review
 * thread on the filter order]: UNO takes top-k first, renormalises over the
 * kept tokens and applies top-p to that distribution (UNO_ORDER_TOPK_FIRST,
 * what the entry points above do); the regular sampler uses the "joint"
 * order, where the top-p cut is taken on the full-vocabulary softmax
 * (UNO_ORDER_JOINT): the cumulative mass of the top-k tokens, in descending
 * order, is divided by the sum of exp((l - l_max) / T) over every finite
 * logit of the row instead of over the top k.  Top-k still bounds the kept
 * set, and the kept probabilities are still renormalised among themselves.
 *
 * temperature, top_k, top_p  device arrays of one entry per request
 *             (4-byte aligned); a row reads the entries of its request
 *             (filter: row / rows_per_request; verifiers: the request whose
 *             target row it is).  Each call reads them when it runs, so they
 *             may change between replays of a captured graph.
 * top_k_max   host value, 1 .. UNO_MAX_TOP_K: an upper bound of the top_k
 *             entries after clamping to the vocabulary.  It sizes the
 *             selection and the workspace (pass it as top_k to the
 *             *_workspace_bytes functions) and `cap` must hold
 *             min(top_k_max, vocab).
 * order       UNO_ORDER_TOPK_FIRST or UNO_ORDER_JOINT.  The joint order adds
 *             one read of each row (its normaliser) before the row kernels.
 * A request whose entries are out of range (temperature negative, NaN or
 * infinite; top_k < 1 or, clamped to the vocabulary, above top_k_max; top_p
 * outside (0, 1]) is not an error of the call: its rows get
 * UNO_FLAG_BAD_PARAMS and no support, and a verifier treats them like
 * non-finite target rows.  Host-side errors (UNO_ERR_INVALID_ARG): rp NULL,
 * a NULL or misaligned array, top_k_max < 1, an unknown order.
 *
 * The four entry points take the same arguments as the ones above, with rp
 * in place of the sampling parameters.
 * ---------------------------------------------------------------------- */
#define UNO_ORDER_TOPK_FIRST 0
#define UNO_ORDER_JOINT 1
typedef struct {
    const float* temperature;
    const int32_t* top_k;
    const float* top_p;
    int32_t top_k_max;
    int32_t order;
} uno_request_params;

uno_status uno_filter_softmax_params(const void* logits, uno_dtype dt, int64_t rows, int64_t vocab,
                                     int64_t row_stride, int32_t rows_per_request, const uno_request_params* rp,
                                     int32_t cap, int32_t* out_ids, float* out_probs, int32_t* out_count,
                                     float* out_dense, const uno_rng* rng, int32_t* out_sample, uint32_t* out_flags,
                                     void* workspace, size_t workspace_bytes, void* stream);
uno_status uno_linear_verify_params(const void* target_logits, uno_dtype dt, int32_t R, int32_t B, int64_t vocab,
                                    const uno_request_params* rp, const int32_t* draft_ids, const int32_t* q_ids,
                                    const float* q_probs, const int32_t* q_count, int32_t q_cap, uno_rng rng,
                                    int32_t* out_tokens, int32_t* out_accept_len, int32_t* out_num_tokens,
                                    uint32_t* out_flags, void* workspace, size_t workspace_bytes, void* stream);
uno_status uno_linear_cycle_params(const void* draft_logits, const void* target_logits, uno_dtype dt, int32_t R,
                                   int32_t B, int64_t vocab, int32_t layout, const uno_request_params* rp,
                                   uno_rng rng, int32_t* out_tokens, int32_t* out_num_accepted,
                                   int32_t* out_num_tokens, uint32_t* out_flags, int32_t* out_draft_ids,
                                   void* workspace, size_t workspace_bytes, void* stream);
uno_status uno_tree_verify_params(const void* target_logits, uno_dtype dt, int32_t R, int32_t B, int32_t V,
                                  int64_t vocab, const uno_request_params* rp, const int32_t* node_token,
                                  const int32_t* node_parent, const int32_t* num_nodes, uno_rng rng,
                                  int32_t* out_tokens, int32_t* out_accept_len, int32_t* out_num_tokens,
                                  int32_t* out_path_nodes, uint32_t* out_flags, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * uno_linear_verify_noalloc -- uno_linear_verify without a caller workspace.
 * This entry point has no counterpart on the method's pages: it only changes
 * where the scratch memory comes from.  It is for callers that cannot
 * allocate device memory for the library -- a serving loop that has given all
 * free memory to its KV-cache pool, or a host that loads this library as a
 * plugin and offers it no allocator.  Its scratch is a library-owned device
 * array of UNO_NOALLOC_SCRATCH_BYTES (8 MiB) that every GPU which loads the
 * library holds until the process exits.
 *
 * Arguments, results and errors are those of uno_linear_verify, minus the
 * workspace.  Sizes whose uno_linear_verify_workspace_bytes exceeds
 * UNO_NOALLOC_SCRATCH_BYTES return UNO_ERR_UNSUPPORTED before anything is
 * enqueued: the 8 MiB hold R*(B+1) * k4 up to about 800,000, k4 being
 * min(top_k, vocab) rounded up to a multiple of 4 (512 requests with B = 16
 * at top_k 50 fit; at top_k 200 they do not).  Each CUDA context that loads
 * the library has its own copy of the array at its own address.  A call made
 * while `stream` is not being captured looks that address up
 * (cudaGetSymbolAddress) in the current context and remembers it for that
 * context; a call made during stream capture uses the remembered address, so
 * make one uncaptured call in a context before capturing one there (a
 * captured call in a context never seen returns UNO_ERR_CUDA if the lookup
 * is refused during capture).  The call itself allocates nothing: it
 * enqueues cudaMemsetAsync of the counters it may use, then its kernels.
 * Every call
 * shares the one array, so calls that overlap on the GPU (other streams,
 * other host threads) race; serialise them.
 * ---------------------------------------------------------------------- */
#define UNO_NOALLOC_SCRATCH_BYTES (8u << 20)
uno_status uno_linear_verify_noalloc(const void* target_logits, uno_dtype dt, int32_t R, int32_t B, int64_t vocab,
                                     uno_sampling_params sp, const int32_t* draft_ids, const int32_t* q_ids,
                                     const float* q_probs, const int32_t* q_count, int32_t q_cap, uno_rng rng,
                                     int32_t* out_tokens, int32_t* out_accept_len, int32_t* out_num_tokens,
                                     uint32_t* out_flags, void* stream);

/* ------------------------------------------------------------------------
 * uno_tree_suffix_attention_merge -- tree-suffix attention of the V tree
 * nodes, merged with the prefix attention state by log-sum-exp.
 * [UNO PR, Modifications]: tree mode verifies its V nodes with EAGLE's
 * cascade attention, and UNO adds a fused kernel for the tree-suffix
 * attention and the LSE merge.  The pages print no formula; the standard
 * cascade split is taken.  Node j's query attends, within the tree, to its
 * ancestors and itself, with scores scale * <q, k>.  That gives a partial
 * state (o_s, l_s), where l_s = log sum exp(scores) in natural logarithms.
 * The prefix part arrives as (o_p, l_p) from another attention kernel.  The
 * result is o = (e^l_p o_p + e^l_s o_s) / (e^l_p + e^l_s) and
 * l = log(e^l_p + e^l_s).  Query head h reads key/value head h / (H / Hkv).
 * Arithmetic is binary32.
 *
 * q            [R][V][H][d]; k and v [R][V][Hkv][d]; dtype dt, contiguous.
 * node_parent  [R][V] int32, with parent[0] = -1 and parent[j] < j;
 *              num_nodes [R].  Both are as written by uno_tree_topk_expand.
 *              Nodes at or past num_nodes[r] are not read; they get o = 0
 *              and lse = -inf.
 * o_prefix     [R][V][H][d] float; lse_prefix [R][V][H] float.  An lse of
 *              -inf marks an empty prefix, and its o_prefix is then not read.
 * out_o        [R][V][H][d] float; out_lse [R][V][H] float.
 * out_flags    nullable [R]: UNO_FLAG_BAD_TREE when a node's parent breaks
 *              the rule above.  That node then attends to itself alone.
 * Kernels: bf16 calls with d a multiple of 16, q, k, v, o_prefix and out_o
 * 16-byte aligned and the operand tiles within 220 KB of shared memory run
 * on the tensor cores (tcgen05, accumulators in tensor memory), one CTA per
 * (request, key/value head, 128 stacked query rows).  Every other call runs
 * on a CUDA-core kernel, one CTA per (request, key/value head), which needs
 * the key and value tiles of one head, 2 * V * (d + 1) floats, within
 * shared memory.  Arrays need only their element alignment.
 * Limits: 1 <= V <= UNO_MAX_TREE_NODES, d <= 256, H a multiple of Hkv;
 * UNO_ERR_UNSUPPORTED when neither kernel applies.  No workspace.
 * ---------------------------------------------------------------------- */
#define UNO_FLAG_BAD_TREE 16u
uno_status uno_tree_suffix_attention_merge(const void* q, const void* k, const void* v, uno_dtype dt, int32_t R,
                                           int32_t V, int32_t H, int32_t Hkv, int32_t d, float scale,
                                           const int32_t* node_parent, const int32_t* num_nodes,
                                           const float* o_prefix, const float* lse_prefix, float* out_o,
                                           float* out_lse, uint32_t* out_flags, void* stream);

/* Text of a status code (static storage). */
const char* uno_status_string(uno_status s);

#ifdef __cplusplus
}
#endif

#endif /* UNO_FILTER_H */
