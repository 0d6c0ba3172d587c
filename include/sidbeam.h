/*
 * sidbeam.h -- C ABI of libsidbeam.so: catalog-constrained wide-beam
 * semantic-ID (SID) expansion on NVIDIA B200 (sm_100a).
 *
 * Sources (web pages; cited by title and section):
 *  [P1] flashrec 0.1.0 (PyPI page). Introduction: a SID is a short fixed-depth
 *       token sequence indexing an item catalog; a request decodes 3-5 steps at
 *       beam widths 50-512+, every continuation restricted to the catalog.
 *       Features > Decoding, "SID constraint": a fused kernel with a dense or
 *       CSR-sparse trie restricts decoding to valid SIDs, lm_head covers only
 *       the SID token range, illegal SIDs are never candidates. Features >
 *       Decoding, "Scheduling": beam rows of several requests share a step.
 *       Features > Serving, "API": deterministic top-k at temperature 0.
 *       Quickstart: beams return ranked best-first with a sequence score; with
 *       no catalog the full vocabulary is decoded.
 *  [P4] SPRINT (paper summary), inference paragraph: valid SIDs of a prefix
 *       trie are scored by a token log-probability sum, then top-K; scoring a
 *       SID is a lookup in an L-by-M table.
 *
 * Conventions shared by every call
 *  - Every pointer named "device" is CUDA device memory owned by the caller;
 *    "host" pointers are ordinary host memory. The library owns only the trie.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call except sid_trie_build and sidbeam_get_device_status is
 *    asynchronous on `stream` and never synchronises the host.
 *  - Return value: SIDBEAM_OK (0) or a negative sidbeam_status. Argument errors
 *    are found on the host before anything is launched; sidbeam_last_error()
 *    then holds a message (thread-local).
 *  - Rows are request-major: row = r * B_in + b, b = the slot of the parent
 *    beam in the previous step's ranked output. At step 0, B_in = 1 and the
 *    single row of each request is the trie root (node 0, score 0).
 *  - Scores are cumulative log-probabilities in fp32: the sum over levels of a
 *    log-softmax taken over the level's FULL codebook of V codes; codes that
 *    are not valid trie children are -inf after normalisation (never
 *    candidates), with no renormalisation over the valid ones.
 *  - Order of candidates: score descending, then parent slot ascending, then
 *    code ascending (a total order; ties are resolved exactly).
 *  - Missing outputs (fewer valid candidates than n) are padded with
 *    score -inf and index -1.
 *  - There is no CPU fallback: without a usable CUDA device every call that
 *    launches work returns SIDBEAM_ERR_CUDA.
 */
#ifndef SIDBEAM_H_
#define SIDBEAM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct sidbeam_trie sidbeam_trie; /* opaque, library-owned */

typedef enum {
  SIDBEAM_OK = 0,
  SIDBEAM_ERR_INVALID_ARG = -1,  /* bad size, NULL pointer, unsupported shape   */
  SIDBEAM_ERR_BAD_CATALOG = -2,  /* a code outside [0, V_l), empty catalog     */
  SIDBEAM_ERR_ALIGNMENT = -3,    /* logits not 16-byte aligned rows            */
  SIDBEAM_ERR_WORKSPACE = -4,    /* workspace NULL or smaller than required    */
  SIDBEAM_ERR_OOM = -5,          /* device or host allocation failed (trie)    */
  SIDBEAM_ERR_CUDA = -6,         /* a CUDA runtime call or launch failed       */
  SIDBEAM_ERR_DEVICE_CHECK = -7, /* the device found a bad node id (status)    */
  SIDBEAM_ERR_TIMEOUT = -8       /* a bounded device wait gave up (status)     */
} sidbeam_status;

typedef enum { SIDBEAM_F32 = 0, SIDBEAM_BF16 = 1 } sidbeam_dtype;

typedef enum {
  SIDBEAM_LAYOUT_AUTO = 0,  /* dense when mean fan-out > V/16, else CSR        */
  SIDBEAM_LAYOUT_DENSE = 1, /* per node: V-bit child bitmask + first child id  */
  SIDBEAM_LAYOUT_CSR = 2    /* per node: child offset range + child codes      */
} sidbeam_layout;

/* Limits of the library. */
#define SIDBEAM_MAX_DEPTH 16
#define SIDBEAM_MAX_V 32768      /* codes per level; also V*sizeof(dtype) <= 64 KiB */
#define SIDBEAM_MAX_BEAM 4096    /* n_out of beam_step, K of catalog_score_topk     */

/* ---------------------------------------------------------------- trie
 * sid_trie_build -- [P1] Features > Decoding ("dense or CSR-sparse trie").
 * Sorts and de-duplicates the catalog, numbers the nodes of every level by
 * lexicographic rank among that level's distinct prefixes (root = node 0 of
 * level 0; at the last level node id = leaf id), and uploads one structure per
 * step t = 0..depth-1 (expanding level-t nodes into level-(t+1) codes):
 *   dense: uint32 bitmask [P_t][ceil(V/32) rounded up to 4 words] + offsets;
 *   CSR  : uint32 offsets [P_t + 1] + uint16 child codes [P_{t+1}].
 *  sids             host int32 [n_sids][depth], row-major; duplicates allowed.
 *  codes_per_level  host int32 [depth]; V_l in [1, SIDBEAM_MAX_V].
 *  layout_per_level host int32 [depth] of sidbeam_layout, or NULL (= AUTO).
 *  stream           used for the uploads; the call synchronises it before
 *                   returning, so the trie is ready on return.
 *  out              receives the new trie; free with sid_trie_free.
 * Errors: INVALID_ARG (NULL, depth outside [1, SIDBEAM_MAX_DEPTH], n_sids < 1,
 * more than 2^31-1 nodes on a level), BAD_CATALOG (a code outside [0, V_l)),
 * OOM, CUDA. On error *out is untouched and nothing is leaked. */
int sid_trie_build(const int32_t* sids, int64_t n_sids, int depth,
                   const int32_t* codes_per_level, const int32_t* layout_per_level,
                   void* stream, sidbeam_trie** out);

/* sid_trie_info -- sizes of the built trie.
 *  level in [0, depth]: *n_nodes = number of distinct length-`level` prefixes
 *  (level 0: 1, level depth: number of leaves). For level < depth, *layout is
 *  the layout used to expand level-`level` nodes and *bytes the device bytes of
 *  that step's structure; for level == depth, *layout = -1 and *bytes = bytes
 *  of the leaf tables (leaf rows + leaf codes). Any output pointer may be NULL. */
int sid_trie_info(const sidbeam_trie* trie, int level, int64_t* n_nodes, int* layout,
                  size_t* bytes);

/* sid_trie_leaf_rows -- device int32 [n_leaves]: for each leaf (in leaf-id
 * order) the first input row of sid_trie_build that carried it (the SID ->
 * item map a catalog file provides). Asynchronous copy on `stream`. */
int sid_trie_leaf_rows(const sidbeam_trie* trie, int32_t* out, void* stream);

/* sid_trie_leaf_codes -- device int32 [n_leaves][depth]: the SID of every leaf
 * in leaf-id (lexicographic) order. Asynchronous on `stream`. */
int sid_trie_leaf_codes(const sidbeam_trie* trie, int32_t* out, void* stream);

/* sid_trie_free -- releases the trie (synchronises the device). NULL is a no-op. */
void sid_trie_free(sidbeam_trie* trie);

/* ---------------------------------------------------------------- beam step
 * beam_step_workspace_size -- bytes of device workspace beam_step needs for
 * this shape on the CURRENT device (the row partition depends on its SM
 * count). The workspace must be zero-filled once after allocation; every
 * beam_step call leaves its counters at zero again, so it can be reused by
 * later calls of any shape whose size fits, but not by two calls that run
 * at the same time. Returns 0 for invalid shapes. */
size_t beam_step_workspace_size(int R, int B_in, int n_out, int V);

/* beam_step -- one expansion step for every beam row of every request
 * ([P1] introduction, Features > Decoding, Features > Serving "API").
 *  trie          built trie, or NULL for the unconstrained mode (every code
 *                valid; out_node is then -1). With a trie, V must equal the
 *                trie's V for level step+1.
 *  step          0..depth-1: rows hold level-`step` nodes, codes are level step+1.
 *  logits        device [R*B_in][ld] of `dtype`, row-major; columns 0..V-1 are
 *                the level's codes (a view into a wider vocabulary is fine).
 *                The base must be 16-byte aligned and ld*sizeof(dtype) a
 *                multiple of 16 (else ALIGNMENT); all R*B_in*ld elements must
 *                be readable. Values must be finite.
 *  parent_scores device f32 [R*B_in]; -inf marks a dead row (skipped; its
 *                logits are not read).
 *  parent_nodes  device i32 [R*B_in]; the row's trie node at level `step`
 *                (negative = dead row). Ignored when trie == NULL. A node id
 *                >= the level's node count makes the row dead and sets the
 *                workspace status (sidbeam_get_device_status -> DEVICE_CHECK).
 *  R, B_in       requests and input rows per request; B_in * V < 2^32.
 *  n_out         output beams per request, 1..SIDBEAM_MAX_BEAM.
 *  out_scores    device f32 [R*n_out]: ranked best-first per request.
 *  out_parent    device i32 [R*n_out]: parent slot b in [0, B_in), or -1.
 *  out_code      device i32 [R*n_out]: chosen code in [0, V), or -1.
 *  out_node      device i32 [R*n_out]: child node id at level step+1, or -1.
 *                out_parent/out_code are this step's back-pointers; pass the
 *                step's slices of a [depth][R][n_out] history to keep them.
 *  workspace     device, >= beam_step_workspace_size(R, B_in, n_out, V) bytes,
 *                zero-filled before its first use, 256-byte aligned.
 * Outputs must not alias the inputs. Errors: INVALID_ARG, ALIGNMENT,
 * WORKSPACE, CUDA. */
int beam_step(const sidbeam_trie* trie, int step, const void* logits, sidbeam_dtype dtype,
              int64_t ld, const float* parent_scores, const int32_t* parent_nodes, int R,
              int B_in, int n_out, int V, float* out_scores, int32_t* out_parent,
              int32_t* out_code, int32_t* out_node, void* workspace, size_t workspace_bytes,
              void* stream);

/* beam_step_ex -- beam_step with options (flags: OR of SIDBEAM_STEP_*).
 *  SIDBEAM_STEP_SKIP_ROWS: row skipping (not a step the pages describe; it
 *  leaves every result unchanged). Every child's score s + (z - lse) is at
 *  most its parent's score s (z <= lse), so a row
 *  whose parent score cannot reach a valid lower bound on the request's n-th
 *  best key that the step already holds can contribute nothing: its logits
 *  are not read. Applies when the request's rows are spread over CTAs that
 *  each hold only that request (R no larger than the GPU's SM count); the
 *  first rows of each CTA are always read. The number of rows passed over
 *  accumulates in the workspace (beam_step_skipped_rows).
 *  out_width: NULL, or device i32 [R] with 0 <= out_width[r] <= n_out: request r
 *  keeps only its out_width[r] best beams; output slots past that are padding
 *  (score -inf, indices -1), so they are dead rows of the next step and are
 *  never read. The kept beams are exactly the first out_width[r] ranks of the
 *  request's top n_out, the same as a step with n_out = out_width[r]: per-request
 *  beam widths in one launch, and so in one captured graph of the whole search
 *  (flashrec 0.1.0, Features > Decoding, "Scheduling": rows of several requests
 *  share a step). Values outside [0, n_out] are undefined.
 *  Other arguments, results and errors: those of beam_step; unknown flag bits
 *  give INVALID_ARG. beam_step(...) is beam_step_ex(..., 0, NULL). */
#define SIDBEAM_STEP_SKIP_ROWS 1u
int beam_step_ex(const sidbeam_trie* trie, int step, const void* logits, sidbeam_dtype dtype,
                 int64_t ld, const float* parent_scores, const int32_t* parent_nodes, int R,
                 int B_in, int n_out, int V, float* out_scores, int32_t* out_parent,
                 int32_t* out_code, int32_t* out_node, void* workspace, size_t workspace_bytes,
                 void* stream, unsigned flags, const int32_t* out_width);

/* beam_step_gumbel -- beam_step at temperature > 0: Gumbel top-k without
 * replacement (flashrec 0.1.0, Features > Serving, "API"). Candidate c of
 * parent slot b in request r, with the usual score x = s_b + (z_c - lse_b), is
 * ranked by the key x + T*G, G = -log(-log U)
 * a standard Gumbel variate: U = (v + 1/2) * 2^-23 with v the top 23 bits of
 * the first output word of Philox4x32-10 (Salmon et al., SC'11) on the counter
 * (r, b, c, step) with key (seed low 32 bits, seed high 32 bits). The n largest
 * keys are kept, ranked by key (ties: parent asc, code asc), which draws n
 * candidates without replacement in proportion to exp(x / T). The beams keep
 * the unperturbed score: out_scores[r][i] = x of the i-th drawn candidate, so
 * the next step adds plain log-probabilities (and out_scores are in draw
 * order, not sorted). temperature = 0 is exactly beam_step; it must be
 * finite and >= 0 (else INVALID_ARG).
 *  workspace >= beam_step_gumbel_workspace_size(R, B_in, n_out, V) bytes
 *  (beam_step's workspace plus every row's lse), zero-filled before first use.
 *  Other arguments, results and errors: those of beam_step. Rows are walked in
 *  shared memory (no register rows), so the step is slower than beam_step. */
size_t beam_step_gumbel_workspace_size(int R, int B_in, int n_out, int V);
int beam_step_gumbel(const sidbeam_trie* trie, int step, const void* logits, sidbeam_dtype dtype,
                     int64_t ld, const float* parent_scores, const int32_t* parent_nodes, int R,
                     int B_in, int n_out, int V, float temperature, uint64_t seed,
                     float* out_scores, int32_t* out_parent, int32_t* out_code,
                     int32_t* out_node, void* workspace, size_t workspace_bytes, void* stream);

/* beam_step_skipped_rows -- rows not read by row skipping since the last call
 * on this workspace (host *count); the counter is reset to zero. `stream`
 * orders the read after the steps that used the workspace (the call
 * synchronises it). Errors: INVALID_ARG, CUDA. */
int beam_step_skipped_rows(void* workspace, uint32_t* count, void* stream);

/* beam_step_noalloc -- the same step as beam_step, for callers that cannot
 * allocate device memory when they run it (a plugin whose host application owns
 * every device allocation or enforces a fixed budget, a serving loop that plans
 * all memory up front and must not call cudaMalloc later). Not in the pages:
 * it has no counterpart there; it only changes where the scratch space lives.
 *  Arguments and results are those of beam_step, without the workspace. The
 *  scratch is a fixed array of SIDBEAM_NOALLOC_SCRATCH_BYTES compiled into the
 *  library: every GPU that loads the library holds it until the process exits.
 *  The call allocates nothing. It clears the array's counters on `stream`
 *  (one memset) and then runs the beam_step kernel on it.
 *  The first call on each device looks the array's device address up
 *  (cudaGetSymbolAddress with that device current); make that first call before
 *  any stream capture.
 *  All calls share the one array and it keeps the last call's contents: calls
 *  whose work overlaps on the GPU (other streams, other host threads) race and
 *  give wrong results; serialise them.
 *  The device status word also lives in the array and is not reported here.
 *  Errors: those of beam_step, and WORKSPACE when the shape needs more scratch
 *  than the array holds (beam_step_workspace_size(R, B_in, n_out, V) >
 *  SIDBEAM_NOALLOC_SCRATCH_BYTES). */
#define SIDBEAM_NOALLOC_SCRATCH_BYTES (4 << 20)
int beam_step_noalloc(const sidbeam_trie* trie, int step, const void* logits,
                      sidbeam_dtype dtype, int64_t ld, const float* parent_scores,
                      const int32_t* parent_nodes, int R, int B_in, int n_out, int V,
                      float* out_scores, int32_t* out_parent, int32_t* out_code,
                      int32_t* out_node, void* stream);

/* beam_finalize -- [P1] Quickstart (beams ranked best-first). Follows the
 * back-pointers of `depth` steps from the last step's ranks.
 *  bp_parent, bp_code device i32 [depth][R][n] (each step's out_parent/out_code).
 *  last_node          device i32 [R][n] (the last step's out_node = leaf id).
 *  out_sids           device i32 [R][n][depth]; a padded beam gives all -1.
 *  out_leaf           device i32 [R][n]; -1 for padded beams.
 *  n                  1..SIDBEAM_MAX_BEAM (the steps' n_out).
 * A beam whose parent slot at some step falls outside [0, n) is reported as
 * padded. Launched as a programmatic dependent of the previous kernel on the
 * stream. The scores are the last step's out_scores (unchanged). Errors:
 * INVALID_ARG, CUDA. */
int beam_finalize(int depth, int R, int n, const int32_t* bp_parent, const int32_t* bp_code,
                  const int32_t* last_node, int32_t* out_sids, int32_t* out_leaf, void* stream);

/* ---------------------------------------------------------------- catalog scorer
 * catalog_score_topk -- [P4] inference paragraph. For every request r and
 * every leaf j: score = sum_l logp[r][l][code_l(j)] in fp32 (levels added in
 * order l = 0..depth-1), then the K best by (score desc, leaf id asc).
 *  logp       device f32 [R][depth][V] with V = max over levels of V_l (code
 *             c of level l reads logp[r][l][c]).
 *  out_scores device f32 [R][K]; out_leaf device i32 [R][K] (leaf ids; -1 pad).
 *  workspace  device, >= catalog_score_workspace_size(trie, R, K) bytes,
 *             zero-filled before first use (the call leaves it zeroed).
 * Errors: INVALID_ARG (K outside 1..SIDBEAM_MAX_BEAM), WORKSPACE, CUDA. */
size_t catalog_score_workspace_size(const sidbeam_trie* trie, int R, int K);
int catalog_score_topk(const sidbeam_trie* trie, const float* logp, int R, int K,
                       float* out_scores, int32_t* out_leaf, void* workspace,
                       size_t workspace_bytes, void* stream);

/* catalog_score_topk_sim -- catalog_score_topk plus the SID-level similarity
 * term of the same page (inference paragraph: token log-probability sum plus
 * SID-level similarity, then top-K; closing paragraph: one pass gives the
 * L-by-M table and a user vector, and scoring a SID is a lookup plus one matrix
 * product). score = sum_l logp[r][l][code_l(j)] + <user[r], sid_emb[j]>, the
 * dot product in fp32 (four partial sums over k = 0, 1, 2, 3 mod 4, added
 * pairwise), added after the lookup sum.
 * The pages give no weight between the terms (a scale of user[r] is one).
 *  user     device f32 [R][d]; sid_emb device bf16 [N][d] (N = the trie's
 *           leaf count, row j = leaf id j as sid_trie_leaf_codes orders them),
 *           16-byte aligned (else ALIGNMENT); d a multiple of 8 in [8, 1024].
 *  Other arguments as catalog_score_topk (same workspace size). Errors:
 *  INVALID_ARG, ALIGNMENT, WORKSPACE, CUDA. */
int catalog_score_topk_sim(const sidbeam_trie* trie, const float* logp, const float* user,
                           const uint16_t* sid_emb, int d, int R, int K, float* out_scores,
                           int32_t* out_leaf, void* workspace, size_t workspace_bytes,
                           void* stream);

/* ---------------------------------------------------------------- SID-range lm_head
 * lmhead_logits -- flashrec 0.1.0, Features > Decoding ("SID constraint"): the
 * lm_head evaluated only over the SID token range. For every row and code:
 *   logits[row][c] = sum_k hidden[row][k] * w_sid[c][k]
 * with bf16 inputs (exact products) and fp32 accumulation on the tensor cores
 * (tcgen05; the summation order is not specified).
 *  hidden     device bf16 [M][d], row-major, 16-byte aligned; d % 8 == 0.
 *  w_sid      device bf16 [V][d], row-major, 16-byte aligned (the rows of the
 *             lm_head weight that belong to the level's SID codes).
 *  logits     device f32 [M][ld], ld >= V, ld % 4 == 0, 16-byte aligned.
 *  workspace  device, >= 256 bytes, zero-filled before first use (status word).
 * Asynchronous on `stream`. Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, CUDA. */
int lmhead_logits(const void* hidden, const void* w_sid, int M, int V, int d, float* logits,
                  int64_t ld, void* workspace, size_t workspace_bytes, void* stream);

/* sidbeam_fused_lmhead_step -- flashrec 0.1.0, Features > Decoding ("SID
 * constraint"): the lm_head over the SID token range feeding the constrained
 * step, without writing the logits out. Computes exactly beam_step's result
 * for logits[row][c] = sum_k hidden[row][k] * w_sid[c][k] (fp32 accumulation
 * on the tensor cores, as lmhead_logits):
 *  hidden          device bf16 [R*B_in][d], row-major, 16-byte aligned, d % 8 == 0.
 *  w_sid           device bf16 [V][d], row-major, 16-byte aligned.
 *  every other argument as for beam_step (no dtype / ld: the logits are made
 *  here); workspace >= fused_lmhead_workspace_size(R, B_in, n_out, V) bytes,
 *  zero-filled before first use (the call leaves the first part zeroed; the
 *  rest is scratch: per-row child bitmaps, per-tile partial sums, child logits).
 * Asynchronous on `stream` (three launches). Errors as for beam_step. */
size_t fused_lmhead_workspace_size(int R, int B_in, int n_out, int V);
int sidbeam_fused_lmhead_step(const sidbeam_trie* trie, int step, const void* hidden,
                              const void* w_sid, int d, const float* parent_scores,
                              const int32_t* parent_nodes, int R, int B_in, int n_out, int V,
                              float* out_scores, int32_t* out_parent, int32_t* out_code,
                              int32_t* out_node, void* workspace, size_t workspace_bytes,
                              void* stream);

/* ---------------------------------------------------------------- status
 * sidbeam_get_device_status -- synchronises `stream`, reads and clears the
 * status word that beam_step / catalog_score_topk keep at the start of
 * `workspace`; returns SIDBEAM_OK, DEVICE_CHECK (a bad node id was seen) or
 * TIMEOUT (a bounded wait inside a kernel gave up). */
int sidbeam_get_device_status(void* workspace, void* stream);

/* sidbeam_last_error -- message for the last non-OK return on this thread. */
const char* sidbeam_last_error(void);

/* sidbeam_version -- "major.minor.patch". */
const char* sidbeam_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SIDBEAM_H_ */
