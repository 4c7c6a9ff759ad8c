/*
 * bsa.h -- C ABI of libbsa.so: query-dependent block-sparse causal attention with per-block key
 * summaries, hand-written for NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page title and the section / equation on it:
 *   [SAS]        review page "SAS: Simple Attention Sparsification via End-to-End Optimization of
 *                Context Ranking": "Background" (Eq. 1-3), "The new approach" (Eq. 4, Eq. 9),
 *                "Why the four design choices matter" (Eq. 5, log g = s - LSE(s)),
 *                "How it works: a worked example", "Decoding efficiency" (Fig. 7).
 *   [FreeSolo]   summary page "FreeSolo가 학습 길이의 64배까지 제로샷 검색을 유지한다": "How it works"
 *                (cells, summaries, cell score, two branches), "How it differs" (FS-L, FS-B).
 *   [Monodratic] article "Monodratic、学習ルーティングによりスパース因果アテンションの選択性を高められると
 *                主張": guaranteed local block + exact causal softmax over the selected tokens.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers named q, k, v, o, dout, mean_k, ... are DEVICE pointers; sizes are host ints.
 *  - Layouts are row-major with the head dimension d fastest:
 *        Q, O, dO  [B, Hq, nq, d]      K, V  [B, Hk, n, d]
 *    Query head h reads kv head h / (Hq / Hk) (contiguous GQA groups).
 *  - Context of n positions is cut into C = ceil(n / b) blocks of b tokens; a short final block
 *    keeps the remaining tokens ([SAS] "Background", Eq. 3).
 *  - Block indices are int32, padding is -1; summaries, scores, lse and dg are float32.
 *  - The caller owns every buffer (allocate with any allocator, e.g. PyTorch).  The library
 *    never allocates or frees device memory and keeps no state between calls.
 *  - Every call is asynchronous on the given cudaStream_t (passed as void*; NULL = legacy
 *    default stream).  Arguments are checked on the host first; a bad argument returns an
 *    error status and launches nothing.  A failed launch returns BSA_ERR_CUDA.
 *  - Kernels that wait on the copy engine bound every wait; when a bound runs out they write a
 *    nonzero word at the start of the workspace and stop.  bsa_workspace_status() reads it
 *    (BSA_ERR_TIMEOUT) and clears it.
 *  - Supported: dtype BSA_F32 or BSA_BF16, head dim d in {64, 128}, Hq % Hk == 0 with
 *    Hq / Hk in {1, 2, 4, 8}, block size b in [1, 128] (decode) / [1, 1024] (summaries).
 *    Other valid values return BSA_ERR_UNSUPPORTED.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSA_OK = 0,
  BSA_ERR_ARG = 1,          /* null pointer, negative size or unknown enum value */
  BSA_ERR_SHAPE = 2,        /* sizes inconsistent with each other (Hq % Hk, K < 1, ...) */
  BSA_ERR_DTYPE = 3,        /* unknown dtype */
  BSA_ERR_UNSUPPORTED = 4,  /* valid request this build has no kernel for (e.g. d = 96) */
  BSA_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed */
  BSA_ERR_TIMEOUT = 6,      /* a bounded device-side wait ran out (reported by status query) */
  BSA_ERR_WORKSPACE = 7     /* workspace missing or smaller than *_workspace_bytes() */
} bsa_status;

typedef enum { BSA_F32 = 0, BSA_BF16 = 1 } bsa_dtype;

/* Training-mode gate of [SAS] "The new approach", Eq. 9. */
/* BSA_GATE_OUTER is the outer-gate variant ([SAS] "Why the four design choices matter", the gate
 * placed outside the softmax): o_i = sum_j g_m(j) p_j v_j with p the ungated softmax and g the
 * same softmax gate; prefill (training) form only. */
typedef enum { BSA_GATE_NONE = 0, BSA_GATE_LOG_SOFTMAX = 1, BSA_GATE_OUTER = 2 } bsa_gate_mode;

/* Set the softmax gate normalises over ([SAS] "Why the four design choices matter"):
 * SELECTED = LSE over the selected history blocks, ALL_HISTORY = LSE over every history block. */
typedef enum { BSA_NORM_SELECTED = 0, BSA_NORM_ALL_HISTORY = 1 } bsa_gate_norm;

/* Variants of bsa_decode_step_ex (bit flags). */
typedef enum {
  /* One selection per kv head: the group's score of a block is the mean of its G query heads'
   * scores (the bsa_score_blocks scores); its Top-K (plus the current block) is attended by every
   * head of the group.  The pages leave per-head versus shared selection under GQA open; the
   * per-head rule is the default. */
  BSA_DECODE_SHARED_SELECTION = 1,
  /* mean_k is bf16 [B, Hk, C, d] (see bsa_round_summaries_bf16): half the summary bytes; the dot
   * products still accumulate in fp32.  Needs dt = BSA_BF16 and b = 64. */
  BSA_DECODE_BF16_SUMMARIES = 2,
  /* bsa_decode_step_ws only: q and o are page-locked host buffers (cudaHostAlloc, or a pinned
   * torch tensor) instead of device memory.  The step reads q itself (once per kv-head group, or
   * through a small staging kernel whose host reads may start before the work queued ahead of it
   * on the stream has finished, so that work must not write q) and its last phase writes o
   * straight to host memory.  As with an asynchronous copy from page-locked memory, the host must
   * leave q unchanged, and must not read o, until the stream has passed the call.  BSA_ERR_ARG if
   * q or o is not page-locked host memory mapped for the device. */
  BSA_DECODE_HOST_IO = 4
} bsa_decode_flags;

/* Human-readable name of a status code (static string, never NULL). */
const char* bsa_status_string(bsa_status s);

/* Library version as 10000*major + 100*minor + patch. */
int bsa_version(void);

/*
 * bsa_build_block_summaries -- per-block key summaries ([FreeSolo] "How it works": mean key of
 * the cell, its centre position, the largest key norm inside it).
 *
 *   k         [B, Hk, n, d] keys (dtype dt).
 *   seq_lens  optional [B] int32 device array of valid lengths (1..n); NULL = n for every row.
 *             Tokens at or after seq_lens[b] are ignored; a block with no valid token gets
 *             mean 0, max norm 0 and the centre of a full block.
 *   b         block (cell) size in tokens.
 *   first_block, num_blocks: compute blocks [first_block, first_block + num_blocks) only;
 *             num_blocks = -1 means "to the end".  first_block = -1 computes, for every batch
 *             row, the one block holding its newest token (position seq_lens[b] - 1): the
 *             decode-time append of the block being filled.
 *   mean_k    [B, Hk, C, d] float32 out:  (1/|c|) * sum_{j in c} k_j
 *   max_norm  [B, Hk, C]    float32 out:  max_{j in c} ||k_j||_2
 *   centre    [B, Hk, C]    float32 out:  mean position of the block's valid tokens
 *   (max_norm and centre may be NULL when not wanted.)
 */
bsa_status bsa_build_block_summaries(const void* k, bsa_dtype dt, int B, int Hk, int n, int d,
                                     int b, const int* seq_lens, int first_block, int num_blocks,
                                     float* mean_k, float* max_norm, float* centre, void* stream);

/*
 * bsa_round_summaries_bf16 -- mean keys for BSA_DECODE_BF16_SUMMARIES: out[i] = bf16(mean_k[i])
 * with round-to-nearest-even (NaN stays NaN, infinities stay infinite).
 *   mean_k    count float32 values (device);  out  count bf16 values (device), 16-byte aligned.
 */
bsa_status bsa_round_summaries_bf16(const float* mean_k, void* out, long long count,
                                    void* stream);

/*
 * bsa_score_blocks -- decode block scores of one query per (batch, query head).
 * The query of row b sits at position pos = seq_lens[b] - 1 (n - 1 if seq_lens is NULL).
 *
 *   s_c = q . kbar_c / sqrt(d)                                   ([SAS] Eq. 3 selector input;
 *       + lambda_h * a_c * erf((pos - p_c) / (2 sigma_h))        [FreeSolo] cell score r_ic)
 *
 *   q         [B, Hq, d] (dtype dt); mean_k/max_norm/centre as written by the summaries call.
 *   lambda_h, sigma_h: optional [Hq] float32 device arrays; both NULL = plain dot score.
 *             max_norm and centre may be NULL when lambda_h is NULL.
 *   prefix_block: 0 = SAS candidates c < pos / b ([SAS] Eq. 4: history blocks only);
 *             P > 0 = FreeSolo candidates, cells lying before floor(pos / P) * P.
 *   scores    [B, Hq, C] float32 out; non-candidate entries are written as -inf.
 *   n_cand    optional [B * Hq] int32 out: number of candidates of each row.
 */
bsa_status bsa_score_blocks(const void* q, bsa_dtype dt, int B, int Hq, int Hk, int n, int d,
                            int b, const int* seq_lens, const float* mean_k,
                            const float* max_norm, const float* centre, const float* lambda_h,
                            const float* sigma_h, int prefix_block, float* scores, int* n_cand,
                            void* stream);

/*
 * bsa_topk_blocks -- I = Top-K(s, K) per row ([SAS] "Background", Eq. 3; worked example step 3).
 *
 *   scores    [rows, ld] float32; only the first C columns take part.
 *   Candidates of a row are its columns c < n_cand(row), where
 *       n_cand(row) = n_cand[row]                        if n_cand != NULL,
 *                   = ((row % units) * q_block) / b      if n_cand == NULL and units > 0
 *                     (prefill: history blocks of the first query of unit row % units),
 *                   = C                                  otherwise.
 *   Order: larger score first; equal scores -> lower index first; NaN ranks below everything
 *   (and -0.0 equals +0.0).  Exactly min(K, n_cand) blocks are selected.
 *   idx       [rows, K] int32 out, selected indices in ascending order, padded with -1.
 *   count     optional [rows] int32 out, min(K, n_cand(row)).
 *   Requires C <= 16384 and K <= 256.
 */
bsa_status bsa_topk_blocks(const float* scores, int rows, int C, int ld, const int* n_cand,
                           int units, int q_block, int b, int K, int* idx, int* count,
                           void* stream);

/*
 * bsa_decode_step -- one whole decode step in a single launch: the composition of
 * bsa_score_blocks, bsa_topk_blocks and bsa_sparse_attn_fwd (nq = 1, no gate), plus the summary
 * append of the block holding each row's newest token ([SAS] "How it works" step 6: score the
 * history blocks, keep Top-K and the current block, exact softmax over their tokens).
 * Selection is per query head; the scores are those bsa_score_blocks writes (same arithmetic),
 * the Top-K the exact order of bsa_topk_blocks.
 *
 *   q [B, Hq, d], k/v [B, Hk, n, d]; query of row b at seq_lens[b] - 1 (n - 1 if NULL).
 *   mean_k, max_norm, centre: block summaries [B, Hk, C, *] of all history blocks (read); with
 *             append != 0 the entry of each row's current block is rewritten from its keys.
 *             max_norm / centre may be NULL unless lambda_h is given.
 *   lambda_h, sigma_h, prefix_block: optional FreeSolo score bias and candidate rule, as in
 *             bsa_score_blocks.
 *   K         history blocks per head, 1..32.
 *   o [B, Hq, d] out, lse [B, Hq] optional out, idx [B, Hq, K] optional out (ascending, -1
 *   padded), count [B, Hq] optional out.
 *   status    optional device int: a bounded wait that runs out writes a nonzero value there.
 * Needs no workspace: the CTAs of one (batch, kv head) group form a thread-block cluster and
 * exchange candidates and partial results through distributed shared memory.
 */
bsa_status bsa_decode_step(const void* q, const void* k, const void* v, bsa_dtype dt, int B,
                           int Hq, int Hk, int n, int d, int b, const int* seq_lens,
                           float* mean_k, float* max_norm, float* centre, int append,
                           const float* lambda_h, const float* sigma_h, int prefix_block, int K,
                           void* o, float* lse, int* idx, int* count, int* status, void* stream);

/*
 * bsa_decode_step_ex -- bsa_decode_step with the variants of bsa_decode_flags: flags = 0 is
 * bsa_decode_step.  With BSA_DECODE_SHARED_SELECTION every head of a group writes the group's
 * selection to idx / count; with BSA_DECODE_BF16_SUMMARIES mean_k is bf16 (read, and with
 * append != 0 the current block's entry rewritten as bf16 of its fp32 mean).  Unknown flag bits
 * are BSA_ERR_ARG; bf16 summaries with dt != BSA_BF16 or b != 64 are BSA_ERR_UNSUPPORTED.
 */
bsa_status bsa_decode_step_ex(const void* q, const void* k, const void* v, bsa_dtype dt, int B,
                              int Hq, int Hk, int n, int d, int b, const int* seq_lens,
                              void* mean_k, float* max_norm, float* centre, int append,
                              const float* lambda_h, const float* sigma_h, int prefix_block, int K,
                              void* o, float* lse, int* idx, int* count, int* status, int flags,
                              void* stream);

/*
 * bsa_decode_step_ws -- bsa_decode_step_ex with a workspace that lets long histories use the
 * whole GPU ([SAS] "Decoding efficiency": at long contexts the block scoring and Top-K dominate
 * the step).  On the 64-token bf16 path with more than 512 history blocks the step runs as two
 * launches: the first scores the history in chunks (about two CTAs per SM) and writes each chunk's
 * Top-K of every selecting head to the workspace; the second merges those lists -- only entries at
 * or above the largest threshold of a full chunk can be among the K largest -- and then forms the
 * union and attends exactly as bsa_decode_step_ex.  Selection, o, lse, idx and count are those of
 * bsa_decode_step_ex (same scores, same order, ties to the lower block).
 *   workspace        device memory, 16-byte aligned, owned by the caller; no initialisation is
 *                    needed and it may be reused once the stream has passed the call.  NULL or
 *                    workspace_bytes = 0: bsa_decode_step_ex (one launch).  With
 *                    BSA_DECODE_HOST_IO it also holds the device copy of q.
 *   workspace_bytes  its size; BSA_ERR_WORKSPACE if nonzero and below
 *                    bsa_decode_step_workspace_bytes().
 */
bsa_status bsa_decode_step_ws(const void* q, const void* k, const void* v, bsa_dtype dt, int B,
                              int Hq, int Hk, int n, int d, int b, const int* seq_lens,
                              void* mean_k, float* max_norm, float* centre, int append,
                              const float* lambda_h, const float* sigma_h, int prefix_block, int K,
                              void* o, float* lse, int* idx, int* count, int* status, int flags,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes bsa_decode_step_ws uses for this shape (dt is a bsa_dtype value): the chunk
 * lists of a long history (none when the step runs as one launch: short histories, other dtypes
 * or block sizes), plus the device copy of q with BSA_DECODE_HOST_IO; 0 for invalid sizes. */
size_t bsa_decode_step_workspace_bytes(int B, int Hq, int Hk, int n, int d, int b, int K,
                                       int flags, int dt);

/*
 * bsa_sparse_attn_fwd -- exact causal softmax over the gathered tokens
 * ([SAS] Eq. 2 and "How it works" step 6; [Monodratic]), optionally with the log-gate of
 * [SAS] Eq. 9.
 *
 * Query i attends the tokens of the selected history blocks of its unit plus the tokens
 * j <= i of its current block cur = i / b (always kept, gate 1):
 *     o_i = sum_j softmax_j(q_i . k_j / sqrt(d) + [gate] log g_m(j)) v_j,  lse_i = log sum exp.
 *
 *   Decode (nq == 1): q [B, Hq, 1, d]; the query of row b sits at seq_lens[b] - 1 (n - 1 if
 *     seq_lens is NULL); idx [B, Hq, K]; scores (gate only) [B, Hq, scores_ld].
 *   Prefill (nq == n, seq_lens must be NULL): queries 0..n-1 in units of q_block consecutive
 *     queries sharing one selection; idx [B, Hq, U, K] with U = ceil(n / q_block);
 *     scores (gate only) [B, Hq, U, scores_ld].  The candidates of unit u are the history
 *     blocks c < (u * q_block) / b of its first query.
 *   idx       selected history blocks (ascending, -1 padded), e.g. from bsa_topk_blocks.
 *   count     optional per-row/per-unit int32 count of valid idx entries; NULL = up to first -1.
 *   gate      BSA_GATE_LOG_SOFTMAX adds log g_m = s_m - LSE(normaliser set) to the logits of
 *             selected history block m; the current block gets 0 ([SAS] Eq. 4).
 *             BSA_GATE_OUTER (prefill only; decode returns BSA_ERR_UNSUPPORTED) multiplies the
 *             value contributions of block m by g_m outside the softmax; lse is then the
 *             log-sum-exp of the ungated logits.
 *   o         [B, Hq, nq, d] out (dtype dt);  lse  optional [B, Hq, nq] float32 out.
 *   workspace device scratch of bsa_sparse_attn_workspace_bytes() bytes, zero-filled before its
 *             first use; each call leaves it reusable (its arrival counters back at zero, also
 *             when a bounded wait ran out).  A wait that ran out writes the status word and the
 *             call then leaves o and lse unwritten; until bsa_workspace_status() reads and clears
 *             that word, later decode calls on the workspace skip their final merge as well.
 *             Calls sharing one workspace must not run concurrently.
 */
bsa_status bsa_sparse_attn_fwd(const void* q, const void* k, const void* v, bsa_dtype dt, int B,
                               int Hq, int Hk, int nq, int n, int d, int b,
                               const int* seq_lens, int q_block, const int* idx,
                               const int* count, int K, bsa_gate_mode gate, bsa_gate_norm norm,
                               const float* scores, int scores_ld, void* o, float* lse,
                               void* workspace, size_t workspace_bytes, void* stream);

size_t bsa_sparse_attn_workspace_bytes(int B, int Hq, int Hk, int nq, int n, int d, int b,
                                       int K);

/*
 * bsa_gate_grad -- closed-form gradient of the loss with respect to the inner gates
 * ([SAS] "Why the four design choices matter", Eq. 5):
 *     dg_m = sum_{i in B_m} (ptilde_i / g_m) * do^T (v_i - o),
 * summed over the queries of the unit that shares gate g_m.  Same layouts as the prefill form of
 * bsa_sparse_attn_fwd; o and lse are that call's gated outputs, dout the upstream gradient.
 *   dg        [B, Hq, U, K] float32 out (0 in padded slots).
 */
/*
 * bsa_gate_grad_outer -- the gradient for the outer gate (BSA_GATE_OUTER forward):
 *     dg_m = sum_{queries i of the unit} sum_{j in B_m} p_ij do_i^T v_j,
 * p the ungated softmax of query i over its token set (lse as written by the outer-gate
 * forward).  Arguments as bsa_gate_grad (o is not read but must be given).
 */
bsa_status bsa_gate_grad_outer(const void* q, const void* k, const void* v, const void* o,
                               const float* lse, const void* dout, bsa_dtype dt, int B, int Hq,
                               int Hk, int n, int d, int b, int q_block, const int* idx,
                               const int* count, int K, bsa_gate_norm norm, const float* scores,
                               int scores_ld, float* dg, void* stream);

bsa_status bsa_gate_grad(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, bsa_dtype dt, int B, int Hq, int Hk,
                         int n, int d, int b, int q_block, const int* idx, const int* count,
                         int K, bsa_gate_norm norm, const float* scores, int scores_ld,
                         float* dg, void* stream);

/*
 * bsa_selector_grad -- gradient of the loss with respect to the selector scores, through the
 * log-softmax gate ([SAS] "Why the four design choices matter": log g_m = s_m - LSE(s) over the
 * normaliser set N).  From dg (bsa_gate_grad):
 *     ds_c = [c selected] g_c dg_c - pi_c * sum_{m selected} g_m dg_m,   pi = softmax over N,
 * pi_c = 0 outside N (N = the row's history blocks c < n_cand for BSA_NORM_ALL_HISTORY, the
 * selected blocks for BSA_NORM_SELECTED).
 *   scores    [rows, scores_ld] float32, the row's history scores in its first n_cand entries.
 *   n_cand    [rows] int32 device array: history blocks of the row (prefill unit u with
 *             q_block = b has u; a decode row at position i has i / b).
 *   idx, count, K   the row's selection as given to the gated forward (K <= 32; count may be
 *             NULL); entries outside [0, n_cand) are ignored.
 *   dg        [rows, K] float32 (per idx slot), as written by bsa_gate_grad.
 *   ds        [rows, ds_ld] float32 out: ds_c for c < n_cand, 0 for c in [n_cand, ds_ld).
 * Rows are the flattened leading dimensions ([B, Hq, U] for prefill units).
 */
bsa_status bsa_selector_grad(const float* scores, int scores_ld, const int* n_cand,
                             const int* idx, const int* count, int K, const float* dg,
                             bsa_gate_norm norm, int rows, float* ds, int ds_ld, void* stream);

/*
 * bsa_fsl_prune -- FS-L pre-query pruning ([FreeSolo] "How it differs", FS-L): before any
 * query arrives, each (batch, head) row keeps its W most recent candidate cells and the P cells
 * of largest maximum key norm among the older ones (lower index on ties, NaN last).
 *   max_norm  [rows, C] float32 (from bsa_build_block_summaries with b = cell).
 *   n_cells   [rows] int32 device array: candidate cells of the row (c < n_cells).
 *   cand      [rows, W + P] int32 out: kept cells ascending, -1 padded; cand_count [rows] out,
 *             min(n_cells, W + P).  Limits: C <= 16384, P <= 256, W + P <= 128.
 */
bsa_status bsa_fsl_prune(const float* max_norm, int rows, int C, const int* n_cells, int W, int P,
                         int* cand, int* cand_count, void* stream);

/*
 * bsa_fsl_select -- FS-L decode selection: the query of each (batch, head) row scores only its
 * kept cells with the FreeSolo cell score
 *     r_c = q . kbar_c / sqrt(d) + lambda_h * a_c * erf((i - p_c) / (2 sigma_h))
 * (plain q . kbar_c / sqrt(d) when lambda_h is NULL) and keeps the K best (ties to the lower cell
 * index, NaN last).
 *   q         [B, H, d] (the decode query of each row); pos [B] int32 device array: its position i.
 *   mean_k [B, H, C, d], max_norm / centre [B, H, C]: cell summaries; lambda_h, sigma_h [H] or NULL.
 *   cand, cand_count, cand_ld  as written by bsa_fsl_prune (cand_ld = W + P <= 128).
 *   idx       [B, H, K] int32 out, ascending, -1 padded; count [B, H] optional out.
 */
bsa_status bsa_fsl_select(const void* q, bsa_dtype dt, int B, int H, int d, const int* pos,
                          const float* mean_k, const float* max_norm, const float* centre, int C,
                          const float* lambda_h, const float* sigma_h, const int* cand,
                          const int* cand_count, int cand_ld, int K, int* idx, int* count,
                          void* stream);

/*
 * bsa_fsl_state_update -- the FS-L state as a fixed-size structure updated in O(P) per new cell
 * ([FreeSolo] "How it differs", FS-L: the prefix is pruned before the query arrives, cost O(N),
 * state of fixed size).  Per row (batch x head) the state is
 *     older       [rows, P] int32: the kept older cells, ascending, -1 padded (in/out),
 *     older_count [rows] int32: how many of them are valid (in/out),
 *     state_cells [rows] int32: the candidate cells the state covers (in/out);
 * a new row starts with older_count = state_cells = 0.  The call grows each row's candidate
 * prefix from state_cells to n_cells[row] (never shrinks it), one cell at a time: the cell leaving
 * the W newest joins the older cells and replaces the lowest-ranked kept one if its maximum key
 * norm ranks higher (larger first, lower index on ties, NaN last), or joins outright while fewer
 * than P are kept.  The result equals bsa_fsl_prune's set for the same n_cells.
 *   max_norm  [rows, C] float32 (bsa_build_block_summaries with b = cell).
 *   n_cells   [rows] int32: candidate cells of the row's current query (cells wholly before its
 *             query block: floor(i / 128) * 128 / cell at query position i).
 *   cand      [rows, W + P] int32 out: the kept cells ascending (older ones, then the W newest),
 *             -1 padded; cand_count [rows] optional out.   Limits: P <= 128, W + P <= 128.
 */
bsa_status bsa_fsl_state_update(const float* max_norm, int rows, int C, const int* n_cells, int W,
                                int P, int* older, int* older_count, int* state_cells, int* cand,
                                int* cand_count, void* stream);

/*
 * bsa_fsl_decode -- FS-L decode output of one query per (batch, head) ([FreeSolo] "How it works"
 * two-branch output, with the long branch's top K taken among the FS-L state's kept cells,
 * "How it differs"):
 *     o = (1 - alpha_h) o_short + alpha_h o_long      (o_short alone when no cell is kept)
 * o_short: softmax of RoPE(q_i) . RoPE(k_j) / sqrt(d) over j in [i - window + 1, i] (base
 * rope_theta, rotate-half pairing, absolute positions) against v_j; o_long: softmax of the raw
 * q_i . k_j / sqrt(d) over the tokens of the K best kept cells by the FreeSolo cell score (as
 * bsa_fsl_select: ties to the lower cell, NaN last).
 *   q [B, H, d], k / v [B, H, n, d] (MHA), pos [B] int32 device: the query position i of each
 *   batch row (its own key at i is in the cache).
 *   mean_k / max_norm / centre: cell summaries [B, H, C, *], C = ceil(n / cell); lambda_h,
 *   sigma_h [H] or NULL (plain dot score); alpha_h [H].
 *   cand, cand_count, cand_ld: the kept cells (bsa_fsl_state_update or bsa_fsl_prune).
 *   o [B, H, d] out; idx [B, H, K] optional out (selected cells ascending, -1 padded); count
 *   [B, H] optional out; status optional device int, set nonzero if a bounded wait ran out.
 *   Limits: K <= 8, window <= 1024, cell <= 128, cand_ld <= 128.  Needs no workspace: four CTAs
 *   per row form a cluster and merge through distributed shared memory.
 */
bsa_status bsa_fsl_decode(const void* q, const void* k, const void* v, bsa_dtype dt, int B, int H,
                          int n, int d, const int* pos, int cell, const float* mean_k,
                          const float* max_norm, const float* centre, const float* lambda_h,
                          const float* sigma_h, const float* alpha_h, const int* cand,
                          const int* cand_count, int cand_ld, int K, int window,
                          float rope_theta, void* o, int* idx, int* count, int* status,
                          void* stream);

/*
 * FS-B ([FreeSolo] "How it differs", FS-B): per (batch, head) two forests of cell summaries --
 * one over every candidate cell, one over the cells of norm at or above the median -- searched by
 * a beam of W_b nodes per level with the node score U_v as an upper bound of the cell scores
 * below v; the cells reached are re-ranked by log-sum-exp over their token keys and the top K
 * are read.  The page gives the node contents (mean key, radius, maximum norm, minimum position)
 * and the search, not the tree shape; this library reads it as follows.  A forest over m cells in
 * position order is the row of perfect binary trees given by the set bits of m (largest first);
 * the "median" forest holds the ceil(m / 2) cells of largest maximum key norm (lower index on
 * ties, NaN last), in position order; a node keeps the mean of its leaves' mean keys, the
 * largest distance of a leaf mean key from it, the largest leaf norm and the smallest leaf
 * centre; U_v = (q . mu_v + ||q|| rho_v) / sqrt(d) + lambda_h a_max erf((i - p_min) / (2 sigma_h)).
 * Level h of the beam holds the W_b best (U as float32, larger first, lower first cell on ties)
 * of the previous beam's children and the root of height h, if any.
 *
 * bsa_fsb_forest_bytes -- bytes of the forest buffer for B x H rows over C cells of head dim d
 * (0 for unsupported sizes: C > 16384, d not in {64, 128}).
 *
 * bsa_fsb_build -- build both forests of every row for its candidate prefix of n_cells[row]
 * cells (cells wholly before the query block: floor(i / 128) * 128 / cell).
 *   mean_k [B, H, C, d], max_norm / centre [B, H, C] float32 (bsa_build_block_summaries, b = cell).
 *   n_cells [B * H] int32 device.   forest: device buffer of bsa_fsb_forest_bytes() bytes, 16-byte
 *   aligned (written; the caller owns it).
 *
 * bsa_fsb_select -- the FS-B selection of one query per (batch, head) over forests built for its
 * candidate prefix.
 *   q [B, H, d], k [B, H, n, d] (the token keys of the re-rank, unrotated), pos [B] int32 device:
 *   query position i (for the erf bias); cell, n: C = ceil(n / cell) must equal the build's C.
 *   lambda_h, sigma_h [H] or NULL (plain dot score in U).   width: W_b (1..16).   K: 1..8.
 *   idx [B, H, K] int32 out (selected cells ascending, -1 padded); count [B, H] optional out;
 *   lse [B, H, K] optional out: the re-rank score of each selected cell.
 * The selected cells feed bsa_fsl_decode as its kept set (cand = idx, cand_count = count, the
 * same K) for the two-branch decode output.
 */
size_t bsa_fsb_forest_bytes(int B, int H, int C, int d);
bsa_status bsa_fsb_build(const float* mean_k, const float* max_norm, const float* centre, int B,
                         int H, int C, int d, const int* n_cells, void* forest,
                         size_t forest_bytes, void* stream);
bsa_status bsa_fsb_select(const void* q, const void* k, bsa_dtype dt, int B, int H, int n, int d,
                          const int* pos, int cell, const void* forest, size_t forest_bytes,
                          const float* lambda_h, const float* sigma_h, int width, int K, int* idx,
                          int* count, float* lse, void* stream);

/*
 * bsa_freesolo_select -- per-query cell selection of the FreeSolo long branch (prefill),
 * [FreeSolo] "How it works": for the query at position i of head h the candidates are the cells
 * c lying wholly before the start of its query block, (c + 1) * cell <= floor(i / q_block) *
 * q_block, scored by
 *     r_ic = q_i . kbar_c / sqrt(d) + lambda_h * a_c * erf((i - p_c) / (2 sigma_h)),
 * and the K best cells are kept (ties to the lower index, NaN last).
 *   q         [B, H, n, d] (MHA: one kv head per query head).
 *   mean_k, max_norm, centre: cell summaries [B, H, C, d] / [B, H, C] / [B, H, C] with
 *             C = ceil(n / cell), from bsa_build_block_summaries with b = cell.
 *   lambda_h, sigma_h: [H] float32 device arrays.
 *   idx       [B, H, n, K] int32 out, ascending, -1 padded; count optional [B, H, n] out.
 *   K <= 8.
 *   workspace device scratch of bsa_freesolo_select_workspace_bytes() bytes, its first int zeroed
 *             before first use (the status word: a bounded wait that runs out writes a nonzero
 *             value there; bsa_workspace_status reads and clears it).  Required (else
 *             BSA_ERR_WORKSPACE) for the tensor-core form: bf16, d in {64, 128}, q_block = 128;
 *             it then holds the mean keys split into bf16 high and low parts.  Other forms take
 *             no workspace (size 0; the pointer may be NULL).
 */
bsa_status bsa_freesolo_select(const void* q, bsa_dtype dt, int B, int H, int n, int d,
                               int cell, int q_block, const float* mean_k, const float* max_norm,
                               const float* centre, const float* lambda_h, const float* sigma_h,
                               int K, int* idx, int* count, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Workspace bytes bsa_freesolo_select needs for these arguments (0: none). */
size_t bsa_freesolo_select_workspace_bytes(bsa_dtype dt, int B, int H, int n, int d, int cell,
                                           int q_block, int K);

/*
 * bsa_freesolo_attn -- FreeSolo two-branch prefill output ([FreeSolo] "How it works"):
 *     o_i = (1 - alpha_h) o_short_i + alpha_h o_long_i      (o_short_i alone when count = 0)
 * o_short: softmax attention of RoPE(q_i) over RoPE(k_j), j in [i - window + 1, i] (RoPE base
 * rope_theta, rotate-half pairing t <-> t + d/2, absolute positions).
 * o_long: softmax attention of the raw q_i over the raw tokens of its selected cells (NoPE).
 *   idx/count as written by bsa_freesolo_select (cells not wholly at or before i are ignored).
 *   alpha_h   [H] float32 device array.   o  [B, H, n, d] out (dtype dt).
 *   workspace device scratch of bsa_freesolo_workspace_bytes() bytes, its first int zeroed before
 *             first use (the status word of the bounded waits, read and cleared by
 *             bsa_workspace_status).  It holds the rotated keys; for bf16 also the rotated queries
 *             and the long branch's scratch.  With bf16, d in {64, 128}, cell in {16, 32, 64} and
 *             K <= 8 the long branch is regrouped by cell: each attended (query, cell) pair gets a
 *             place in its cell's list, tiles of 128 such queries attend to the cell's tokens on
 *             the tensor cores, and an unnormalised output row with its (max, sum) per pair
 *             (B * H * n * K * (d + 2) floats) is merged per query at the end.  With other cell
 *             sizes (powers of two up to 64) the scratch holds, per 64-query unit, the sorted
 *             union of the 64-key blocks holding the unit's selected cells.  A slot is attended
 *             once: a cell repeated within a query's slots counts once.
 */
bsa_status bsa_freesolo_attn(const void* q, const void* k, const void* v, bsa_dtype dt, int B,
                             int H, int n, int d, int cell, int window, float rope_theta,
                             const float* alpha_h, const int* idx, const int* count, int K,
                             void* o, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes bsa_freesolo_attn needs for these arguments (0 for invalid sizes). */
size_t bsa_freesolo_workspace_bytes(bsa_dtype dt, int B, int H, int n, int d, int cell, int K);

/*
 * bsa_sparse_attn_decode_noalloc -- the decode form of bsa_sparse_attn_fwd (nq == 1) for callers
 * that cannot provide device memory: an engine that plans all device memory ahead and forbids
 * any other allocation, or a plugin whose host framework owns the allocator and gives it none.
 * The pages have no counterpart to this call; it exists for those callers only.
 *
 * Arguments, layouts and results are those of bsa_sparse_attn_fwd with nq = 1, minus the
 * workspace.  Instead of a workspace it uses one fixed 4 MiB device array inside the library,
 * which every GPU that loads the library keeps until the process exits.  Nothing is allocated:
 * no cudaMalloc, cudaFree or allocating library routine is called.
 *  - Limit: a problem whose split-K scratch (see bsa_sparse_attn_workspace_bytes with nq = 1)
 *    exceeds 4 MiB is rejected with BSA_ERR_WORKSPACE, before any launch.
 *  - The first call on a device looks up the array's device address (once per device, with the
 *    device current); make that first call before any CUDA stream capture.
 *  - Every call shares the one array, which keeps the previous call's contents; each call zeroes
 *    the parts that must start at zero.  Calls that overlap on the GPU (other streams, other
 *    threads, concurrent graph launches) race on the array and give wrong results.
 *  - A bounded wait that runs out writes the array's status word; o and lse are then left
 *    unwritten.  bsa_noalloc_status() reads and clears that word (the next call on the device
 *    also clears it when it starts).
 */
bsa_status bsa_sparse_attn_decode_noalloc(const void* q, const void* k, const void* v,
                                          bsa_dtype dt, int B, int Hq, int Hk, int n, int d,
                                          int b, const int* seq_lens, const int* idx,
                                          const int* count, int K, bsa_gate_mode gate,
                                          bsa_gate_norm norm, const float* scores, int scores_ld,
                                          void* o, float* lse, void* stream);

/* Status of the last bsa_sparse_attn_decode_noalloc call on the current device: reads and clears
 * the status word of the library's fixed array (synchronises the stream; no counterpart in the
 * pages).  Returns BSA_OK, BSA_ERR_TIMEOUT (a bounded wait of that call ran out; its o and lse
 * were not written) or BSA_ERR_CUDA. */
bsa_status bsa_noalloc_status(void* stream);

/* Read and clear the status word a bounded device wait writes into a workspace
 * (synchronises the stream).  Returns BSA_OK or BSA_ERR_TIMEOUT (or BSA_ERR_CUDA). */
bsa_status bsa_workspace_status(void* workspace, void* stream);

/* Failure-path self-test (no counterpart in the pages): one thread waits on an mbarrier that is
 * never completed, gives up after `polls` polls and writes the timeout into the status word of
 * `workspace` (>= 256 bytes, device).  A following bsa_workspace_status() returns
 * BSA_ERR_TIMEOUT; the CUDA context stays usable. */
bsa_status bsa_selftest_bounded_wait(void* workspace, int polls, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H_ */
