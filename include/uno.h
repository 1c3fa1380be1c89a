/*
 * uno.h -- C ABI of the B200 (sm_100a) hot path of one Psi-Spec decode step.
 *
 * Source of the operations: "Unlocking Lossless Speedups in LLMs via Discrete
 * Diffusion" (Uno). The picx.dev summary page, "Methodology / Architecture",
 * and the paperglide reader page, "The Uno Framework", define the dual-pathway
 * linear; the reader's "The Psi-Speculative Sampler" and "Sampler Extensions"
 * (linear sampler) define the verification step, with the standard speculative
 * rejection-sampling rule the pages cite (Leviathan et al. 2023; Chen et al.
 * 2023). The same sections, with the worked (B, K, V) = (3, 2, 2) example and
 * the summary page's "Psi-Speculative Sampler", define drafting and the tree
 * sampler. Each entry point below names its passage.
 *
 * Conventions shared by every entry point:
 *  - Every buffer argument is a DEVICE pointer owned by the caller. The library
 *    never allocates, frees or keeps a reference to caller memory after a call.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and never synchronise the host. The return value reports argument
 *    errors (checked on the host before anything is launched) and launch errors.
 *  - Matrices are dense and row-major with no padding between rows.
 *  - Base pointers of logits, activations, weights and outputs must be 16-byte
 *    aligned (cudaMalloc and PyTorch allocations are 256-byte aligned); the
 *    draft and tree samplers need only element alignment. Workspaces must be
 *    16-byte aligned (the tree draft's 256-byte aligned).
 *  - On an error nothing is launched and no output is written.
 */
#ifndef UNO_H_
#define UNO_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of logits, activations and weights. */
typedef enum {
  UNO_BF16 = 0, /* bfloat16 storage, float32 arithmetic                       */
  UNO_F32 = 1   /* float32 storage; the GEMM runs on the TF32 tensor-core path */
} uno_dtype;

/* Status codes (negative = error). */
typedef enum {
  UNO_OK = 0,
  UNO_ERR_NULL = -1,      /* a required pointer is NULL                         */
  UNO_ERR_SIZE = -2,      /* a size is negative or beyond a documented limit    */
  UNO_ERR_ALIGN = -3,     /* a pointer or a row stride breaks the 16-byte rule  */
  UNO_ERR_DTYPE = -4,     /* dtype is not a uno_dtype value                     */
  UNO_ERR_WORKSPACE = -5, /* workspace is NULL or smaller than required         */
  UNO_ERR_CUDA = -6,      /* a CUDA runtime/driver call or a launch failed      */
  UNO_ERR_DEVICE = -7     /* the current device is not an sm_100 GPU            */
} uno_status;

/* Human-readable name of a status code. Never returns NULL. */
const char* uno_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
int uno_version(void);

/* ------------------------------------------------------------------------ *
 * Block verifier (linear Psi-Spec sampler, verification step)
 *
 * For each sequence b in [0, B) with drafted ids x_0..x_{K-1}:
 *   p_i = softmax(p_logits[b, i, :]), q_i = softmax(q_logits[b, i, :])
 *   (temperature 1, float32 arithmetic on device).
 *   u_i, u'_i = uniforms of Philox4x32-10 (Salmon et al., SC'11) with
 *   key = (seed lo32, seed hi32) and counter = (b, i, step lo32, step hi32);
 *   u_i = (word0 >> 8) * 2^-24, u'_i = (word1 >> 8) * 2^-24.
 *   accept_i  <=>  u_i * q_i(x_i) < p_i(x_i)
 *   n = index of the first rejected position, or K when all are accepted.
 *   n < K : y ~ max(0, p_n - q_n) (normalised; p_n if that is all zero)
 *   n = K : y ~ p_K (the bonus row).
 *   y is drawn by inverse CDF in index order: the smallest v whose running
 *   weight sum exceeds u'_n times the total.
 *   out_tokens[b] = (x_0, ..., x_{n-1}, y, -1, ..., -1); accepted_len[b] = n.
 * A draft id outside [0, V) in sequence b is reported on the device:
 * accepted_len[b] = -1 and out_tokens[b, :] = -1 (the call still returns
 * UNO_OK; the caller reads accepted_len to see it).
 * ------------------------------------------------------------------------ */

/* Workspace bytes uno_verify_block needs for (B, K, V, dtype); 0 on bad sizes. */
size_t uno_verify_workspace_bytes(int B, int K, int V, int dtype);

/*
 * p_logits      [B, K+1, V] dtype  AR (verifier) logits; row K is the bonus row
 * q_logits      [B, K,   V] dtype  draft logits
 * draft_tokens  [B, K]      int32  drafted ids
 * B             0 <= B <= 2^20     (B = 0 launches nothing and returns UNO_OK)
 * K             1 <= K <= 256      drafted positions per sequence
 * V             1 <= V <= 2^28     vocabulary size (any value; no alignment rule)
 * seed, step    Philox key and counter words (see above)
 * out_tokens    [B, K+1]    int32  emitted tokens, -1 padded        (required)
 * accepted_len  [B]         int32  accepted draft count n (or -1)   (required)
 * p_at_draft    [B, K]      float  p_i(x_i)                         (optional, NULL)
 * q_at_draft    [B, K]      float  q_i(x_i)                         (optional, NULL)
 * row_lse       [B, 2K+1]   float  log-sum-exp of every row: p rows 0..K,
 *                                  then q rows 0..K-1               (optional, NULL)
 * workspace     device scratch of at least uno_verify_workspace_bytes(B,K,V,dtype)
 *               bytes, 16-byte aligned; its contents on entry do not matter.
 *               Two calls that share a workspace must be ordered on one stream.
 * stream        cudaStream_t
 * Returns UNO_OK or a negative uno_status.
 */
int uno_verify_block(const void* p_logits, const void* q_logits, const int32_t* draft_tokens,
                     int B, int K, int V, int dtype, uint64_t seed, uint64_t step,
                     int32_t* out_tokens, int32_t* accepted_len, float* p_at_draft,
                     float* q_at_draft, float* row_lse, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * uno_verify_block_noalloc -- the same verification, with no workspace
 * argument and no allocation. The paper has no counterpart to this entry
 * point; it exists for callers that cannot allocate device memory when they
 * call, such as a plug-in whose host engine owns all device memory through its
 * own pool, a latency-critical path that cannot afford cudaMalloc (it may
 * synchronise the device), or a caller from another language with no device
 * allocator at hand.
 *
 * Scratch: one fixed 4 MiB array in the library's device memory. It is
 * reserved on a device once the library's module is loaded there -- with
 * CUDA's default lazy module loading, at this entry point's first call on that
 * device -- and stays reserved until the process exits. Calls whose
 * uno_verify_workspace_bytes(B, K, V, dtype) exceeds 4 MiB are rejected with
 * UNO_ERR_SIZE (for example B = 64, K = 16, V = 151936 needs about 51 KB).
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * The array keeps the previous call's contents; the verifier does not depend
 * on them (it rewrites whatever it reads), so nothing is cleared. All calls
 * on a device share the array, so calls that may overlap on the GPU
 * (different streams, or different host threads without ordering) race and
 * corrupt each other's results: order them on one stream.
 * The library calls no cudaMalloc, cudaFree or other allocating routine here.
 * Arguments, outputs and errors are those of uno_verify_block.
 */
int uno_verify_block_noalloc(const void* p_logits, const void* q_logits,
                             const int32_t* draft_tokens, int B, int K, int V, int dtype,
                             uint64_t seed, uint64_t step, int32_t* out_tokens,
                             int32_t* accepted_len, float* p_at_draft, float* q_at_draft,
                             float* row_lse, void* stream);

/* ------------------------------------------------------------------------ *
 * Dual-pathway linear (one pass over the frozen weight W)
 *
 *   y_ar    = x W^T                       (verification pathway, theta_AR)
 *   T       = scale * x A^T               (LoRA down projection, scale = alpha/r)
 *   y_draft = y_ar + T Bm^T               (drafting pathway, theta_AR + theta_Delta)
 *
 * Arithmetic: tcgen05 tensor cores, float32 accumulation. With UNO_BF16
 * operands T is rounded to bfloat16 before the adapter product (it is a
 * bfloat16 tensor-core operand); with UNO_F32 operands every product runs in
 * TF32 and T stays float32. Outputs are stored in dtype, rounded to nearest.
 * ------------------------------------------------------------------------ */

/* Workspace bytes uno_dualpath_linear needs; 0 on bad sizes. */
size_t uno_dualpath_workspace_bytes(int M, int d_in, int d_out, int r, int dtype);

/*
 * x        [M, d_in]      dtype  activations
 * W        [d_out, d_in]  dtype  frozen AR weight (nn.Linear layout)
 * A        [r, d_in]      dtype  LoRA down weight
 * Bm       [d_out, r]     dtype  LoRA up weight
 * scale    alpha / r
 * y_ar     [M, d_out]     dtype  output, or NULL to skip it
 * y_draft  [M, d_out]     dtype  output, or NULL to skip it (and the adapter)
 * M        0 <= M <= 2^24 rows (M = 0 launches nothing)
 * d_in     >= 1, multiple of 8 (bf16) / 4 (f32) so rows are 16-byte strided
 * d_out    >= 1, multiple of 8 (bf16) / 4 (f32)
 * r        1 <= r <= 256, multiple of 8 (bf16) / 4 (f32)
 * workspace  device scratch of at least uno_dualpath_workspace_bytes(...) bytes,
 *            16-byte aligned, contents irrelevant on entry. Two calls that
 *            share a workspace must be ordered on one stream.
 * Returns UNO_OK or a negative uno_status. At least one of y_ar / y_draft
 * must be non-NULL.
 *
 * Schedule: one persistent launch; when its last round of tiles would leave
 * most SMs idle, each tile of that round is accumulated as 3 or 4 K-pieces
 * whose float32 partials are added before the epilogue. Results are
 * deterministic for a given device and call; the split depends on the SM
 * count, so the last bits of those tiles can differ between devices.
 */
int uno_dualpath_linear(const void* x, const void* W, const void* A, const void* Bm,
                        float scale, void* y_ar, void* y_draft, int M, int d_in, int d_out,
                        int r, int dtype, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * Grouped dual-pathway linear: n (1..4) projections of the same activations x
 * in one launch, e.g. the q, k and v projections of a layer, or gate and up.
 * The summary page's "Methodology / Architecture" adds the LoRA to every
 * attention and MLP projection; projections that read the same x share one
 * launch, so small ones (k, v) fill the GPU together with a large one.
 *
 * Projection g has its own W[g] [d_out[g], d_in], A[g] [r, d_in],
 * Bm[g] [d_out[g], r], scale[g], y_ar[g] and y_draft[g] [M, d_out[g]]; M,
 * d_in, r and dtype are shared, with the limits of uno_dualpath_linear.
 * Either every y_draft[g] is NULL (no adapter anywhere) or none is; y_ar[g]
 * may be NULL per projection. gate [M] (or NULL) is the per-row adapter gate of
 * uno_dualpath_linear_gated, shared by all projections. The results equal n
 * separate single calls bit for bit, except when a last, partial round of
 * tiles is split along K (see uno_dualpath_linear): the grouped launch may
 * split other tiles than the single calls, and those tiles then differ in
 * float32 summation order only.
 * workspace  at least uno_dualpath_grouped_workspace_bytes(...) bytes, 16-byte
 *            aligned, contents irrelevant on entry (n single-call workspaces
 *            back to back).
 * The pointer arrays are host arrays, read during the call only.
 * Returns UNO_OK or a negative uno_status (UNO_ERR_SIZE for n outside 1..4).
 */
size_t uno_dualpath_grouped_workspace_bytes(int n, int M, int d_in, const int* d_out, int r,
                                            int dtype);
int uno_dualpath_linear_grouped(int n, const void* x, const void* const* W,
                                const void* const* A, const void* const* Bm,
                                const float* scale, const uint8_t* gate, void* const* y_ar,
                                void* const* y_draft, int M, int d_in, const int* d_out,
                                int r, int dtype, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * Gated dual-pathway linear. gate [M] uint8 on the device (or NULL: every row
 * on): a row with gate 0 gets no adapter, so its y_draft equals its y_ar bit
 * for bit; a row with a nonzero gate is the ungated result. This is the gated
 * LoRA of the reader page, "The Psi-Speculative Sampler": when a draft block
 * is computed, token 1 uses the AR weights alone and tokens 2..B the gated
 * LoRA-augmented weights ("Supplementary Details": the first position's
 * clean-token distribution uses theta_AR only), so one pass serves the block.
 * The grouped call above takes the same gate for all its projections.
 * Everything else is as for uno_dualpath_linear.
 */
int uno_dualpath_linear_gated(const void* x, const void* W, const void* A, const void* Bm,
                              float scale, const uint8_t* gate, void* y_ar, void* y_draft,
                              int M, int d_in, int d_out, int r, int dtype, void* workspace,
                              size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------ *
 * LM head with the verifier's row statistics, and the verifier that uses them
 *
 * The last dual-path linear of a decode step is the LM head: y_ar holds the
 * verifier's logits p, y_draft the draft logits q (reader page, "The Uno
 * Framework": drafting uses theta_AR + theta_Delta, verification theta_AR
 * alone). uno_dualpath_linear_stats is uno_dualpath_linear_gated (same
 * arguments, same outputs bit for bit) that also writes, for every output
 * row, the softmax partials of the values it stored, each over a part of the
 * row: m = max(value) * log2(e) and z = sum of 2^(value * log2(e) - m)
 * (float pairs; a part with no values is (-inf, 0)). uno_verify_block_head then verifies without reading every
 * logit again: it merges those partials instead of streaming the rows and
 * reads only the logits at the drafted ids and the one p (and q) row that
 * the final draw needs per sequence.
 *
 * uno_dualpath_stats_tiles(M, d_out) = T, the partials per row: for M > 256
 *   (CTA pairs, one per 256-column tile) ceil(d_out / 256), the partial of
 *   tile t covering columns [256 t, 256 t + 256); for 1 <= M <= 256 (swapped
 *   operands, one partial per CTA, which accumulates over every column tile
 *   it computes) 148, slots of CTAs the launch does not start holding
 *   (-inf, 0); 0 when M < 1 or d_out < 1.
 * uno_dualpath_linear_stats: as uno_dualpath_linear_gated, plus
 *   stats_ar     [M, T, 2] f32 out (T = uno_dualpath_stats_tiles), or null;
 *                needs y_ar
 *   stats_draft  [M, T, 2] f32 out, or null; needs y_draft
 *   A row's logsumexp is the merge of its T partials, whatever the layout.
 * uno_verify_block_head: as uno_verify_block, with
 *   y_ar         [B, K+1, V] dtype: p, row i of sequence b = LM-head row
 *                b * (K+1) + i
 *   y_draft      [B, K+1, V] dtype: q_i of sequence b = row b * (K+1) + i for
 *                i < K (row K, the bonus position, is not read)
 *   stats_ar, stats_draft  the partials of those rows, stats_tiles per row
 *   The accept tests, the draw and every output follow uno_verify_block;
 *   the row statistics are summed in tile order instead of slab order, so
 *   probabilities can differ from uno_verify_block's by float32 rounding.
 *   Workspace: uno_verify_workspace_bytes(B, K, V, dtype).
 * ------------------------------------------------------------------------ */
int uno_dualpath_stats_tiles(int M, int d_out);
int uno_dualpath_linear_stats(const void* x, const void* W, const void* A, const void* Bm,
                              float scale, const uint8_t* gate, void* y_ar, void* y_draft,
                              float* stats_ar, float* stats_draft, int M, int d_in, int d_out,
                              int r, int dtype, void* workspace, size_t workspace_bytes,
                              void* stream);
int uno_verify_block_head(const void* y_ar, const void* y_draft, const float* stats_ar,
                          const float* stats_draft, int stats_tiles, const int32_t* draft_tokens,
                          int B, int K, int V, int dtype, uint64_t seed, uint64_t step,
                          int32_t* out_tokens, int32_t* accepted_len, float* p_at_draft,
                          float* q_at_draft, float* row_lse, void* workspace,
                          size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------ *
 * Drafting a block (linear Psi-Spec sampler)
 *
 * Reader page, "The Psi-Speculative Sampler": the block's candidates are
 * sampled from the joint proposal; the linear sampler draws every position in
 * parallel from its own marginal. Here draft_tokens[b][i] ~ softmax(q[b][i])
 * (temperature 1) by the inverse CDF over exp(q - max) in index order: the
 * smallest v with C_v > u * C_{V-1}. The uniform u is word 2 of the Philox
 * block of counter (b, i, step lo, step hi), key (seed lo, seed hi); words 0
 * and 1 of the same block are the accept test and the resample of
 * uno_verify_block, so one (seed, step) gives independent uniforms to both.
 *
 * q_logits      [B, K, V] dtype (bf16 or f32), rows need not be aligned
 * draft_tokens  [B, K] int32 output; -1 for a row with no finite logit
 * Limits: 0 <= B <= 2^20, 1 <= K <= 256, 1 <= V <= 2^28. No workspace.
 * Asynchronous on `stream`; returns UNO_OK or a negative uno_status.
 * ------------------------------------------------------------------------ */
int uno_sample_drafts(const void* q_logits, int B, int K, int V, int dtype, uint64_t seed,
                      uint64_t step, int32_t* draft_tokens, void* stream);

/* The same draws from logits laid out in blocks of block_rows >= K rows per
 * sequence ([B, block_rows, V], for example the LM head's draft-pathway output
 * of K + 1 rows per block): draft_tokens[b][i] ~ softmax(logits[b][i]) for
 * i < K; rows K..block_rows-1 of each block are not read. With block_rows = K
 * this is uno_sample_drafts. Limits as above, and K <= block_rows <= 4096,
 * B * block_rows <= 2^28 (else UNO_ERR_SIZE). */
int uno_sample_drafts_blocks(const void* logits, int B, int K, int block_rows, int V, int dtype,
                             uint64_t seed, uint64_t step, int32_t* draft_tokens, void* stream);

/* ------------------------------------------------------------------------ *
 * Tree sampler
 *
 * Reader page, "The Psi-Speculative Sampler" (worked example with
 * (B, K, V) = (3, 2, 2): the K^(B-1) candidate sequences of the positions
 * after the block's first token are ranked by joint log-probability, the top V
 * are kept, every prefix is verified by the frozen AR model and the longest
 * valid one is accepted) and "Sampler Extensions"; summary page,
 * "Psi-Speculative Sampler" (top-K at each position). The pages' (B, K, V)
 * are depth D = B - 1, top_k and budget here.
 *
 * uno_tree_nodes(D, budget) = 1 + D * budget: the node rows N of a tree
 * (root + one node per position of every kept sequence, at most); 0 when D
 * or budget is out of range.
 *
 * uno_tree_draft:
 *   q_logits     [B, D, V] dtype: draft logits of positions 1..D
 *   topk_ids     [B, D, top_k] int32 out: per position the top_k ids by
 *                logit, larger first, ties to the smaller id; -inf logits
 *                are never candidates (-1 fills missing slots)
 *   topk_logq    [B, D, top_k] f32 out: log softmax(q)(id) (-inf when -1)
 *   node_token   [B, N] int32 out: token of each node (root, padding: -1)
 *   node_parent  [B, N] int32 out: parent node (root, padding: -1)
 *   node_depth   [B, N] int32 out: 0 root, j for a prefix of length j
 *                (padding: -1)
 *   n_nodes      [B] int32 out
 *   workspace    device scratch of at least
 *                uno_tree_draft_workspace_bytes(B, D, V, top_k) bytes,
 *                256-byte aligned (each row's logits are split over several
 *                CTAs at small B; their partial lists meet there); contents
 *                on entry do not matter
 *   The kept set is the budget best of the top_k^D sequences by the sum of
 *   topk_logq over positions (float32, position order), ties by the
 *   sequence of ranks (lexicographic, smaller first); the nodes are their
 *   distinct prefixes, by depth, then by rank sequence.
 *   Limits: 0 <= B <= 2^20, 1 <= D <= 16, 1 <= top_k <= 16,
 *   1 <= budget <= 64, 1 <= V <= 2^28.
 *
 * uno_tree_verify: the lossless walk of each sequence's tree.
 *   p_logits     [B, N, V] dtype: AR logits after each node's prefix (rows
 *                n >= n_nodes[b] are not read)
 *   node_*, n_nodes  the tree (as uno_tree_draft writes it)
 *   node_draw    [B, N] int32 out: the draw of every node in use (-1 for
 *                rows not in use and rows with no finite logit)
 *   out_tokens   [B, D+1] int32 out: accepted tree tokens, then the token
 *                drawn where the walk stopped; -1 padding
 *   accepted_len [B] int32 out: accepted tree tokens (0..D), -1 when a row
 *                on the walk has no finite logit (then all tokens are -1)
 *   At node n (depth j) the draw is the inverse CDF of softmax(p[b][n]) at
 *   the uniform of Philox word 1 of the block (b, j, step) under (seed); the
 *   walk follows it while it is the token of a child of the current node and
 *   emits it either way, so every emitted token is an exact draw of the AR
 *   distribution given the tokens before it.
 *
 * uno_tree_verify takes no workspace. Both are asynchronous on `stream` and
 * return UNO_OK or a negative uno_status (UNO_ERR_WORKSPACE for a missing,
 * short or misaligned draft workspace).
 * ------------------------------------------------------------------------ */
int uno_tree_nodes(int depth, int budget);
size_t uno_tree_draft_workspace_bytes(int B, int D, int V, int top_k);
int uno_tree_draft(const void* q_logits, int B, int D, int V, int dtype, int top_k, int budget,
                   int32_t* topk_ids, float* topk_logq, int32_t* node_token,
                   int32_t* node_parent, int32_t* node_depth, int32_t* n_nodes, void* workspace,
                   size_t workspace_bytes, void* stream);
int uno_tree_verify(const void* p_logits, const int32_t* node_token, const int32_t* node_parent,
                    const int32_t* node_depth, const int32_t* n_nodes, int B, int D, int budget,
                    int V, int dtype, uint64_t seed, uint64_t step, int32_t* node_draw,
                    int32_t* out_tokens, int32_t* accepted_len, void* stream);

/* ------------------------------------------------------------------------ *
 * Device fault flags
 *
 * Every wait inside the kernels is bounded in time. A wait that gives up
 * (which correct code never does) sets a bit here, abandons its work and lets
 * the kernel exit instead of hanging the GPU: bit 0 TMA producer, bit 1 MMA
 * issuer, bit 2 epilogue. This call synchronises the device, writes the
 * current flags to *flags and clears them when `clear` is non-zero.
 * ------------------------------------------------------------------------ */
int uno_device_fault_flags(int clear, unsigned int* flags);

/* Failure-path test hook of the dual-path linear (for tests, not for use):
 * the calls that follow in this process bound every wait of the GEMM by
 * wait_ns nanoseconds instead of one second, and, when t_flag_skew is non-zero,
 * make its TMA producers wait for a T-tile flag value that no tile writes (the
 * call's value plus the skew), so that those waits run out: the kernel then
 * sets fault bits, abandons its work (outputs undefined) and exits normally,
 * and the context stays usable. (0, 0) restores normal operation. Always
 * returns UNO_OK. */
int uno_dualpath_test_hooks(uint64_t wait_ns, uint32_t t_flag_skew);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* UNO_H_ */
