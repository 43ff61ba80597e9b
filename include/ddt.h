/*
 * ddt.h -- C ABI of libddt.so: the DDTree verification round on B200 (sm_100a).
 *
 * The round (DDTree page, a curated summary of the authors' announcement of
 * "Diffusion Draft Tree"; section 運作流程 "workflow", steps 1-4):
 *   1. ddt_topk        per-position softmax normaliser and top-k candidates of
 *                      the drafter's marginals q_i (step 1);
 *      ddt_topk_noalloc  the same without a caller workspace;
 *   2. ddt_build_tree  the B most probable prefixes of the factorised draft
 *                      (step 2; section 理論基礎 "theory", Propositions 1-2),
 *                      compiled to token / parent / depth / position /
 *                      ancestor-mask tensors (step 3);
 *   3. ddt_tree_attn   one attention pass of every tree row against the KV
 *                      cache and its own ancestors (step 3; section 核心創新
 *                      "core innovation", ancestor-only attention mask);
 *   4. ddt_tree_walk   the greedy walk over the target's logits that accepts
 *                      matching children and returns the bonus token (step 4);
 *      ddt_tree_walk_sample  the same walk under temperature sampling;
 *      ddt_lm_head_walk      the greedy walk straight from the target's
 *                            hidden states (LM head on the tensor cores);
 *   5. ddt_kv_commit   appends the root's and the accepted rows' K/V to the
 *                      committed context for the next round.
 *   ddt_plan_budget    splits a batch's node budget between its sequences
 *                      (between a first and a second ddt_build_tree).
 *
 * Conventions shared by every entry point:
 *   - Every tensor pointer is a DEVICE pointer owned by the caller.  The
 *     library allocates no device memory; scratch comes from a caller-owned
 *     workspace sized by the matching *_workspace_size() function.
 *   - Every workspace starts with a counter region of DDT_WS_COUNTER_BYTES
 *     that must be zero-filled before the workspace's first use; every call
 *     that returns DDT_OK leaves it zero again when its kernels finish.  The
 *     rest of a workspace may hold anything.  One workspace can therefore
 *     serve calls of any stage and shape one after another on one stream;
 *     calls that share a workspace must not overlap on the GPU.
 *   - Calls are asynchronous on `stream` and perform no host synchronisation,
 *     so they can be captured into a CUDA graph.
 *   - Kernels are launched with programmatic stream serialization: a call's
 *     kernel may be scheduled while the previous kernel on the stream is
 *     still running, but it waits for that kernel to complete (and its
 *     writes to be visible) before it reads any input; no input is read
 *     early.  Launched after a non-kernel operation, it runs as usual.
 *   - Arguments are validated on the host before any launch: an invalid
 *     argument returns DDT_ERR_INVALID_ARG / DDT_ERR_UNSUPPORTED /
 *     DDT_ERR_WORKSPACE and launches nothing.  Problems only visible on the
 *     device (e.g. a per-sequence budget above the maximum) are clamped and
 *     reported through the optional `dev_status` word (0 = fine, otherwise a
 *     ddt_status code); the word is only ever raised, never cleared.
 *   - A launch failure returns DDT_ERR_CUDA.  No C++ exception crosses the ABI.
 *   - "bf16" means IEEE bfloat16 stored in 2 bytes; all layouts are dense,
 *     row-major, innermost index last.
 */
#ifndef DDT_H
#define DDT_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ddt_status {
  DDT_OK = 0,
  DDT_ERR_INVALID_ARG = 1, /* null pointer, negative size, inconsistent shapes */
  DDT_ERR_UNSUPPORTED = 2, /* valid but outside the implemented range (dtype, d, k, B, L) */
  DDT_ERR_WORKSPACE = 3,   /* workspace missing, misaligned (256 B) or too small */
  DDT_ERR_CUDA = 4,        /* a CUDA call failed; see cudaGetLastError() */
  DDT_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up (reported via dev_status) */
} ddt_status;

typedef enum ddt_dtype { DDT_BF16 = 0, DDT_F32 = 1 } ddt_dtype;

/* Size of the counter region at the start of every workspace. */
#define DDT_WS_COUNTER_BYTES (256u << 10)

/* Implementation limits. */
#define DDT_TOPK_K_MAX 32     /* candidates per position */
#define DDT_TREE_L_MAX 64     /* draft positions (tree depth) */
#define DDT_TREE_B_MAX 1023   /* draft nodes; rows N = B + 1 <= 1024 */

/* Human-readable name of a status code (static storage; never NULL). */
const char* ddt_status_string(ddt_status s);

/* Number of 32-bit mask words per tree row: ceil(n_max / 32). */
int ddt_mask_words(int n_max);

/* Test hook for the timeout path.  The tensor-core kernels (ddt_tree_attn on
 * its tensor-core paths, ddt_lm_head_walk) bound every wait on an on-chip
 * barrier; a wait that runs out raises DDT_ERR_TIMEOUT in dev_status, after
 * which the kernel lets its copies and MMAs in flight complete, frees its
 * tensor memory and returns, leaving the context usable.  By default a wait
 * gives up after about one second (2e9 clock cycles).  This call sets the
 * bound, in clock cycles, for every later launch in the process (cycles <= 0
 * restores the default) and returns the previous setting (0 = default).
 * A bound of a few cycles makes the waits run out on purpose.  It is not
 * synchronised with launches on other host threads. */
long long ddt_debug_set_wait_limit(long long cycles);

/* Tuning and test hook: which tensor-core attention kernel ddt_tree_attn
 * uses.  0 (default): the planner chooses; 1: the one-query-tile kernel
 * only; 2: the two-query-tile kernel wherever a kv head has at least two
 * query tiles (the one-tile kernel elsewhere).  The KV split is planned for
 * the chosen kernel as usual, and ddt_tree_attn_plan and
 * ddt_tree_attn_workspace_size follow the same choice.  Applies to every
 * later call in the process; returns the previous setting, or -1 (nothing
 * changed) for a value outside 0..2.  Not synchronised with calls on other
 * host threads. */
int ddt_debug_set_attn_kernel(int which);

/* ------------------------------------------------------------------------
 * Stage 1: per-position softmax normaliser and top-k.
 * DDTree page, 運作流程 step 1: the drafter returns one marginal q_i per
 * position i = 1..L (conditioned on the previous block only).  The tree's
 * candidates at depth i are the k most likely tokens of q_i.
 *
 * logits   [batch][L] rows of V logits, row r = b*L + i starting at
 *          logits + r*row_stride elements; dtype DDT_BF16 or DDT_F32.
 *          row_stride >= V.  BF16 rows need logits and row_stride*2 bytes
 *          aligned to 16 bytes for the vector path (otherwise a scalar path
 *          is used).
 * k        1..DDT_TOPK_K_MAX, k <= V.
 * inv_temperature  > 0: q_i = softmax(inv_temperature * z).
 * Outputs (all [batch][L][k] unless noted), in candidate order: logit
 * descending, ties by smaller token id first:
 *   ids  int32 token ids;   zk  float, the raw logit z (an exact copy);
 *   logp float, inv_temperature*z - lse (may be NULL);
 *   lse  float [batch][L], log sum_v exp(inv_temperature*z_v).
 * The ordering is decided on raw z, so temperature never reorders it.
 * ------------------------------------------------------------------------ */
size_t ddt_topk_workspace_size(int batch, int L, int V, int k);
ddt_status ddt_topk(const void* logits, ddt_dtype dtype, int batch, int L, int V,
                    int64_t row_stride, int k, float inv_temperature, int32_t* ids, float* zk,
                    float* logp, float* lse, void* workspace, size_t workspace_bytes,
                    cudaStream_t stream);

/* ------------------------------------------------------------------------
 * ddt_topk_noalloc: ddt_topk for callers that cannot allocate device memory.
 * The DDTree page has no counterpart to this entry point; it is a service of
 * this library for code that runs where obtaining device memory is not
 * allowed at the point of the call (an allocator-free region under a custom
 * memory manager that owns the heap, an embedded runtime with a fixed memory
 * plan, a plug-in whose host forbids cudaMalloc), so that it cannot supply
 * the workspace ddt_topk needs.
 *
 * Same arguments, outputs, results and status codes as ddt_topk, minus the
 * workspace; arguments are checked before anything is enqueued.
 * Its scratch is a fixed array in device global memory owned by libddt.so:
 * DDT_TOPK_NOALLOC_SCRATCH_BYTES on every GPU that loads the library, held
 * until the process exits.  Shapes whose ddt_topk_workspace_size exceeds it
 * are rejected with DDT_ERR_WORKSPACE before anything is launched.
 * A call made outside stream capture (with its device current) looks up the
 * array's device address and remembers it for that device; a call made
 * during capture uses the remembered address, so make the first call on a
 * device before any stream capture.  A device reset (or a new primary
 * context) moves the array; the next call made outside capture looks up the
 * new address.
 * Every call on a device shares the array; each call clears the part it uses
 * (an asynchronous memset on `stream`), so consecutive calls on one stream
 * are independent, while calls that overlap on the GPU race on the array.
 * Never calls cudaMalloc, cudaFree or any allocating library routine.
 * ------------------------------------------------------------------------ */
#define DDT_TOPK_NOALLOC_SCRATCH_BYTES (4u << 20)
ddt_status ddt_topk_noalloc(const void* logits, ddt_dtype dtype, int batch, int L, int V,
                            int64_t row_stride, int k, float inv_temperature, int32_t* ids,
                            float* zk, float* logp, float* lse, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Stage 2: build and compile the draft tree (one CTA per sequence).
 * DDTree page, 核心創新 and 運作流程 step 2: under a budget of B draft nodes
 * the tree is the set of B most probable prefixes of the factorised draft
 * prod_i q_i (it maximises the expected acceptance length under the draft,
 * 理論基礎 Proposition 1, and is prefix-closed, Proposition 2).  Step 3: the
 * tree is compiled into target-model inputs.
 *
 * Candidates: ids / zk / lse exactly as produced by ddt_topk
 * ([batch][L][k], [batch][L]).  Sequence b uses the first k_b candidates of
 * each position (k_per_seq[b], or k when k_per_seq is NULL) and the budget
 * B_b (budget_per_seq[b], or B_max when NULL).  Out-of-range device values
 * are clamped to [1,k] and [0,B_max] and flagged in dev_status.
 *
 * Total order (best first) on prefixes p of depth t with logit sum
 * s(p) = sum of raw z along p and score(p) = inv_temperature*s(p) - sum_{i<=t} lse_i
 * (fp64): at equal depth, larger s(p) first (exact: the lse terms cancel),
 * then the smaller token id at the deepest position, then at the one above,
 * and so on; at different depths, larger score first, then the shallower.
 *
 * Compiled outputs, N_max = B_max + 1 rows per sequence, breadth-first
 * order (depth, parent row, candidate rank); row 0 is the root carrying
 * root_token[b] (the bonus token of the previous round):
 *   tok, parent (root: -1), depth (root: 0), pos = ctx_len[b] + depth
 *        int32 [batch][N_max]; rows >= n_nodes[b] are -1;
 *   mask uint32 [batch][N_max][W], W = ddt_mask_words(N_max): bit i of row j
 *        set iff row i is row j or one of its ancestors; padding rows 0;
 *   n_nodes int32 [batch] = 1 + number of selected prefixes;
 *   surrogate double [batch] (may be NULL): sum of exp(score) over the
 *        draft nodes, the expected acceptance length under the draft.
 * ctx_len may be NULL (treated as 0).  Limits: L <= DDT_TREE_L_MAX,
 * k <= DDT_TOPK_K_MAX, B_max <= DDT_TREE_B_MAX.  The builder relies on the
 * fp64 sums of logits along every path being exact (children of a node then
 * come in candidate order); it checks that the binary exponents of the
 * nonzero finite candidate logits of a sequence span at most
 * 29 - ceil(log2 L) and raises DDT_ERR_UNSUPPORTED in dev_status when they
 * do not (e.g. 1e-30 or subnormal logits beside 3.0): the tree it then
 * writes may differ from the exact order at the budget's cut.
 * ------------------------------------------------------------------------ */
ddt_status ddt_build_tree(const int32_t* ids, const float* zk, const float* lse, int batch, int L,
                          int k, float inv_temperature, const int32_t* k_per_seq,
                          const int32_t* budget_per_seq, int B_max, const int32_t* root_token,
                          const int32_t* ctx_len, int32_t* tok, int32_t* parent, int32_t* depth,
                          int32_t* pos, uint32_t* mask, int32_t* n_nodes, double* surrogate,
                          int32_t* dev_status, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Between stage 2 and a second build: node budgets across the batch.
 * DDTree page, section 實驗結果與權衡: acceptance grows with the node budget
 * and so does the verifier's cost; section 理論基礎, Proposition 1: a tree's
 * expected acceptance length is the sum of its nodes' prefix probabilities,
 * and a smaller budget's best tree is the best-first part of a larger one's.
 *
 * Input: every sequence's tree built with the largest budget it may get
 * (tok, parent, depth, n_nodes of ddt_build_tree, n_max rows) and the
 * candidates it was built from (ids, zk, lse of ddt_topk, [batch][L][k]).
 * A draft node of depth d with tokens t_1..t_d on its path has the score
 * invT*(z_1 + ... + z_d) - (lse_1 + ... + lse_d) (fp64, depth order) and the
 * probability exp(score).  The batch's nodes ranked by score (ties: smaller
 * sequence, then smaller row) give the split of any total n that maximises
 * the expected acceptance: the first n.  The call takes the n in
 * [0, total_budget] (total_budget < 0: every node) that maximises
 * (batch + the first n probabilities) / (cost_fixed + cost_per_node * n),
 * the expected emitted tokens per unit of round cost (smallest n on ties);
 * with cost_per_node <= 0 it takes n = min(total_budget, all nodes).
 * Outputs: budget_per_seq int32 [batch], sequence b's share (feed it to
 * ddt_build_tree's budget_per_seq); expected_tokens double [batch] (may be
 * NULL): 1 + the sum of the probabilities of its share.
 * Limits: batch * (n_max - 1) <= 8192 nodes.  cost_per_node > 0 needs
 * cost_fixed > 0.  A row that is not a node of these candidates raises
 * DDT_ERR_INVALID_ARG in dev_status and counts for nothing.
 * ------------------------------------------------------------------------ */
ddt_status ddt_plan_budget(const int32_t* tok, const int32_t* parent, const int32_t* depth,
                           const int32_t* n_nodes, const int32_t* ids, const float* zk,
                           const float* lse, int batch, int L, int k, int n_max,
                           float inv_temperature, int total_budget, double cost_fixed,
                           double cost_per_node, int32_t* budget_per_seq, double* expected_tokens,
                           int32_t* dev_status, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Stage 3: tree attention.
 * DDTree page, 核心創新 third bullet and 運作流程 step 3: one target forward
 * scores the whole tree; each tree row attends to the committed context and
 * to its own ancestors (and itself) only.
 *
 * For sequence b, tree row j < n_nodes[b] and query head h (kv head
 * h / (hq/hkv)):  out = softmax(scale * q K^T) V  over the context
 * positions 0..ctx_len[b]-1 and the tree rows i with mask bit (j, i) set.
 * Accumulation is fp32; out is bf16.  Rows j >= n_nodes[b] are written as 0
 * (and lse_out as -inf).
 *
 *   q       bf16 [batch][n_max][hq][d]
 *   k_cache, v_cache  dense (page_table == NULL): bf16 [batch][t_max][hkv][d];
 *           paged: bf16 [pages][page_size][hkv][d], context position t of
 *           sequence b lives in page page_table[b*max_pages + t/page_size],
 *           slot t % page_size.
 *   k_tree, v_tree  bf16 [batch][n_max][hkv][d]  (the tree rows' own K/V)
 *   mask    uint32 [batch][n_max][W] as produced by ddt_build_tree
 *   out     bf16 [batch][n_max][hq][d];  lse_out optional f32 [batch][n_max][hq]
 *           (natural log of the softmax normaliser of the scaled scores).
 *   max_ctx host-side upper bound of ctx_len[] (sizes the KV-split grid);
 *           a ctx_len above it is clamped and flagged in dev_status.
 * Limits: d in {64, 128}; hq % hkv == 0; n_max <= 1024; all base pointers
 * 16-byte aligned; page_size a multiple of 16.
 * Paths: d = 128 with (hq/hkv) dividing 128, at least 64 query rows per kv
 * head and (paged) num_pages > 0 with page_size dividing 128 or a multiple of
 * 128 runs on the tensor cores (tcgen05, TMA); everything else on CUDA cores.
 * ------------------------------------------------------------------------ */
typedef struct ddt_attn_args {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* page_table; /* NULL: dense cache */
  int page_size;
  int max_pages;
  int num_pages;             /* paged: pages in the pool (bounds the page loads); 0 = unknown */
  int64_t t_max;             /* dense: tokens per sequence in k_cache/v_cache */
  const int32_t* ctx_len;
  int max_ctx;
  const void* k_tree;
  const void* v_tree;
  const uint32_t* mask;
  const int32_t* n_nodes;
  int batch, n_max, hq, hkv, d;
  float scale;
  void* out;
  float* lse_out;            /* may be NULL */
  int32_t* dev_status;       /* may be NULL */
} ddt_attn_args;

size_t ddt_tree_attn_workspace_size(const ddt_attn_args* a);
ddt_status ddt_tree_attn(const ddt_attn_args* a, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream);

/* How ddt_tree_attn would run this call on the current device (a query: it
 * launches nothing).  *path: DDT_ATTN_PATH_SIMT (CUDA cores), _TC (tensor
 * cores, one query tile of 128 rows per CTA, one pass over the KV range),
 * _TC_CLUSTER (KV splits of a query tile run as one thread-block cluster and
 * merge through distributed shared memory), _TC_COMBINE (KV splits write
 * partials to the workspace and a second kernel merges them), _TC_PAIRS
 * (two query tiles of one kv head per CTA, sharing every K/V tile, one pass)
 * or _TC_PAIRS_COMBINE (the same with workspace-combined KV splits);
 * *kv_splits: the number of KV splits per query tile (either pointer may be
 * NULL).  Returns the status ddt_tree_attn's argument check would return. */
enum { DDT_ATTN_PATH_SIMT = 0, DDT_ATTN_PATH_TC = 1, DDT_ATTN_PATH_TC_CLUSTER = 2,
       DDT_ATTN_PATH_TC_COMBINE = 3, DDT_ATTN_PATH_TC_PAIRS = 4,
       DDT_ATTN_PATH_TC_PAIRS_COMBINE = 5 };
ddt_status ddt_tree_attn_plan(const ddt_attn_args* a, int* path, int* kv_splits);

/* ------------------------------------------------------------------------
 * Stage 4: greedy tree walk.
 * DDTree page, 運作流程 step 4: starting at the root, take the target's
 * next token under its decoding rule (greedy: argmax, smaller token id on
 * ties); if the current row has a child carrying that token, accept the
 * child and continue from it; otherwise that token is the bonus token of
 * the next round (also when the walk reaches a row of depth L).
 *
 *   logits  [batch][n_max] rows of V target logits, row (b, j) at
 *           logits + (b*n_max + j)*row_stride elements; DDT_F32 or DDT_BF16.
 *   tok, parent, depth, n_nodes: the compiled tree of ddt_build_tree.
 *   L       the draft length (the deepest a row can be).
 *   mode    how the rows' argmaxes are taken (same outputs for every mode):
 *           DDT_WALK_ALL_ROWS  every tree row's argmax in one scan of all
 *                              batch*n_max rows, then the walk: one pass at
 *                              full bandwidth, reading rows the walk never
 *                              visits;
 *           DDT_WALK_LAZY      only the rows the walk visits (at most L + 1
 *                              per sequence), one after another: one
 *                              thread-block cluster per sequence;
 *           DDT_WALK_AUTO      the library picks, from the sizes, the one
 *                              that is faster on this device even when the
 *                              walk goes down to depth L
 *                              (ddt_tree_walk_resolve_mode tells which).
 * Outputs: acc_len int32 [batch] (0..L), acc_nodes / acc_tok int32
 * [batch][L] (accepted rows and their tokens in walk order; unused -1),
 * bonus int32 [batch].  Tokens emitted this round = acc_len + 1.
 * Limits: row_stride < V, an unknown mode or a null pointer give
 * DDT_ERR_INVALID_ARG; L <= DDT_TREE_L_MAX, n_max <= DDT_TREE_B_MAX + 1,
 * batch <= 65535 and batch * (n_max + 1) + 1 <= DDT_WS_COUNTER_BYTES / 4
 * (the tickets) give DDT_ERR_UNSUPPORTED otherwise.
 * ------------------------------------------------------------------------ */
enum { DDT_WALK_ALL_ROWS = 0, DDT_WALK_LAZY = 1, DDT_WALK_AUTO = 2 };
size_t ddt_tree_walk_workspace_size(int batch, int n_max, int V);
ddt_status ddt_tree_walk(const void* logits, ddt_dtype dtype, int batch, int n_max, int V,
                         int64_t row_stride, const int32_t* tok, const int32_t* parent,
                         const int32_t* depth, const int32_t* n_nodes, int L, int mode,
                         int32_t* acc_len, int32_t* acc_nodes, int32_t* acc_tok, int32_t* bonus,
                         void* workspace, size_t workspace_bytes, int32_t* dev_status,
                         cudaStream_t stream);
/* The mode (DDT_WALK_ALL_ROWS or DDT_WALK_LAZY) that ddt_tree_walk runs for
 * `mode` and these sizes on the current device; -1 for invalid arguments. */
int ddt_tree_walk_resolve_mode(int mode, ddt_dtype dtype, int batch, int n_max, int V, int L);

/* ------------------------------------------------------------------------
 * Stage 4 from the target's hidden states (greedy): LM head, argmax, walk.
 * DDTree page, 運作流程 step 4: the target's greedy token after tree row j
 * is the argmax of its LM-head logits h_j W^T.  This call computes those
 * logits on the tensor cores tile by tile (bf16 inputs, fp32 accumulation),
 * keeps only each row's argmax (smaller token id on equal logits), and walks
 * the trees as ddt_tree_walk does; the [rows x V] logits are never stored.
 *
 *   hidden  bf16 [batch][n_max][K]: the target's final hidden state of every
 *           tree row (after its final norm), row-major
 *   weight  bf16 [V][K]: the LM head (the nn.Linear [out][in] layout)
 *   tok, parent, depth, n_nodes, L: the compiled tree (as ddt_tree_walk)
 * Outputs: acc_len, acc_nodes, acc_tok, bonus as ddt_tree_walk; row_token
 * (optional) int32 [batch][n_max]: every row's argmax.
 * Limits: K a multiple of 8; batch*n_max <= ddt_lm_head_max_rows(); base
 * pointers 16-byte aligned.  Rows beyond a sequence's n_nodes are computed
 * but not used by the walk.  The workspace is the counter region only.
 * ------------------------------------------------------------------------ */
typedef struct ddt_lm_head_walk_args {
  const void* hidden;
  const void* weight;
  int K, V;
  const int32_t* tok;
  const int32_t* parent;
  const int32_t* depth;
  const int32_t* n_nodes;
  int batch, n_max, L;
  int32_t* acc_len;
  int32_t* acc_nodes;
  int32_t* acc_tok;
  int32_t* bonus;
  int32_t* row_token;        /* may be NULL */
  int32_t* dev_status;       /* may be NULL */
} ddt_lm_head_walk_args;

int ddt_lm_head_max_rows(void);
size_t ddt_lm_head_walk_workspace_size(const ddt_lm_head_walk_args* a);
ddt_status ddt_lm_head_walk(const ddt_lm_head_walk_args* a, void* workspace,
                            size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * After stage 4: commit the accepted path's K/V to the context.
 * DDTree page, 運作流程 (workflow): a round starts from the bonus token the
 * target produced but has not run yet, runs it as the tree's root with the
 * draft rows, and the walk accepts a path.  The root and the accepted rows
 * are therefore forwarded; their K/V join the committed context at the
 * positions they were scored at, and the new bonus token (not forwarded)
 * stays out.  For sequence b with a = acc_len[b] and c = ctx_len[b]:
 * context position c + i receives the tree K/V of row 0 (i = 0) or of row
 * acc_nodes[b][i-1] (i = 1..a), for every kv head; then ctx_len[b] = c + a + 1.
 *
 *   k_tree, v_tree  bf16 [batch][n_max][hkv][d] (as for ddt_tree_attn)
 *   acc_len [batch], acc_nodes [batch][L]: the walk's outputs
 *   ctx_len [batch]  read, then advanced in place
 *   k_cache, v_cache dense (page_table == NULL): bf16 [batch][t_max][hkv][d];
 *           paged: bf16 [pages][page_size][hkv][d] through
 *           page_table [batch][max_pages] (as for ddt_tree_attn); pages the
 *           new positions fall in must already be in the table.
 * A position outside the cache (dense: >= t_max; paged: beyond max_pages, a
 * negative page id or one >= num_pages when num_pages > 0), an acc_len
 * outside [0, L] or an accepted row outside [0, n_max) is not written and
 * raises DDT_ERR_INVALID_ARG in dev_status; ctx_len still advances by
 * acc_len + 1.  Limits: hkv * d a multiple of 8 and at most 2^20, and
 * L <= DDT_TREE_L_MAX (DDT_ERR_UNSUPPORTED otherwise); all base pointers
 * 16-byte aligned (DDT_ERR_INVALID_ARG otherwise).  No workspace.
 * ------------------------------------------------------------------------ */
typedef struct ddt_kv_commit_args {
  const void* k_tree;
  const void* v_tree;
  const int32_t* acc_len;
  const int32_t* acc_nodes;
  int32_t* ctx_len;
  void* k_cache;
  void* v_cache;
  const int32_t* page_table; /* NULL: dense cache */
  int page_size;
  int max_pages;
  int num_pages;             /* paged: pages in the pool; 0 = unknown */
  int64_t t_max;             /* dense: tokens per sequence */
  int batch, n_max, hkv, d, L;
  int32_t* dev_status;       /* may be NULL */
} ddt_kv_commit_args;

ddt_status ddt_kv_commit(const ddt_kv_commit_args* a, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Stage 4 under a sampling decoding rule (target temperature T > 0).
 * DDTree page, 運作流程 step 4 (the walk follows the target's decoding
 * rule) and 核心創新 (the target's output distribution is preserved): each
 * visited row x draws its token from softmax(z_x / T), and the walk accepts
 * and descends exactly as ddt_tree_walk does.  One fresh uniform per row
 * keeps the walk lossless: every emitted token is a draw from the target's
 * conditional given the accepted prefix.
 *
 * The draw of row j of sequence b is by inversion over token ids in
 * increasing order: the token is the smallest v whose cumulative weight
 * exceeds u * sum(w), where u = (w0 >> 12) + 1/2 times 2^-52 and w0 is word
 * 0 of Philox4x64-10 (Salmon, Moraes, Dror and Shaw, SC'11) at counter
 * (j, b, 0, 0) under key (seed, step).  The weights are fp32 evaluations
 * of exp(z/T - max) with a fixed arithmetic (a = fl32(log2(e)/T),
 * t = fl32(a*z), k = round(t), w = P(t - k) * (1 + ln2 * e) * 2^(k - K)
 * with P the fp32 Horner form of the degree-7 Taylor polynomial of 2^r,
 * e the part of z*log2(e)/T that t lost, K = round of the row's largest
 * t; 0 below 2^-120), so they are reproducible exactly and each is within
 * about 3e-7 (relative) of the exact weight whatever the size of z/T;
 * their sums are at least double-float (~48-bit) accurate.  Logits must
 * be finite or -inf, with |z/T| < 2^21; a row with no finite logit draws
 * token 0.
 *
 *   inv_temperature  1/T, finite and > 0 (larger -> closer to greedy)
 *   seed, step       the Philox key: a stream per request (seed) and a
 *                    fresh draw per round (step)
 *   step_counter     optional device uint64 (8-byte aligned), or NULL.  When
 *                    given, the key's second word is step + *step_counter,
 *                    and the call adds one to *step_counter after its last
 *                    draw: a captured CUDA graph then draws fresh uniforms on
 *                    every replay.  Calls sharing a counter must not overlap.
 * Every other argument, the outputs and the workspace
 * (ddt_tree_walk_workspace_size) are those of ddt_tree_walk; the draws scan
 * every row (as DDT_WALK_ALL_ROWS).
 * ------------------------------------------------------------------------ */
ddt_status ddt_tree_walk_sample(const void* logits, ddt_dtype dtype, int batch, int n_max, int V,
                                int64_t row_stride, const int32_t* tok, const int32_t* parent,
                                const int32_t* depth, const int32_t* n_nodes, int L,
                                float inv_temperature, uint64_t seed, uint64_t step,
                                uint64_t* step_counter, int32_t* acc_len, int32_t* acc_nodes,
                                int32_t* acc_tok, int32_t* bonus, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DDT_H */
