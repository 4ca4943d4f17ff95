/*
 * tpc.h -- C ABI of the B200 (sm_100a) tree-packed chunkwise KDA library.
 *
 * The operation: chunkwise gated delta-rule ("KDA") linear attention,
 * forward and backward, run once over a prefix-shared rollout tree instead
 * of once per root-to-leaf trajectory (HARTS: "A Prefix-Sharing Training
 * System for Agentic RL with Hybrid-Attention Models", abstract; Figure 1;
 * Figure 2; Figure C.1).  Per token t and head, with g_t = log(alpha_t):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * Conventions shared by every call
 *  - Trees are parent-pointer forests of fork-free segments (HARTS Figure
 *    2(a)).  parent[i] = -1 (root) or a smaller id; length[i] >= 1.  The
 *    trajectories are the root-to-leaf paths, ordered by leaf id.
 *  - Token tensors use the plan's compact layout (HARTS Figure C.1(a): one
 *    physical row per unique token): segment v occupies rows
 *    row_offset[v] .. row_offset[v] + length[v] - 1 (tpc_plan_export).
 *    Row-major [N_unique, H, d]; beta is [N_unique, H].
 *  - All device memory (tensors, plan tables, workspace) is owned by the
 *    caller and passed as raw pointers.  The library owns only the opaque
 *    host-side plan object.
 *  - Device calls are asynchronous on the given stream and never
 *    synchronise; a zero stream means the legacy default stream.
 *  - Every call returns a status code (TPC_OK = 0).  tpc_last_error()
 *    gives a message for the calling thread.  Nothing aborts and no C++
 *    exception crosses this boundary.  Kernel-side checks (gate range,
 *    table bounds) record a code in the workspace status word; read it with
 *    tpc_status().
 */
#ifndef TPC_H_
#define TPC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* tpc_stream_t; /* == cudaStream_t */

enum tpc_status_code {
  TPC_OK = 0,
  TPC_ERR_INVALID_TREE = 1, /* parent order, range or zero-length segment */
  TPC_ERR_BAD_SHAPE = 2,    /* inconsistent sizes */
  TPC_ERR_UNSUPPORTED = 3,  /* head dims / chunk size not built */
  TPC_ERR_NULL = 4,         /* required pointer is NULL */
  TPC_ERR_WORKSPACE = 5,    /* workspace too small or misaligned */
  TPC_ERR_CUDA = 6,         /* a CUDA runtime call failed */
  TPC_ERR_DEVICE_CHECK = 7, /* a kernel-side check failed (see tpc_status) */
  TPC_ERR_TIMEOUT = 8,      /* a bounded device wait ran out */
  TPC_ERR_RANGE = 9,        /* gates outside the supported range */
  TPC_ERR_STATE = 10        /* plan not uploaded / wrong call order */
};

/*
 * Element types.  TPC_F32_SPLIT is an input type of the KDA calls only: fp32 tensors that the
 * tensor-core kernels (chunk 64, d 128) take as bf16 pairs hi + lo, each product formed as
 * hi*hi + lo*hi + hi*lo in fp32 (about 1e-4 of the output RMS in max error).  TPC_F32 inputs run
 * the fp32 CUDA-core kernels, whose results match the fp64 recurrence to about 1e-6.
 */
enum tpc_dtype { TPC_F32 = 0, TPC_BF16 = 1, TPC_F32_SPLIT = 2 };

/* Returns the message of the last failed call on this thread ("" if none). */
const char* tpc_last_error(void);
/* Library version string. */
const char* tpc_version(void);

/* ------------------------------------------------------------------ plan */
typedef struct tpc_plan tpc_plan;

/*
 * Round planner (HARTS abstract: a linear-time planner reaching the minimum
 * number of sequential packed linear-attention calls; Figure 2: direct
 * continuations, replay-started side sequences, a boundary state usable
 * only by a later call).  Runs on the host in O(n_nodes + tokens/chunk).
 *   parent, length: host arrays of n_nodes int32 (see conventions).
 *   chunk: chunk size C (16, 32 or 64).
 *   *out: receives a new plan; free it with tpc_plan_destroy.
 * Errors: TPC_ERR_NULL, TPC_ERR_INVALID_TREE, TPC_ERR_UNSUPPORTED.
 */
int tpc_plan_create(const int32_t* parent, const int32_t* length, int32_t n_nodes,
                    int32_t chunk, tpc_plan** out);
void tpc_plan_destroy(tpc_plan* plan);

/*
 * Planner modes.  TPC_PLAN_MIN_ROUNDS is tpc_plan_create's plan.  The other two are the ablations
 * the HARTS pages compare against (Figure 4: node-wise linear attention; Figure 5: no replay):
 *   TPC_PLAN_NODEWISE  every segment is a sequence of its own (no direct continuations); each starts
 *                      at its aligned boundary b_v with the same bounded replay, one round after the
 *                      segment holding token b_v - 1, so the call count is the depth of that chain
 *                      and every trajectory keeps its chunkwise numerical path.
 *   TPC_PLAN_NO_REPLAY side sequences start exactly at their fork point s_v from the state after
 *                      token s_v - 1 (no replay): the producing sequence cuts a chunk at s_v to
 *                      export that state, the side sequence's chunk grid starts at s_v.  Chunk
 *                      boundaries then differ from the trajectory-expanded grid, so results differ
 *                      from the per-trajectory chunkwise path in the last bits.
 * Every other call accepts a plan of any mode.
 */
enum tpc_plan_mode { TPC_PLAN_MIN_ROUNDS = 0, TPC_PLAN_NODEWISE = 1, TPC_PLAN_NO_REPLAY = 2 };
/* tpc_plan_create with a planner mode (above).  Errors as tpc_plan_create; an unknown mode is
 * TPC_ERR_UNSUPPORTED. */
int tpc_plan_create_mode(const int32_t* parent, const int32_t* length, int32_t n_nodes, int32_t chunk, int32_t mode,
                         tpc_plan** out);

/*
 * Plan with external boundary-state exports, for sharing windows across microbatches (HARTS
 * abstract: within a sharing window, gradients from dependent microbatches accumulate before one
 * backward pass through the shared prefix; Figure 3: the producer's backward runs after its
 * consumers').  Export e asks for the state after token export_pos[e] - 1 on the path of node
 * export_node[e], which must hold that token (s < pos <= s + length) at a position that is a
 * multiple of the chunk, so that a consumer microbatch can start there and keep its trajectories'
 * chunkwise numerical path (its replayed rows, pos .. fork - 1, are its own first segment).
 * The forward writes each export's state into the workspace (tpc_kda_export_states copies it out);
 * tpc_kda_backward_window adds the consumers' gradients of those states to the reverse scan where
 * it crosses them, in export order after the in-tree consumers.
 * Errors: as tpc_plan_create_mode; TPC_ERR_INVALID_TREE for an export that breaks the rule above.
 */
int tpc_plan_create_window(const int32_t* parent, const int32_t* length, int32_t n_nodes, int32_t chunk, int32_t mode,
                           int32_t n_exports, const int32_t* export_node, const int64_t* export_pos, tpc_plan** out);

typedef struct tpc_plan_info {
  int64_t n_unique;     /* unique token rows N */
  int64_t n_expanded;   /* sum of trajectory lengths */
  int64_t replay_total; /* replayed rows over all sequences (R) */
  int64_t n_seq_tokens; /* rows processed by the packed calls = N + R */
  int32_t n_nodes, n_rounds, n_seqs, n_chunks, n_slots, n_leaves, n_roots, chunk;
  int32_t max_seq_chunks; /* longest sequence, in chunks */
  int32_t n_replay_targets;
  int32_t n_exports;      /* external boundary-state exports (tpc_plan_create_window) */
} tpc_plan_info;
int tpc_plan_get_info(const tpc_plan* plan, tpc_plan_info* info);

/*
 * Host tables (bit-exact comparison surface).  Every member is a
 * caller-owned host array or NULL (skipped).  Sizes: per node n_nodes,
 * leaves n_leaves, expanded_rows n_expanded, traj_offset n_leaves + 1.
 *   round        1-based round of the packed call that computes the node
 *   is_cont      1 if the node continues its parent's sequence
 *   anchor       node holding token b_v - 1 (b_v = floor(s_v/C)*C), -1 if b_v = 0
 *   replay_start first position of a sequence head (b_v, 0 for roots), -1 otherwise
 *   replay_len   replayed rows of a sequence head (s_v - b_v), -1 otherwise
 *   row_offset   first compact row of the node
 *   occurrence   number of trajectories through the node (HARTS Figure 1: q_B)
 *   leaves       leaf node ids in trajectory order
 *   expanded_rows compact row of every trajectory position, trajectories concatenated
 *   traj_offset  start of each trajectory in expanded_rows
 */
typedef struct tpc_plan_tables {
  int32_t* round;
  int32_t* is_cont;
  int32_t* anchor;
  int32_t* replay_start;
  int32_t* replay_len;
  int64_t* row_offset;
  int32_t* occurrence;
  int32_t* leaves;
  int64_t* expanded_rows;
  int64_t* traj_offset;
} tpc_plan_tables;
int tpc_plan_export(const tpc_plan* plan, tpc_plan_tables* tables);

/*
 * Device index tables: bytes needed, and the upload.  The caller allocates
 * `bytes` of device memory (256-byte aligned); tpc_plan_upload copies the
 * sequence, chunk, slot and replay tables there (async on `stream`) and
 * records the address in the plan, which every later device call uses.
 * The memory must stay valid while the plan is used.
 */
/*
 * Diagnostics: the device-facing tables as int32 rows (caller-owned host arrays, NULL skips one):
 *   seqs   [n_seqs][8]   chunk_begin, n_chunks, import (slot >= 0, or -(root ordinal + 1)),
 *                        leaf ordinal (-1: the chain ends at an internal node), head node, round,
 *                        start position, replayed rows
 *   chunks [n_chunks][8] sequence, rows, replayed rows, first own compact row, replay base, export
 *                        slot (-1 none), first position, index in the sequence
 *   slots  [n_slots][4]  producing sequence, exporting chunk, first consumer, consumers
 *   slot_cons [sum of consumers] consumer sequences (n_seqs + e for external export e)
 *   replay_rows [replay_total] compact row of every replayed row
 */
int tpc_plan_debug_tables(const tpc_plan* plan, int32_t* seqs, int32_t* chunks, int32_t* slots, int32_t* slot_cons,
                          int32_t* replay_rows);

size_t tpc_plan_device_bytes(const tpc_plan* plan);
int tpc_plan_upload(tpc_plan* plan, void* dev, size_t bytes, tpc_stream_t stream);

/* ------------------------------------------------------------------ microbatches (L1) */
/*
 * First-level (L1) microbatch planner: compression-oriented packing of the trajectories of many
 * rollout trees under a budget of unique token rows per microbatch (HARTS abstract: a two-level
 * planner first constructs compression-oriented microbatches; Figure 1(c); Table 4).  The pages
 * give no algorithm; this one keeps a tree whole when its unique tokens fit the budget, cuts a
 * larger tree along its depth-first leaf order (so that trajectories sharing the longest prefixes
 * stay together; a piece closes before the leaf whose new path tokens would exceed the budget, and
 * a trajectory longer than the budget is a piece alone), and places pieces first-fit in decreasing
 * cost order (ties: smaller first leaf id).  Host only, deterministic.
 *   parent, length: the forest of all trees of the step (conventions above), n nodes.
 *   budget: unique token rows per microbatch (>= 1).
 *   leaf_mb: host [n_leaves] (leaves in id order) receives each trajectory's microbatch.
 *   mb_unique, mb_expanded: host [max_mb] or NULL: per microbatch the tokens of the union of its
 *   trajectories' paths, and the sum of their lengths.
 *   stats: totals, compression = expanded / unique, balance = mean unique / max unique.
 * Errors: TPC_ERR_NULL, TPC_ERR_INVALID_TREE, TPC_ERR_BAD_SHAPE (budget < 1, or more microbatches
 * than max_mb while mb_unique or mb_expanded is given; stats->n_microbatches then holds the count).
 */
typedef struct tpc_microbatch_stats {
  int32_t n_microbatches;
  int64_t unique_tokens, expanded_tokens, max_unique;
  double compression, balance;
} tpc_microbatch_stats;
int tpc_microbatch_plan(const int32_t* parent, const int32_t* length, int32_t n_nodes, int64_t budget,
                        int32_t* leaf_mb, int64_t* mb_unique, int64_t* mb_expanded, int32_t max_mb,
                        tpc_microbatch_stats* stats);

/* ------------------------------------------------------------------ KDA */
typedef struct tpc_kda_shape {
  int32_t H;          /* heads */
  int32_t dk, dv;     /* head dims; dk == dv in {32, 64, 128} */
  int32_t in_dtype;   /* tpc_dtype of q, k, v, g, beta, d_o (TPC_F32_SPLIT: fp32 data) */
  int32_t out_dtype;  /* tpc_dtype of o, dq, dk, dv */
} tpc_kda_shape;

/*
 * Workspace bytes for tpc_kda_forward + tpc_kda_backward on this plan.
 * The forward leaves in it what the backward reads (chunk-start states,
 * U, W, boundary-state slots); do not reuse it in between.  256-byte
 * aligned.  Returns 0 for an unsupported shape.
 */
size_t tpc_kda_workspace_bytes(const tpc_plan* plan, const tpc_kda_shape* shape);

typedef struct tpc_kda_fwd_io {
  const void* q;          /* [N, H, dk] in_dtype */
  const void* k;          /* [N, H, dk] in_dtype, any norm */
  const void* v;          /* [N, H, dv] in_dtype */
  const void* g;          /* [N, H, dk] in_dtype, log(alpha) <= 0 */
  const void* beta;       /* [N, H]     in_dtype */
  const float* init_state;/* [n_roots, H, dk, dv] fp32 or NULL (= 0) */
  void* o;                /* [N, H, dv] out_dtype */
  float* final_state;     /* [n_leaves, H, dk, dv] fp32 or NULL */
} tpc_kda_fwd_io;

/*
 * Tree-packed forward: for each round, one packed launch over every
 * sequence of the round (HARTS Figure 2(c)); sequences start from the
 * initial state or from a boundary state exported by an earlier round and
 * replay the rows between the aligned boundary and their first own row
 * without writing outputs (Figure C.1(b)).  Outputs equal the per-trajectory
 * recurrence (the chunk grid is aligned to trajectory positions).
 * Errors: TPC_ERR_NULL, TPC_ERR_STATE (plan not uploaded),
 * TPC_ERR_UNSUPPORTED, TPC_ERR_WORKSPACE, TPC_ERR_CUDA.
 * Streams: on the tensor-core path (chunk 64, d 128) the sequential state scans run on a
 * library-owned high-priority stream, ordered against `stream` by events (one per round), so that
 * the per-chunk kernels of neighbouring rounds on `stream` overlap them; `stream` waits for every
 * scan before the call's last work, so everything is complete when work queued on `stream` after
 * the call runs (stream capture sees the fork and the join).  tpc_kda_backward does the same.
 */
int tpc_kda_forward(const tpc_plan* plan, const tpc_kda_shape* shape, const tpc_kda_fwd_io* io,
                    void* ws, size_t ws_bytes, tpc_stream_t stream);

typedef struct tpc_kda_bwd_io {
  const void* q; const void* k; const void* v; const void* g; const void* beta; /* as forward */
  const float* init_state;  /* as forward */
  const void* d_o;          /* [N, H, dv] in_dtype: output gradient per unique row */
  const float* d_final;     /* [n_leaves, H, dk, dv] fp32 or NULL */
  void* dq; void* dk; void* dv; /* [N, H, d] out_dtype */
  float* dg;                /* [N, H, dk] fp32 (gradient w.r.t. log alpha) */
  float* dbeta;             /* [N, H] fp32 */
  float* d_init;            /* [n_roots, H, dk, dv] fp32 or NULL */
} tpc_kda_bwd_io;

/*
 * Backward of sum <d_o, o> + sum <d_final, final_state>: rounds in reverse;
 * the gradient of each boundary state is the sum of its consumers'
 * gradients, in a fixed order, added before the producer's reverse scan
 * crosses that boundary (HARTS abstract: gradients from dependent work
 * accumulate before one backward pass through the shared prefix).
 * Replayed rows contribute to the gradients of their own rows in a fixed
 * order; results are bitwise reproducible.  Requires the workspace of a
 * tpc_kda_forward on the same inputs.
 */
int tpc_kda_backward(const tpc_plan* plan, const tpc_kda_shape* shape, const tpc_kda_bwd_io* io,
                     void* ws, size_t ws_bytes, tpc_stream_t stream);

/*
 * After tpc_kda_forward on a plan with exports: states [n_exports, H, dk, dv] fp32 receives each
 * exported boundary state (device to device copies on `stream`).
 */
int tpc_kda_export_states(const tpc_plan* plan, const tpc_kda_shape* shape, const void* ws, float* states,
                          tpc_stream_t stream);
/*
 * tpc_kda_backward with the gradients of the exported states (export_grads [n_exports, H, dk, dv]
 * fp32, e.g. the d_init of the consumer microbatches, summed per export) added to the reverse scan;
 * NULL means zero.  tpc_kda_backward is this call with NULL.
 */
int tpc_kda_backward_window(const tpc_plan* plan, const tpc_kda_shape* shape, const tpc_kda_bwd_io* io,
                            const float* export_grads, void* ws, size_t ws_bytes, tpc_stream_t stream);

/*
 * Reads (after synchronising `stream`) and clears the status word that
 * kernels write in `ws`.  Returns TPC_OK or the first recorded error.
 */
int tpc_status(const tpc_plan* plan, const tpc_kda_shape* shape, void* ws, tpc_stream_t stream);

/* ------------------------------------------------------------------ row maps */
/*
 * Deterministic occurrence sum (HARTS Figure 1: one row serves every
 * trajectory through it): x_unique[r] = sum over occurrences of r, in
 * trajectory order, of x_exp[j].  x_exp is [n_expanded, width] and
 * x_unique [N, width], both fp32.
 */
int tpc_reduce_expanded_to_unique(const tpc_plan* plan, const float* x_exp, float* x_unique,
                                  int64_t width, tpc_stream_t stream);
/* Gather to the trajectory-expanded layout: x_exp[j] = x_unique[expanded_rows[j]];
 * elem_bytes 2 or 4, width elements per row. */
int tpc_gather_expanded(const tpc_plan* plan, const void* x_unique, void* x_exp, int64_t width,
                        int32_t elem_bytes, tpc_stream_t stream);
/* Occurrence count per compact row (int32 [N]). */
int tpc_occurrence_counts(const tpc_plan* plan, int32_t* counts, tpc_stream_t stream);
/* Row gather dst[i] = src[rows[i]] (rows of `width` elements of elem_bytes 2 or 4; n_rows rows). */
int tpc_gather_rows(const void* src, const int32_t* rows, void* dst, int64_t n_rows, int64_t width, int32_t elem_bytes,
                    tpc_stream_t stream);
/* Row accumulation dst[rows[i]] += src[i] (fp32, `width` per row); the rows of one call must be
 * distinct (one writer per row), so repeated calls in a fixed order sum deterministically.  Used to
 * return a consumer microbatch's replayed-row gradients to the producer's rows. */
int tpc_add_rows(const float* src, const int32_t* rows, float* dst, int64_t n_rows, int64_t width, tpc_stream_t stream);

/* ------------------------------------------------------------------ dense products */
/*
 * bf16 GEMM on tensor cores (the projections of the hybrid layer group and the vocabulary
 * products of log-probability recovery, HARTS Figure C.1(d)):
 *   C = alpha * op(A) op(B) + beta * C,  op(A) M x K, op(B) K x N, fp32 accumulation.
 *   a_mn = 0: A stored [M][lda] (K contiguous); a_mn = 1: A stored [K][lda] (M contiguous).
 *   b_mn = 0: B stored [N][ldb] (K contiguous); b_mn = 1: B stored [K][ldb] (N contiguous).
 *   C: [M][ldc], c_dtype TPC_F32 (beta allowed) or TPC_BF16 (beta must be 0).
 *   A, B 16-byte aligned with lda, ldb multiples of 8.  status: optional device int receiving
 *   TPC_ERR_TIMEOUT if a bounded pipeline wait runs out.
 */
int tpc_gemm_bf16(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
                  int64_t ldc, int32_t a_mn, int32_t b_mn, int32_t c_dtype, float alpha, float beta, int32_t* status,
                  tpc_stream_t stream);

/*
 * Split-precision form of tpc_gemm_bf16 for fp32 operands held as two bf16 matrices, X_hi = bf16(X)
 * and X_lo = bf16(X - X_hi) (X = X_hi + X_lo to 2^-17 relative):
 *   C = alpha * (A B + A_lo B + A B_lo) + beta * C,
 * where A_lo and B_lo are optional (NULL: term left out; B_lo requires A_lo) and share A's and B's
 * layout and leading dimensions.  With A_lo only (fp32 activations times bf16 weights) the result
 * is the fp32 product to about 2^-16 relative; with both (two fp32 operands) the dropped
 * A_lo B_lo term is below 2^-16 of the product.  Costs one tensor-core pass per term.
 */
int tpc_gemm_split(const void* A, const void* A_lo, const void* B, const void* B_lo, void* C, int64_t M, int64_t N,
                   int64_t K, int64_t lda, int64_t ldb, int64_t ldc, int32_t a_mn, int32_t b_mn, int32_t c_dtype,
                   float alpha, float beta, int32_t* status, tpc_stream_t stream);

/* ------------------------------------------------------------------ tree-masked attention */
/*
 * Softmax attention in which each token reads only its ancestors' keys and values and the earlier
 * tokens of its own segment (HARTS Figure 1(b); Figure C.1(c): diagonal blocks causal, outputs
 * return to compact rows).  Along any trajectory this is causal attention over the trajectory's
 * prefix.  Compact-row tensors, bf16 inputs:
 *   q, k: [N][H][d_qk], v: [N][H][d_v]; o: [N][H][d_v] and (backward) dq, dk, dv in io_dtype;
 *   lse: fp32 [N][H] (natural log of the softmax normaliser of scale * q.k).
 *   delta: caller scratch fp32 [N][H] (backward).  Built for d_qk = 192, d_v = 128.
 *   q, k, v, d_o and their low parts are read by TMA: base pointers 16-byte aligned (a tensor map
 *   that cannot be encoded returns TPC_ERR_CUDA before any launch).
 * Deterministic: the backward sums every gradient in a fixed order without atomics.
 */
typedef struct tpc_attn_shape {
  int32_t H;
  int32_t d_qk, d_v;
  float scale;
  int32_t io_dtype; /* dtype of o (forward) and of o, dq, dk, dv (backward) */
} tpc_attn_shape;
/*
 * Optional bf16 low parts (NULL = zero) of inputs given as hi/lo pairs: an fp32 tensor x is passed
 * as hi = bf16(x) in the main argument and lo = bf16(x - hi) here (x = hi + lo to 2^-17 relative).
 * With any low part present, every product takes the three partial products hi hi + lo hi + hi lo,
 * so fp32 inputs and upstream gradients enter without a bf16 rounding of their own.  lo may be NULL.
 */
typedef struct tpc_attn_lo {
  const void* q; const void* k; const void* v; /* layouts of q, k, v */
  const void* d_o;                             /* backward only, layout of d_o */
} tpc_attn_lo;
int tpc_tree_attn_forward(const tpc_plan* plan, const tpc_attn_shape* shape, const void* q, const void* k,
                          const void* v, const tpc_attn_lo* lo, void* o, float* lse, int32_t* status,
                          tpc_stream_t stream);
int tpc_tree_attn_backward(const tpc_plan* plan, const tpc_attn_shape* shape, const void* q, const void* k,
                           const void* v, const tpc_attn_lo* lo, const void* o, const float* lse, const void* d_o,
                           void* dq, void* dk, void* dv, float* delta, int32_t* status, tpc_stream_t stream);
/* Trajectory position (depth from the root) of every compact row, int32 [N] (rotary positions). */
int tpc_rope_positions(const tpc_plan* plan, int32_t* pos, tpc_stream_t stream);

/* ------------------------------------------------------------------ log-probability recovery */
/*
 * Log-probabilities of every original trajectory position from one logit row per unique row
 * (HARTS abstract: log-probabilities recovered for each original trajectory position; Figure 1:
 * one logit row z_B supplies every trajectory's target log-probability; Figure C.1(d): no
 * expanded vocabulary-sized logits).  For compact row u with hidden state h_u and output matrix
 * W [V][Dh]: z_u = W h_u, lse_u = log sum exp z_u, and for each occurrence j of u (trajectory
 * order, tpc_plan_export's expanded_rows) with target y_j: logp_j = z_u[y_j] - lse_u.
 * No logit matrix is stored: the tensor-core GEMM's epilogue reduces each 256-column tile of z to
 * its (max, sum of exponentials) per row, lse combines those in a fixed order, and every target
 * logit is its own fp32 dot product W_{y_j} . h_u.
 *   h: bf16 [N_unique][Dh] (compact order), W: bf16 [V][Dh], targets: int32 [n_expanded] in [0, V).
 *   logp: fp32 [n_expanded], lse: fp32 [N_unique].  V and Dh multiples of 8, V < 2^31.
 *   scratch: caller device memory of tpc_logprob_scratch_bytes(plan, V, chunk_rows) bytes
 *   (256-aligned); the GEMMs run chunk_rows unique rows at a time.
 *   status: optional device int; a target outside [0, V) records TPC_ERR_DEVICE_CHECK.
 * Backward of sum_j dlogp_j logp_j: dh fp32 [N_unique][Dh] and dW fp32 [V][Dh] (overwritten), from
 * the forward's lse.  dz_u = sum_j dlogp_j onehot(y_j) - s_u softmax(z_u) (s_u: u's weight sum):
 * the dense part comes out of the recomputed logit tile's epilogue as bf16 and enters one
 * tensor-core pass each of dh = dz W and dW = dz^T h; the one-hot part is added exactly in fp32
 * (occurrences grouped by target for dW).  Deterministic (fixed chunk and occurrence order).
 */
size_t tpc_logprob_scratch_bytes(const tpc_plan* plan, int64_t V, int32_t chunk_rows);
int tpc_logprob_forward(const tpc_plan* plan, const void* h, const void* W, int64_t V, int64_t Dh,
                        const int32_t* targets, float* logp, float* lse, void* scratch, size_t scratch_bytes,
                        int32_t chunk_rows, int32_t* status, tpc_stream_t stream);
int tpc_logprob_backward(const tpc_plan* plan, const void* h, const void* W, int64_t V, int64_t Dh,
                         const int32_t* targets, const float* dlogp, const float* lse, float* dh, float* dW,
                         void* scratch, size_t scratch_bytes, int32_t chunk_rows, int32_t* status,
                         tpc_stream_t stream);

/* ------------------------------------------------------------------ compact MoE routing */
/*
 * Deterministic top-k routing of the unique rows with occurrence counts (HARTS abstract: for
 * deterministic top-k routing without token dropping, occurrence counts restore MoE objective
 * weights and expert-load statistics; Figure 1: q_B = 2 restores them without repeating routing or
 * expert computation; Figure C.1(d): multiplicity-weighted router losses and expert-load counts).
 * Every unique row u is routed once; each of its q_u trajectory positions would route identically,
 * so statistics over positions are q_u-weighted sums over unique rows.
 *   tpc_moe_route: z_u = W_r h_u (fp32, a fixed-order sum over the hidden dimension of separately
 *     rounded products, so the top-k decision is reproducible), lse_u, the top-k experts (larger
 *     logit first, ties to the lower expert index) and their gates (softmax renormalised over the
 *     top-k), expert_load_e = sum_u q_u [e in topk(u)] (exact integers) and
 *     prob_sum_e = sum_u q_u softmax(z_u)_e.
 *     h: bf16 [N_unique][Dh] (compact rows), w_router: bf16 [E][Dh], Dh a multiple of 64, E <= 256,
 *     1 <= k <= min(E, 8).  logits fp32 [N][E], lse fp32 [N], topk_idx int32 [N][k], topk_gate fp32
 *     [N][k], expert_load int64 [E], prob_sum fp32 [E].
 *   tpc_moe_router_loss: with n = n_expanded positions, L_aux = E / (k n^2) sum_e load_e P_e and
 *     L_z = (1/n) sum over positions of lse^2 (losses[0], losses[1], device fp32), and dlogits fp32
 *     [N][E] = the gradient of a L_aux + b L_z with respect to each unique row's logits (the
 *     occurrence-weighted sum of the per-position gradients; the routing is held fixed).
 *   scratch: tpc_moe_scratch_bytes(plan, E) bytes of caller device memory.  All reductions run in a
 *   fixed order.  The expert FFNs themselves are ordinary per-row products and are not part of this.
 */
size_t tpc_moe_scratch_bytes(const tpc_plan* plan, int32_t E);
int tpc_moe_route(const tpc_plan* plan, const void* h, const void* w_router, int64_t Dh, int32_t E, int32_t k,
                  float* logits, float* lse, int32_t* topk_idx, float* topk_gate, int64_t* expert_load,
                  float* prob_sum, void* scratch, size_t scratch_bytes, tpc_stream_t stream);
int tpc_moe_router_loss(const tpc_plan* plan, const float* logits, const float* lse, const int64_t* expert_load,
                        const float* prob_sum, int32_t E, int32_t k, float a, float b, float* losses, float* dlogits,
                        void* scratch, size_t scratch_bytes, tpc_stream_t stream);

/* ------------------------------------------------------------------ hybrid layer group */
/*
 * A group of n_kda KDA layers followed by one latent-attention (MLA) layer on the compact rows of
 * the plan's tree (HARTS Table 1: KDA and MLA layers in a 3:1 group; Figure C.1: each layer runs
 * once per unique row; Table 7 and Section 4: activations recomputed in the backward pass).  The
 * pages give no layer formulas; this library fixes the plainest pre-norm residual layers:
 *   KDA layer: xn = RMSNorm(x) (unit weight, eps 1e-6); [q | k | v | g | beta] = xn W_in^T with
 *     W_in [4 D + H][D] (rows: q, k, v, g blocks of D = H d_head, then H beta rows);
 *     k L2-normalised per head (eps 1e-6), g = -0.1 softplus(.), beta = sigmoid(.);
 *     y = x + KDA(q, k, v, g, beta) W_o^T, W_o [D][D].
 *   MLA layer: xn = RMSNorm(x); [q | c | kr] = xn W_a^T, W_a [H (d_head + d_rope) + d_latent + d_rope][D]
 *     (per head d_head no-position dims then d_rope rotary dims; c the latent; kr the rotary key
 *     shared by every head); [k_nope | v] = c W_b^T, W_b [2 D][d_latent]; rotary half-split rotation
 *     (base 10000) of q's and kr's rotary dims at the row's trajectory depth; k = [k_nope | kr];
 *     tree-masked softmax attention with scale 1/sqrt(d_head + d_rope); y = x + o W_o^T, W_o [D][D].
 * Precision: weights bf16; activations and gradients fp32.  Tensor-core products take fp32
 * operands as bf16 hi/lo pairs (tpc_gemm_split, tpc_attn_lo), so no activation or gradient is
 * rounded to bf16; the KDA recurrence runs on fp32 inputs.
 * Built for D = 2048, H = 16, d_head = 128, d_rope = 64, d_latent = 512, chunk-64 plans.
 */
#define TPC_GROUP_MAX_KDA 8
typedef struct tpc_group_shape {
  int32_t D, H, d_head, d_rope, d_latent;
  int32_t n_kda;         /* KDA layers before the MLA layer, 0..TPC_GROUP_MAX_KDA */
  int32_t reuse_forward; /* backward only: 1 = the workspace still holds this group's forward on the
                            same inputs (tpc_group_forward was the last call to use it); the last
                            (MLA) layer, whose activations are then still resident, is not recomputed.
                            0 = recompute every layer.  Results are bitwise the same either way. */
} tpc_group_shape;
typedef struct tpc_group_kda_weights { const void* w_in; const void* w_o; } tpc_group_kda_weights;
typedef struct tpc_group_mla_weights { const void* w_a; const void* w_b; const void* w_o; } tpc_group_mla_weights;
typedef struct tpc_group_weights {
  tpc_group_kda_weights kda[TPC_GROUP_MAX_KDA]; /* bf16, first n_kda used */
  tpc_group_mla_weights mla;
} tpc_group_weights;
/* weight gradients, fp32, same shapes as the weights; overwritten by the backward */
typedef struct tpc_group_kda_grads { float* w_in; float* w_o; } tpc_group_kda_grads;
typedef struct tpc_group_mla_grads { float* w_a; float* w_b; float* w_o; } tpc_group_mla_grads;
typedef struct tpc_group_grads {
  tpc_group_kda_grads kda[TPC_GROUP_MAX_KDA];
  tpc_group_mla_grads mla;
} tpc_group_grads;

/* Workspace bytes for tpc_group_forward / tpc_group_backward on this plan (0 if unsupported). */
size_t tpc_group_workspace_bytes(const tpc_plan* plan, const tpc_group_shape* shape);
/*
 * Forward.  x: fp32 [N][D] (compact rows); h: fp32 [n_kda][N][D] receives each KDA layer's output
 * (= the next layer's input, the only activations kept for the backward); y: fp32 [N][D].
 * Errors: TPC_ERR_NULL, TPC_ERR_STATE, TPC_ERR_UNSUPPORTED, TPC_ERR_WORKSPACE, TPC_ERR_CUDA;
 * device-side failures (GEMM or attention wait timeouts, KDA gate range) are read by
 * tpc_group_status.
 */
int tpc_group_forward(const tpc_plan* plan, const tpc_group_shape* shape, const tpc_group_weights* w,
                      const float* x, float* h, float* y, void* ws, size_t ws_bytes, tpc_stream_t stream);
/*
 * Backward of sum <dy, y>: recomputes every layer from its kept input (x, h), then runs its adjoint
 * in reverse layer order.  dy fp32 [N][D] (occurrence-summed upstream gradient per compact row);
 * dx fp32 [N][D] (may equal dy); weight gradients into g.  The workspace need not hold a forward,
 * unless shape->reuse_forward is set (see tpc_group_shape).
 */
int tpc_group_backward(const tpc_plan* plan, const tpc_group_shape* shape, const tpc_group_weights* w,
                       const float* x, const float* h, const float* dy, float* dx, const tpc_group_grads* g,
                       void* ws, size_t ws_bytes, tpc_stream_t stream);
/* Synchronises `stream`, returns and clears the first device-side error of the group's kernels. */
int tpc_group_status(const tpc_plan* plan, const tpc_group_shape* shape, void* ws, tpc_stream_t stream);

/* ------------------------------------------------------------------ allocation-free forward */
/* Bytes of device scratch built into the library for tpc_kda_forward_static (64 MiB). */
#define TPC_STATIC_SCRATCH_BYTES (64u << 20)

/*
 * tpc_kda_forward with no device allocation at all (the HARTS pages have no counterpart; this is
 * a deployment convenience).  It is for callers that may not allocate device memory themselves:
 * code running inside a host runtime whose own pool owns the whole device, or a latency-critical
 * path that must not pay the device-wide synchronisation a fresh cudaMalloc can cause.  The plan
 * tables and the forward workspace go into one device array of TPC_STATIC_SCRATCH_BYTES that is
 * compiled into this library, so every GPU that loads the library holds those bytes until the
 * process exits.  The plan does not need tpc_plan_upload for this call.
 *   io: as tpc_kda_forward (caller-owned inputs and outputs); the call allocates nothing and calls
 *       no allocating routine.
 *   Sizes: problems whose tables + workspace exceed TPC_STATIC_SCRATCH_BYTES are rejected with
 *       TPC_ERR_WORKSPACE and a message giving the bytes needed.
 *   Set-up: the first call on a device looks up the array's device address (with that device
 *       current).
 *   Sharing: every call uses the same array and it keeps the previous call's contents; the call
 *       clears its status word itself (tpc_kda_static_status reads it).  Calls that overlap on the GPU (other streams, other host
 *       threads) race on the array: serialise them.  tpc_kda_backward cannot follow this call (the
 *       workspace it needs is not kept).
 */
int tpc_kda_forward_static(const tpc_plan* plan, const tpc_kda_shape* shape, const tpc_kda_fwd_io* io,
                           tpc_stream_t stream);
/*
 * Reads (after synchronising `stream`) and clears the status word of the allocation-free forward
 * on the current device: kernel-side checks of tpc_kda_forward_static (the gate range) record
 * their code there, since that call has no caller workspace.  Returns TPC_OK, TPC_ERR_RANGE or
 * TPC_ERR_DEVICE_CHECK.  Allocates nothing.
 */
int tpc_kda_static_status(tpc_stream_t stream);

/* ------------------------------------------------------------------ diagnostics */
/* Per-kernel timing: when enabled, every launch is bracketed by CUDA events recorded on
 * its stream (adds a few microseconds per launch).  Not thread safe. */
void tpc_profile_enable(int on);
/* Synchronises the recorded events and writes "name launches total_ms" lines into buf
 * (truncated to len), then clears the records. */
int tpc_profile_read(char* buf, size_t len);
/* Number of kernels this library has launched in the process. */
long long tpc_launch_count(void);
/*
 * Check of the device-side timeout path: one CTA runs the bounded mbarrier wait that every
 * tensor-core kernel of this library uses, on a barrier that nothing arrives on (no copy or MMA in
 * flight), with a limit of timeout_ns (1e3 .. 1e8).  The wait runs out, the kernel writes
 * TPC_ERR_TIMEOUT into *status (a caller-owned device int) and returns; the context stays usable.
 */
int tpc_debug_wait_timeout(int32_t* status, int64_t timeout_ns, tpc_stream_t stream);

/* ------------------------------------------------------------------ index and bounds mode */
/*
 * Every kernel of this library indexes rows, chunks, boundary-state slots and replayed rows through
 * the plan's uploaded tables (HARTS Figure 2(c): the rounds' packed calls, the exported and imported
 * boundary states, the replay from the last aligned boundary).  With the mode on, each call that
 * reads those tables (KDA forward / backward / export, attention, the layer group, log-prob
 * recovery, MoE routing, the row maps) first bounds every index field of every table on the device
 * with one kernel and waits for it: a bad entry makes the call return TPC_ERR_DEVICE_CHECK (the
 * message names the table, the record and the bound) before any compute kernel is launched.  The
 * check reads only inside the tables.  The mode costs one launch and one host synchronisation per
 * call.  Off by default; the environment variable TPC_CHECKS=1 turns it on at the first call.
 */
void tpc_checks_enable(int on);
int tpc_checks_enabled(void);
/* Runs the table check once, whatever the mode: TPC_OK, TPC_ERR_DEVICE_CHECK or TPC_ERR_STATE
 * (tables not uploaded).  Synchronises `stream`. */
int tpc_plan_check_device(const tpc_plan* plan, tpc_stream_t stream);
/* The same checks on the host copy of the tables (no GPU, no upload needed), with word `word` of
 * table `table` (numbering of tpc_debug_poke_table) replaced by `value` when table >= 0: TPC_OK or
 * TPC_ERR_DEVICE_CHECK (same message as the device check); TPC_ERR_BAD_SHAPE for a word outside
 * the table. */
int tpc_plan_check_host(const tpc_plan* plan, int32_t table, int64_t word, int32_t value);
/*
 * Test hook: overwrites int32 word `word` of uploaded table `table` (blob order: 0 sequences
 * (8 words per record), 1 chunks (8), 2 slots (4), 3 slot consumers, 4 root-consumer offsets,
 * 5 root consumers, 6 replayed rows, 7 replay-target rows, 8 target offsets, 9 target parts,
 * 10 row-to-target map, 11 expanded rows, 12 occurrence offsets, 13 occurrence list,
 * 14 occurrence counts, 15 attention nodes (8), 16 attention ranges (2), 17 query tiles (4),
 * 18 key tiles (4)) with `value`, returning the previous value in *old_value (may be NULL).
 * `table` and `word` are checked against the plan on the host (TPC_ERR_BAD_SHAPE).  Synchronises
 * `stream`.  A plan whose tables were changed this way is only safe to use with the mode on.
 */
int tpc_debug_poke_table(tpc_plan* plan, int32_t table, int64_t word, int32_t value, int32_t* old_value,
                         tpc_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* TPC_H_ */
