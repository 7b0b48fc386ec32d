/*
 * recsa.h -- C ABI of the B200 (sm_100a) RecSA hot path.
 *
 * Recursive Sparse Attention ("Recursive Sparse Attention: Million-Token Length
 * Extrapolation at Logarithmic Cost", abstract) keeps a tree over one layer's
 * KV cache.  Every node summarises its span with one key, pooled by one
 * per-layer pooler shared by all levels, and one mean-pooled value.  A query
 * walks the tree top-down keeping at most k candidates per level; the
 * summaries of the unselected candidates join the exact tokens of the kept
 * leaf blocks and of a local window in one softmax, and every entry is rotated
 * (RoPE) to its index among the candidates of its level.
 *
 * Conventions for every entry point:
 *   - All tensors are caller-owned device memory; the library allocates
 *     nothing, and its only global state is the fixed scratch array of
 *     recsa_prefill_static.  Pointers to K, V, Q, O, k_new, v_new
 *     must be 16-byte aligned, the tree 256-byte aligned.
 *   - Layouts are row-major:
 *       K, V          [batch][n_kv_heads][capacity][head_dim]   (dtype)
 *       Q, O          [batch][n_q][n_q_heads][head_dim]         (dtype)
 *       k_new, v_new  [batch][n_kv_heads][head_dim]             (dtype)
 *       pooler_r      [n_kv_heads][n_ref][head_dim] fp32 with a head stride
 *                     in elements (0 = one set shared by every KV head);
 *                     n_ref = 1 unless the geometry sets n_ref > 1
 *       len           int64 [batch]: tokens currently in each sequence
 *     Query head h reads KV head h / (n_q_heads / n_kv_heads).
 *   - Work is enqueued on `stream` (a cudaStream_t, 0 = legacy default) and
 *     runs asynchronously.  Argument and launch errors are returned at once;
 *     errors found on the device (a full cache on append) set a flag in the
 *     tree header, read with recsa_tree_error().
 *   - Inputs are assumed finite.
 */
#ifndef RECSA_H_
#define RECSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum recsa_status {
  RECSA_OK = 0,
  RECSA_ERR_INVALID_GEOMETRY = 1, /* a geometry field is out of range */
  RECSA_ERR_NULL = 2,             /* a required pointer is NULL */
  RECSA_ERR_MISALIGNED = 3,       /* a pointer breaks the alignment rule */
  RECSA_ERR_CAPACITY = 4,         /* a length or query range exceeds capacity */
  RECSA_ERR_UNSUPPORTED = 5,      /* valid geometry outside the kernels' limits */
  RECSA_ERR_CUDA = 6,             /* a CUDA runtime call or launch failed */
  RECSA_ERR_DEVICE = 7            /* the tree header carries a device error */
} recsa_status;

enum { RECSA_DTYPE_F32 = 0, RECSA_DTYPE_BF16 = 1 };

/* k value meaning "keep every candidate" (the shared softmax then covers every
 * token up to the query: dense causal attention). */
#define RECSA_KEEP_ALL 2147483647

/* Deepest tree the kernels walk (levels of summaries above the tokens). */
#define RECSA_MAX_LEVELS 16
/* Largest k for which a selection trace is recorded. */
#define RECSA_TRACE_MAX_K 64

/* recsa_geometry.mode */
#define RECSA_MODE_RECSA 0
#define RECSA_MODE_ZHA 1
#define RECSA_MODE_GROUP 2

/* recsa_geometry.key_format: storage of the summary keys */
#define RECSA_KEYS_F32 0 /* fp32 rows */
#define RECSA_KEYS_FP8 1 /* FP8 E4M3 codes with one fp32 scale per row (ZHA mode only) */
#define RECSA_KEYS_NVFP4 2 /* E2M1 codes, E4M3 scale per 16, fp32 scale per row (ZHA only) */

/* Device error flags in the tree header (recsa_tree_error). */
#define RECSA_DEVERR_APPEND_FULL 0x1u /* recsa_append on a full sequence */
#define RECSA_DEVERR_WAIT_TIMEOUT 0x2u /* a bounded wait of the decode kernel on its own
                                         asynchronous copies expired (the output of
                                         that launch is not valid) */

/*
 * Tree geometry and attention shape.
 *   leaf_block (B): tokens per level-1 node.  branching (b): children per node
 *   above level 1.  A level-l node spans B * b^(l-1) tokens; only complete nodes
 *   exist, so a cache of T tokens holds floor(T / (B b^(l-1))) level-l nodes
 *   ("Subquadratic Attention with a Hierarchical Tree-Structured Indexer",
 *   Table VIII), and a level exists while it holds at least one node.
 *   k: candidates kept per level (RecSA abstract); RECSA_KEEP_ALL keeps all.
 *   window (W >= 1): the exact local window.  For a query at position t it is
 *   [a*B, t] with a = floor(max(0, t + 1 - W) / B), and only nodes whose span
 *   ends at or before a*B are visible to that query.
 *   rope_enabled / rope_base: rotate-half RoPE at candidate-local indices
 *   (RecSA abstract), inverse frequencies base^(-2j/d).
 *   mode: RECSA_MODE_RECSA (the method above) or RECSA_MODE_ZHA, the routing
 *   variant of "Subquadratic Attention with a Hierarchical Tree-Structured
 *   Indexer" (Figure 3): the same tree and candidates, but each level expands
 *   the smallest set of highest-scoring candidates whose softmax mass reaches
 *   top_p (at most k of them), scores are q . key / sqrt(d) without rotation,
 *   and the attention covers only the tokens of the reached leaves and the
 *   window, at their true positions with standard RoPE (no summaries; the
 *   tree's RoPE table then covers every position, so capacity < 2^24, else
 *   RECSA_ERR_UNSUPPORTED); or
 *   RECSA_MODE_GROUP, RecSA with one selection per KV group (the "per KV
 *   group" convention of the same page's Table IX): the G query heads of a
 *   KV head score the shared candidates with their own RecSA logits, a
 *   candidate's group score is the sum over the G heads of its softmax
 *   probability among the level's candidates, the top min(k, c) group scores
 *   are kept (ties -> lower index) for all G heads, and each head then
 *   attends as in RecSA.
 *   n_ref: with R = n_ref > 1 (ZHA mode only) every node holds R keys, one per
 *   reference query of the pooler, and a node's routing score is the largest
 *   of its R scores q . key_j / sqrt(d).
 *   key_format: RECSA_KEYS_FP8 (ZHA mode only) stores every summary key row
 *   as FP8 E4M3 codes (OCP format, ties to even, saturated at +-448) of
 *   key / scale with scale = max|key| / 448 in fp32: a low-precision router
 *   key cache ("Subquadratic Attention with a Hierarchical Tree-Structured
 *   Indexer", Figure 16 caption).  A parent key pools its children's stored
 *   (decoded) keys; values stay fp32; the routing score is
 *   scale * (q . codes) / sqrt(d).  RECSA_KEYS_NVFP4 stores E2M1 codes (two
 *   per byte, the lower element in the low nibble) with one E4M3 scale per 16
 *   elements and one fp32 scale per row: row scale = max|key| / (6 * 448),
 *   block scale = E4M3(block max / (6 * row scale)), code = E2M1(key /
 *   (block scale * row scale)), nearest, ties to even, saturated.
 */
typedef struct recsa_geometry {
  int32_t dtype;        /* RECSA_DTYPE_F32 or RECSA_DTYPE_BF16: K, V, Q, O, k_new, v_new */
  int32_t head_dim;     /* d: 64 or 128 */
  int32_t n_q_heads;    /* query heads */
  int32_t n_kv_heads;   /* KV heads; n_q_heads / n_kv_heads in {1, 2, 4, 8} */
  int32_t leaf_block;   /* B, 1..1024 */
  int32_t branching;    /* b, 2..64 */
  int32_t k;            /* 1..RECSA_KEEP_ALL */
  int32_t window;       /* W >= 1 */
  int32_t rope_enabled; /* 0 or 1 */
  float rope_base;      /* > 1 */
  int32_t batch;        /* sequences, >= 1 */
  int32_t mode;         /* RECSA_MODE_RECSA (0), RECSA_MODE_ZHA (1), RECSA_MODE_GROUP (2) */
  int64_t capacity;     /* tokens each sequence's K/V cache (and tree) can hold, < 2^31 */
  float top_p;          /* ZHA: routing mass in (0, 1]; ignored in RECSA mode */
  int32_t n_ref;        /* reference queries per pooler: 0 or 1 = one; 2..64 (ZHA mode only) */
  int32_t key_format;   /* RECSA_KEYS_F32, _FP8 or _NVFP4 (the last two: ZHA mode only) */
  int32_t reserved;     /* must be 0 */
} recsa_geometry;

/* Human-readable name of a status code (static string). */
const char* recsa_status_string(recsa_status s);

/* Check a geometry without touching the device. */
recsa_status recsa_validate(const recsa_geometry* geom);

/* Summary levels a cache of `length` tokens holds under `geom` (0 if length < B). */
recsa_status recsa_num_levels(const recsa_geometry* geom, int64_t length, int32_t* levels);

/*
 * Bytes of the tree buffer for `geom` at its capacity: a 256-byte header
 * (device error flags), the RoPE cos/sin table of the indices a traversal can
 * reach, and per level l: keys [batch][n_kv_heads][n_l][n_ref][head_dim] and
 * values [batch][n_kv_heads][n_l][head_dim] in fp32, n_l the level's node
 * count at capacity.  With RECSA_KEYS_FP8 the keys are one byte per element,
 * followed by their fp32 scales [batch][n_kv_heads][n_l][n_ref]; with
 * RECSA_KEYS_NVFP4 half a byte per element, then the E4M3 block scales
 * [batch][n_kv_heads][n_l][n_ref][head_dim / 16], then the fp32 row scales.
 */
recsa_status recsa_tree_bytes(const recsa_geometry* geom, size_t* bytes);

/*
 * Build the tree (RecSA abstract: one key and one mean-pooled value per node).
 * For each sequence s, every complete node over its first len_host[s] tokens
 * is written: level 1 pools each leaf block of B tokens, level l > 1 pools b
 * consecutive level-(l-1) summary keys ("Subquadratic Attention with a
 * Hierarchical Tree-Structured Indexer", Figure 3).  Pooling: weights =
 * softmax_i(r . k_i / sqrt(d)), key = sum_i weight_i k_i; value = mean of the
 * children's values.  With n_ref > 1 reference queries r_1..r_R the keys of
 * each are built in parallel (ZHA, Figure 3 caption): reference j's parent
 * key pools reference j's child keys.  Also clears the error flags and writes
 * the RoPE table.
 *   len_host: HOST int64 [batch], each in [0, capacity].
 */
recsa_status recsa_build(const recsa_geometry* geom, const void* K, const void* V,
                         const int64_t* len_host, const float* pooler_r,
                         int64_t pooler_head_stride, void* tree, void* stream);

/*
 * Append one token per sequence (decode-time tree maintenance): writes k_new,
 * v_new at position len_dev[s] of K and V, increments len_dev[s], and, when the
 * token completes a leaf block, pools that leaf and every ancestor it
 * completes (the cost is amortised over node completions: ZHA, Table VIII).
 * A sequence already at capacity is left unchanged and sets
 * RECSA_DEVERR_APPEND_FULL.
 *   len_dev: DEVICE int64 [batch].
 */
recsa_status recsa_append(const recsa_geometry* geom, void* K, void* V, const void* k_new,
                          const void* v_new, int64_t* len_dev, const float* pooler_r,
                          int64_t pooler_head_stride, void* tree, void* stream);

/*
 * Decode attention: n_q queries per sequence, all at position len_dev[s] - 1
 * (the newest token, already appended).  O[s][i][h] = RecSA output of
 * Q[s][i][h].  Sequences with len_dev[s] == 0 get O = 0.
 *   trace: NULL, or DEVICE int32 [batch][n_q][n_q_heads][recsa_trace_ints()]
 *   (requires k <= RECSA_TRACE_MAX_K).
 */
recsa_status recsa_decode(const recsa_geometry* geom, const void* Q, const void* K,
                          const void* V, const void* tree, const int64_t* len_dev,
                          int32_t n_q, void* O, int32_t* trace, void* stream);

/*
 * One decode step in a single launch: recsa_append of k_new, v_new followed by
 * recsa_decode of the n_q queries at the new token's position, with the same
 * results (the new token is read from k_new/v_new by the attention, written
 * to K/V, and the leaf and ancestors it completes are pooled; none of those
 * nodes is visible to the step's own query, whose window holds them).  A
 * sequence at capacity is flagged (RECSA_DEVERR_APPEND_FULL) and decoded
 * without the append, as the two separate calls would do.
 *   len_dev: DEVICE int64 [batch], incremented for every appended sequence.
 *   Per-sequence step counters live in the tree header (zeroed by
 *   recsa_build); for batch > 48 the step runs as the two separate launches.
 *   Steps on one tree must not overlap on the device.
 */
recsa_status recsa_decode_step(const recsa_geometry* geom, const void* Q, void* K, void* V,
                               const void* k_new, const void* v_new, int64_t* len_dev,
                               const float* pooler_r, int64_t pooler_head_stride, void* tree,
                               int32_t n_q, void* O, int32_t* trace, void* stream);

/*
 * Prefill attention: query i of sequence s sits at position q_start + i,
 * i < n_q, causal.  The tree must have been built over at least q_start + n_q
 * tokens of every sequence (a node is a pure function of its span, so a tree
 * built over more tokens serves every earlier query: each query sees only the
 * nodes that end before its window).
 *   workspace: NULL, or DEVICE memory of at least
 *   recsa_prefill_workspace_bytes(geom, n_q) bytes (16-byte aligned) given as
 *   workspace_bytes.  With a workspace and bf16 data the exact window runs on
 *   the tensor cores and its partial softmax (per query head an fp32 row of
 *   head_dim + 2: the window's normalised output, max and sum) is kept there
 *   until the tree kernel merges it and writes O once; without one, the window
 *   is attended by the tree kernel itself.  Both give the same result within
 *   rounding.  This holds in RECSA_MODE_RECSA and RECSA_MODE_ZHA (both attend
 *   the window at true distances); RECSA_MODE_GROUP ignores the workspace.
 *   The workspace is only read and written by this call; calls that share one
 *   must not overlap on the device.
 */
recsa_status recsa_prefill(const recsa_geometry* geom, const void* Q, const void* K,
                           const void* V, const void* tree, int64_t q_start, int32_t n_q,
                           void* O, int32_t* trace, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * recsa_prefill without a workspace argument, for callers that cannot hand
 * the library any device memory beyond the call's tensors: a runtime whose
 * device memory is planned ahead and owned by its own arena, or a C host with
 * no device allocator on its call path.  (The pages have no counterpart: it
 * is a packaging variant of recsa_prefill, same arguments and result.)
 *   Scratch: the window partials live in a fixed 4 MiB device array, which
 *   every GPU that loads the library holds until the process exits.  A call
 *   needs batch * n_q * n_q_heads * (head_dim + 2) * 4 bytes of it (8065 query
 *   heads at head_dim 128, e.g. 252 queries of 32 heads); a larger call is
 *   rejected with RECSA_ERR_CAPACITY (and a message on stderr): split the
 *   query range.  RECSA_MODE_ZHA uses no window partials and no scratch.
 *   The array needs no clearing (each call writes what it reads), but every
 *   call shares it: calls that overlap on the device race.
 *   Set-up: every call made outside stream capture looks up the array's
 *   device address on the current device (so a call after a device reset,
 *   which reloads the library's module, finds the array again); a call during
 *   capture uses the address found by the last call outside capture on that
 *   device, so make the first call on each device before any stream capture
 *   (a device never called outside capture is refused with RECSA_ERR_CUDA).
 *   Nothing is allocated by this call.
 */
recsa_status recsa_prefill_static(const recsa_geometry* geom, const void* Q, const void* K,
                                  const void* V, const void* tree, int64_t q_start, int32_t n_q,
                                  void* O, int32_t* trace, void* stream);

/* Workspace bytes recsa_prefill needs for n_q queries per sequence. */
recsa_status recsa_prefill_workspace_bytes(const recsa_geometry* geom, int32_t n_q,
                                           size_t* bytes);

/*
 * Trace record length in int32 per (sequence, query, head):
 *   [0] visible levels  [1] softmax entries  [2] keys read  [3] exact tokens
 *   [4 + l - 1]                      candidates at level l   (l = 1..16)
 *   [4 + 16 + l - 1]                 kept at level l
 *   [4 + 32 + (l - 1) * k + j]       j-th kept node id at level l, in position order
 */
recsa_status recsa_trace_ints(const recsa_geometry* geom, int32_t* ints);

/*
 * Re-read the environment switches that force a kernel variant (the tests use
 * them to run every kernel of a call on the same inputs):
 *   RECSA_DECODE_GENERIC, RECSA_PREFILL_GENERIC, RECSA_ZHA_GENERIC   (set: use
 *     the generic one-CTA-per-query kernel), RECSA_DECODE_SPLIT="hpc,s" (decode
 *     launch shape: query heads per CTA, candidate shares per head group),
 *     RECSA_PREFILL_PATH (unset or 0: automatic; 1: the CUDA-core paths only --
 *     the prefill's kept leaves attended by its traversal kernel, several
 *     reference queries pooled by warps; 2: the tensor-core kept-leaf path
 *     with the warp-per-query-head traversal; 3: the tensor-core kept-leaf
 *     path with the tree levels as tensor-core tiles, the automatic choice
 *     when the geometry and the workspace allow it),
 *     RECSA_TEST_EXPIRE_WAIT (set: the decode kernel ends with a bounded wait
 *     that nothing completes, to test the timeout status).
 * The library reads them once, at its first call; this entry point makes a
 * change of the environment take effect.  It must not run concurrently with
 * other calls into the library.  Not part of the method (no passage defines it).
 */
void recsa_reload_switches(void);

/* Read (and optionally clear) the device error flags of a tree; synchronises `stream`. */
recsa_status recsa_tree_error(const recsa_geometry* geom, void* tree, int32_t clear,
                              uint32_t* flags, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RECSA_H_ */
