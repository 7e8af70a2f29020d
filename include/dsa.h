/*
 * dsa.h -- C ABI of the DeepSeek Sparse Attention (DSA) forward path on one
 * NVIDIA B200 (sm_100a).
 *
 * DSA replaces dense causal attention by three steps per query token
 * (DeepSeek-V3.2-Exp report read-through on 53ai.com, section "Innovative
 * architecture: core design of DSA", and its Figure 1):
 *   1. a lightning indexer scores the query against every preceding token:
 *        I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]),   s <= t,
 *      multi-head and ReLU-gated, with FP8 inputs;
 *   2. fine-grained selection keeps the k best-scoring tokens (k = 2048 in
 *      DeepSeek-V3.2: paperbridge.wiki summary, section "DeepSeek Sparse
 *      Attention"; juhe.plus read-through, step 2);
 *   3. attention runs in MLA's MQA mode -- one latent KV row shared by all
 *      query heads -- over the selected rows only.
 *
 * Conventions shared by every call
 *   - Every tensor pointer is a DEVICE pointer owned by the caller. The
 *     library never allocates device memory on these paths; scratch space is
 *     the caller's workspace, sized by dsa_workspace_size(). The one
 *     exception is dsa_select_noalloc, which takes no workspace and keeps its
 *     score rows in a fixed 16 MiB scratch array that the library holds on
 *     each GPU that loads it (see its declaration).
 *   - Every call is asynchronous on the given CUDA stream (a cudaStream_t;
 *     NULL is the legacy default stream). Host-side argument checks run before
 *     any launch and return an error without launching anything. A call's
 *     first kernel starts after all earlier work on the stream; inside one
 *     dsa_select / dsa_select_noalloc / dsa_forward the indexer and top-k
 *     launches may overlap one another's start-up (programmatic dependent
 *     launch), never their reads and writes of shared buffers, and the work
 *     after the call sees all of its results.
 *   - Errors found on the device (an index or page id out of range, a bounded
 *     wait that ran out) are recorded in a per-device status word; read it
 *     with dsa_check_status(), which synchronises the stream. Device code
 *     never traps: bad indices are skipped (treated as masked) and reported.
 *   - Positions. CONTIGUOUS layout: keys are rows 0..n_keys-1 of one
 *     sequence and query i sits at position n_keys - n_q + i (n_q == n_keys is
 *     a plain prefill; n_q < n_keys is a chunk of a longer prefill). PAGED
 *     layout: query i belongs to sequence b = q_seq ? q_seq[i] : i, whose
 *     ctx_lens[b] cached tokens include the query's own, and sits at position
 *     q_pos ? q_pos[i] : ctx_lens[b] - 1. In both cases the query sees keys
 *     0..pos of its sequence (inclusive: the pages say "preceding tokens"; the
 *     token itself is kept so that every row has at least one key). A query
 *     whose sequence, length or position is out of range is reported as
 *     DSA_ERR_DEVICE_BOUNDS and gets an empty selection.
 *   - Supported combinations (others return DSA_ERR_UNSUPPORTED):
 *       E4M3 indexer (H_I=64, d_I=128) + BF16 attention (H=128, d_qk=576,
 *       d_v=512, V = first 512 columns of the KV row), CONTIGUOUS or PAGED
 *       with 64-token pages;
 *       F32 indexer (H_I<=64, d_I<=128, d_I%4==0) + F32 attention (H<=128,
 *       d_qk<=256, d_v<=256, separate V allowed), CONTIGUOUS only.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

/* A cudaStream_t. */
typedef struct CUstream_st* dsa_stream_t;

typedef enum dsa_status {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,          /* null pointer, bad size/stride/alignment, k out of [1,2048] */
  DSA_ERR_UNSUPPORTED = 2,          /* dtype/dims/layout combination not built */
  DSA_ERR_WORKSPACE_TOO_SMALL = 3,  /* ws_bytes < dsa_workspace_size() */
  DSA_ERR_CUDA = 4,                 /* a CUDA runtime call failed; see dsa_last_cuda_error() */
  DSA_ERR_DEVICE_BOUNDS = 5,        /* device saw an index/page id out of range (skipped) */
  DSA_ERR_TIMEOUT = 6               /* a bounded device wait ran out; results are invalid */
} dsa_status;

typedef enum dsa_dtype {
  DSA_F32 = 0,   /* float32 */
  DSA_E4M3 = 1,  /* OCP FP8 e4m3 codes (uint8) + one float32 scale per token */
  DSA_BF16 = 2   /* bfloat16 */
} dsa_dtype;

typedef enum dsa_kv_kind {
  DSA_KV_CONTIGUOUS = 0,
  DSA_KV_PAGED = 1
} dsa_kv_kind;

/* Where the keys live. For PAGED, logical token p of sequence b is slot
 * p % page_size of page block_table[b * ld_block_table + p / page_size].
 * A PAGED query belongs to one sequence and sits at one position in it (see
 * "Positions" above): with q_seq and q_pos NULL, query b is the newest token
 * of sequence b (decode); with them, several queries may share a sequence
 * (multi-token decode, a chunk of a prefill against the paged cache). */
typedef struct dsa_kv_layout {
  int32_t kind;                 /* dsa_kv_kind */
  int32_t page_size;            /* PAGED: tokens per page, must be 64 */
  const int32_t* block_table;   /* PAGED: device [n_seq, ld_block_table] page ids */
  int64_t ld_block_table;       /* PAGED: elements between rows of block_table */
  int32_t max_pages;            /* PAGED: columns of block_table usable per row */
  int32_t num_pages;            /* PAGED: pages in the caches (page ids must be < this) */
  const int32_t* ctx_lens;      /* PAGED: device [n_seq] cached tokens per sequence, in [1, max_pages*page_size] */
  const int32_t* q_seq;         /* PAGED, nullable: device [n_q] sequence of each query, in [0, n_seq) (NULL: query b -> sequence b) */
  const int32_t* q_pos;         /* PAGED, nullable: device [n_q] position of each query in its sequence, in [0, ctx_lens[seq]) (NULL: ctx_lens[seq] - 1) */
  int32_t n_seq;                /* PAGED: sequences (rows of block_table, entries of ctx_lens); 0 means n_q. Without q_seq, n_seq >= n_q */
} dsa_kv_layout;

/* Indexer inputs (step 1). Token-major rows; all strides in ELEMENTS.
 * E4M3: q/k hold e4m3 codes, the real value of an entry is
 *       decode(code) * q_scale[token] (resp. k_scale[key token]), scales > 0.
 * F32 : q/k hold the real values; q_scale/k_scale must be NULL. */
typedef struct dsa_indexer_in {
  int32_t dtype;        /* DSA_E4M3 or DSA_F32 */
  int32_t n_q;          /* query tokens */
  int32_t n_keys;       /* CONTIGUOUS: key tokens (>= n_q); PAGED: ignored */
  int32_t heads;        /* H_I */
  int32_t dim;          /* d_I */
  const void* q;        /* [n_q, heads, dim]; heads contiguous within a token */
  int64_t ld_q;         /* elements between query tokens (>= heads*dim) */
  const float* q_scale; /* E4M3: [n_q] */
  const void* k;        /* CONTIGUOUS: [n_keys, dim]; PAGED: [num_pages, page_size, dim] */
  int64_t ld_k;         /* elements between key tokens (>= dim) */
  const float* k_scale; /* E4M3: CONTIGUOUS [n_keys]; PAGED [num_pages * page_size] */
  const float* w;       /* [n_q, heads] per-query head weights */
  int64_t ld_w;         /* elements between query tokens of w (>= heads) */
  dsa_kv_layout kv;
} dsa_indexer_in;

/* Attention inputs (step 3). V defaults to the first d_v columns of each KV
 * row (MLA latent); a separate V is accepted for F32 only. */
typedef struct dsa_attn_in {
  int32_t dtype;        /* DSA_BF16 or DSA_F32 */
  int32_t n_q;          /* query tokens (same as the indexer's) */
  int32_t n_keys;       /* CONTIGUOUS: KV rows; PAGED: ignored */
  int32_t heads;        /* H */
  int32_t d_qk;         /* key/query width */
  int32_t d_v;          /* value width */
  float scale;          /* softmax scale on q.k (e.g. 1/sqrt(d_qk)) */
  const void* q;        /* [n_q, heads, d_qk], heads contiguous */
  int64_t ld_q;         /* elements between query tokens (>= heads*d_qk) */
  const void* kv;       /* CONTIGUOUS: [n_keys, d_qk]; PAGED: [num_pages, page_size, d_qk] */
  int64_t ld_kv;        /* elements between KV rows (>= d_qk) */
  const void* v;        /* NULL, or F32 only: [n_keys, d_v] */
  int64_t ld_v;
  dsa_kv_layout kv_layout;
} dsa_attn_in;

typedef enum dsa_op {
  DSA_OP_INDEXER_SCORES = 0,
  DSA_OP_TOPK = 1,
  DSA_OP_SPARSE_MQA = 2,
  DSA_OP_FORWARD = 3,
  DSA_OP_SELECT = 4
} dsa_op;

/* Step 1 alone: lightning-indexer scores for selected query rows.
 * Row r of `scores` (row stride ld_scores floats) belongs to query
 * rows ? rows[r] : r (device array, values in [0, n_q)). Columns 0..n_cols-1
 * are written: the score for keys s <= pos(query), -INFINITY for s > pos.
 * Scores are float32 and bit-identical to those the fused dsa_forward ranks.
 * Requires n_cols >= 1, ld_scores >= n_cols; for PAGED n_cols <=
 * max_pages*page_size. ws / ws_bytes are reserved and unused by this version
 * (dsa_workspace_size(DSA_OP_INDEXER_SCORES) is 0): pass NULL / 0. */
DSA_API dsa_status dsa_indexer_scores(const dsa_indexer_in* in, const int32_t* rows,
                                      int32_t n_rows, float* scores, int64_t ld_scores,
                                      int32_t n_cols, void* ws, size_t ws_bytes,
                                      dsa_stream_t stream);

/* Step 2 alone: exact top-k of each score row.
 * Row r considers scores[r*ld_scores + s] for s in [0, row_pos[r]] (device
 * array). It keeps the min(k, row_pos[r]+1) entries with the largest score,
 * ties to the lower s, -0.0 equal to +0.0, NaN below every number, and writes
 * their s in ascending order to idx[r*ld_idx + 0..], padding with -1 up to k.
 * Needs no workspace. 1 <= k <= 2048; 0 <= row_pos[r] < 2^31-1. */
DSA_API dsa_status dsa_topk(const float* scores, int64_t ld_scores, const int32_t* row_pos,
                            int32_t n_rows, int32_t k, int32_t* idx, int64_t ld_idx,
                            dsa_stream_t stream);

/* Step 3 alone: sparse MQA attention.
 * For query i, idx[i*ld_idx + 0..k-1] lists key positions (logical positions
 * for PAGED); entries < 0 are skipped, entries > pos(query) are reported as
 * DSA_ERR_DEVICE_BOUNDS and skipped. Every row must hold at least one valid
 * entry. out: [n_q, heads, d_v] contiguous, same dtype as q; lse: [n_q, heads]
 * float32 natural-log log-sum-exp of the scaled logits (may be NULL).
 * ws / ws_bytes are reserved and unused by this version
 * (dsa_workspace_size(DSA_OP_SPARSE_MQA) is 0): pass NULL / 0. */
DSA_API dsa_status dsa_sparse_mqa_fwd(const dsa_attn_in* in, const int32_t* idx, int64_t ld_idx,
                                      int32_t k, void* out, float* lse, void* ws,
                                      size_t ws_bytes, dsa_stream_t stream);

/* Dense causal MLA-MQA attention: the baseline that DSA replaces, in which
 * every query attends to all of its preceding tokens (paperbridge.wiki
 * summary, section on dense attention; the pages compare DSA's prefill and
 * decode cost per token position against it: juhe.plus read-through, sparse
 * training stage; 53ai.com read-through, Figure 3). Query i (position pos, as
 * in "Positions") attends to keys 0..pos with the same inputs and outputs as
 * dsa_sparse_mqa_fwd, as if its selection held every key. Results equal
 * dsa_sparse_mqa_fwd with idx = 0..pos (ascending) bit for bit when pos < k.
 * BF16: CONTIGUOUS or PAGED; a PAGED query with a page id out of range among
 * its pages is reported as DSA_ERR_DEVICE_BOUNDS and gets a zero output.
 * F32: CONTIGUOUS, n_keys <= 4096. No workspace. */
DSA_API dsa_status dsa_dense_mqa_fwd(const dsa_attn_in* in, void* out, float* lse,
                                     dsa_stream_t stream);

/* Steps 1-2 fused: the selection alone (indexer -> top-k), streamed over
 * bounded blocks of queries so the n_q x n_keys score matrix never exists.
 * idx: [n_q, ld_idx] int32 (ld_idx >= k), same contents and rules as
 * dsa_topk(dsa_indexer_scores(...)) bit for bit.
 * Workspace: dsa_workspace_size(DSA_OP_SELECT): one block of float32 score
 * rows, min(n_q, max(128, rows that fit in 80 MiB)) rows of n_keys (CONTIGUOUS)
 * or max_pages*page_size (PAGED) columns, so it does not grow with n_q. */
DSA_API dsa_status dsa_select(const dsa_indexer_in* indexer, int32_t k, int32_t* idx,
                              int64_t ld_idx, void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Steps 1-3 fused: indexer -> top-k -> sparse attention without ever holding
 * the n_q x n_keys score matrix (prefill streams the indexer over bounded
 * blocks of queries). idx_out (nullable, [n_q, k] int32) receives the
 * selection, identical to dsa_topk(dsa_indexer_scores(...)).
 * Workspace: dsa_workspace_size(DSA_OP_FORWARD). */
DSA_API dsa_status dsa_forward(const dsa_indexer_in* indexer, const dsa_attn_in* attn,
                               int32_t k, int32_t* idx_out, void* out, float* lse,
                               void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Steps 1-2 fused like dsa_select, also writing the indexer score of every
 * kept key: sel_scores[r*ld_sel + i] is the score of key idx[r*ld_idx + i]
 * (-INFINITY where idx is -1), the very value the selection ranked -- bit for
 * bit what dsa_indexer_scores gives for that key. These are the indexer-side
 * inputs of dsa_indexer_kl. Workspace as dsa_select. */
DSA_API dsa_status dsa_select_scored(const dsa_indexer_in* indexer, int32_t k, int32_t* idx,
                                     int64_t ld_idx, float* sel_scores, int64_t ld_sel,
                                     void* ws, size_t ws_bytes, dsa_stream_t stream);

/* The indexer's KL training signal over each query's selected keys. The
 * indexer is trained to match the main attention's distribution with a
 * KL-divergence loss, over every preceding key in the dense warm-up and with
 * only the top-k keys selected in sparse training (wiki-for-amaranth report,
 * section "DeepSeek Sparse Attention (DSA)"; juhe.plus read-through, stages
 * "Dense Warm-up" and "Sparse Training"; 53ai.com read-through, continued
 * pre-training). For query i with selected keys j (idx row i, entries < 0 or
 * past the query's position skipped):
 *   p_j = (1/H) sum_h exp(scale * q[i,h] . kv[key_j] - lse[i,h])  (main attention, heads averaged)
 *   r_j = softmax_j(sel_scores[i, j])                               (the indexer)
 *   loss[i] = sum_j p_j (log p_j - log r_j),  grad[i*ld_grad + j] = r_j - p_j (0 when skipped),
 * the gradient of the loss with respect to the indexer scores (p held fixed).
 * attn: the forward's attention inputs (BF16, H=128, d_qk=576, CONTIGUOUS or
 * PAGED); lse: [n_q, 128] the forward's log-sum-exp (dsa_sparse_mqa_fwd /
 * dsa_forward) of this selection; sel_scores: from dsa_select_scored. With a
 * selection of every key 0..pos (k >= pos + 1) this is the dense warm-up
 * signal. No workspace. */
DSA_API dsa_status dsa_indexer_kl(const dsa_attn_in* attn, const int32_t* idx, int64_t ld_idx,
                                  int32_t k, const float* lse, const float* sel_scores,
                                  int64_t ld_sel, float* loss, float* grad, int64_t ld_grad,
                                  dsa_stream_t stream);

/* Gradient of step 3 for sparse training: the main model is trained through
 * the attention over the selected keys only, the indexer's input being detached
 * (wiki-for-amaranth report, section "DeepSeek Sparse Attention (DSA)", stage
 * B), so no gradient reaches the selection. For query i (position
 * n_keys - n_q + i) with selected rows j (idx row i, entries < 0 skipped,
 * entries past the query's position reported as DSA_ERR_DEVICE_BOUNDS and
 * skipped), K_j = kv[key_j, 0:576], V_j = kv[key_j, 0:512] and the upstream
 * gradient dO = d loss / d out:
 *   P[h,j]  = exp(scale * q[i,h] . K_j - lse[i,h])
 *   D[h]    = dO[i,h] . out[i,h]   (its halves over value dims [0,256) and
 *             [256,512) written to delta[(i*128 + h)*2 + 0] and [... + 1])
 *   dZ[h,j] = scale * P[h,j] * (dO[i,h] . V_j - D[h])
 *   d_q[i,h]     = sum_j dZ[h,j] K_j                                  (written)
 *   d_kv[key_j] += sum_h dZ[h,j] q[i,h];  d_kv[key_j, 0:512] += sum_h P[h,j] dO[i,h]
 * (d_kv is ACCUMULATED: zero it first for a plain gradient).
 * in: the forward's attention inputs, BF16, H=128, d_qk=576, d_v=512,
 * CONTIGUOUS only (DSA_ERR_UNSUPPORTED otherwise). out, lse: the forward's
 * outputs for this selection; d_out: [n_q, 128, 512] bf16; d_q: [n_q, 128, 576]
 * bf16; out, d_out, d_q contiguous and 16-byte aligned. d_kv: float32 rows
 * ld_dkv >= 576 apart (columns 0..575 used); delta: [n_q, 128, 2] float32
 * scratch, written. The reductions into d_kv make its low-order bits depend
 * on the order in which queries finish. No workspace. */
DSA_API dsa_status dsa_sparse_mqa_bwd(const dsa_attn_in* in, const int32_t* idx, int64_t ld_idx,
                                      int32_t k, const void* out, const float* lse,
                                      const void* d_out, void* d_q, float* d_kv, int64_t ld_dkv,
                                      float* delta, dsa_stream_t stream);

/* Workspace bytes for `op` with these inputs (arguments an op does not use may
 * be NULL/0). The workspace must be 256-byte aligned device memory. */
DSA_API dsa_status dsa_workspace_size(int32_t op, const dsa_indexer_in* indexer,
                                      const dsa_attn_in* attn, int32_t n_rows, int32_t n_cols,
                                      int32_t k, size_t* bytes);

/* Synchronises `stream`, returns the first device-side error recorded on the
 * current device since the last call (DSA_OK if none) and clears it. */
DSA_API dsa_status dsa_check_status(dsa_stream_t stream);

/* Static description of a status code. */
DSA_API const char* dsa_status_string(dsa_status status);

/* The cudaError_t value behind the last DSA_ERR_CUDA on this thread (0 if none). */
DSA_API int32_t dsa_last_cuda_error(void);

/* Allocation-free form of dsa_select (the paper has no counterpart; this is a
 * service for callers that cannot allocate device memory).
 *
 * Some callers cannot hand this library a workspace: a plugin that a host
 * application (a serving engine, another language's runtime) loads and gives
 * only its input and output buffers, because the host owns every byte of
 * device memory through its own pool; or a latency-critical loop that must not
 * call cudaMalloc, which can synchronise the whole device. This entry point
 * takes no workspace and allocates nothing: its score rows live in a fixed
 * 16 MiB scratch array that the library keeps in device memory (one per GPU
 * that loads the library, held until the process exits).
 *
 * Same arguments and results as dsa_select (bit-identical idx), minus the
 * workspace. Query rows are processed in blocks that fit the scratch, so one
 * score row -- n_keys floats (CONTIGUOUS) or max_pages*page_size floats
 * (PAGED) -- must fit in 16 MiB, i.e. at most 4,194,304 keys; larger problems
 * return DSA_ERR_WORKSPACE_TOO_SMALL without launching anything.
 *
 * The first call on each device looks up the scratch array's device address
 * (with that device current); make that first call before any stream capture.
 * Every call on a device shares the one scratch array and leaves its last
 * contents in it; no call relies on what an earlier call left there. Calls
 * whose kernels overlap on the same device (other streams or threads) race on
 * the scratch and give wrong results: order them. */
#define DSA_NOALLOC_SCRATCH_BYTES (16u << 20)
DSA_API dsa_status dsa_select_noalloc(const dsa_indexer_in* indexer, int32_t k, int32_t* idx,
                                      int64_t ld_idx, dsa_stream_t stream);

/* Failure detection: every wait inside the kernels (on a TMA copy, an MMA, a
 * peer CTA) is bounded; a wait that runs out records DSA_ERR_TIMEOUT in the
 * device status word (read it with dsa_check_status), the waiting role gives
 * up, the kernel lets the copies and MMAs it already issued complete, frees its
 * tensor memory and returns -- the GPU context stays usable, but the results of
 * that call are invalid. No legitimate wait lasts more than microseconds.
 * This sets the bound of the lightning-indexer kernel's pipeline waits for
 * launches issued after the call (process-wide, all devices); ns <= 0 restores
 * the default of 1 second. The other kernels keep the 1 s bound. A bound far
 * below the copies' latency makes the indexer give up on purpose, which is
 * how the failure path is tested. */
DSA_API dsa_status dsa_set_wait_limit_ns(int64_t ns);

/* Number of kernel launches this process has issued through the library so
 * far (all devices, all threads). Lets a caller count launches in a region. */
DSA_API int64_t dsa_launch_counter(void);

/* Library version, major*10000 + minor*100 + patch. */
DSA_API int32_t dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
