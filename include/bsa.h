/*
 * bsa.h -- C ABI of libbsa: query-aware top-k block-sparse causal attention
 * on NVIDIA B200 (sm_100a).
 *
 * The method, as the source pages state it:
 *   - a cheap selector scores every KV block (or chunk gist) against the
 *     query -- "粗粒度 Block 打分" (coarse block scoring), 稀疏注意力 tutorial
 *     §4.6; SAS page, 核心模块 1; SSA page, 推理时的关键模块 1;
 *   - the top-k blocks are kept per query block or decode token, per KV-head
 *     group, with the current block always kept -- SAS page, 核心洞察 and
 *     核心模块 3 ("始终保留的当前块"), and its 推理 paragraph;
 *   - FlashAttention-style attention runs over the kept blocks only -- the
 *     tutorial §2 (real speed-up needs the skipped region never computed) and
 *     §7 (Block-Sparse FlashAttention);
 *   - the gated variant adds log g_j to the logits of every token of block j,
 *     g = softmax of the selector scores over the kept blocks -- SAS page,
 *     核心模块 2-3.
 *
 * Conventions shared by every call
 *   Layout     all tensors are dense and contiguous, head-major [B, H, N, d]
 *              with d innermost; block j of a sequence is tokens
 *              [j*block, (j+1)*block).  Query head h belongs to KV group
 *              h / (Hq/Hkv) (GQA grouping).
 *   Pointers   all data pointers are DEVICE pointers, 16-byte aligned, owned
 *              by the caller.  The library never allocates, frees or
 *              synchronises device memory on these paths; scratch space is
 *              passed in by the caller (see bsa_workspace_bytes).
 *   Streams    `stream` is a cudaStream_t (NULL = legacy default stream).
 *              Every compute call only enqueues work on it and returns.
 *   Errors     arguments are checked on the host before anything is launched:
 *              malformed -> BSA_ERR_INVALID_ARG, legal but not built ->
 *              BSA_ERR_UNSUPPORTED, a failed launch -> BSA_ERR_CUDA.  Nothing is
 *              enqueued when a check fails.  Device-side problems (an index
 *              out of range, a bounded wait that expired) never trap: the
 *              kernel records a flag in the device status word, skips the bad
 *              work and returns; read it with bsa_device_status().
 *   Threads    calls are thread-safe; the only global state is the tensor-map
 *              entry point, the device status word and the overrides of
 *              the testing hooks below.
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
  BSA_ERR_INVALID_ARG = 1,
  BSA_ERR_UNSUPPORTED = 2,
  BSA_ERR_CUDA = 3,
  BSA_ERR_TIMEOUT = 4,      /* device status: a bounded wait expired */
  BSA_ERR_DEVICE = 5        /* device status: bad index or shape seen by a kernel */
} bsa_status_t;

typedef enum { BSA_F32 = 0, BSA_BF16 = 1 } bsa_dtype_t;

/* Problem shape.  Nq = query tokens (prefill: Nq == Nk; decode: Nq == 1),
 * Nk = key/value tokens, block = KV block size (or gist chunk size). */
typedef struct {
  int B, Hq, Hkv, Nq, Nk, d, block;
  bsa_dtype_t dtype;
} bsa_shape_t;

/* selector modes for bsa_score_blocks */
enum { BSA_SCORE_PREFILL = 0, BSA_SCORE_DECODE = 1, BSA_SCORE_GIST = 2, BSA_SCORE_DECODE_HEADS = 3 };
/* candidate rules for bsa_topk_select */
enum { BSA_TOPK_CAUSAL_BLOCK = 0, BSA_TOPK_LAST_BLOCK = 1, BSA_TOPK_PLAIN = 2 };
/* operations for bsa_workspace_bytes */
enum { BSA_OP_DECODE = 0, BSA_OP_GIST_DECODE = 1, BSA_OP_DECODE_HEADS = 2 };

/*
 * bsa_score_blocks -- the cheap selector (block pooling + scoring).
 * Cite: 稀疏注意力 tutorial §4.5 (a block = consecutive tokens) and §4.6
 * (coarse block scoring instead of a full QK^T); SAS page 核心模块 1
 * (continuous per-unit score); SSA page 推理时的关键模块 1 (score the query
 * against every gist).  Score s = pooled-q . pooled-k / sqrt(d), in fp32 in
 * a fixed order: pooling sums heads ascending then tokens ascending and
 * divides once; the dot product runs over the channel ascending with every
 * product and sum rounded to fp32; then one multiply by fp32(1/sqrt(d)).
 *
 * mode BSA_SCORE_PREFILL  (dtype BF16 or F32, Nq == Nk, Nk % block == 0)
 *   q [B,Hq,Nq,d], k [B,Hkv,Nk,d]           (dtype)
 *   pooled_q_out [B,Hkv,nb,d] fp32          (required) group query means
 *   pooled_k_out [B,Hkv,nb,d] fp32          (required) block key means
 *   pooled_k_in                              must be NULL
 *   scores [B,Hkv,nb,nb] fp32: s[i][j] for j <= i, -inf for j > i.
 * mode BSA_SCORE_DECODE   (one query token per sequence)
 *   q [B,Hq,d]; pooled_k_in [B,Hkv,nb,d] fp32, the block-mean summary kept
 *   next to the KV cache.  If pooled_k_in is NULL, k [B,Hkv,Nk,d] is pooled
 *   into pooled_k_out (required then) first.
 *   pooled_q_out [B,Hkv,d] fp32 (optional) receives the group query means.
 *   scores [B,Hkv,nb] fp32.
 * mode BSA_SCORE_GIST     (SSA: per query head, no pooling)
 *   q [B,Hq,d]; k = gist keys [B,Hkv,nc,d] with nc = Nk/block;
 *   scores [B,Hq,nc] fp32.  pooled_* must be NULL.
 * mode BSA_SCORE_DECODE_HEADS  (one score row per query head, for a budget
 *   shared across the heads: Sparse Frontier review §2.3.2, Ada-KV)
 *   q [B,Hq,d] (d in {64,128}); pooled_k_in [B,Hkv,nb,d] fp32 (required);
 *   scores [B,Hq,nb] fp32: q_h . pooled_k_j / sqrt(d) in the same fixed
 *   order.  k, pooled_q_out and pooled_k_out must be NULL.
 */
bsa_status_t bsa_score_blocks(const bsa_shape_t* shape, int mode, const void* q, const void* k,
                              const float* pooled_k_in, float* pooled_q_out, float* pooled_k_out,
                              float* scores, void* stream);

/*
 * bsa_topk_select -- hard top-k selection of history blocks.
 * Cite: SAS page, 推理 paragraph (each query keeps the k highest-scoring
 * units) and 核心模块 3 (the current block is always kept); gated-sparse
 * essay §四, pseudo-code step 2 (top-k blocks form the sparse index).
 * scores [rows, ncols] fp32 (row-major).  Per row, candidates and the forced
 * block depend on `mode`:
 *   BSA_TOPK_CAUSAL_BLOCK  row r is query block i = r % ncols: candidates
 *                          j < i, block i always kept (prefill);
 *   BSA_TOPK_LAST_BLOCK    candidates j < ncols-1, block ncols-1 kept (decode);
 *   BSA_TOPK_PLAIN         candidates j < ncols, nothing forced (gist).
 * Order: larger score first, equal scores -> lower index first, NaN below
 * every number.  min(kb, #candidates) are kept.
 * idx_out [rows, idx_stride] int32: kept indices ascending, then -1;
 *   idx_stride >= kb + (mode != PLAIN).  count_out [rows] int32 (optional).
 * Limits: ncols <= 8192.
 */
bsa_status_t bsa_topk_select(const float* scores, int rows, int ncols, int mode, int kb,
                             int* idx_out, int idx_stride, int* count_out, void* stream);

/*
 * bsa_topk_select_pattern -- prefill selection with a fixed part and a
 * dynamic part.
 * Cite: Sparse Frontier review §2.2.3 (MInference block-sparse: each query
 * block keeps the local blocks, the first block and a set of dynamically
 * selected blocks; StreamingLLM's attention sinks: the first tokens) and its
 * §3.2 method table (局部 + 首块 + 动态选择块).
 * scores [rows, ncols] as for BSA_TOPK_CAUSAL_BLOCK (row r is query block
 * i = r % ncols).  Kept for row r: blocks j < sink (j <= i), the `local` most
 * recent blocks i-local < j <= i (current included), and the kb best of the
 * blocks in between by the order of bsa_topk_select.  sink >= 0, local >= 1,
 * kb >= 0.  idx_out [rows, idx_stride], idx_stride >= sink + local + kb:
 * kept blocks ascending, then -1; count_out [rows] (optional).
 * Limits: ncols <= 8192.  With sink = 0 and local = 1 it is
 * bsa_topk_select(BSA_TOPK_CAUSAL_BLOCK).
 */
bsa_status_t bsa_topk_select_pattern(const float* scores, int rows, int ncols, int sink, int local, int kb,
                                     int* idx_out, int idx_stride, int* count_out, void* stream);

/*
 * bsa_topk_select_joint_heads -- decode selection under one budget shared by
 * the query heads of a KV group.
 * Cite: Sparse Frontier review §2.3.2 (Ada-KV: the top (k x h) units over
 * all h heads, so important heads keep more keys and others fewer).
 * scores [rows, heads, ncols] fp32: per-head decode scores of one (batch, KV
 * group) row each (bsa_score_blocks mode BSA_SCORE_DECODE_HEADS).  Candidates:
 * the pairs (h, j), j < ncols-1; the kb_total best are kept (equal scores:
 * the lower h*(ncols-1)+j first; NaN below every number); the last block
 * ncols-1 is kept by every head.  idx_out [rows, heads, idx_stride]: each
 * head's kept blocks ascending, then -1, idx_stride >= min(kb_total,
 * ncols-1) + 1; count_out [rows, heads] (optional).
 * Limits: heads <= 16, heads*(ncols-1) <= 8192.  With one head it is
 * bsa_topk_select(BSA_TOPK_LAST_BLOCK).
 */
bsa_status_t bsa_topk_select_joint_heads(const float* scores, int rows, int heads, int ncols, int kb_total,
                                         int* idx_out, int idx_stride, int* count_out, void* stream);

/*
 * bsa_decode_select -- the decode selector in one call: the group query
 * mean, its scores against the pooled-key summary kept next to the cache,
 * and the top-kb history blocks with the last block kept.
 * Cite: 稀疏注意力 tutorial §4.6 (coarse block scoring) and §5 (decode: one
 * new query against the history); SAS page, 推理 paragraph (the k best units
 * kept) and 核心模块 3 (the current block always kept).
 * Results equal bsa_score_blocks(BSA_SCORE_DECODE, pooled_k_in = pooled_k)
 * followed by bsa_topk_select(BSA_TOPK_LAST_BLOCK) bit for bit; with d = 128
 * and at most 2048 blocks they come from one kernel that keeps the scores
 * on chip between the two steps.
 * q [B,Hq,d] (dtype); pooled_k [B,Hkv,nb,d] fp32 with nb = Nk/block; Nq = 1.
 * scores [B,Hkv,nb] fp32 (required, written); idx_out [B,Hkv,idx_stride]
 * int32, idx_stride >= kb + 1; count_out [B,Hkv] int32 and pooled_q_out
 * [B,Hkv,d] fp32 are optional.  Limits: nb <= 8192.
 */
bsa_status_t bsa_decode_select(const bsa_shape_t* shape, const void* q, const float* pooled_k, int kb,
                               float* pooled_q_out, float* scores, int* idx_out, int idx_stride,
                               int* count_out, void* stream);

/*
 * bsa_sparse_attn_prefill -- block-sparse causal attention (prefill).
 * Cite: 稀疏注意力 tutorial §1 (softmax(QK^T/sqrt(d))V), §2 (additive mask
 * M in {0,-inf}; skip the masked region instead of computing it), §4.5
 * (block-sparse pattern), §7 (Block-Sparse FlashAttention: online softmax).
 * q [B,Hq,N,d], k/v [B,Hkv,N,d] (dtype), N = Nq = Nk, N % block == 0.
 * idx [B,Hkv,nb,idx_stride] int32: for query block i of group g, the kept
 *   blocks ascending, ended by -1 (or by idx_stride).  Entries must satisfy
 *   0 <= j <= i; a kernel that finds another value skips it and sets
 *   BSA_DEV_BAD_INDEX.  Inside block i, key u is masked for query t when u > t.
 * softmax_scale: usually 1/sqrt(d).
 * o [B,Hq,N,d] (dtype) output; lse [B,Hq,N] fp32 natural-log row LSE of the
 *   scaled logits (optional, NULL to skip).
 * Built: BF16 with d = 128 and block in {64,128} (tcgen05 + TMA kernel);
 *   F32 with d in {64,128} and block in {64,128} (fp32 SIMT kernel).
 */
bsa_status_t bsa_sparse_attn_prefill(const bsa_shape_t* shape, const void* q, const void* k,
                                     const void* v, const int* idx, int idx_stride,
                                     float softmax_scale, void* o, float* lse, void* stream);

/*
 * bsa_gated_attn_fwd -- SAS gated sparse attention (inner log-gate).
 * Cite: SAS page, 核心模块 2 (the selector's continuous score enters the
 * softmax logits in log form) and 核心模块 3 (the gate is a normalised softmax
 * over the kept history blocks and the always-kept current block).
 * As bsa_sparse_attn_prefill, plus sel_scores [B,Hkv,nb,nb] fp32 (the prefill
 * selector scores, as bsa_score_blocks writes them): for query block i the
 * logit of every key of kept block j gains log g_j with
 *   g_j = exp(s[i][j]) / sum_{l kept} exp(s[i][l]).
 * All heads of a KV group share the group's gate.
 */
bsa_status_t bsa_gated_attn_fwd(const bsa_shape_t* shape, const void* q, const void* k,
                                const void* v, const int* idx, int idx_stride,
                                const float* sel_scores, float softmax_scale, void* o, float* lse,
                                void* stream);

/*
 * bsa_gated_attn_bwd -- backward of bsa_sparse_attn_prefill (sel_scores =
 * NULL) or bsa_gated_attn_fwd: the gradients of sum(dO * O) with respect to
 * q, k, v and, gated, the selector scores.
 * Cite: SAS page, 核心洞察 (the continuous score injected into the attention
 * logits lets the language-modelling loss update the context ranking by
 * standard back-propagation) and 核心模块 2-3 (the log-form gate inside the
 * softmax, normalised over the kept blocks and the current block).
 * Inputs: the forward's q, k, v, idx, idx_stride, sel_scores, softmax_scale;
 * its natural-log row LSE lse [B,Hq,N] fp32 (required); the upstream
 * gradient d_o [B,Hq,N,d] (dtype).  The forward's output O is not an input:
 * the row term D_t = dO_t . O_t is formed as sum_u P_{t,u} (dO_t . v_u) from
 * the recomputed probabilities, so the bf16 rounding of the stored O does not
 * enter the gradients.
 * Outputs (fp32, written whole): dq [B,Hq,N,d], dk and dv [B,Hkv,N,d]; dsel
 * [B,Hkv,nb,nb] (optional, gated only): for query block i of group g and its
 * kept block l, d/ds[i][l] through log g_l = s_l - log sum_{kept} exp(s),
 * zero elsewhere.  The selection itself (the hard top-k) passes no gradient.
 * workspace: bsa_workspace_bytes_bwd(shape, idx_stride) bytes, 256-byte
 * aligned.  Built: BF16, d = 128, block in {64, 128}, idx_stride <= 256
 * (BSA_ERR_UNSUPPORTED otherwise); tcgen05 MMAs with fp32 accumulation, P and
 * dS rounded to bf16 as MMA operands, D and the selector-score gradient
 * summed in fp32 from the unrounded values.
 */
bsa_status_t bsa_gated_attn_bwd(const bsa_shape_t* shape, const void* q, const void* k, const void* v,
                                const float* lse, const void* d_o, const int* idx, int idx_stride,
                                const float* sel_scores, float softmax_scale, float* dq, float* dk, float* dv,
                                float* dsel, void* workspace, size_t workspace_bytes, void* stream);

/* Scratch bytes of bsa_gated_attn_bwd; 0 on a bad shape. */
size_t bsa_workspace_bytes_bwd(const bsa_shape_t* shape, int idx_stride);

/*
 * bsa_sparse_attn_decode -- one query token per sequence over a retained KV
 * cache, reading only the kept blocks.
 * Cite: 稀疏注意力 tutorial §5 (decode: one new query against the history);
 * Sparse Frontier review §2.4.2 (full cache retained, selective loading, as
 * Quest does with query-aware pages).
 * q [B,Hq,d] (dtype BF16), k_cache/v_cache [B,Hkv,Nk,d], Nk % block == 0,
 * idx [B,Hkv,idx_stride] int32 kept blocks ascending, -1 ended; every cached
 * token is history of the query (no causal mask).  All heads of a group
 * share one gather of the kept blocks.
 * workspace: device scratch of at least
 *   bsa_workspace_bytes(BSA_OP_DECODE, shape, idx_stride) bytes, 256-byte
 *   aligned; its contents on entry do not matter.
 * o [B,Hq,d] (dtype); lse [B,Hq] fp32 (optional).
 * Built: BF16, d = 128, block = 64, at most 16 query heads per KV group
 * (BSA_ERR_UNSUPPORTED otherwise).
 */
bsa_status_t bsa_sparse_attn_decode(const bsa_shape_t* shape, const void* q, const void* k_cache,
                                    const void* v_cache, const int* idx, int idx_stride,
                                    float softmax_scale, void* workspace, size_t workspace_bytes,
                                    void* o, float* lse, void* stream);

/*
 * bsa_gist_expand_decode -- SSA gist scoring + selective expansion decode.
 * Cite: SSA page, 推理时的关键模块: (1) score the query against every chunk's
 * gist key, (2) expand the top-k chunks back to their tokens -- under GQA
 * each query head chooses its own chunks, (3) attend over the expanded tokens
 * together with the gists of the chunks that were not expanded.
 * q [B,Hq,d], k_cache/v_cache [B,Hkv,Nk,d] (tokens), gist_k/gist_v
 * [B,Hkv,nc,d] with nc = Nk/block (one gist per chunk), all BF16.
 * topk: chunks expanded per query head (0 <= topk <= nc).
 * idx_in [B,Hq,topk] int32 (optional): if given, these chunks are expanded
 *   and no scoring/selection runs (the way to inject a known index set).
 * idx_out [B,Hq,topk] int32 (optional): receives the chosen chunks ascending
 *   (with idx_in, a copy of it; idx_out may be idx_in itself).
 * workspace: bsa_workspace_bytes(BSA_OP_GIST_DECODE, shape, topk) bytes.
 * o [B,Hq,d] (dtype); lse [B,Hq] fp32 (optional).
 * Built: BF16, d = 128, block = 64, at most 16 query heads per KV group
 * (BSA_ERR_UNSUPPORTED otherwise).
 */
bsa_status_t bsa_gist_expand_decode(const bsa_shape_t* shape, const void* q, const void* k_cache,
                                    const void* v_cache, const void* gist_k, const void* gist_v,
                                    int topk, const int* idx_in, int* idx_out,
                                    float softmax_scale, void* workspace, size_t workspace_bytes,
                                    void* o, float* lse, void* stream);

/*
 * bsa_sparse_attn_decode_heads -- decode where every query head has its own
 * kept blocks (e.g. from bsa_topk_select_joint_heads).
 * Cite: 稀疏注意力 tutorial §5 (decode over the history); Sparse Frontier
 * review §2.3.2 (Ada-KV: per-head budgets) and §2.4.2 (full cache retained,
 * selective loading).
 * As bsa_sparse_attn_decode, but idx [B,Hq,idx_stride] holds one ascending,
 * -1 ended list per query head.  The union of a group's lists is gathered
 * once and each head masks the blocks it did not keep.
 * workspace: bsa_workspace_bytes(BSA_OP_DECODE_HEADS, shape, idx_stride).
 * Built: BF16, d = 128, block = 64, nb = Nk/64 a multiple of 32 and at most
 * 8192, at most 16 query heads per KV group.
 */
bsa_status_t bsa_sparse_attn_decode_heads(const bsa_shape_t* shape, const void* q, const void* k_cache,
                                          const void* v_cache, const int* idx, int idx_stride,
                                          float softmax_scale, void* workspace, size_t workspace_bytes,
                                          void* o, float* lse, void* stream);

/*
 * bsa_sparse_attn_decode_paged -- bsa_sparse_attn_decode over a paged KV
 * cache.
 * Cite: 稀疏注意力 tutorial §7 (PagedAttention: the logically contiguous KV
 * cache is mapped onto physical blocks that need not be contiguous) and §5
 * (decode); Sparse Frontier review §2.4.2 (full cache retained, selective
 * loading).
 * k_pool/v_pool [num_pages, Hkv, 64, d] bf16: physical blocks of 64 tokens.
 * block_table [B, table_stride] int32: sequence b's logical block j is
 * physical block block_table[b*table_stride + j] (the same for every KV
 * head); table_stride >= nb = Nk/64, shape->Nk = the logical cache length.
 * idx [B,Hkv,idx_stride] holds LOGICAL block ids (as the selector gives them
 * from the logical pooled summary); a logical id out of range or a table
 * entry outside [0, num_pages) is skipped and flagged (BSA_DEV_BAD_INDEX).
 * Otherwise as bsa_sparse_attn_decode (workspace: bsa_workspace_bytes(
 * BSA_OP_DECODE, shape, idx_stride)); with the identity table the result is
 * that of bsa_sparse_attn_decode on the contiguous cache, bit for bit.
 */
bsa_status_t bsa_sparse_attn_decode_paged(const bsa_shape_t* shape, const void* q, const void* k_pool,
                                          const void* v_pool, int num_pages, const int* block_table,
                                          int table_stride, const int* idx, int idx_stride, float softmax_scale,
                                          void* workspace, size_t workspace_bytes, void* o, float* lse,
                                          void* stream);

/*
 * bsa_paged_append -- append shape->Nq new tokens to every sequence of a
 * paged cache and keep the decode selector's block-mean summary current.
 * Cite: 稀疏注意力 tutorial §7 (PagedAttention) and §4.6 (one pooled key per
 * block for coarse scoring); Sparse Frontier review §2.4.2 (the retained
 * cache grows as decoding proceeds).
 * k_new/v_new [B, Hkv, Nq, d] bf16; seq_lens [B] int32: the tokens each
 * sequence holds before the append (left unchanged: the caller advances
 * them); token t goes to logical position seq_lens[b] + t, i.e. logical block
 * (seq_lens[b]+t)/64 through block_table [B, table_stride].  pooled_k
 * [B, Hkv, table_stride, d] fp32 (optional): every block that this append
 * completes gets its mean key (tokens ascending, fp32, one division --
 * the arithmetic of bsa_score_blocks' pooling, so equal to pooling the
 * whole logical cache).  Incomplete blocks are not pooled.  Built: BF16,
 * block 64.  A position past the table or a table entry outside
 * [0, num_pages) is skipped and flagged (BSA_DEV_BAD_INDEX).
 */
bsa_status_t bsa_paged_append(const bsa_shape_t* shape, const void* k_new, const void* v_new, const int* seq_lens,
                              const int* block_table, int table_stride, int num_pages, void* k_pool,
                              void* v_pool, float* pooled_k, void* stream);

/*
 * bsa_hssa_decode -- two-level gist routing (H-SSA) decode.
 * Cite: SSA page, 层级扩展：H-SSA (meta-gist tokens, "gist-of-gist", make a
 * coarse selection; inside the selected groups the ordinary gists score the
 * chunks finely and the best are expanded) and 推理时的关键模块 1-3 (per-head
 * selection under GQA; mixed attention over tokens and summaries).
 * Groups are 64 consecutive chunks; meta_k/meta_v [B,Hkv,nm,d] hold one
 * meta-gist per group, nm = nc/64 (nc = Nk/block chunks, gist_k/gist_v
 * [B,Hkv,nc,d]).  Per query head: score the nm meta-gists, keep the km best
 * groups; score the gists of the kept groups' chunks, expand the topk best
 * chunks.  Keys of the head (a reading: SSA's mixed attention one level
 * up): the tokens of its expanded chunks, the gists of the other chunks of
 * its kept groups, the meta-gists of the groups it did not keep.
 * Scores and order as bsa_score_blocks / bsa_topk_select (fixed-order fp32;
 * larger first, ties to the lower index, nothing forced).
 * meta_out [B,Hq,km] and idx_out [B,Hq,topk] int32 (optional): the kept
 * groups and expanded chunks, ascending.  workspace:
 * bsa_workspace_bytes_hssa(shape, km, topk) bytes, 256-byte aligned.
 * Built: BF16, d = 128, block = 64, nc a multiple of 64 and at most 4096,
 * 1 <= km <= nm, 0 <= topk <= 64*km, at most 16 query heads per KV group.
 */
bsa_status_t bsa_hssa_decode(const bsa_shape_t* shape, const void* q, const void* k_cache, const void* v_cache,
                             const void* gist_k, const void* gist_v, const void* meta_k, const void* meta_v,
                             int km, int topk, int* meta_out, int* idx_out, float softmax_scale,
                             void* workspace, size_t workspace_bytes, void* o, float* lse, void* stream);

/* Scratch bytes of bsa_hssa_decode; 0 on a bad shape. */
size_t bsa_workspace_bytes_hssa(const bsa_shape_t* shape, int km, int topk);

/*
 * bsa_sparse_attn_decode_noalloc -- bsa_sparse_attn_decode for callers that
 * cannot allocate device memory (no counterpart on the source pages; it is a
 * deployment convenience).  Some callers have no way to provide the decode
 * scratch buffer: a server that reserves all its device memory at start-up
 * and allocates nothing afterwards, or a plugin whose host framework owns
 * every device buffer.  This call takes no workspace; it uses a fixed
 * 4 MiB array built into the library, held on every GPU that loads the
 * library until the process exits.
 * Arguments, layouts and results are those of bsa_sparse_attn_decode.
 * Returns BSA_ERR_UNSUPPORTED, before launching anything, when the shape
 * needs more than 4 MiB of scratch (bsa_workspace_bytes(BSA_OP_DECODE, ...)).
 * The first call on a device (and the first after a device reset, which
 * reloads the library's module) looks up the array's device address; make
 * that first call before any stream capture.  All calls on a device share the
 * array: calls whose work may overlap on the GPU (unordered streams) race.
 * Nothing in the array needs to start zeroed between calls.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
bsa_status_t bsa_sparse_attn_decode_noalloc(const bsa_shape_t* shape, const void* q, const void* k_cache,
                                            const void* v_cache, const int* idx, int idx_stride,
                                            float softmax_scale, void* o, float* lse, void* stream);

/* Scratch bytes a decode call needs (op = BSA_OP_*; budget = idx_stride for
 * BSA_OP_DECODE and BSA_OP_DECODE_HEADS, topk for BSA_OP_GIST_DECODE).  0 on
 * a bad shape. */
size_t bsa_workspace_bytes(int op, const bsa_shape_t* shape, int budget);

/* Human-readable name of a status code (static string). */
const char* bsa_status_string(bsa_status_t status);

/* Reads (and, if reset != 0, clears) the current device's status word.
 * Synchronises the device.  flags may be NULL.  Returns BSA_ERR_TIMEOUT or
 * BSA_ERR_DEVICE when a flag is set, BSA_OK otherwise. */
bsa_status_t bsa_device_status(unsigned int* flags, int reset);

/* Library ABI version (major*100 + minor). */
int bsa_version(void);

/*
 * Testing and tuning hooks (no counterpart on the source pages).
 *
 * bsa_decode_split_override -- fixes the number of split-K ranges the decode
 * calls cut a batch's kept-block lists into (num_splits > 0), or restores the
 * default of one range per SM (num_splits <= 0).  Process-wide; returns the
 * previous setting (0 = default).  It changes bsa_workspace_bytes() for the
 * decode operations too, so set it before sizing a workspace, and do not
 * change it while a decode call is being enqueued on another thread.  The
 * result of a decode does not depend on it beyond fp32 rounding order.
 */
int bsa_decode_split_override(int num_splits);

/*
 * bsa_prefill_kernel_override -- selects which bf16 prefill kernel the
 * prefill and gated calls run: 0 = chosen by shape (default), 1 = paired
 * tiles (two 128-row tiles per SM), 2 = one 128-row tile per SM with split
 * key halves, 3 = SM pair (two SMs per 256 rows, MMAs of M = 256).
 * Process-wide; returns the previous setting.  All kernels compute the same
 * result up to fp32 rounding order; the hook exists to test and time each.
 */
int bsa_prefill_kernel_override(int kernel);

/*
 * bsa_selftest_wait_expiry -- enqueues a one-thread kernel that waits, with
 * a budget of budget_cycles SM cycles, on a shared-memory barrier nothing
 * arrives on, through the same bounded-wait helper every kernel uses.  The
 * wait expires, BSA_DEV_TIMEOUT is raised in the device status word and the
 * kernel returns; bsa_device_status() then reports BSA_ERR_TIMEOUT.  It
 * exists to test that expiry path; it faults nothing and leaves the device
 * usable.  budget_cycles < 0 -> BSA_ERR_INVALID_ARG.
 */
bsa_status_t bsa_selftest_wait_expiry(long long budget_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H_ */
