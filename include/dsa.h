/*
 * dsa.h -- C ABI of libdsa.so, the DeepSeek Sparse Attention (DSA) layer
 * step on one NVIDIA B200 (sm_100a).
 *
 * The step has three parts, each a CUDA kernel of this library:
 *   1. Lightning-indexer scores of every query against every previous key of
 *      the single-head indexer key cache (DeepSeek-V3.2 model doc,
 *      Transformers, section "DeepSeek Sparse Attention (DSA)", item 1, and
 *      the paragraph on the indexer's own key cache);
 *   2. per-query top-index_topk selection (same section, item 2);
 *   3. MLA attention over the selected latent rows only (same section,
 *      item 2: O(index_topk) per query instead of O(L)).
 * Shapes follow section DeepseekV32Config (index_n_heads 64, index_head_dim
 * 128, index_topk 2048, num_attention_heads 128, kv_lora_rank 512,
 * qk_rope_head_dim 64).
 *
 * Conventions for every entry point
 *   - All tensor arguments are DEVICE pointers to row-major, contiguous
 *     buffers in the layouts stated below, owned by the caller, except where
 *     an argument is marked HOST.  The library keeps no pointer after a call.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  No call synchronises unless stated; none allocates device
 *     memory; scratch space comes from the caller's `workspace`, sized with
 *     dsa_workspace_bytes().
 *   - Argument errors are reported synchronously by the return value and
 *     nothing is enqueued.  A failed launch returns DSA_ERR_CUDA.  Errors
 *     found by a kernel while it runs (a bounded wait that expired, an index
 *     out of range) are recorded in a per-device error word inside the
 *     library and read with dsa_get_error().
 *   - Pointers fed to the tensor-memory-accelerator paths (q_idx, k_idx for
 *     BF16 / E4M3) must be 16-byte aligned.
 *   - Query t of sequence b sits at position pos = q_pos0[b] + t, and
 *     0 <= q_pos0[b], q_pos0[b] + n_q <= ctx_len[b] <= s_max.  A query sees
 *     the keys s <= pos ("previous keys" is read as including its own
 *     position; a decode query is the newest token, already in the cache).
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer */
    DSA_ERR_UNSUPPORTED = 2,  /* valid but not implemented shape/dtype combination */
    DSA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than dsa_workspace_bytes() */
    DSA_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
    DSA_ERR_TIMEOUT = 5,      /* (device) a bounded wait inside a kernel expired */
    DSA_ERR_BAD_INDEX = 6,    /* (device) an attention index was >= ctx_len and was skipped */
    DSA_ERR_HIST_MISMATCH = 7 /* (device) dsa_topk_hist was given partial histograms that do not
                                 describe its scores (not from the dsa_indexer_scores_hist call
                                 that wrote them); the affected rows' indices are undefined */
} dsa_status_t;

typedef enum {
    DSA_F32 = 0,   /* IEEE fp32 */
    DSA_BF16 = 1,  /* bfloat16 */
    DSA_E4M3 = 2   /* OCP FP8 E4M3 codes (uint8) with fp32 per-row scales */
} dsa_dtype_t;

/* Shape and numeric options shared by every call (plain data, by pointer). */
typedef struct {
    int32_t batch;      /* B, sequences */
    int32_t n_q;        /* queries per sequence (1 = decode) */
    int32_t s_max;      /* cache capacity: rows per sequence of every cache */
    int32_t idx_heads;  /* H_I, index_n_heads (64) */
    int32_t idx_dim;    /* D_I, index_head_dim (128) */
    int32_t topk;       /* k, index_topk (2048) */
    int32_t heads;      /* H, attention heads (128) */
    int32_t d_qk;       /* query/key width per head: 576 = kv_lora_rank 512 + rope 64 */
    int32_t d_v;        /* value/output width per head (512, the latent) */
    int32_t kv_heads;   /* 1 = absorbed MLA (one shared latent row per token, value = its
                           first d_v columns); > 1 = MHA/GQA with a separate v tensor */
    int32_t idx_dtype;  /* dsa_dtype_t of the indexer inputs: F32, BF16 or E4M3 */
    int32_t attn_dtype; /* dsa_dtype_t of q, kv, v and out: F32 or BF16 */
    float idx_scale;    /* > 0: multiplies each head's dot product inside the ReLU (1.0) */
    float sm_scale;     /* softmax scale of the attention logits (1/sqrt(192) for MLA) */
    int32_t q_chunk;    /* dsa_forward only: queries per sequence processed per round of
                           indexer -> top-k -> attention; 0 = all n_q at once */
    int32_t idx_rescore;/* step with the E4M3 indexer only: > 0 keeps the top
                           (topk + idx_rescore) keys of the FP8 scores, re-scores them
                           from the BF16 key cache (dsa_indexer_rescore) and selects the
                           final topk among them; 0 = select on the FP8 scores */
} dsa_shape_t;

/* Which workspace dsa_workspace_bytes() sizes. */
enum { DSA_WS_TOPK = 0, DSA_WS_ATTN = 1, DSA_WS_FORWARD = 2, DSA_WS_FORWARD_HOST = 3, DSA_WS_HIST = 4 };

/*
 * Lightning-indexer scores (section DSA, item 1; key cache paragraph).
 *   I[b,t,s] = sum_h w[b,t,h] * max(0, idx_scale * <q_idx[b,t,h,:], k_idx[b,s,:]>)
 *              for s <= pos(b,t);  -inf for pos(b,t) < s < ctx_len[b].
 * The per-head ReLU and the weights_proj weighting are this library's
 * reading; the pages name the score but do not print its formula.
 * Arguments
 *   q_idx   [B][n_q][H_I][D_I]  idx_dtype (E4M3: codes of the Hadamard-rotated query)
 *   q_scale [B][n_q][H_I] fp32  E4M3 only (else NULL): per (query, head) scale
 *   k_idx   [B][s_max][D_I]     idx_dtype (E4M3: codes of the rotated key)
 *   k_scale [B][s_max] fp32     E4M3 only (else NULL): per key scale
 *   w       [B][n_q][H_I] fp32  head weights (the weights_proj output)
 *   ctx_len, q_pos0 [B] int32   device
 *   scores  [B][n_q][ld_scores] fp32 output; columns s < ctx_len[b] are
 *           written, the rest of each row is left untouched.
 *   ld_scores >= s_max, a multiple of 4.
 * BF16 and E4M3 run on the tensor cores (tcgen05) and need D_I = 128 and
 * H_I in {16, 32, 64, 128}; F32 runs on the CUDA cores for any D_I <= 256,
 * H_I <= 128.  E4M3 scores equal the scores of the dequantised inputs.
 */
dsa_status_t dsa_indexer_scores(const dsa_shape_t *shape,
                                const void *q_idx, const float *q_scale,
                                const void *k_idx, const float *k_scale,
                                const float *w,
                                const int32_t *ctx_len, const int32_t *q_pos0,
                                float *scores, int64_t ld_scores,
                                void *stream);

/*
 * Fine-grained token selection (section DSA, item 2): for each query, the
 * min(topk, pos+1) keys s <= pos with the largest scores; among equal scores
 * the lower index wins (the pages are silent on ties; -0.0 equals +0.0).
 * Arguments
 *   scores [B][n_q][ld_scores] fp32, finite for s <= pos.
 *   idx    [B][n_q][topk] int32 output: the kept indices in ascending order,
 *          then -1 padding.
 *   workspace: dsa_workspace_bytes(shape, DSA_WS_TOPK) bytes (may be 0).
 * The selection is exact: it is decided on the fp32 bit patterns.
 */
dsa_status_t dsa_topk(const dsa_shape_t *shape,
                      const float *scores, int64_t ld_scores,
                      const int32_t *ctx_len, const int32_t *q_pos0,
                      int32_t *idx,
                      void *workspace, size_t workspace_bytes,
                      void *stream);

/*
 * The indexer's projections, which produce the step's indexer inputs
 * (DeepSeek-V3.2 model doc: the note on the query LoRA path -- the indexer
 * scores queries from the low-rank latent q_a_layernorm(q_a_proj(x)) through
 * its `wq_b` projection, sized by q_lora_rank = 1536; section DeepseekV32Config
 * -- index_n_heads 64, index_head_dim 128, hidden_size 7168; section "Usage
 * example" -- weights_proj stays out of FP8).  Each is a plain linear map
 * Y = X W^T on the tensor cores: bf16 operands, fp32 accumulation.
 * Normalisations and rotary embeddings around them are the caller's.
 *
 * dsa_indexer_proj_q: q_idx[t, h, d] = sum_j q_latent[t, j] * wq_b[h * D_I + d, j]
 *   q_latent [n_tokens][q_lora_rank] BF16, wq_b [H_I * D_I][q_lora_rank] BF16,
 *   q_idx    [n_tokens][H_I][D_I] BF16 output (rounded to nearest even).
 *   q_lora_rank a multiple of 64; H_I * D_I a multiple of 256 (or 64, 128, 192).
 */
dsa_status_t dsa_indexer_proj_q(const dsa_shape_t *shape, int32_t n_tokens, int32_t q_lora_rank,
                                const void *q_latent, const void *wq_b, void *q_idx, void *stream);

/*
 * dsa_indexer_proj_kw: the single-head index key and the head weights of
 * each token, from its hidden state, in one pass over x:
 *   k_new[t, d] = sum_j x[t, j] * w_kw[d, j]          (d < D_I; BF16 out)
 *   w[t, h]     = sum_j x[t, j] * w_kw[D_I + h, j]    (h < H_I; fp32 out)
 *   x [n_tokens][hidden] BF16; w_kw [D_I + H_I][hidden] BF16: the key
 *   projection's rows followed by weights_proj's rows.  hidden a multiple of
 *   64; D_I + H_I in {64, 128, 192} or a multiple of 256, D_I a multiple of 32.
 *   k_new feeds dsa_cache_append, w feeds the indexer (any constant factor of
 *   the score goes into shape->idx_scale or into w_kw).
 * All pointers 16-byte aligned.
 */
dsa_status_t dsa_indexer_proj_kw(const dsa_shape_t *shape, int32_t n_tokens, int32_t hidden,
                                 const void *x, const void *w_kw, void *k_new, float *w, void *stream);

/*
 * The indexer -> top-k pair with a handoff (section DSA, items 1-2: the
 * index score exists to feed the per-query top-index_topk selection).
 * dsa_indexer_scores_hist computes exactly what dsa_indexer_scores computes
 * and, where the indexer's schedule allows it (tensor-core indexer, one
 * query per sequence, i.e. decode, on rows of at least a few thousand keys),
 * its epilogue also counts the first 11-bit radix digit of every score into
 * `hist`; dsa_topk_hist then selects exactly what dsa_topk selects, starting
 * from those counts instead of a first pass over each score row.  Elsewhere
 * the pair behaves as dsa_indexer_scores + dsa_topk (hist unused).
 * Arguments as in those two calls, plus
 *   hist  device buffer of dsa_workspace_bytes(shape, DSA_WS_HIST) bytes,
 *         16-byte aligned, opaque; written by the indexer call, read by the
 *         top-k call.  The two calls must be made with the same shape on the
 *         same device, with the top-k reading the scores the indexer call
 *         wrote, and nothing else writing `hist` in between.  The top-k
 *         checks the counts against the scores it reads: where they differ
 *         it records DSA_ERR_HIST_MISMATCH in the device error word and the
 *         row's indices are undefined (no access outside the buffers).
 */
dsa_status_t dsa_indexer_scores_hist(const dsa_shape_t *shape,
                                     const void *q_idx, const float *q_scale,
                                     const void *k_idx, const float *k_scale,
                                     const float *w,
                                     const int32_t *ctx_len, const int32_t *q_pos0,
                                     float *scores, int64_t ld_scores,
                                     void *hist, size_t hist_bytes,
                                     void *stream);
dsa_status_t dsa_topk_hist(const dsa_shape_t *shape,
                           const float *scores, int64_t ld_scores,
                           const int32_t *ctx_len, const int32_t *q_pos0,
                           const void *hist, size_t hist_bytes,
                           int32_t *idx, void *stream);

/*
 * Selection among listed candidates (section DSA, item 2, applied to a
 * candidate list): for each query, the min(topk, n) entries of
 * cand[b,t,0:n] with the largest cand_scores, n = min(n_cand, pos+1,
 * ctx_len[b]) -- the first n entries are the candidates.  The candidates
 * are key indices in ascending order (as dsa_topk writes them), so "ties go
 * to the lower index" is "ties go to the earlier entry".
 * Arguments
 *   cand_scores [B][n_q][cand_ld] fp32, finite for the n listed entries;
 *   cand        [B][n_q][cand_ld] int32 ascending key indices;
 *   cand_ld >= n_cand, a multiple of 4.
 *   idx         [B][n_q][topk] int32 output: the kept key indices (values of
 *               cand), ascending, then -1 padding.
 * The E4M3 step uses it after dsa_indexer_rescore.  No workspace.
 */
dsa_status_t dsa_topk_candidates(const dsa_shape_t *shape,
                                 const float *cand_scores, const int32_t *cand,
                                 int64_t cand_ld, int32_t n_cand,
                                 const int32_t *ctx_len, const int32_t *q_pos0,
                                 int32_t *idx, void *stream);

/*
 * Index scores of listed keys from BF16 rows (section DSA, item 1: the
 * reference indexer runs in FP8 after the Hadamard rotation, and FP8 is only
 * a precision optimisation of this same score).  For each query and each of
 * its first n = min(n_cand, pos+1, ctx_len[b]) listed keys s = cand[b,t,j]:
 *   scores[b,t,j] = sum_h w[b,t,h] * max(0, idx_scale * <q_idx[b,t,h,:], k_idx[b,s,:]>)
 * computed as dsa_indexer_scores computes it for BF16 inputs (tensor cores,
 * fp32 accumulation).  Used by the E4M3 step (shape->idx_rescore > 0) to
 * re-score the FP8 indexer's top (topk + idx_rescore) keys before the final
 * selection, so that the selection matches the BF16 indexer's.
 * Arguments
 *   q_idx [B][n_q][H_I][D_I] BF16 and k_idx [B][s_max][D_I] BF16, whatever
 *         shape->idx_dtype says; 16-byte aligned.  D_I = 128,
 *         H_I in {16, 32, 64, 128}.
 *   w     [B][n_q][H_I] fp32;  ctx_len, q_pos0 [B] int32.
 *   cand  [B][n_q][cand_ld] int32: listed key indices, each in [0, ctx_len[b])
 *         (an entry outside is scored as an all-zero key and sets
 *         DSA_ERR_BAD_INDEX in the device error word).
 *   scores [B][n_q][ld_scores] fp32 output, entries j < n written;
 *         cand_ld, ld_scores >= n_cand.
 */
dsa_status_t dsa_indexer_rescore(const dsa_shape_t *shape,
                                 const void *q_idx, const void *k_idx, const float *w,
                                 const int32_t *cand, int64_t cand_ld, int32_t n_cand,
                                 const int32_t *ctx_len, const int32_t *q_pos0,
                                 float *scores, int64_t ld_scores, void *stream);

/*
 * Attention over the selected keys only (section DSA, item 2).  For head h
 * of query (b,t), over the listed keys j (entries < 0 are skipped):
 *   l_j = sm_scale * <q[b,t,h,:], K[b,idx_j,:]>,  O = sum_j softmax(l)_j V[b,idx_j,:]
 * kv_heads == 1 (absorbed MLA): K = kv[b,s,:] (d_qk wide), V = kv[b,s,:d_v],
 * shared by all heads (v must be NULL).  kv_heads > 1: K = kv[b,s,g,:],
 * V = v[b,s,g,:] with g = h / (H / kv_heads).
 * Arguments
 *   q   [B][n_q][H][d_qk]          attn_dtype
 *   kv  [B][s_max][kv_heads][d_qk] attn_dtype
 *   v   [B][s_max][kv_heads][d_v]  attn_dtype, or NULL when kv_heads == 1
 *   idx [B][n_q][topk] int32; an entry >= ctx_len[b] is skipped and flagged
 *       DSA_ERR_BAD_INDEX in the device error word.
 *   out [B][n_q][H][d_v] attn_dtype output (BF16: rounded to nearest even)
 *   lse [B][n_q][H] fp32 output or NULL: log-sum-exp of the scaled logits
 *       (-inf, with out = 0, when no key is listed).
 *   workspace: dsa_workspace_bytes(shape, DSA_WS_ATTN) bytes.
 * BF16 with d_qk = 576, d_v = 512, kv_heads = 1, H a multiple of 64 runs on
 * the tensor cores; F32 runs on the CUDA cores for d_qk, d_v in {32, 64,
 * 128} (and the MLA sizes).
 */
dsa_status_t dsa_sparse_mla_attn(const dsa_shape_t *shape,
                                 const void *q, const void *kv, const void *v,
                                 const int32_t *idx, const int32_t *ctx_len,
                                 void *out, float *lse,
                                 void *workspace, size_t workspace_bytes,
                                 void *stream);

/*
 * Hadamard rotation + FP8 quantisation of rows (section DSA, item 1: the
 * reference indexer runs in FP8 after the orthogonal `rotate_activation`,
 * Hq.Hk = q.k).  For each row r of `rows` rows of `dim` (= 128) elements:
 *   y = H x (orthonormal Sylvester-Hadamard, entries +-1/sqrt(dim)),
 *   scale[r] = max|y| / 448 (1 for an all-zero row),
 *   x_fp8[r,:] = e4m3(y / scale[r]), round to nearest even, saturating.
 * x: [rows][dim] in x_dtype (BF16 or F32); x_fp8 [rows][dim] uint8;
 * scale [rows] fp32.  Used on keys when they enter the cache and on the
 * indexer queries of each step.
 */
dsa_status_t dsa_hadamard_quant_fp8(const void *x, int32_t x_dtype, int64_t rows, int32_t dim,
                                    uint8_t *x_fp8, float *scale, void *stream);

/*
 * Cache append, the update before the step scores (DeepSeek-V3.2 model doc,
 * section "DeepSeek Sparse Attention (DSA)": the indexer keeps its own small
 * per-token key cache -- single head, index_head_dim wide -- beside the main
 * K/V cache, updated through update_indexer(); the reference indexer runs in
 * FP8 after the Hadamard rotation).  New token i of sequence b goes to cache
 * row pos[b] + i:
 *   k_new   [B][n_new][idx_dim] in idx_dtype (F32/BF16), or BF16 when
 *           idx_dtype is E4M3;
 *   kv_new  [B][n_new][kv_heads][d_qk] attn_dtype; v_new [B][n_new][kv_heads][d_v]
 *           for the separate-V form, else NULL;
 *   pos     [B] int32, DEVICE: the first cache row of each sequence's new tokens;
 *   k_cache the indexer key cache as read by dsa_indexer_scores: the row is
 *           copied (F32/BF16), or (E4M3, idx_dim 128) rotated by the 128-point
 *           Hadamard and quantised exactly as dsa_hadamard_quant_fp8 does, codes
 *           into k_cache [B][s_max][128] and the row scale into k_scale [B][s_max];
 *   kv_cache, v_cache as read by dsa_sparse_mla_attn (v_cache NULL iff v_new is).
 * All pointers are DEVICE pointers, 4-byte aligned; the caller owns them and
 * advances its own ctx_len.  Rows that fall outside [0, s_max) are skipped
 * and set DSA_ERR_BAD_INDEX in the device error word.  Nothing is allocated;
 * the work is enqueued on `stream`.
 */
dsa_status_t dsa_cache_append(const dsa_shape_t *shape, int32_t n_new,
                              const void *k_new, const void *kv_new, const void *v_new,
                              const int32_t *pos,
                              void *k_cache, float *k_scale, void *kv_cache, void *v_cache,
                              void *stream);

/*
 * The whole layer step: indexer scores -> top-k -> sparse attention, in
 * rounds of shape->q_chunk queries per sequence (scores of one round live in
 * the workspace).  Inputs as in the calls above, except with
 * idx_dtype == E4M3: q_idx is BF16 [B][n_q][H_I][D_I] and is rotated and
 * quantised inside the step (q_scale must be NULL), while k_idx/k_scale are
 * the FP8 key cache as written by dsa_hadamard_quant_fp8 (or dsa_cache_append).
 *   k_rescore  E4M3 with shape->idx_rescore > 0: the BF16 key cache
 *              [B][s_max][D_I] (the same keys before rotation and
 *              quantisation), from which the FP8 indexer's top
 *              (topk + idx_rescore) candidates are re-scored before the final
 *              top-k; otherwise NULL.
 *   idx_out [B][n_q][topk] int32 or NULL: the selected indices.
 *   workspace: dsa_workspace_bytes(shape, DSA_WS_FORWARD) bytes.
 */
dsa_status_t dsa_forward(const dsa_shape_t *shape,
                         const void *q_idx, const float *q_scale,
                         const void *k_idx, const float *k_scale,
                         const void *k_rescore,
                         const float *w,
                         const void *q, const void *kv, const void *v,
                         const int32_t *ctx_len, const int32_t *q_pos0,
                         void *out, float *lse, int32_t *idx_out,
                         void *workspace, size_t workspace_bytes,
                         void *stream);

/*
 * dsa_forward with the per-step tensors in HOST memory: q_idx, w, q,
 * ctx_len, q_pos0 (inputs) and out, lse (outputs; lse may be NULL) are HOST
 * pointers (page-locked memory gives asynchronous copies; pinned on the
 * GPU's own NUMA node -- e.g. allocated from a thread bound to the CPUs
 * NVML reports as nearest the GPU -- host-to-device copies run at the link
 * rate, pinned on the far socket they can run at a fraction of it), while
 * the caches k_idx, k_scale, k_rescore, kv, v stay on the device as the
 * layer's resident state.
 * The call copies the inputs in (one cudaMemcpyAsync each), runs the step,
 * copies the outputs back and synchronises `stream` before returning.
 * workspace: dsa_workspace_bytes(shape, DSA_WS_FORWARD_HOST) bytes: the
 * scratch of dsa_forward, two input staging slots (consecutive host-buffer
 * calls on a device alternate between them) and the output staging.  The
 * inputs are copied on a stream of the library's own, which waits for the
 * last call that used the same slot; it waits for `stream` too when the
 * workspace address differs from the previous host-buffer call's.  So
 * between two host-buffer calls with the same workspace, the caller must
 * not use that memory for anything else.
 */
dsa_status_t dsa_forward_host(const dsa_shape_t *shape,
                              const void *h_q_idx, const float *h_w, const void *h_q,
                              const int32_t *h_ctx_len, const int32_t *h_q_pos0,
                              const void *k_idx, const float *k_scale, const void *k_rescore,
                              const void *kv, const void *v,
                              void *h_out, float *h_lse,
                              void *workspace, size_t workspace_bytes,
                              void *stream);

/*
 * dsa_forward_host for a loop of steps whose copies overlap one another's
 * compute (the pages have no counterpart; it is the serving-loop form of the
 * call above).  Arguments as in dsa_forward_host, plus:
 *   done_event  a cudaEvent_t (passed as void*) created by the caller on the
 *               same device, or NULL.  It is recorded once this call's
 *               outputs are in h_out / h_lse.
 * The call returns once the work is enqueued; it does not synchronise.
 *   - The inputs are copied in on a stream of the library's own into the
 *     call's staging slot (as in dsa_forward_host): the indexer waits for
 *     its inputs, the attention for the queries, and the copies need not
 *     wait for the previous call's compute, only for the call before it
 *     (the last one that used the slot) to finish its attention.
 *   - The outputs are copied back on a second stream of the library's own
 *     after the step's attention, so that the copy runs under the next
 *     call's indexer and top-k.  The next host-buffer call on the device
 *     (either form) waits for that copy before its attention rewrites the
 *     device output, so one workspace serves consecutive calls.
 *   - Host buffers: the inputs must stay unchanged, and h_out / h_lse must
 *     not be read, until done_event has completed (or the device has been
 *     synchronised).
 *   - Errors: argument errors return before anything is enqueued; device
 *     errors are read with dsa_get_error.
 *   - Threads: host-buffer calls (either form) may come from several host
 *     threads; the library's staging slots, streams and events are per
 *     device, and a per-device lock makes each call's enqueue atomic, so
 *     concurrent calls run one after the other in the order they take it.
 */
dsa_status_t dsa_forward_host_async(const dsa_shape_t *shape,
                                    const void *h_q_idx, const float *h_w, const void *h_q,
                                    const int32_t *h_ctx_len, const int32_t *h_q_pos0,
                                    const void *k_idx, const float *k_scale, const void *k_rescore,
                                    const void *kv, const void *v,
                                    void *h_out, float *h_lse,
                                    void *workspace, size_t workspace_bytes,
                                    void *done_event, void *stream);

/*
 * dsa_sparse_mla_attn without a workspace argument: the scratch memory that
 * the split-K combine needs comes from a fixed array inside the library.
 * The pages have no counterpart to this call; it exists for callers that
 * cannot hand the library device memory on their decode path -- a serving
 * loop whose device memory is planned once up front and may not grow, or a
 * host program without a device allocator of its own (cudaMalloc, which can
 * synchronise the whole device, is no substitute there).
 * Arguments and results are those of dsa_sparse_mla_attn.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - The array is 32 MiB and lives on every GPU that loads the library until
 *     the process exits.  A shape that would need more returns
 *     DSA_ERR_WORKSPACE before anything is enqueued (on a 148-SM B200 no
 *     shape needs more than about 20 MB).
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   - Every call shares the one array and leaves the last call's partial
 *     results in it; nothing in it has to start at zero.  Calls that overlap
 *     on the GPU (different streams, or devices sharing a context) race on
 *     it: serialise them.
 */
dsa_status_t dsa_sparse_mla_attn_static(const dsa_shape_t *shape,
                                        const void *q, const void *kv, const void *v,
                                        const int32_t *idx, const int32_t *ctx_len,
                                        void *out, float *lse,
                                        void *stream);

/* Bytes of device workspace a call needs (DSA_WS_*); 0 for an invalid shape. */
size_t dsa_workspace_bytes(const dsa_shape_t *shape, int32_t which);

/*
 * Reads (and, if clear != 0, resets) the device error word of the current
 * device.  Synchronises the device.  Returns DSA_OK, DSA_ERR_TIMEOUT,
 * DSA_ERR_BAD_INDEX or DSA_ERR_HIST_MISMATCH (the first recorded kind in that
 * order), or DSA_ERR_CUDA if the read
 * itself failed.  `detail`, if not NULL, receives the raw word.
 * Sharing: the word lives in the library's own device memory, one per
 * device, not in a caller's workspace -- several entry points that can
 * record an error (dsa_indexer_scores, dsa_cache_append,
 * dsa_sparse_mla_attn_static) take no workspace.  So every caller and every
 * stream on a device records into the same word (bits are OR-ed, nothing is
 * lost), and a clear by one caller also clears what another caller's kernels
 * recorded: a program with several independent users of one device should
 * read with clear = 0 and clear at an agreed point.
 */
dsa_status_t dsa_get_error(int32_t clear, uint32_t *detail);

/*
 * Diagnostic with no counterpart on the pages: enqueues a one-thread kernel
 * whose bounded wait on a barrier is never completed.  After the library's
 * wait limit (about 2 s) it gives up, records DSA_ERR_TIMEOUT in the device
 * error word and returns, exactly as a stalled pipeline wait in the other
 * kernels would; the context stays usable.  Read the result with
 * dsa_get_error().
 */
dsa_status_t dsa_selftest_wait_timeout(void *stream);

/* Static English text for a status code. */
const char *dsa_status_string(dsa_status_t status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
