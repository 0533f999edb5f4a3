/*
 * lsa.h -- C ABI of the token-level sparse-attention hot path on B200 (sm_100a).
 *
 * One long-context attention layer, three stages:
 *   1. lightning-indexer scores        lsa_index_score   (bf16 or FP8-e4m3 keys)
 *   2. per-query selection             lsa_topk_select   (top-K + sink/window union)
 *                                      lsa_topk_refine   (FP8 scan's top-2K re-ranked exactly in bf16)
 *                                      lsa_bucket_select, lsa_bucket_select_split, lsa_bucket_select_noalloc
 *                                                        (Flat buckets / 4-token micro-blocks)
 *                                      lsa_tree_select, lsa_tree_select_split
 *                                                        (two-level tree search over the Flat buckets)
 *                                      lsa_hi_select     (pages, then tokens: hierarchical index)
 *                                      lsa_msa_select    (group-wise 128-token blocks)
 *      precompute, cached once:        lsa_pool_keys, lsa_split_representatives, lsa_tree_parents
 *   3. sparse attention over the gathered MLA latent rows
 *                                      lsa_sparse_attn   (one pass over the selected rows)
 *                                      lsa_hybrid_attn   (sink + window and sparse rows on two streams,
 *                                                         merged by log-sum-exp)
 *                                      lsa_msa_attn      (each head group over its own blocks)
 *   Scratch sizes: lsa_workspace_size and the per-call *_workspace_size functions.
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library keeps
 *     no pointer after the call returns.  Row-major layouts; "[B, H]" means B rows of H.
 *   - Positions are 0-based.  q_pos[b] (device int64) is the position of query b; it
 *     sees the keys s in [0, q_pos[b]] (decode: q_pos = L - 1; causal prefill: q_pos = t).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Every
 *     call only enqueues work on that stream: nothing synchronises with the host.
 *   - Scratch memory ("ws") is caller-allocated device memory of at least
 *     lsa_workspace_size(...) bytes, 256-byte aligned.  Contents need no initialisation.
 *   - Return value: LSA_OK (0) or a negative lsa_status.  Arguments are validated
 *     before anything is launched; a failed check launches nothing.  A launch failure
 *     returns LSA_ERR_CUDA (the CUDA error string is kept for lsa_last_error()).
 *     Nothing throws across this ABI.
 *   - All calls are deterministic: the same inputs give the same bytes.
 */
#ifndef LSA_H_
#define LSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LSA_OK = 0,
  LSA_ERR_INVALID_ARG = -1,  /* a pointer, size or parameter is out of range        */
  LSA_ERR_UNSUPPORTED = -2,  /* valid request this build does not handle (e.g. dims) */
  LSA_ERR_WORKSPACE = -3,    /* ws is NULL, misaligned or smaller than required      */
  LSA_ERR_CUDA = -4,         /* a CUDA runtime/driver call failed                    */
  LSA_ERR_DEVICE_CHECK = -5, /* a device-side check recorded a bad index              */
  LSA_ERR_TIMEOUT = -6       /* a bounded device-side wait gave up                    */
} lsa_status;

typedef enum {
  LSA_BF16 = 0,     /* bfloat16 elements                                            */
  LSA_FP8_E4M3 = 1  /* OCP e4m3fn codes with one fp32 scale per row (value = code*scale) */
} lsa_dtype;

typedef enum {
  LSA_OP_TOPK = 1,
  LSA_OP_BUCKET = 2,
  LSA_OP_ATTN = 3,
  LSA_OP_REFINE = 4,
  LSA_OP_BUCKET_MIN = 5, /* the smaller lsa_bucket_select workspace: CUDA-core representative scoring */
  LSA_OP_HYBRID_ATTN = 6
} lsa_op;

/*
 * lsa_index_score -- lightning-indexer scores.
 *   Source: "LongCat Sparse Attention（LSA）完全拆解", section "DSA 基线：闪电索引器是怎么工作的",
 *   equation I_{t,s} = sum_{j<H_I} w_{t,j} * ReLU(q^I_{t,j} . k^I_s): H_I index heads share one
 *   MQA index key k^I_s, ReLU instead of softmax, FP8-capable.
 *
 *   scores[b*ld + s] = sum_j w[b,j] * max(0, q[b,j,:] . k[s,:])   for s <= q_pos[b]
 *                    = -inf                                        for q_pos[b] < s < L
 *   q_idx   [B, H_I, d_I]  bf16, or e4m3 codes with q_scale [B, H_I] fp32 (value = code*scale)
 *   w       [B, H_I]       fp32 head weights
 *   k_idx   [L, d_I]       bf16, or e4m3 codes with k_scale [L] fp32
 *   q_scale, k_scale       must be NULL for LSA_BF16 and non-NULL for LSA_FP8_E4M3
 *   scores  [B, ld]        fp32, ld >= L; entries s >= L are not touched
 *   Supported: d_I in {32, 64, 128}; H_I in [1, 64] with H_I*d_I <= 8192 (bf16);
 *   FP8 needs d_I multiple of 32.  q_idx/k_idx 16-byte aligned, scores 16-byte aligned,
 *   ld a multiple of 4.  Accumulation is fp32 (products of bf16/e4m3 are exact in fp32).
 */
int lsa_index_score(const void* q_idx, const float* q_scale, const float* w,
                    const void* k_idx, const float* k_scale, int dtype,
                    int64_t B, int H_I, int d_I, int64_t L, const int64_t* q_pos,
                    float* scores, int64_t ld, void* stream);

/*
 * lsa_topk_select -- per-query top-K, unioned with attention-sink and sliding-window positions.
 *   Source: same page, S_t = arg topK({I_{t,s}}_{s<=t}, K) (section "DSA 基线"), and section
 *   "机制一：流式感知索引（SI）/ 预算分解": S_t = S_sink u S_swa u S_sparse, S_sink = the first
 *   K_sink positions, S_swa = {t-K_swa+1 .. t}, S_sparse = arg topK over s outside S_sink u S_swa.
 *
 *   For each query b (visible keys [0, q_pos[b]], q_pos[b] < L):
 *     sink   = {0 .. min(sink, q_pos+1)-1}
 *     window = {max(0, q_pos-window+1) .. q_pos} minus sink
 *     cand   = visible positions outside sink u window
 *     sparse = the min(K, |cand|) candidates with the largest scores; equal scores are
 *              ordered by ascending position (exact: fp32 bit patterns are compared)
 *   idx[b*idx_ld + i], i < count[b]: the union, ascending (sink, then sparse, then window);
 *   idx[b*idx_ld + i] = -1 for count[b] <= i < min(idx_ld, K+sink+window).
 *   scores [B, ld] fp32 (16-byte aligned, ld % 4 == 0); idx int32 [B, idx_ld] with
 *   idx_ld >= K + sink + window; count int32 [B].  K >= 1, sink >= 0, window >= 0, L < 2^31.
 *   Needs no scratch memory.
 */
int lsa_topk_select(const float* scores, int64_t ld, int64_t B, int64_t L, int K,
                    int sink, int window, const int64_t* q_pos,
                    int32_t* idx, int64_t idx_ld, int32_t* count, void* stream);

/*
 * lsa_topk_refine -- exact re-ranking of a coarse candidate set (second stage after an FP8 pass).
 *   Source: "LongCat Sparse Attention（LSA）完全拆解", section "机制三：层级索引（HI）": a cheap first stage
 *   recalls candidate tokens, then the standard token-level score I_{t,s} runs on the recalled tokens
 *   only and the final arg topK is taken there.  Here the first stage is lsa_index_score in FP8 mode
 *   followed by lsa_topk_select with K' > K (same sink / window); this call re-scores the K' dynamic
 *   candidates from the bf16 index queries and keys and keeps the top K of them.
 *
 *   cand [B, cand_ld] int32 / cand_count [B]: a row written by lsa_topk_select(..., K', sink, window)
 *   (sink entries, then the dynamic candidates ascending, then the window entries).
 *   For each query b: kept = the min(K, #dynamic) dynamic candidates with the largest
 *   sum_j w[b,j] max(0, q[b,j,:] . k[s,:]) (fp32 from bf16; ties -> lower position);
 *   idx row = sink entries, kept (ascending), window entries; -1 padded up to K + sink + window.
 *   q_idx [B, H_I, d_I] bf16, w [B, H_I] fp32, k_idx [L, d_I] bf16; d_I in {32, 64, 128}, H_I <= 64.
 *   idx_ld >= K + sink + window.  ws: lsa_workspace_size(LSA_OP_REFINE, B, cand_ld, K, 0, 0, 0) bytes.
 */
int lsa_topk_refine(const void* q_idx, const float* w, const void* k_idx, int64_t B, int H_I, int d_I,
                    int64_t L, const int32_t* cand, int64_t cand_ld, const int32_t* cand_count, int K,
                    int sink, int window, const int64_t* q_pos, int32_t* idx, int64_t idx_ld,
                    int32_t* count, void* ws, size_t ws_bytes, void* stream);

/*
 * lsa_pool_keys -- bucket / micro-block representatives (computed once per sequence, cached).
 *   Source: "LongCat Sparse Attention（LSA）完全拆解", section "机制三：层级索引（HI）" (mean of the
 *   sub-block's index keys, computed once and cached); lecture "从两本账看懂长上下文注意力", section
 *   "Qwen Sparse Attention" (index keys mean-pooled in 4-token micro-blocks); "LSA 稀疏注意力會省顯存嗎",
 *   section 二 step 2 (each bucket keeps a representative vector and its member positions).
 *
 *   centroids[c, :] = (1/bsz) * sum_{i<bsz} k[m(c,i), :]  in fp32, members summed in order
 *   m(c,i) = members[c*bsz + i]   (explicit buckets; every entry in [0, L))
 *          = c*bsz + i            (members == NULL: contiguous micro-blocks; NB <= L/bsz)
 *   k_idx [L, d_I] bf16, or e4m3 codes with k_scale [L] (value = code*scale).
 *   centroids [NB, d_I] fp32.  1 <= bsz <= 1024, d_I % 4 == 0.
 */
int lsa_pool_keys(const void* k_idx, int dtype, const float* k_scale, int64_t L, int d_I,
                  const int32_t* members, int bsz, int64_t NB, float* centroids, void* stream);

/*
 * lsa_bucket_select -- Flat bucket or micro-block selection.
 *   Source: "LSA 稀疏注意力會省顯存嗎", section 二 steps 2-4 (Flat compares the bucket
 *   representatives, expands the kept buckets to member positions, adds sink and window);
 *   lecture "从两本账看懂长上下文注意力", sections "Qwen Sparse Attention" and "尾部计数与 query 自身"
 *   (complete micro-blocks are ranked; visible tokens of the incomplete tail block are read
 *   directly); the representative score uses the indexer formula of lsa_index_score.
 *
 *   For each query b:
 *     bscore[c] = sum_j w[b,j] * max(0, q[b,j,:] . centroids[c,:])   (fp32 centroids)
 *     ranked    = all NB buckets (members != NULL), or the complete visible micro-blocks
 *                 c < min(NB, (q_pos+1)/bsz) (members == NULL)
 *     kept      = the M ranked buckets with the largest bscore (ties -> lower bucket id)
 *     idx row   = sorted, de-duplicated union of the kept buckets' positions, the tail
 *                 {bsz*floor((q_pos+1)/bsz) .. q_pos} (micro-block mode only), sink and
 *                 window, restricted to [0, q_pos]; -1 padded up to idx_ld.
 *   q_idx [B, H_I, d_I] bf16 (dtype must be LSA_BF16), w [B, H_I] fp32, centroids [NB, d_I]
 *   fp32, members int32 [NB, bsz] or NULL.  idx int32 [B, idx_ld] with
 *   idx_ld >= M*bsz + sink + window (+ bsz-1 for the micro-block tail); count int32 [B].
 *   1 <= M <= 1024, M*bsz + bsz + sink + window <= 8192.
 *   ws: lsa_workspace_size(LSA_OP_BUCKET, B, NB, M, 0, 0, 0) bytes; at least
 *   lsa_workspace_size(LSA_OP_BUCKET_MIN, B, NB, M, 0, 0, 0) bytes (else LSA_ERR_WORKSPACE).
 *   Scoring: with the full workspace and d_I = 128, H_I in {32, 64}, NB >= 128 the representatives are
 *   scored on the tensor cores from their exact three-part bf16 split (written into the workspace each
 *   call: every product with the bf16 query is exact, the sums are fp32); otherwise on the CUDA cores
 *   (fp32).  Both are fp32-accurate; they can keep different buckets only where two representatives'
 *   scores lie within fp32 rounding of the M-th.
 */
int lsa_bucket_select(const void* q_idx, const float* q_scale, const float* w, int dtype,
                      int64_t B, int H_I, int d_I, const float* centroids, int64_t NB,
                      const int32_t* members, int bsz, int M, int sink, int window, int64_t L,
                      const int64_t* q_pos, int32_t* idx, int64_t idx_ld, int32_t* count,
                      void* ws, size_t ws_bytes, void* stream);

/*
 * lsa_tree_parents -- the level-2 centres of the tree search (untimed precompute, beside the bucket centres).
 *   Source: "超长上下文LSA注意力技术开源", section "Qwen LSA注意力优化原理与核心创新" (keys clustered into a
 *   tree of cluster centres).  The pages give no construction; the reading here: parent p covers buckets
 *   [p*F, min((p+1)*F, NB)) and its centre is their centres' plain mean,
 *     parents[p, d] = (sum_{c in p} centroids[c, d], summed in order) / (number of children)   (fp32)
 *   centroids [NB, d_I] fp32, parents [ceil(NB/F), d_I] fp32.  1 <= d_I <= 128, F >= 1.
 */
int lsa_tree_parents(const float* centroids, int64_t NB, int d_I, int F, float* parents, void* stream);

/*
 * lsa_tree_select -- two-level tree search over the Flat buckets (the Tree form of lsa_bucket_select).
 *   Source: "LSA 稀疏注意力會省顯存嗎", section 二 step 3 (the Tree version searches level by level, keeping
 *   candidates at each level); the same page's step 4 and lsa_bucket_select for the expansion.
 *
 *   For each query b (scores: the indexer formula on a centre, fp32, as lsa_bucket_select):
 *     level 2   kept parents  = the M2 parents with the largest score (ties -> lower parent id)
 *     level 1   candidates    = the kept parents' children, in ascending bucket id
 *               kept buckets  = the M candidates with the largest score (ties -> lower bucket id)
 *     idx row   = sorted, de-duplicated union of the kept buckets' members, sink and window, restricted to
 *                 [0, q_pos]; -1 padded up to idx_ld.  count[b] entries.
 *   With M2 >= NP every bucket is a candidate and the result is lsa_bucket_select's (Flat).
 *   q_idx [B, H_I, d_I] bf16, w [B, H_I] fp32, centroids [NB, d_I] fp32, parents [NP, d_I] fp32 from
 *   lsa_tree_parents (NP = ceil(NB/F)), members int32 [NB, bsz].  d_I in {32, 64, 128}, H_I <= 64,
 *   1 <= M2, M <= 1024; M*bsz + sink + window <= min(8192, idx_ld).
 *   ws: lsa_tree_workspace_size(B, NP, F, M2, M) bytes.
 */
int lsa_tree_select(const void* q_idx, const float* w, int64_t B, int H_I, int d_I, const float* centroids,
                    int64_t NB, const float* parents, int64_t NP, int F, const int32_t* members, int bsz, int M2,
                    int M, int sink, int window, int64_t L, const int64_t* q_pos, int32_t* idx, int64_t idx_ld,
                    int32_t* count, void* ws, size_t ws_bytes, void* stream);

/*
 * lsa_tree_select_split -- lsa_tree_select with the children scored on the tensor cores.
 *   Same search, arguments and result as lsa_tree_select, except that the bucket centres are given as their
 *   exact three-part bf16 split (lsa_split_representatives of the fp32 centroids, split [3, NB, 128] bf16,
 *   cached beside them) instead of the fp32 centres.  A kept parent's children are F consecutive centre rows,
 *   so two kept parents form one 128-row tile against the query's 64 heads; each product is exact and the sums
 *   are fp32, as in lsa_tree_select (results equal up to the order of the fp32 sums).
 *   Requires F = 64, H_I = 64, d_I = 128 (LSA_ERR_UNSUPPORTED otherwise).  ws: lsa_tree_workspace_size.
 */
int lsa_tree_select_split(const void* q_idx, const float* w, int64_t B, int H_I, int d_I, const void* split,
                          int64_t NB, const float* parents, int64_t NP, int F, const int32_t* members, int bsz,
                          int M2, int M, int sink, int window, int64_t L, const int64_t* q_pos, int32_t* idx,
                          int64_t idx_ld, int32_t* count, void* ws, size_t ws_bytes, void* stream);

/* lsa_tree_workspace_size -- scratch bytes of lsa_tree_select(_split); (size_t)-1 for invalid sizes. */
size_t lsa_tree_workspace_size(int64_t B, int64_t NP, int F, int M2, int M);

/*
 * lsa_split_representatives -- the exact three-part bf16 split of fp32 representatives, for
 *   lsa_bucket_select_split: computed once with the representatives (lsa_pool_keys) and cached beside
 *   them.  Not on the pages: a layout of the pages' representative for the tensor cores.
 *
 *   split[p*NB*d_I + c*d_I + d], p = 0, 1, 2, are bf16 with
 *     centroids[c*d_I + d] = split0 + split1 + split2   exactly
 *   (each part is the round-to-nearest bf16 of what the earlier parts leave; 8 + 8 + 8 significand bits).
 *   centroids [NB, d_I] fp32, split bf16 [3, NB, d_I] (6*NB*d_I bytes); both 16-byte aligned; d_I % 4 == 0.
 *   Values must not exceed the largest bf16 (about 3.39e38) in magnitude (means of bf16 keys never do);
 *   larger ones make the first part infinite.
 */
int lsa_split_representatives(const float* centroids, int64_t NB, int d_I, void* split, void* stream);

/*
 * lsa_bucket_select_split -- lsa_bucket_select with the representatives given as their cached split
 *   (lsa_split_representatives), so no per-call conversion.  Same selection rule, arguments and results
 *   as lsa_bucket_select with its full workspace (tensor-core scoring), with `split` in place of
 *   `centroids` (and no q_scale / dtype: q_idx is bf16).  Shapes: d_I = 128, H_I in {32, 64}, NB >= 128
 *   (others: LSA_ERR_UNSUPPORTED).
 *   ws: lsa_workspace_size(LSA_OP_BUCKET_MIN, B, NB, M, 0, 0, 0) bytes.
 */
int lsa_bucket_select_split(const void* q_idx, const float* w, int64_t B, int H_I, int d_I, const void* split,
                            int64_t NB, const int32_t* members, int bsz, int M, int sink, int window, int64_t L,
                            const int64_t* q_pos, int32_t* idx, int64_t idx_ld, int32_t* count,
                            void* ws, size_t ws_bytes, void* stream);

/*
 * lsa_hi_select -- hierarchical (two-stage) selection: pages, then tokens.
 *   Source: "LongCat Sparse Attention（LSA）完全拆解", section "机制三：层级索引（HI）": pages of P tokens,
 *   sub-blocks of Bsub tokens with cached mean index keys; page score
 *     I_page(b, p) = sum_j w[b,j] sum_{n in page p} max(0, q[b,j,:] . kmean_n);
 *   the M best pages are recalled; the token score I(b, s) (lsa_index_score's formula) then runs on the
 *   recalled tokens only, with lsa_topk_select's sink / window union and arg topK over them.
 *
 *   For each query b (q_pos[b] < L):
 *     ranked pages = p with p*P <= q_pos[b]; a page's score sums its complete sub-blocks that end at or
 *                    before q_pos[b] (fp32 sums of fp32-accurate sub-block scores); ties -> lower page
 *     recalled     = tokens of the min(M, #ranked) best pages, plus the visible tokens
 *                    {Bsub*floor((q_pos+1)/Bsub) .. q_pos} of the sub-block holding q_pos when that
 *                    sub-block is not entirely visible (it has no mean key), clipped to [0, q_pos]
 *     idx row      = sink, the min(K, #recalled outside sink u window) recalled tokens with the largest
 *                    I(b, s) (fp32 from bf16; ties -> lower position), window; ascending; -1 padded up to
 *                    K + sink + window (lsa_topk_select's row layout).
 *   q_idx [B, H_I, 128] bf16, w [B, H_I] fp32, k_idx [L, 128] bf16 (the token keys), sub_split = the exact
 *   bf16 split (lsa_split_representatives) of the sub-block means lsa_pool_keys(k_idx, Bsub) gives:
 *   bf16 [3, floor(L/Bsub), 128].  H_I in {32, 64}; floor(L/Bsub) >= 128 (else LSA_ERR_UNSUPPORTED).
 *   P % Bsub == 0, 1 <= M <= 1024.  idx int32 [B, idx_ld], idx_ld >= K + sink + window; count int32 [B].
 *   ws: lsa_hi_workspace_size(B, L, P, Bsub, M, K, sink, window) bytes.
 *   With M*P >= L every visible token is recalled and the result is lsa_index_score + lsa_topk_select's.
 */
int lsa_hi_select(const void* q_idx, const float* w, const void* k_idx, int64_t B, int H_I, int d_I,
                  int64_t L, const void* sub_split, int P, int Bsub, int M, int K, int sink, int window,
                  const int64_t* q_pos, int32_t* idx, int64_t idx_ld, int32_t* count,
                  void* ws, size_t ws_bytes, void* stream);

/* lsa_hi_workspace_size -- scratch bytes of lsa_hi_select; (size_t)-1 for invalid sizes. */
size_t lsa_hi_workspace_size(int64_t B, int64_t L, int P, int Bsub, int M, int K, int sink, int window);

/*
 * lsa_msa_select -- group-wise block selection.
 *   Source: lecture "从两本账看懂长上下文注意力", section "MiniMax Sparse Attention": the index branch scores
 *   tokens, a block's score is the max of its tokens' scores, each GQA group picks its own top-k blocks (the
 *   group's query heads share them) and the current local block is always kept.
 *
 *   Blocks of 128 tokens.  For each query b and group g (index heads [g*64/G, (g+1)*64/G)):
 *     token score  = sum_{j in g} w[b,j] max(0, q[b,j,:] . k[s,:])           (fp32 from bf16)
 *     block score  = max over the block's tokens (blocks before the local block, lb = q_pos[b] / 128)
 *     kept(b, g)   = the min(KB, lb) blocks with the largest block score (ties -> lower block), plus lb
 *   idx row b: the tokens of the union of kept(b, g) over g, ascending (the local block up to q_pos[b]);
 *   gmask[b*idx_ld + i]: bit g set when group g kept the block of idx[b*idx_ld + i]; count[b] entries.
 *   q_idx [B, 64, 128] bf16, w [B, 64] fp32, k_idx [L, 128] bf16; G in {1, 2, 4, 8}; G*KB + 1 <= 1024;
 *   L >= 128.  idx int32 / gmask uint8 [B, idx_ld], idx_ld >= (G*KB + 1) * 128.
 *   ws: lsa_msa_workspace_size(B, L, G, KB) bytes.  The block scores come from the indexer's tensor-core
 *   kernel with a grouped block-max epilogue (no token scores are written).
 */
int lsa_msa_select(const void* q_idx, const float* w, const void* k_idx, int64_t B, int H_I, int d_I,
                   int64_t L, int G, int KB, const int64_t* q_pos, int32_t* idx, uint8_t* gmask,
                   int64_t idx_ld, int32_t* count, void* ws, size_t ws_bytes, void* stream);

/* lsa_msa_workspace_size -- scratch bytes of lsa_msa_select; (size_t)-1 for invalid sizes. */
size_t lsa_msa_workspace_size(int64_t B, int64_t L, int G, int KB);

/*
 * lsa_msa_attn -- attention over a group-wise selection: each head attends to its own group's rows.
 *   Source: the same section (a group's query heads share its blocks).
 *   out[b,h] / lse[b,h] = lsa_sparse_attn's attention of head h (group g = h / (128 / G)) over the entries of
 *   idx[b, :count[b]] whose gmask has bit g.  G = 2, 4, 8: one CTA per (query, 16-head slice of one group) reads
 *   the union row's blocks whose mask has bit g and runs each 128-token block with its rows on the MMA's M side (the
 *   slice's 16 heads on N), no scratch; this needs idx / gmask as lsa_msa_select writes them (whole 128-token
 *   blocks, then the partial local block) and reports LSA_ERR_DEVICE_CHECK (lsa_device_status) for a block whose
 *   entries are not consecutive tokens.  G = 1 (every head shares the union): the rows are compacted
 *   (k_msa_group_rows) and run through the 128-head tensor-core attention.
 *   q [B, 128, 576] bf16, kv [L, 576] bf16 (value = first 512 dims), idx / gmask / count as lsa_msa_select
 *   writes them (idx_ld <= 65536), out [B, 128, 512] bf16, lse [B, 128] fp32 or NULL; all 16-byte aligned.
 *   H = 128, d_qk = 576, d_v = 512, G in {1, 2, 4, 8}, B*G <= 65535.
 *   ws: lsa_msa_attn_workspace_size(B, idx_ld, G) bytes (0 for G = 2, 4, 8: ws may be NULL).
 */
int lsa_msa_attn(const void* q, const void* kv, int64_t L, const int32_t* idx, const uint8_t* gmask,
                 int64_t idx_ld, const int32_t* count, int64_t B, int H, int d_qk, int d_v, int G,
                 float scale, void* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/* lsa_msa_attn_workspace_size -- scratch bytes of lsa_msa_attn; (size_t)-1 for invalid sizes. */
size_t lsa_msa_attn_workspace_size(int64_t B, int64_t idx_ld, int G);

/*
 * lsa_bucket_select_noalloc -- lsa_bucket_select for callers that cannot allocate device memory.
 *   The pages have no counterpart: this is a packaging variant of lsa_bucket_select.
 *
 *   Same arguments, layouts and results as lsa_bucket_select given the smaller workspace
 *   (LSA_OP_BUCKET_MIN: CUDA-core scoring), minus ws / ws_bytes.  It is meant for
 *   callers that may not call cudaMalloc (or any allocating library routine) where they select: a
 *   plugin inside a host framework that owns every device allocation, a thread that must stay out of
 *   the CUDA allocator, or a process with no allocation budget left.  The scratch comes from an 8 MiB
 *   buffer compiled into the library as a __device__ array; the CUDA runtime creates it on every GPU
 *   that loads the library, and it stays allocated there until the process exits.  The call itself
 *   allocates nothing.
 *   - Limit: lsa_workspace_size(LSA_OP_BUCKET_MIN, B, NB, M, 0, 0, 0) must be <= 8 MiB (8388608 bytes);
 *     larger requests return LSA_ERR_WORKSPACE before anything is launched (lsa_last_error() gives
 *     the sizes).  Flat selection over 156250 buckets fits up to B = 13 queries.
 *   - Set-up: the first call on a device looks up the buffer's device address (cudaGetSymbolAddress,
 *     with that device current) and caches it; make that first call before any stream capture.  Under
 *     lazy module loading (the CUDA 12 default) that lookup also loads the library's module on the
 *     device, which is when the runtime creates the 8 MiB buffer: a caller that must not see any
 *     allocation at selection time makes one warm-up call beforehand.  Later calls allocate nothing.
 *     The cached address belongs to the device's primary context; after cudaDeviceReset on that
 *     device, calling this entry point there again is not supported.
 *   - Sharing: every call on a device uses the same buffer, which keeps the last call's contents
 *     (nothing in it needs clearing: each call writes what it reads).  Calls whose work overlaps on
 *     the GPU (concurrent streams, or threads without ordering between their streams) race on it;
 *     order them on one stream.
 */
int lsa_bucket_select_noalloc(const void* q_idx, const float* q_scale, const float* w, int dtype,
                              int64_t B, int H_I, int d_I, const float* centroids, int64_t NB,
                              const int32_t* members, int bsz, int M, int sink, int window, int64_t L,
                              const int64_t* q_pos, int32_t* idx, int64_t idx_ld, int32_t* count,
                              void* stream);

/*
 * lsa_sparse_attn -- sparse attention over the gathered MLA latent rows (absorbed MQA).
 *   Source: "LongCat Sparse Attention（LSA）完全拆解", section "DSA 基线", u_t = Attn(h_t, {c_s |
 *   s in S_t}) with c_s the MLA latent shared by every query head; the 1152-byte bf16 latent row
 *   (section "瓶颈一"); "LSA 稀疏注意力會省顯存嗎", section 四 (scores q.k scaled, softmax, weighted V).
 *
 *   For each query b and head h, with S = {idx[b*idx_ld + i] : i < count[b]}:
 *     z_s      = scale * q[b,h,:] . kv[s, 0:d_qk]
 *     out[b,h] = sum_s softmax(z)_s * kv[s, 0:d_v]          (bf16, fp32 accumulation)
 *     lse[b,h] = log sum_s exp(z_s)                          (natural log; -inf if S empty)
 *   An empty set gives out = 0.  Entries of idx must lie in [0, L) (an entry outside is clamped, so the
 *   access stays in bounds, and lsa_device_status reports LSA_ERR_DEVICE_CHECK); the call does not read
 *   idx past count[b].
 *   Kernels: decode-sized batches (every query's rows in units of at most 256, at most 148 units) run one
 *   unit per SM in two passes (logits and softmax, then P.V) and a merge of the units; larger batches run
 *   the value-half kernel.  H < 128 runs the same kernels on zero-padded 128-head queries.  Programmatic
 *   dependent launch: the decode kernel may start loading q while the kernel before it on `stream` is
 *   still running, when that kernel signalled its dependents early (the library's own kernels do, and none
 *   of them writes a query); every other input is read after that kernel has completed.
 *   q   [B, H, d_qk] bf16;  kv [L, d_qk] bf16 (row stride d_qk);  out [B, H, d_v] bf16;
 *   lse [B, H] fp32 or NULL.  Supported: d_qk = 576, d_v = 512, H in {16, 32, 64, 128},
 *   idx_ld >= max count, max count <= 65536.  q, kv, out 16-byte aligned.
 *   ws: lsa_workspace_size(LSA_OP_ATTN, B, L, Kmax=idx_ld, H, 0, 0) bytes.
 */
int lsa_sparse_attn(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                    const int32_t* count, int64_t B, int H, int d_qk, int d_v, float scale,
                    void* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * lsa_hybrid_attn -- lsa_sparse_attn over a selection row split into its two parts, run concurrently.
 *   Source: "LongCat Sparse Attention（LSA）完全拆解", section "训练与 kernel：混合稀疏注意力算子（HFA）": the
 *   core attention is split into a sparse-gather operator over S_sparse and a sliding-window operator over
 *   the contiguous positions, dispatched on separate non-blocking streams and merged by online-softmax
 *   (log-sum-exp) rescaling -- mathematically one attention over the union.
 *
 *   idx / count: rows in lsa_topk_select's layout (sink entries, then the sparse entries, then the window
 *   entries, for the same sink / window / q_pos).  The fixed part (sink {0..} and window {..q_pos}) is read
 *   as contiguous positions; the sparse part from the row.  out / lse: as lsa_sparse_attn over the whole row
 *   (equal up to fp32 rounding of the merge).  The fixed part runs on a library-owned second stream (created
 *   on the first call on a device: make that call before any stream capture), forked from and joined back
 *   into `stream` with events.  H other than 128: one pass over the union on `stream`.
 *   ws: lsa_workspace_size(LSA_OP_HYBRID_ATTN, B, L, idx_ld, H, sink, window) bytes.
 */
int lsa_hybrid_attn(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                    const int32_t* count, int64_t B, int H, int d_qk, int d_v, int sink, int window,
                    const int64_t* q_pos, float scale, void* out, float* lse, void* ws, size_t ws_bytes,
                    void* stream);

/*
 * lsa_workspace_size -- scratch bytes a call needs (0 if none).
 *   op = LSA_OP_TOPK:   0.
 *   op = LSA_OP_BUCKET: (B, L=NB, K=M) -> per-query bucket scores and kept-bucket lists, plus the
 *                       representatives' bf16 split for tensor-core scoring (NB * 768 bytes).
 *   op = LSA_OP_BUCKET_MIN: the same without the split (CUDA-core scoring).
 *   op = LSA_OP_ATTN:   (B, L, K=idx_ld, H) -> split-K partial outputs.
 *   op = LSA_OP_HYBRID_ATTN: (B, L, K=idx_ld, H, sink, window) -> both branches' partials and index rows.
 *   op = LSA_OP_REFINE: (B, L=cand_ld, K) -> re-ranked scores and kept lists.
 *   Returns (size_t)-1 for an unknown op or negative sizes.
 */
size_t lsa_workspace_size(int op, int64_t B, int64_t L, int K, int H, int sink, int window);

/* lsa_strerror -- static description of a status code (never NULL). */
const char* lsa_strerror(int status);

/* lsa_last_error -- the last CUDA error message seen by this thread ("" if none). */
const char* lsa_last_error(void);

/* lsa_version -- library version string. */
const char* lsa_version(void);

/*
 * lsa_device_status -- whether a kernel gave up a bounded wait or failed a device-side check.
 *   Every wait of the tensor-core kernels (indexer, re-rank re-score, attention) on an mbarrier is bounded
 *   (2 s of globaltimer); a wait that runs out sets a device flag, the kernel's other roles stop at their next
 *   wait, the issuing threads wait (bounded) for the copies and MMAs they started, TMEM is freed and the
 *   outputs of that launch are not valid.  The decode attention kernel also checks every selected index
 *   against [0, L): an index outside it is clamped (the access stays in bounds) and flagged.
 *   This call synchronises `stream`, then reads and clears the flags: LSA_ERR_TIMEOUT if a wait gave up since
 *   the previous call, else LSA_ERR_DEVICE_CHECK if an index check failed (lsa_last_error names the kernel),
 *   LSA_ERR_CUDA if the stream or the flag read failed, else LSA_OK.  Not part of the hot path (it blocks the
 *   host); meant for a serving loop's periodic health check.
 */
int lsa_device_status(void* stream);

/*
 * lsa_selftest_wait -- exercises the bounded-wait give-up path that lsa_device_status reports.
 *   The pages have no counterpart: this is a health check of the library's failure reporting.
 *   Launches one thread that waits on an mbarrier nothing ever completes, for at most limit_ns nanoseconds
 *   of globaltimer (1 <= limit_ns <= 10^9); the wait runs out, the kernel records the give-up in the same
 *   way as the tensor-core kernels and returns.  No copy, MMA or TMEM is involved, so nothing is left in
 *   flight.  The next lsa_device_status on `stream` returns LSA_ERR_TIMEOUT naming "k_selftest_wait", and
 *   the one after it LSA_OK.  Returns LSA_ERR_INVALID_ARG for a limit outside the range.
 */
int lsa_selftest_wait(uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H_ */
