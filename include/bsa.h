/*
 * bsa.h -- C ABI of the B200 (sm_100a) dynamic block-sparse attention library.
 *
 * The library implements the selection-then-attention path for video
 * diffusion transformers:
 *
 *   bsa_block_scores   block centroids of Q and K, then the cluster-size-
 *                      weighted softmax P' over key blocks
 *   bsa_build_mask     per-row top-p over P', text-block keep, frame-0 dense
 *                      override, per-head entropy, compacted key-block lists
 *   bsa_attention_fwd  exact softmax attention over the listed key blocks only
 *   bsa_dense_fwd      the same kernel with every key block listed
 *
 * Sources (pages by title and section):
 *   "Attention matrix view: make only frame-0 query rows dense"
 *       s1 token packing [text] + frame0 + frame1 + ...; s2 dense rows vs
 *       sparse rows; s4 block-level override of the query blocks that overlap
 *       frame 0; s7 keep text/global blocks.
 *   "Competition Domains Matter: Selective Head Globalization for
 *    Training-Free Sparse Attention in Video Diffusion Transformers"
 *       s3: centroids with cluster sizes n_i, n_j; cluster-size-weighted
 *       softmax P' (Eq. 1; rows sum to one); per-head entropy H_h (Eq. 3)
 *       and H_h / log C_k; per-row local top-p (domain 1, Eq. 2).
 *   "AB-Attention: accurate block-sparse attention for video diffusion"
 *       TL;DR: exact attention computed only on the selected K/V blocks; key
 *       blocks smaller than a tensor-core tile gathered into full tiles.
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, row-major, and live in device memory that the caller
 *     allocated.  The library allocates nothing, frees nothing and keeps no
 *     state between calls beyond a cached driver entry point.
 *   - Q, K, V and O are bf16 [batch, heads, seq_pad, head_dim].  Token t of
 *     (b, h) is row t; rows seq_len..seq_pad-1 are padding and are never read
 *     as keys.  Every other array is described at its entry point.
 *   - Query block i covers tokens [i*q_block, (i+1)*q_block); key block j
 *     covers [j*k_block, (j+1)*k_block).  C_q = seq_pad / q_block,
 *     C_k = seq_pad / k_block.  n_j = number of tokens of block j below
 *     seq_len.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and never synchronises.
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check returns BSA_ERR_INVALID_ARG (or BSA_ERR_UNSUPPORTED for a
 *     valid shape the library has no kernel for) and launches nothing.
 *   - A launch failure returns BSA_ERR_LAUNCH; a failure of the CUDA driver's
 *     tensor-map encoder returns BSA_ERR_DRIVER.
 *   - Bad data found on the device (a list entry outside [0, C_k), a count
 *     outside [0, C_k], a wait that timed out) never traps: the kernel skips
 *     the offending item and ORs a BSA_DEVERR_* bit into *err_flag when the
 *     caller passed one (a device int32 the caller zeroes beforehand).
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Problem geometry ("Attention matrix view ..." s1 and s4). */
typedef struct bsa_layout {
    int32_t batch;            /* B >= 1 */
    int32_t heads;            /* H, 1..256 */
    int32_t seq_len;          /* S valid tokens, >= 1 */
    int32_t seq_pad;          /* padded length: a multiple of max(q_block, k_block),
                                 seq_pad - seq_len < min(q_block, k_block) so that
                                 every block holds at least one valid token */
    int32_t head_dim;         /* D: 64 or 128 */
    int32_t q_block;          /* 64 or 128 */
    int32_t k_block;          /* 64 or 128 */
    int32_t text_len;         /* text tokens at the front of the sequence, >= 0 */
    int32_t tokens_per_frame; /* latent_h * latent_w, >= 0 */
    int32_t num_frames;       /* >= 0; text_len + num_frames*tokens_per_frame <= seq_len */
} bsa_layout;

enum bsa_status {
    BSA_OK = 0,
    BSA_ERR_INVALID_ARG = 1,
    BSA_ERR_UNSUPPORTED = 2,
    BSA_ERR_LAUNCH = 3,
    BSA_ERR_DRIVER = 4
};

/* bsa_build_mask flags */
enum bsa_flags {
    BSA_TEXT_KEEP = 1u,     /* keep every key block that holds a text token ("... s7") */
    BSA_FRAME0_DENSE = 2u   /* every key block for query blocks overlapping frame 0 ("... s4") */
};

/* Bits ORed into *err_flag by device code. */
enum bsa_device_error {
    BSA_DEVERR_BAD_INDEX = 1,  /* a kv_index entry outside [0, C_k): entry skipped */
    BSA_DEVERR_BAD_COUNT = 2,  /* a kv_count outside [0, C_k]: clamped */
    BSA_DEVERR_TIMEOUT = 4     /* an internal pipeline wait gave up: the tile's output is invalid */
};

/*
 * Block centroids and block scores ("Competition Domains Matter" s3, Eq. 1).
 *
 *   q_centroids[b,h,i,:] = mean of Q rows of query block i below seq_len
 *   k_centroids[b,h,j,:] = mean of K rows of key block j below seq_len
 *   s_ij  = q_centroids_i . k_centroids_j / sqrt(head_dim)
 *   probs[b,h,i,j] = P'_ij = n_j exp(s_ij) / sum_j' n_j' exp(s_ij')
 *
 * q, k          bf16 [B,H,seq_pad,D], 16-byte aligned (read only)
 * q_centroids   fp32 [B,H,C_q,D], 16-byte aligned (written)
 * k_centroids   fp32 [B,H,C_k,D], 16-byte aligned (written)
 * probs         fp32 [B,H,C_q,C_k], 16-byte aligned (written; each row sums to 1)
 * Accumulation is fp32.  Supports C_k up to 2048.
 */
int bsa_block_scores(const bsa_layout *layout, const void *q, const void *k,
                     float *q_centroids, float *k_centroids, float *probs, void *stream);

/*
 * Block scores from intra-block query clusters ("AB-Attention: accurate
 * block-sparse attention for video diffusion", TL;DR fix (1): the queries of
 * each query block are clustered among themselves, tokens stay in place, so
 * the importance estimate is finer than one block mean).  The page gives no
 * procedure; this one is used.  Per query block: k-means (Lloyd) on its valid
 * query tokens with n_sub clusters, seeded with the tokens at positions
 * floor(c * n / n_sub) (n = valid tokens), squared Euclidean distance, ties
 * to the lower cluster, `iters` rounds of (assign, move every non-empty
 * cluster to its mean; an empty one keeps its centroid and has size 0), in
 * fp32.  The block's row of P' is the size-weighted mixture of the
 * sub-centroids' cluster-size-weighted softmax rows,
 *   P'_ij = sum_c (n_c / n_i) n_j exp(s_cj) / sum_j' n_j' exp(s_cj'),
 *   s_cj = q_c . k_j / sqrt(D),
 * so rows sum to one and n_sub = 1 is bsa_block_scores.  P' then feeds
 * bsa_build_mask / bsa_build_mask_eg / bsa_build_mask_sampled unchanged.
 *
 * n_sub          1, 2, 4, 8 or 16 (else BSA_ERR_UNSUPPORTED)
 * iters          1 .. 1000
 * sub_centroids  fp32 [B,H,C_q,n_sub,D], 16-byte aligned (written)
 * sub_sizes      int32 [B,H,C_q,n_sub] (written)
 * k_centroids    fp32 [B,H,C_k,D], 16-byte aligned (written)
 * probs          fp32 [B,H,C_q,C_k], 16-byte aligned (written)
 * workspace      device scratch of
 *                bsa_block_scores_clustered_workspace_bytes(layout, n_sub)
 *                bytes (the sub-centroid rows), 256-byte aligned
 */
int bsa_block_scores_clustered(const bsa_layout *layout, const void *q, const void *k, int n_sub,
                               int iters, float *sub_centroids, int32_t *sub_sizes,
                               float *k_centroids, float *probs, void *workspace, void *stream);

/* Bytes of device workspace bsa_block_scores_clustered needs (0: invalid). */
size_t bsa_block_scores_clustered_workspace_bytes(const bsa_layout *layout, int n_sub);

/* Bytes of device workspace bsa_build_mask needs (per-row entropies). */
size_t bsa_build_mask_workspace_bytes(const bsa_layout *layout);

/*
 * Selection ("Competition Domains Matter" s3 domain 1 and Eq. 3;
 * "Attention matrix view ..." s4, s6, s7).  For every row (b,h,i):
 *   1. top-p: order the row by (P' descending, j ascending) and keep the
 *      shortest prefix whose running sum reaches top_p[h] (the entry that
 *      reaches it included); keep the whole row if it never does;
 *   2. BSA_TEXT_KEEP: also keep key blocks j < ceil(text_len / k_block);
 *   3. BSA_FRAME0_DENSE: keep every key block when
 *      text_len / q_block <= i <= (text_len + tokens_per_frame - 1) / q_block;
 *   4. write the kept key blocks in ascending order to kv_index[b,h,i,0..n-1]
 *      and n to kv_count[b,h,i]; entries from n on are left unspecified.
 * Per head: entropy[b,h] = (1/C_q) sum_i -sum_j P'_ij ln(P'_ij + eps) and
 * entropy_norm[b,h] = entropy[b,h] / ln C_k.
 *
 * probs         fp32 [B,H,C_q,C_k] (read only)
 * top_p         HOST fp32 [H], per-head p (read during the call only)
 * flags         BSA_TEXT_KEEP | BSA_FRAME0_DENSE
 * eps           entropy stabiliser (e.g. 1e-8)
 * mask          u8 [B,H,C_q,C_k] 0/1 block mask, or NULL to skip it
 * kv_index      int32 [B,H,C_q,C_k], 4-byte aligned (written)
 * kv_count      int32 [B,H,C_q] (written)
 * entropy       fp32 [B,H], or NULL to skip the entropy
 * entropy_norm  fp32 [B,H], or NULL
 * workspace     device scratch of bsa_build_mask_workspace_bytes(layout) bytes,
 *               16-byte aligned; required when entropy or entropy_norm is set;
 *               its contents on entry do not matter and are clobbered
 * Supports C_k up to 2048.
 */
int bsa_build_mask(const bsa_layout *layout, const float *probs, const float *top_p,
                   uint32_t flags, float eps, uint8_t *mask, int32_t *kv_index,
                   int32_t *kv_count, float *entropy, float *entropy_norm,
                   void *workspace, void *stream);

/*
 * bsa_build_mask without a workspace, for callers that cannot allocate device
 * memory (a framework allocator or memory-planning pass, a process whose device
 * memory is reserved up front, a plugin whose host owns every allocation).
 * The pages have no counterpart: this is a deployment variant of
 * bsa_build_mask, not a step of the method.
 *
 * Same arguments and results as bsa_build_mask minus `workspace`: the
 * per-row entropies go to a fixed array inside the library (4 bytes per row,
 * BSA_NOALLOC_MAX_MASK_ROWS rows, resident on every GPU that loads the
 * library until the process exits).  When entropy or entropy_norm is given,
 * returns BSA_ERR_UNSUPPORTED if batch * heads * (seq_pad / q_block) exceeds
 * BSA_NOALLOC_MAX_MASK_ROWS and BSA_ERR_LAUNCH if the array's device address
 * cannot be obtained; a call that asks for neither uses no workspace, so the
 * array neither caps it nor is touched.  The call allocates and frees nothing.
 * All calls on a device share the array (it keeps the last call's contents;
 * nothing in it needs clearing), so calls that overlap on the GPU race.
 * The first call on each device that asks for entropies looks the array up
 * (cudaGetSymbolAddress) with that device current.  Under CUDA's default lazy
 * module loading that lookup also loads the module holding the array, so the
 * array's 1 MB is reserved by that first call: make it before reserving the
 * rest of device memory and before any stream capture.  The address is cached
 * per device with the current context's id; after a device reset (a new
 * context) the next call looks it up again.
 */
#define BSA_NOALLOC_MAX_MASK_ROWS 262144
int bsa_build_mask_noalloc(const bsa_layout *layout, const float *probs, const float *top_p,
                           uint32_t flags, float eps, uint8_t *mask, int32_t *kv_index,
                           int32_t *kv_count, float *entropy, float *entropy_norm, void *stream);

/*
 * Value-centroid norms for the value-aware score of the entropy-guided
 * selection ("Competition Domains Matter ..." s4): for every key block j of
 * every (b, h), the centroid c^V = mean of V over the block's valid tokens
 * (as for the key centroid) and vnorm[b,h,j] = ||c^V||_2.
 *
 * v      bf16 [B,H,seq_pad,D], 16-byte aligned (read)
 * vnorm  fp32 [B,H,C_k] (written)
 */
int bsa_value_norms(const bsa_layout *layout, const void *v, float *vnorm, void *stream);

/*
 * Entropy-guided selection (EG-Sparse; "Competition Domains Matter ..."
 * s3.3 domain 3 "grouped cross-head", the one-key-per-row safeguard, s4 the
 * value-aware score).  Per batch entry the heads are split at the median of
 * their entropy H_h: ordered by (H_h ascending, h ascending), the first
 * floor(H/2) are pooled, the others keep the per-row local top-p of
 * bsa_build_mask with their top_p[h].  All pairs (h, i, j) of the pooled heads
 * of one batch entry compete in one pool, ranked by the score
 * I = P'[b,h,i,j] * vnorm[b,h,j] (the fp32 product; P' alone when vnorm is
 * NULL) in (I descending, h, i, j ascending) order; the pool keeps the
 * shortest prefix whose running sum reaches pool_p times the pool's total
 * score (everything if it never does; its first pair if pool_p <= 0).  A
 * pooled row left empty then keeps its single highest-scoring key block
 * (lowest j on ties).  The text-keep and frame-0 overrides and the lists
 * follow as in bsa_build_mask.  The cut is found without sorting by an exact
 * radix select over the scores' bit patterns with integer significand sums.
 *
 * probs         fp32 [B,H,C_q,C_k] (read)
 * vnorm         fp32 [B,H,C_k] from bsa_value_norms, or NULL (rank by P')
 * top_p         HOST fp32 [H]: p of the per-row heads
 * pool_p        p of the cross-head pools
 * flags, eps    as for bsa_build_mask
 * mask, kv_index, kv_count   as for bsa_build_mask (mask may be NULL)
 * entropy, entropy_norm      fp32 [B,H], or NULL (always computed)
 * low_heads     u8 [B,H]: 1 for the pooled heads, or NULL
 * workspace     device scratch of bsa_build_mask_eg_workspace_bytes(layout)
 *               bytes, 256-byte aligned; contents on entry do not matter
 */
int bsa_build_mask_eg(const bsa_layout *layout, const float *probs, const float *vnorm,
                      const float *top_p, float pool_p, uint32_t flags, float eps, uint8_t *mask,
                      int32_t *kv_index, int32_t *kv_count, float *entropy, float *entropy_norm,
                      uint8_t *low_heads, void *workspace, void *stream);

/*
 * Competition domains ("Competition Domains Matter ..." s3): which pairs
 * (h, i, j) of one batch entry compete for one top-p budget.
 *   BSA_DOMAIN_ROW      per-row local: no pools, every row the rule of bsa_build_mask
 *   BSA_DOMAIN_HEAD     per-head global: pool g = head g (G = H pools)
 *   BSA_DOMAIN_GROUPED  grouped cross-head with both groups pooled: the floor(H/2)
 *                       lowest-entropy heads form pool 0, the rest pool 1 (G = 2)
 *   BSA_DOMAIN_ALL      all-head global: one pool of every head (G = 1)
 *   BSA_DOMAIN_EG       EG-Sparse: the low-entropy half pooled (pool 0), the
 *                       rest per-row (G = 1); bsa_build_mask_eg
 * The entropy split is the one of bsa_build_mask_eg.
 */
enum bsa_domain {
    BSA_DOMAIN_ROW = 0,
    BSA_DOMAIN_HEAD = 1,
    BSA_DOMAIN_GROUPED = 2,
    BSA_DOMAIN_ALL = 3,
    BSA_DOMAIN_EG = 4
};

/* Bytes of device scratch bsa_build_mask_domain needs for `domain` (0 on a bad
 * layout or domain). */
size_t bsa_build_mask_domain_workspace_bytes(const bsa_layout *layout, int domain);

/*
 * Pooled top-p over a competition domain: as bsa_build_mask_eg, with the pools
 * of `domain` (enum bsa_domain).  Every pool ranks its pairs by the score I of
 * bsa_build_mask_eg in (I descending, h, i, j ascending) order, keeps the
 * shortest prefix reaching pool_p times its total score, and then gives a row
 * it left empty its best key block; rows of unpooled heads keep their per-row
 * top_p[h].  BSA_DOMAIN_EG gives exactly bsa_build_mask_eg.
 *
 * pool_of       i8 [B,H]: each head's pool (-1 = per-row), or NULL
 * workspace     device scratch of bsa_build_mask_domain_workspace_bytes(layout,
 *               domain) bytes, 256-byte aligned
 * other arguments as for bsa_build_mask_eg.  Returns BSA_ERR_INVALID_ARG for a
 * domain outside the enum.
 */
int bsa_build_mask_domain(const bsa_layout *layout, int domain, const float *probs,
                          const float *vnorm, const float *top_p, float pool_p, uint32_t flags,
                          float eps, uint8_t *mask, int32_t *kv_index, int32_t *kv_count,
                          float *entropy, float *entropy_norm, int8_t *pool_of, void *workspace,
                          void *stream);

/* Bytes of device workspace bsa_build_mask_eg needs (0: invalid layout). */
size_t bsa_build_mask_eg_workspace_bytes(const bsa_layout *layout);

/*
 * Importance sampling of key blocks ("AB-Attention: accurate block-sparse
 * attention for video diffusion", TL;DR fix (2): blocks are sampled in
 * proportion to importance and reweighted by the inverse inclusion
 * probability, so that one pass is an unbiased estimate of dense attention).
 * The page gives no sampling law; this one is used: every pair (b, h, i, j)
 * is included independently with probability pi = min(1, fp32(budget * P'))
 * (negative or NaN P' as 0; a row keeps at most `budget` blocks in
 * expectation since its P' sums to one).  The draw of pair
 * idx = ((b*H + h)*C_q + i)*C_k + j is u = (z >> 40) * 2^-24, z the idx-th
 * output (from 0) of SplitMix64 started from state `seed`; the pair is
 * included iff u < pi, and then carries the weight w = 1/pi (fp32, correctly
 * rounded).  With BSA_TEXT_KEEP / BSA_FRAME0_DENSE the text key columns /
 * frame-0 query blocks are included with pi = 1, w = 1.  Same seed, same
 * draw, on any device.
 *
 * probs      fp32 [B,H,C_q,C_k] (read)
 * budget     finite, >= 0 (else BSA_ERR_INVALID_ARG)
 * mask       u8 [B,H,C_q,C_k] (written) or NULL
 * kv_index   int32 [B,H,C_q,C_k]: included key blocks ascending in the first
 *            kv_count entries (written)
 * kv_weight  fp32 [B,H,C_q,C_k]: w of kv_index's entries, same positions (written)
 * kv_count   int32 [B,H,C_q] (written)
 * C_k above 2048: BSA_ERR_UNSUPPORTED.
 */
int bsa_build_mask_sampled(const bsa_layout *layout, const float *probs, float budget,
                           uint64_t seed, uint32_t flags, uint8_t *mask, int32_t *kv_index,
                           float *kv_weight, int32_t *kv_count, void *stream);

/*
 * Block-sparse exact attention ("Attention matrix view ..." s2;
 * "AB-Attention ..." TL;DR).  For every valid query token t of query block i:
 *   U = tokens u < seq_len of the key blocks kv_index[b,h,i,0..kv_count-1]
 *   O_t = sum_{u in U} softmax_u(softmax_scale * Q_t . K_u) V_u
 *   lse_t = ln sum_{u in U} exp(softmax_scale * Q_t . K_u)
 * computed with bf16 tensor-core products and fp32 softmax/accumulation.
 * Padded query rows (t >= seq_len) get O = 0 and lse = -inf; a row with no
 * valid key gets the same.  With k_block = 64, consecutive list entries are
 * paired into one 128-key tensor-core tile.
 *
 * One CTA per SM walks the (batch, head, query block) work items in
 * head-major order.  With a workspace the CTAs claim items from a counter in
 * it, which balances rows of very different list lengths (dense frame-0 rows
 * next to sparse ones); without one, CTA c takes items c, c + #SMs, ...
 *
 * q, k, v       bf16 [B,H,seq_pad,D], 16-byte aligned (read only)
 * kv_index      int32 [B,H,C_q,C_k], ascending within a row (read only)
 * kv_count      int32 [B,H,C_q] (read only)
 * softmax_scale usually 1/sqrt(D)
 * out           bf16 [B,H,seq_pad,D], 16-byte aligned (written)
 * lse           fp32 [B,H,seq_pad], or NULL
 * err_flag      device int32, or NULL (see BSA_DEVERR_*)
 * workspace     device scratch of bsa_attention_workspace_bytes(layout) bytes,
 *               16-byte aligned, or NULL.  Its contents on entry do not matter
 *               (the call clears it on `stream` first); two calls that share
 *               one workspace must not run at the same time.
 */
int bsa_attention_fwd(const bsa_layout *layout, const void *q, const void *k, const void *v,
                      const int32_t *kv_index, const int32_t *kv_count, float softmax_scale,
                      void *out, float *lse, int32_t *err_flag, void *workspace, void *stream);

/*
 * bsa_attention_fwd with inverse-inclusion-probability weights
 * ("AB-Attention ..." TL;DR fix (2)): every exp term of a key of list entry e
 * is multiplied by kv_weight[b,h,i,e], in the numerator and in the sum alike:
 *   O_t = sum_u w_u exp(s_u) V_u / sum_u w_u exp(s_u),
 *   lse_t = ln sum_u w_u exp(s_u),  s_u = softmax_scale * Q_t . K_u,
 * which with the weights of bsa_build_mask_sampled makes the numerator and the
 * sum unbiased estimates of the dense ones.  Weights must be positive and
 * finite.  Everything else as for bsa_attention_fwd.
 *
 * kv_weight  fp32 [B,H,C_q,C_k], entry e beside kv_index's entry e (read only)
 */
int bsa_attention_fwd_weighted(const bsa_layout *layout, const void *q, const void *k,
                               const void *v, const int32_t *kv_index, const float *kv_weight,
                               const int32_t *kv_count, float softmax_scale, void *out, float *lse,
                               int32_t *err_flag, void *workspace, void *stream);

/*
 * Head profiling for autoregressive video generation ("Efficient
 * Autoregressive Video Diffusion with Dummy Head", Step 0 frame attention
 * score).  The layout describes the key window: num_frames >= 2 frames of
 * tokens_per_frame tokens, text_len 0, seq_len = num_frames *
 * tokens_per_frame; frame 0 is the sink, frames 1 .. F-2 the neighbor window,
 * frame F-1 the current frame.  For every (b, h) and every query_stride-th
 * token t of the current frame (from its first token), the softmax of
 * softmax_scale * Q_t . K_u over the whole window is summed per group, and
 * alpha[b,h,:] = [alpha_sink, alpha_neighbor, alpha_current] is the mean over
 * those queries (it sums to one).  Computed on the tensor cores as the
 * attention of the current frame's query blocks over a one-hot V of the key
 * groups (bf16 P: expect ~1e-3 absolute error).
 *
 * q, k       bf16 [B,H,seq_pad,D], 16-byte aligned (read)
 * alpha      fp32 [B,H,3] device (written)
 * workspace  device scratch of bsa_frame_scores_workspace_bytes(layout) bytes,
 *            256-byte aligned
 * A layout that is not such a window: BSA_ERR_INVALID_ARG.
 */
int bsa_frame_scores(const bsa_layout *layout, const void *q, const void *k, float softmax_scale,
                     int query_stride, float *alpha, void *workspace, void *stream);

/* Bytes of device workspace bsa_frame_scores needs (0: invalid layout). */
size_t bsa_frame_scores_workspace_bytes(const bsa_layout *layout);

enum { BSA_HEAD_SINK = 0, BSA_HEAD_NEIGHBOR = 1, BSA_HEAD_DUMMY = 2 };

/*
 * Dynamic Head Programming ("... Dummy Head", Step 1), on the HOST: from
 * alpha [heads][3] (host memory, e.g. one (b) slice of bsa_frame_scores'
 * output), the n_dummy heads with the smallest l_h = max(alpha_sink,
 * alpha_neighbor) (lower h on ties) are labelled BSA_HEAD_DUMMY, every other
 * head BSA_HEAD_SINK if alpha_sink > alpha_neighbor, else BSA_HEAD_NEIGHBOR.
 * labels: int32 [heads] host memory (written).  NaN entries, n_dummy outside
 * [0, heads]: BSA_ERR_INVALID_ARG.  No CUDA call is made.
 */
int bsa_dhp_labels(const float *alpha, int heads, int n_dummy, int32_t *labels);

/* Bytes of device workspace bsa_attention_fwd / bsa_dense_fwd can use. */
size_t bsa_attention_workspace_bytes(const bsa_layout *layout);

/*
 * Dense exact attention: bsa_attention_fwd with every key block selected for
 * every query block ("Attention matrix view ..." s2, the dense rows).
 * Arguments as for bsa_attention_fwd.
 */
int bsa_dense_fwd(const bsa_layout *layout, const void *q, const void *k, const void *v,
                  float softmax_scale, void *out, float *lse, int32_t *err_flag, void *workspace,
                  void *stream);

/*
 * The whole path for host-resident tensors: bsa_block_scores, bsa_build_mask
 * (mask bytes not kept) and bsa_attention_fwd, with the host<->device copies
 * overlapped with the kernels.  The path is independent per (b, h) ("Competition
 * Domains Matter ..." s3 domain 1 selects per head and query row; attention is
 * per head), so the heads of each batch entry are cut into groups of
 * heads_per_group: while group c computes on compute_stream, Q, K, V of group
 * c+1 travel in on h2d_stream and O of group c-1 travels out on d2h_stream,
 * through two device slots inside `workspace`.  Results equal those of the
 * three device entry points called on the same data.
 *
 * heads_per_group  heads per group (>= 1; larger than H means all heads)
 * q, k, v          HOST bf16 [B,H,seq_pad,D] (read).  Page-locked memory
 *                  (cudaHostAlloc / cudaHostRegister) is needed for the copies
 *                  to overlap anything; pageable memory works but serialises.
 * top_p            host fp32 [H]; flags, eps, softmax_scale as above
 * out              HOST bf16 [B,H,seq_pad,D] (written)
 * entropy          HOST fp32 [B,H], or NULL; entropy_norm likewise
 * kv_count         HOST int32 [B,H,C_q] (the list lengths), or NULL
 * err_flag         HOST int32, or NULL: receives the OR of the BSA_DEVERR_*
 *                  bits of every attention launch of the call
 * workspace        device memory, 256-byte aligned, of at least
 *                  bsa_pipeline_workspace_bytes(layout, heads_per_group)
 *                  bytes; owned by the call until it completes
 * compute_stream, h2d_stream, d2h_stream
 *                  cudaStream_t values; they may coincide (no overlap then).
 *
 * Asynchronous: everything is ordered after the work already queued on
 * compute_stream, and compute_stream is made to wait for the last copy, so
 * synchronising compute_stream (or an event recorded on it after the call)
 * means every output is on the host.  The host buffers must stay valid until
 * then.  The call creates and releases a few CUDA events; it allocates no
 * memory.  On an error return some copies may already be queued: synchronise
 * all three streams before reusing the buffers.
 */
int bsa_sparse_attention_host(const bsa_layout *layout, int heads_per_group, const void *q,
                              const void *k, const void *v, const float *top_p, uint32_t flags,
                              float eps, float softmax_scale, void *out, float *entropy,
                              float *entropy_norm, int32_t *kv_count, int32_t *err_flag,
                              void *workspace, size_t workspace_bytes, void *compute_stream,
                              void *h2d_stream, void *d2h_stream);

/* Device workspace bytes bsa_sparse_attention_host needs (0: invalid layout). */
size_t bsa_pipeline_workspace_bytes(const bsa_layout *layout, int heads_per_group);

/*
 * Limit of every internal pipeline wait (mbarrier) of the attention kernel
 * (bsa_attention_fwd, bsa_attention_fwd_weighted, bsa_dense_fwd,
 * bsa_frame_scores, and the attention launches of bsa_sparse_attention_host),
 * in nanoseconds, for the launches made after the call; ns = 0 restores the
 * default of 2 s.  A wait that outlives the limit makes the kernel stop: every
 * copy and product already started is waited for (under the default limit),
 * the tensor memory is released, the outputs of the rows not finished are
 * undefined (lse NaN where the row had started) and BSA_DEVERR_TIMEOUT is ORed
 * into err_flag; the stream and the context stay usable.  The pages have no counterpart: this is a diagnostic
 * setting, process-wide, meant for tests of that stop path (a limit far below
 * the kernel's own latency makes it fire).  Always returns BSA_OK.
 */
int bsa_set_wait_limit_ns(unsigned long long ns);

/* Human-readable name of a bsa_status value (static storage). */
const char *bsa_status_string(int status);

/* ABI version: major * 100 + minor. */
int bsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H */
