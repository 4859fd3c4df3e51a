// internal.h -- launchers shared between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bsa.h"

namespace bsa {

constexpr int kMaxHeads = 256;
constexpr int kMaxScoreCk = 2048;  // bsa_block_scores
constexpr int kMaxMaskCk = 2048;   // bsa_build_mask

struct Geometry {
    int B, H, S, S_pad, D, bq, bk, Cq, Ck;
    int text_kblocks;       // key blocks holding text tokens
    int f0_first, f0_last;  // frame-0 query-block range, f0_last < f0_first when empty
};

Geometry make_geometry(const bsa_layout &L);

// cuTensorMapEncodeTiled, looked up once through the runtime (nullptr if the
// driver lacks it), and the current device's SM count (0 on error).
typedef CUresult (*TensorMapEncoder)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                     const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                     const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
TensorMapEncoder tensor_map_encoder();
int sm_count();

// Host-side validation of a layout shared by every entry point: BSA_OK,
// BSA_ERR_INVALID_ARG or BSA_ERR_UNSUPPORTED.
int check_layout(const bsa_layout *L);

cudaError_t launch_pool(const Geometry &g, const void *q, const void *k, float *qc, float *kc,
                        cudaStream_t st);
// P' rows of the centroid rows qc.  With mix_out: qc holds nsub sub-centroid
// rows per query block (g.Cq = blocks * nsub) and the block's mixed row
// sum_c (n_c / n) P'_c (sizes n_c in mix_size) goes to mix_out; probs then
// only holds intermediate values.
cudaError_t launch_scores(const Geometry &g, const float *qc, const float *kc, float *probs,
                          cudaStream_t st, const int32_t *mix_size = nullptr, int nsub = 1,
                          float *mix_out = nullptr);

struct TopP {
    float p[kMaxHeads];
};

cudaError_t launch_mask(const Geometry &g, const float *probs, const TopP &tp, uint32_t flags,
                        float eps, uint8_t *mask, int32_t *kv_index, int32_t *kv_count,
                        float *row_entropy, cudaStream_t st);
cudaError_t launch_entropy_reduce(const Geometry &g, const float *row_entropy, float *entropy,
                                  float *entropy_norm, cudaStream_t st);

// ---- pooled top-p over a competition domain ("Competition Domains Matter ..."
// s3: per-row, per-head, grouped cross-head, all-head, and the entropy-guided
// EG-Sparse of s3.3 with the s4 value-aware score): the shared state of one
// pool, written by the radix-select kernels of eg.cu and read by the final
// per-row pass of mask.cu.
struct PoolState {
    double target;                // pool_p * (total score of the pool)
    double above;                 // score mass of the pool above the current range
    unsigned long long pad2;
    uint32_t pre;                 // bit-pattern prefix of the current range
    int shift;                    // low bits below the prefix (0 once the cut value is found)
    int keep_all;                 // the pool never reaches target: every pair is kept
    int empty;                    // the pool has no head
    uint32_t ucut;                // the cut score's bit pattern
    int pad0;
    unsigned long long need;      // pairs with score == ucut to keep, in (h, i, j) order
    long long cut_row;            // flat row holding the last kept tie (-1: none)
    int cut_rank;                 // ties kept in that row
    int pad1;
};

// Value-centroid norms ||c^V_{h,j}||_2, fp32 [B,H,C_k].
cudaError_t launch_value_norms(const Geometry &g, const void *v, float *vnorm, cudaStream_t st);

// Pools per batch entry of a BSA_DOMAIN_* value (0 for per-row).
int eg_pools(int H, int domain);

// Workspace layout of the pooled selection (byte offsets; all 256-aligned).
struct EgWorkspace {
    size_t ent_part, heads_h, pool_of, pool_heads, pool_nh, state;
    size_t zero_begin, zero_bytes;  // cleared at the start of every call
    size_t hist1, hist, tiecnt, counters, bytes;
};
EgWorkspace eg_workspace(const Geometry &g, int domain);

// Pooled selection up to the final pass: row entropies, per-head entropy (into
// `entropy` / `entropy_norm` when given, always into the workspace), the
// domain's pools (into `low_heads` as pooled-or-not and `pool_out` as the pool
// id, when given) and every pool's cut.
cudaError_t launch_eg_prepare(const Geometry &g, int domain, const float *probs, const float *vnorm,
                              float pool_p, float eps, float *entropy, float *entropy_norm,
                              uint8_t *low_heads, int8_t *pool_out, uint8_t *workspace, cudaStream_t st);
// The final pass: per-row top-p for the per-row heads, the pool cut and the
// one-key-per-row safeguard for the pooled heads, overrides and lists.
// pool_of [B,H] (-1 = per-row), state [B,G].
cudaError_t launch_mask_eg(const Geometry &g, const float *probs, const float *vnorm,
                           const TopP &tp, uint32_t flags, uint8_t *mask, int32_t *kv_index,
                           int32_t *kv_count, const int8_t *pool_of, int G, const PoolState *state,
                           cudaStream_t st);

// Returns BSA_* status.
// kv_weight (optional, with kv_index): every exp term of list entry e is scaled by kv_weight[e].
int launch_attention(const Geometry &g, const void *q, const void *k, const void *v,
                     const int32_t *kv_index, const float *kv_weight, const int32_t *kv_count,
                     float softmax_scale, void *out, float *lse, int32_t *err_flag,
                     void *workspace, cudaStream_t st);

// Key centroids only (the pool kernel with no query blocks).
cudaError_t launch_pool_keys(const Geometry &g, const void *k, float *kc, cudaStream_t st);

// Intra-block clustering selector: sub-clusters per query block (n_sub in
// {1, 2, 4, 8, 16}) and their size-weighted block scores.
constexpr int kMaxSubclusters = 16;
size_t cluster_workspace_bytes(const Geometry &g, int nsub);
cudaError_t launch_scores_clustered(const Geometry &g, const void *q, const void *k, int nsub,
                                    int iters, float *cent, int32_t *size, float *kc, float *probs,
                                    void *workspace, cudaStream_t st);

// Head profiling for autoregressive generation: frame attention scores over a
// key window of F frames of T tokens (frame 0 sink, 1 .. F-2 neighbors, F-1
// current), computed with the attention kernel and a one-hot V.
struct ProfileWorkspace {
    size_t v, out, kv_index, kv_count, sched, bytes;
};
ProfileWorkspace profile_workspace(const Geometry &g);
int launch_frame_scores(const Geometry &g, int T, int F, const void *q, const void *k,
                        float softmax_scale, int query_stride, float *alpha, uint8_t *workspace,
                        cudaStream_t st);

// Importance sampling of key blocks with inverse-inclusion-probability weights.
cudaError_t launch_sample(const Geometry &g, const float *probs, float budget, uint64_t seed,
                          uint32_t flags, uint8_t *mask, int32_t *kv_index, float *kv_weight,
                          int32_t *kv_count, cudaStream_t st);

constexpr size_t kAttnWorkspaceBytes = 256;

}  // namespace bsa
