// api.cu -- the C ABI: host-side validation, geometry, dispatch to the kernels.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "bsa.h"
#include "internal.h"

namespace bsa {

Geometry make_geometry(const bsa_layout &L) {
    Geometry g;
    g.B = L.batch;
    g.H = L.heads;
    g.S = L.seq_len;
    g.S_pad = L.seq_pad;
    g.D = L.head_dim;
    g.bq = L.q_block;
    g.bk = L.k_block;
    g.Cq = L.seq_pad / L.q_block;
    g.Ck = L.seq_pad / L.k_block;
    // "Attention matrix view ..." s7: key blocks that hold a text token.
    g.text_kblocks = (L.text_len + L.k_block - 1) / L.k_block;
    if (g.text_kblocks > g.Ck) g.text_kblocks = g.Ck;
    // "Attention matrix view ..." s4: query blocks that overlap frame 0.
    if (L.tokens_per_frame > 0 && L.num_frames > 0) {
        g.f0_first = L.text_len / L.q_block;
        g.f0_last = (L.text_len + L.tokens_per_frame - 1) / L.q_block;
        if (g.f0_last > g.Cq - 1) g.f0_last = g.Cq - 1;
    } else {
        g.f0_first = 0;
        g.f0_last = -1;
    }
    return g;
}

TensorMapEncoder tensor_map_encoder() {
    static TensorMapEncoder fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<TensorMapEncoder>(ptr);
    });
    return fn;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

int check_layout(const bsa_layout *L) {
    if (!L) return BSA_ERR_INVALID_ARG;
    if (L->batch < 1 || L->heads < 1 || L->seq_len < 1 || L->seq_pad < L->seq_len)
        return BSA_ERR_INVALID_ARG;
    if (L->heads > bsa::kMaxHeads) return BSA_ERR_UNSUPPORTED;
    if (L->head_dim != 64 && L->head_dim != 128) return BSA_ERR_UNSUPPORTED;
    if ((L->q_block != 64 && L->q_block != 128) || (L->k_block != 64 && L->k_block != 128))
        return BSA_ERR_UNSUPPORTED;
    const int big = L->q_block > L->k_block ? L->q_block : L->k_block;
    const int small = L->q_block < L->k_block ? L->q_block : L->k_block;
    if (L->seq_pad % big != 0) return BSA_ERR_INVALID_ARG;
    if (L->seq_pad - L->seq_len >= small) return BSA_ERR_INVALID_ARG;  // a block with no token
    if (L->text_len < 0 || L->tokens_per_frame < 0 || L->num_frames < 0) return BSA_ERR_INVALID_ARG;
    const long long covered =
        static_cast<long long>(L->text_len) + static_cast<long long>(L->num_frames) * L->tokens_per_frame;
    if (covered > L->seq_len) return BSA_ERR_INVALID_ARG;
    const long long elems = static_cast<long long>(L->batch) * L->heads * L->seq_pad;
    if (elems > (1ll << 40)) return BSA_ERR_UNSUPPORTED;
    if (static_cast<long long>(L->batch) * L->heads * (L->seq_pad / L->q_block) > 0x7FFFFFFFll)
        return BSA_ERR_UNSUPPORTED;
    return BSA_OK;
}

}  // namespace bsa

namespace {

using bsa::check_layout;
using bsa::Geometry;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int launch_status(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ERR_LAUNCH; }

}  // namespace

extern "C" {

int bsa_version(void) { return 100; }

const char *bsa_status_string(int status) {
    switch (status) {
        case BSA_OK: return "BSA_OK";
        case BSA_ERR_INVALID_ARG: return "BSA_ERR_INVALID_ARG";
        case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED";
        case BSA_ERR_LAUNCH: return "BSA_ERR_LAUNCH";
        case BSA_ERR_DRIVER: return "BSA_ERR_DRIVER";
        default: return "BSA_ERR_UNKNOWN";
    }
}

int bsa_block_scores(const bsa_layout *layout, const void *q, const void *k, float *q_centroids,
                     float *k_centroids, float *probs, void *stream) {
    int rc = check_layout(layout);
    if (rc != BSA_OK) return rc;
    if (!q || !k || !q_centroids || !k_centroids || !probs) return BSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(q_centroids, 16) || !aligned(k_centroids, 16) ||
        !aligned(probs, 16))
        return BSA_ERR_INVALID_ARG;
    const Geometry g = bsa::make_geometry(*layout);
    if (g.Ck > bsa::kMaxScoreCk) return BSA_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = launch_status(bsa::launch_pool(g, q, k, q_centroids, k_centroids, st));
    if (rc != BSA_OK) return rc;
    return launch_status(bsa::launch_scores(g, q_centroids, k_centroids, probs, st));
}

size_t bsa_block_scores_clustered_workspace_bytes(const bsa_layout *layout, int n_sub) {
    if (check_layout(layout) != BSA_OK) return 0;
    if (n_sub < 1 || n_sub > bsa::kMaxSubclusters || (n_sub & (n_sub - 1))) return 0;
    return ((bsa::cluster_workspace_bytes(bsa::make_geometry(*layout), n_sub) + 255) / 256) * 256;
}

int bsa_block_scores_clustered(const bsa_layout *layout, const void *q, const void *k, int n_sub,
                               int iters, float *sub_centroids, int32_t *sub_sizes,
                               float *k_centroids, float *probs, void *workspace, void *stream) {
    int rc = check_layout(layout);
    if (rc != BSA_OK) return rc;
    if (!q || !k || !sub_centroids || !sub_sizes || !k_centroids || !probs || !workspace)
        return BSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(sub_centroids, 16) ||
        !aligned(k_centroids, 16) || !aligned(probs, 16) || !aligned(sub_sizes, 4) ||
        !aligned(workspace, 256))
        return BSA_ERR_INVALID_ARG;
    if (iters < 1 || iters > 1000) return BSA_ERR_INVALID_ARG;
    if (n_sub < 1 || n_sub > bsa::kMaxSubclusters || (n_sub & (n_sub - 1))) return BSA_ERR_UNSUPPORTED;
    const Geometry g = bsa::make_geometry(*layout);
    if (g.Ck > bsa::kMaxScoreCk) return BSA_ERR_UNSUPPORTED;
    if (static_cast<long long>(g.B) * g.H * g.Cq * n_sub > 0x7FFFFFFFll) return BSA_ERR_UNSUPPORTED;
    return launch_status(bsa::launch_scores_clustered(g, q, k, n_sub, iters, sub_centroids, sub_sizes,
                                                      k_centroids, probs, workspace,
                                                      static_cast<cudaStream_t>(stream)));
}

size_t bsa_build_mask_workspace_bytes(const bsa_layout *layout) {
    if (check_layout(layout) != BSA_OK) return 0;
    const size_t rows = static_cast<size_t>(layout->batch) * layout->heads *
                        (layout->seq_pad / layout->q_block);
    return ((rows * sizeof(float) + 255) / 256) * 256;
}

int bsa_build_mask(const bsa_layout *layout, const float *probs, const float *top_p, uint32_t flags,
                   float eps, uint8_t *mask, int32_t *kv_index, int32_t *kv_count, float *entropy,
                   float *entropy_norm, void *workspace, void *stream) {
    int rc = check_layout(layout);
    if (rc != BSA_OK) return rc;
    if (!probs || !top_p || !kv_index || !kv_count) return BSA_ERR_INVALID_ARG;
    if (flags & ~static_cast<uint32_t>(BSA_TEXT_KEEP | BSA_FRAME0_DENSE)) return BSA_ERR_INVALID_ARG;
    if (!aligned(probs, 4) || !aligned(kv_index, 4) || !aligned(kv_count, 4)) return BSA_ERR_INVALID_ARG;
    const bool want_entropy = entropy || entropy_norm;
    if (want_entropy && (!workspace || !aligned(workspace, 16))) return BSA_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !isfinite(eps)) return BSA_ERR_INVALID_ARG;
    const Geometry g = bsa::make_geometry(*layout);
    if (g.Ck > bsa::kMaxMaskCk) return BSA_ERR_UNSUPPORTED;
    bsa::TopP tp;
    memset(&tp, 0, sizeof tp);
    for (int h = 0; h < g.H; ++h) {
        if (isnan(top_p[h])) return BSA_ERR_INVALID_ARG;
        tp.p[h] = top_p[h];
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *row_ent = want_entropy ? static_cast<float *>(workspace) : nullptr;
    rc = launch_status(bsa::launch_mask(g, probs, tp, flags, eps, mask, kv_index, kv_count, row_ent, st));
    if (rc != BSA_OK || !want_entropy) return rc;
    return launch_status(bsa::launch_entropy_reduce(g, row_ent, entropy, entropy_norm, st));
}

int bsa_value_norms(const bsa_layout *layout, const void *v, float *vnorm, void *stream) {
    int rc = check_layout(layout);
    if (rc != BSA_OK) return rc;
    if (!v || !vnorm || !aligned(v, 16) || !aligned(vnorm, 4)) return BSA_ERR_INVALID_ARG;
    const Geometry g = bsa::make_geometry(*layout);
    return launch_status(bsa::launch_value_norms(g, v, vnorm, static_cast<cudaStream_t>(stream)));
}

// The pooled selections: bsa_build_mask_eg and bsa_build_mask_domain.
static int build_mask_pooled(const bsa_layout *layout, int domain, const float *probs,
                             const float *vnorm, const float *top_p, float pool_p, uint32_t flags,
                             float eps, uint8_t *mask, int32_t *kv_index, int32_t *kv_count,
                             float *entropy, float *entropy_norm, uint8_t *low_heads, int8_t *pool_of,
                             void *workspace, void *stream) {
    int rc = check_layout(layout);
    if (rc != BSA_OK) return rc;
    if (!probs || !top_p || !kv_index || !kv_count || !workspace) return BSA_ERR_INVALID_ARG;
    if (flags & ~static_cast<uint32_t>(BSA_TEXT_KEEP | BSA_FRAME0_DENSE)) return BSA_ERR_INVALID_ARG;
    if (!aligned(probs, 4) || !aligned(kv_index, 4) || !aligned(kv_count, 4) ||
        (vnorm && !aligned(vnorm, 4)) || !aligned(workspace, 256))
        return BSA_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !isfinite(eps) || isnan(pool_p)) return BSA_ERR_INVALID_ARG;
    const Geometry g = bsa::make_geometry(*layout);
    if (g.Ck > bsa::kMaxMaskCk) return BSA_ERR_UNSUPPORTED;
    bsa::TopP tp;
    memset(&tp, 0, sizeof tp);
    for (int h = 0; h < g.H; ++h) {
        if (isnan(top_p[h])) return BSA_ERR_INVALID_ARG;
        tp.p[h] = top_p[h];
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    rc = launch_status(bsa::launch_eg_prepare(g, domain, probs, vnorm, pool_p, eps, entropy, entropy_norm,
                                              low_heads, pool_of, ws, st));
    if (rc != BSA_OK) return rc;
    const bsa::EgWorkspace w = bsa::eg_workspace(g, domain);
    return launch_status(bsa::launch_mask_eg(
        g, probs, vnorm, tp, flags, mask, kv_index, kv_count, reinterpret_cast<const int8_t *>(ws + w.pool_of),
        bsa::eg_pools(g.H, domain), reinterpret_cast<const bsa::PoolState *>(ws + w.state), st));
}

static bool valid_domain(int domain) { return domain >= BSA_DOMAIN_ROW && domain <= BSA_DOMAIN_EG; }

size_t bsa_build_mask_eg_workspace_bytes(const bsa_layout *layout) {
    return bsa_build_mask_domain_workspace_bytes(layout, BSA_DOMAIN_EG);
}

size_t bsa_build_mask_domain_workspace_bytes(const bsa_layout *layout, int domain) {
    if (check_layout(layout) != BSA_OK || !valid_domain(domain)) return 0;
    return bsa::eg_workspace(bsa::make_geometry(*layout), domain).bytes;
}

int bsa_build_mask_eg(const bsa_layout *layout, const float *probs, const float *vnorm,
                      const float *top_p, float pool_p, uint32_t flags, float eps, uint8_t *mask,
                      int32_t *kv_index, int32_t *kv_count, float *entropy, float *entropy_norm,
                      uint8_t *low_heads, void *workspace, void *stream) {
    return build_mask_pooled(layout, BSA_DOMAIN_EG, probs, vnorm, top_p, pool_p, flags, eps, mask, kv_index,
                             kv_count, entropy, entropy_norm, low_heads, nullptr, workspace, stream);
}

int bsa_build_mask_domain(const bsa_layout *layout, int domain, const float *probs,
                          const float *vnorm, const float *top_p, float pool_p, uint32_t flags,
                          float eps, uint8_t *mask, int32_t *kv_index, int32_t *kv_count,
                          float *entropy, float *entropy_norm, int8_t *pool_of, void *workspace,
                          void *stream) {
    if (!valid_domain(domain)) return BSA_ERR_INVALID_ARG;
    return build_mask_pooled(layout, domain, probs, vnorm, top_p, pool_p, flags, eps, mask, kv_index,
                             kv_count, entropy, entropy_norm, nullptr, pool_of, workspace, stream);
}

size_t bsa_attention_workspace_bytes(const bsa_layout *layout) {
    if (check_layout(layout) != BSA_OK) return 0;
    return bsa::kAttnWorkspaceBytes;
}

int bsa_attention_fwd(const bsa_layout *layout, const void *q, const void *k, const void *v,
                      const int32_t *kv_index, const int32_t *kv_count, float softmax_scale,
                      void *out, float *lse, int32_t *err_flag, void *workspace, void *stream) {
    int rc = check_layout(layout);
    if (rc != BSA_OK) return rc;
    if (!q || !k || !v || !out || !kv_index || !kv_count) return BSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
        return BSA_ERR_INVALID_ARG;
    if (!aligned(kv_index, 4) || !aligned(kv_count, 4) || (lse && !aligned(lse, 4)) ||
        (err_flag && !aligned(err_flag, 4)))
        return BSA_ERR_INVALID_ARG;
    if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return BSA_ERR_INVALID_ARG;
    if (workspace && !aligned(workspace, 16)) return BSA_ERR_INVALID_ARG;
    const Geometry g = bsa::make_geometry(*layout);
    return bsa::launch_attention(g, q, k, v, kv_index, nullptr, kv_count, softmax_scale, out, lse, err_flag,
                                 workspace, static_cast<cudaStream_t>(stream));
}

int bsa_attention_fwd_weighted(const bsa_layout *layout, const void *q, const void *k,
                               const void *v, const int32_t *kv_index, const float *kv_weight,
                               const int32_t *kv_count, float softmax_scale, void *out, float *lse,
                               int32_t *err_flag, void *workspace, void *stream) {
    int rc = check_layout(layout);
    if (rc != BSA_OK) return rc;
    if (!q || !k || !v || !out || !kv_index || !kv_weight || !kv_count) return BSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
        return BSA_ERR_INVALID_ARG;
    if (!aligned(kv_index, 4) || !aligned(kv_weight, 4) || !aligned(kv_count, 4) ||
        (lse && !aligned(lse, 4)) || (err_flag && !aligned(err_flag, 4)))
        return BSA_ERR_INVALID_ARG;
    if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return BSA_ERR_INVALID_ARG;
    if (workspace && !aligned(workspace, 16)) return BSA_ERR_INVALID_ARG;
    const Geometry g = bsa::make_geometry(*layout);
    return bsa::launch_attention(g, q, k, v, kv_index, kv_weight, kv_count, softmax_scale, out, lse,
                                 err_flag, workspace, static_cast<cudaStream_t>(stream));
}

int bsa_build_mask_sampled(const bsa_layout *layout, const float *probs, float budget,
                           uint64_t seed, uint32_t flags, uint8_t *mask, int32_t *kv_index,
                           float *kv_weight, int32_t *kv_count, void *stream) {
    int rc = check_layout(layout);
    if (rc != BSA_OK) return rc;
    if (!probs || !kv_index || !kv_weight || !kv_count) return BSA_ERR_INVALID_ARG;
    if (flags & ~static_cast<uint32_t>(BSA_TEXT_KEEP | BSA_FRAME0_DENSE)) return BSA_ERR_INVALID_ARG;
    if (!aligned(probs, 4) || !aligned(kv_index, 4) || !aligned(kv_weight, 4) || !aligned(kv_count, 4))
        return BSA_ERR_INVALID_ARG;
    if (!(budget >= 0.f) || !isfinite(budget)) return BSA_ERR_INVALID_ARG;
    const Geometry g = bsa::make_geometry(*layout);
    if (g.Ck > bsa::kMaxMaskCk) return BSA_ERR_UNSUPPORTED;
    return launch_status(bsa::launch_sample(g, probs, budget, seed, flags, mask, kv_index, kv_weight,
                                            kv_count, static_cast<cudaStream_t>(stream)));
}

size_t bsa_frame_scores_workspace_bytes(const bsa_layout *layout) {
    if (check_layout(layout) != BSA_OK) return 0;
    return bsa::profile_workspace(bsa::make_geometry(*layout)).bytes;
}

int bsa_frame_scores(const bsa_layout *layout, const void *q, const void *k, float softmax_scale,
                     int query_stride, float *alpha, void *workspace, void *stream) {
    int rc = check_layout(layout);
    if (rc != BSA_OK) return rc;
    if (!q || !k || !alpha || !workspace) return BSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(alpha, 4) || !aligned(workspace, 256))
        return BSA_ERR_INVALID_ARG;
    if (!(softmax_scale > 0.f) || !isfinite(softmax_scale) || query_stride < 1)
        return BSA_ERR_INVALID_ARG;
    const int T = layout->tokens_per_frame, F = layout->num_frames;
    if (layout->text_len != 0 || F < 2 || T < 1 ||
        static_cast<long long>(F) * T != static_cast<long long>(layout->seq_len))
        return BSA_ERR_INVALID_ARG;
    const Geometry g = bsa::make_geometry(*layout);
    return bsa::launch_frame_scores(g, T, F, q, k, softmax_scale, query_stride, alpha,
                                    static_cast<uint8_t *>(workspace),
                                    static_cast<cudaStream_t>(stream));
}

int bsa_dhp_labels(const float *alpha, int heads, int n_dummy, int32_t *labels) {
    if (!alpha || !labels || heads < 1 || n_dummy < 0 || n_dummy > heads) return BSA_ERR_INVALID_ARG;
    // l_h = max(alpha_sink, alpha_neighbor); the n_dummy smallest (lower h on ties) are dummy
    for (int h = 0; h < heads; ++h) {
        const float s = alpha[3 * h], nb = alpha[3 * h + 1];
        if (s != s || nb != nb) return BSA_ERR_INVALID_ARG;
        labels[h] = s > nb ? BSA_HEAD_SINK : BSA_HEAD_NEIGHBOR;
    }
    for (int r = 0; r < n_dummy; ++r) {
        int best = -1;
        float bl = 0.f;
        for (int h = 0; h < heads; ++h) {
            if (labels[h] == BSA_HEAD_DUMMY) continue;
            const float l = alpha[3 * h] > alpha[3 * h + 1] ? alpha[3 * h] : alpha[3 * h + 1];
            if (best < 0 || l < bl) {
                best = h;
                bl = l;
            }
        }
        labels[best] = BSA_HEAD_DUMMY;
    }
    return BSA_OK;
}

int bsa_dense_fwd(const bsa_layout *layout, const void *q, const void *k, const void *v,
                  float softmax_scale, void *out, float *lse, int32_t *err_flag, void *workspace,
                  void *stream) {
    int rc = check_layout(layout);
    if (rc != BSA_OK) return rc;
    if (!q || !k || !v || !out) return BSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
        return BSA_ERR_INVALID_ARG;
    if ((lse && !aligned(lse, 4)) || (err_flag && !aligned(err_flag, 4))) return BSA_ERR_INVALID_ARG;
    if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return BSA_ERR_INVALID_ARG;
    if (workspace && !aligned(workspace, 16)) return BSA_ERR_INVALID_ARG;
    const Geometry g = bsa::make_geometry(*layout);
    return bsa::launch_attention(g, q, k, v, nullptr, nullptr, nullptr, softmax_scale, out, lse, err_flag,
                                 workspace, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
