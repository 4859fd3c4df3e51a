// cluster.cu -- the intra-block clustering selector's block scores.
//
// "AB-Attention: accurate block-sparse attention for video diffusion", TL;DR
// fix (1): the queries of each query block are clustered among themselves
// (tokens stay in place), so the block's importance comes from several
// sub-centroids instead of one coarse mean.  The page gives no procedure;
// this file takes the plain one:
//   - k-means (Lloyd) on the block's valid query tokens, n_sub clusters,
//     seeds = the tokens at positions floor(c * n / n_sub), squared Euclidean
//     distance with ties to the lower cluster, `iters` rounds of (assign,
//     move each non-empty cluster to its mean); an empty cluster keeps its
//     centroid and has size 0;
//   - the block's score row is the size-weighted mixture of the
//     sub-centroids' cluster-size-weighted softmax rows:
//       P'_ij = sum_c (n_c / n_i) softmax_j(q_c . k_j / sqrt(D) + ln n_j).
//
// Launches: pool_kernel (key centroids only), subcluster_kernel (one CTA per
// query block, the block's tokens in shared memory), score_kernel of
// scores.cu on the C_q * n_sub sub-centroid rows (split-tf32 tcgen05 GEMM with
// the fused row softmax) into a workspace, mix_kernel (one warp per block row:
// the size-weighted sum of its n_sub rows).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace bsa {

namespace {

constexpr int kClusterThreads = 128;

// k-means of one query block.  Thread t holds token t in registers and picks
// its cluster by the smallest ||c_k||^2 - 2 x.c_k (the distance without the
// token's own ||x||^2; one independent FMA chain per centroid, centroids read
// as broadcast float4).  Ballots then group the tokens by cluster into a
// permutation (ascending token order inside a cluster), and thread d sums
// dimension d over each cluster's segment from a dimension-major copy of the
// tokens (row stride odd, so a column read is conflict-free).
template <int D, int NSUB>
__global__ void __launch_bounds__(kClusterThreads) subcluster_kernel(
    const uint16_t *__restrict__ q, float *__restrict__ cent, int32_t *__restrict__ size, int S,
    int S_pad, int bq, int Cq, int iters) {
    constexpr int LDT = kClusterThreads + 1;
    constexpr int kWarps = kClusterThreads / 32;
    __shared__ __align__(16) float c[NSUB * D];
    __shared__ float cn[NSUB];                 // ||c_k||^2
    __shared__ int perm[kClusterThreads];      // tokens grouped by cluster
    __shared__ int seg[NSUB + 1];              // cluster k = perm[seg[k] .. seg[k+1])
    __shared__ int wcnt[kWarps][NSUB];
    extern __shared__ float xt[];              // [D][LDT]: xt[d][t]

    const long long blk = blockIdx.x;
    const long long bh = blk / Cq;
    const int i = static_cast<int>(blk % Cq);
    const int n = max(0, min(bq, S - i * bq));
    const int tid = threadIdx.x, lane = tid % 32, wid = tid / 32;
    float xr[D];
    {
        const uint4 *src = reinterpret_cast<const uint4 *>(
            q + (bh * S_pad + static_cast<long long>(i) * bq + min(tid, max(n - 1, 0))) * D);
#pragma unroll
        for (int v8 = 0; v8 < D / 8; ++v8) {
            const uint4 v = tid < n ? __ldg(src + v8) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                xr[v8 * 8 + 2 * m] = __uint_as_float(w[m] << 16);
                xr[v8 * 8 + 2 * m + 1] = __uint_as_float(w[m] & 0xFFFF0000u);
            }
        }
#pragma unroll
        for (int d = 0; d < D; ++d) xt[d * LDT + tid] = xr[d];
    }
    __syncthreads();
    // seeds: the tokens at floor(c * n / NSUB); their squared norms
    for (int e = tid; e < NSUB * D; e += kClusterThreads) {
        const int k = e / D, d = e % D;
        const int t0 = n > 0 ? static_cast<int>((static_cast<long long>(k) * n) / NSUB) : 0;
        c[e] = n > 0 ? xt[d * LDT + t0] : 0.f;
    }
    __syncthreads();
    if (tid < NSUB) {
        float s2 = 0.f;
        for (int d = 0; d < D; ++d) s2 = fmaf(c[tid * D + d], c[tid * D + d], s2);
        cn[tid] = s2;
    }
    __syncthreads();
    int best = 0;
    for (int it = 0; it < iters; ++it) {
        best = 0;
        if (NSUB > 1 && tid < n) {  // nearest centroid, ties to the lower index
            float dot[NSUB];
#pragma unroll
            for (int k = 0; k < NSUB; ++k) dot[k] = 0.f;
#pragma unroll
            for (int d4 = 0; d4 < D / 4; ++d4) {
#pragma unroll
                for (int k = 0; k < NSUB; ++k) {
                    const float4 cv = reinterpret_cast<const float4 *>(c + k * D)[d4];
                    dot[k] = fmaf(xr[4 * d4], cv.x, dot[k]);
                    dot[k] = fmaf(xr[4 * d4 + 1], cv.y, dot[k]);
                    dot[k] = fmaf(xr[4 * d4 + 2], cv.z, dot[k]);
                    dot[k] = fmaf(xr[4 * d4 + 3], cv.w, dot[k]);
                }
            }
            float bd = INFINITY;
#pragma unroll
            for (int k = 0; k < NSUB; ++k) {
                const float dist = fmaf(-2.f, dot[k], cn[k]);
                if (dist < bd) {
                    bd = dist;
                    best = k;
                }
            }
        }
        // group by cluster: per-warp counts, then each token's slot
        const bool live = tid < n;
        int rank_in_warp = 0;
#pragma unroll
        for (int k = 0; k < NSUB; ++k) {
            const unsigned bal = __ballot_sync(0xffffffffu, live && best == k);
            if (best == k) rank_in_warp = __popc(bal & ((1u << lane) - 1u));
            if (lane == 0) wcnt[wid][k] = __popc(bal);
        }
        __syncthreads();
        if (tid == 0) {
            int off = 0;
            for (int k = 0; k < NSUB; ++k) {
                seg[k] = off;
                for (int w = 0; w < kWarps; ++w) {
                    const int m = wcnt[w][k];
                    wcnt[w][k] = off;  // now the warp's first slot in cluster k
                    off += m;
                }
            }
            seg[NSUB] = off;
        }
        __syncthreads();
        if (live) perm[wcnt[wid][best] + rank_in_warp] = tid;
        __syncthreads();
        // move the centroids: thread d sums dimension d over each cluster
        if (tid < D) {
#pragma unroll
            for (int k = 0; k < NSUB; ++k) {
                const int a = seg[k], b = seg[k + 1];
                if (b > a) {
                    float s = 0.f;
                    for (int idx = a; idx < b; ++idx) s += xt[tid * LDT + perm[idx]];
                    c[k * D + tid] = s / static_cast<float>(b - a);
                }
            }
        }
        __syncthreads();
        if (tid < NSUB) {
            float s2 = 0.f;
            for (int d = 0; d < D; ++d) s2 = fmaf(c[tid * D + d], c[tid * D + d], s2);
            cn[tid] = s2;
        }
        __syncthreads();
    }
    for (int e = tid; e < NSUB * D; e += kClusterThreads) cent[blk * NSUB * D + e] = c[e];
    if (tid < NSUB) size[blk * NSUB + tid] = iters > 0 ? seg[tid + 1] - seg[tid] : 0;
}

// P'[r, :] = sum_c (n_c / n) P_sub[r * NSUB + c, :], one warp per row, in
// ascending c; the weights are fixed per row, the column loop keeps several
// rows' loads in flight.
template <int NSUB>
__global__ void __launch_bounds__(256) mix_kernel(const float *__restrict__ psub,
                                                  const int32_t *__restrict__ size,
                                                  float *__restrict__ probs, long long rows, int Ck) {
    const int lane = threadIdx.x % 32;
    const long long r = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
    if (r >= rows) return;
    float wk[NSUB];
    int ntot = 0;
#pragma unroll
    for (int k = 0; k < NSUB; ++k) ntot += __ldg(size + r * NSUB + k);
    const float inv = ntot > 0 ? 1.f / static_cast<float>(ntot) : 0.f;
#pragma unroll
    for (int k = 0; k < NSUB; ++k) wk[k] = static_cast<float>(__ldg(size + r * NSUB + k)) * inv;
    const float *src = psub + r * NSUB * Ck;
#pragma unroll 4
    for (int j = lane; j < Ck; j += 32) {
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < NSUB; ++k)
            if (wk[k] > 0.f) acc = fmaf(wk[k], __ldg(src + k * Ck + j), acc);
        probs[r * Ck + j] = acc;
    }
}

template <int D, int NSUB>
cudaError_t launch_sub_t(const uint16_t *q, float *cent, int32_t *size, const Geometry &g,
                         long long blocks, int iters, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(D) * (kClusterThreads + 1) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(subcluster_kernel<D, NSUB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    subcluster_kernel<D, NSUB><<<static_cast<unsigned>(blocks), kClusterThreads, smem, st>>>(
        q, cent, size, g.S, g.S_pad, g.bq, g.Cq, iters);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_subclusters(const uint16_t *q, float *cent, int32_t *size, const Geometry &g,
                               long long blocks, int nsub, int iters, cudaStream_t st) {
    switch (nsub) {
        case 1: return launch_sub_t<D, 1>(q, cent, size, g, blocks, iters, st);
        case 2: return launch_sub_t<D, 2>(q, cent, size, g, blocks, iters, st);
        case 4: return launch_sub_t<D, 4>(q, cent, size, g, blocks, iters, st);
        case 8: return launch_sub_t<D, 8>(q, cent, size, g, blocks, iters, st);
        case 16: return launch_sub_t<D, 16>(q, cent, size, g, blocks, iters, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

size_t cluster_workspace_bytes(const Geometry &g, int nsub) {
    return static_cast<size_t>(g.B) * g.H * g.Cq * nsub * g.Ck * sizeof(float);
}

cudaError_t launch_scores_clustered(const Geometry &g, const void *q, const void *k, int nsub,
                                    int iters, float *cent, int32_t *size, float *kc, float *probs,
                                    void *workspace, cudaStream_t st) {
    cudaError_t e = launch_pool_keys(g, k, kc, st);
    if (e != cudaSuccess) return e;
    const long long blocks = static_cast<long long>(g.B) * g.H * g.Cq;
    const uint16_t *q16 = static_cast<const uint16_t *>(q);
    if (g.D == 128)
        e = launch_subclusters<128>(q16, cent, size, g, blocks, nsub, iters, st);
    else
        e = launch_subclusters<64>(q16, cent, size, g, blocks, nsub, iters, st);
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // the sub-centroid rows as C_q * nsub query rows of the score kernel
    Geometry gs = g;
    gs.Cq = g.Cq * nsub;
    float *psub = static_cast<float *>(workspace);
    if ((e = launch_scores(gs, cent, kc, psub, st)) != cudaSuccess) return e;
    const unsigned grid = static_cast<unsigned>((blocks + 7) / 8);
    switch (nsub) {
        case 1: mix_kernel<1><<<grid, 256, 0, st>>>(psub, size, probs, blocks, g.Ck); break;
        case 2: mix_kernel<2><<<grid, 256, 0, st>>>(psub, size, probs, blocks, g.Ck); break;
        case 4: mix_kernel<4><<<grid, 256, 0, st>>>(psub, size, probs, blocks, g.Ck); break;
        case 8: mix_kernel<8><<<grid, 256, 0, st>>>(psub, size, probs, blocks, g.Ck); break;
        default: mix_kernel<16><<<grid, 256, 0, st>>>(psub, size, probs, blocks, g.Ck); break;
    }
    return cudaGetLastError();
}

}  // namespace bsa
