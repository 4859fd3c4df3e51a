// scores.cu -- block centroids and the cluster-size-weighted softmax P'.
//
// "Competition Domains Matter: Selective Head Globalization for Training-Free
// Sparse Attention in Video Diffusion Transformers", s3: queries and keys are
// grouped into clusters with sizes n_i / n_j and centroids; P'_ij weights each
// key cluster by its size, P'_ij = n_j exp(q_i.k_j/sqrt(d)) / sum_j' (...), so
// every row sums to one.  Here a cluster is one contiguous block of tokens
// ("AB-Attention ..." TL;DR: importance from block summaries without
// permuting tokens).
//
// pool_kernel   HBM-bound: streams Q and K exactly once with 16-byte loads and
//               writes fp32 centroids.
// score_kernel  fp32 register-tiled centroid GEMM (C_q x C_k x D per head)
//               with the row softmax fused: a CTA owns TM full rows, keeps
//               their logits in shared memory and writes P' once.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace bsa {

namespace {

__device__ __forceinline__ void bf16x8_add(const uint4 &v, float (&acc)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        acc[2 * m] += __uint_as_float(w[m] << 16);
        acc[2 * m + 1] += __uint_as_float(w[m] & 0xFFFF0000u);
    }
}

// One CTA per block: CTAs [0, nq) pool query blocks, the rest key blocks.
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const uint4 *__restrict__ q,
                                                   const uint4 *__restrict__ k,
                                                   float *__restrict__ qc, float *__restrict__ kc,
                                                   int S, int S_pad, int bq, int bk, int Cq, int Ck,
                                                   long long nq) {
    constexpr int CH = D / 8;      // 16-byte chunks per token row
    constexpr int RPI = 256 / CH;  // rows covered per pass of the CTA
    constexpr int PASSES = 128 / RPI;
    __shared__ float red[RPI][D];

    long long item = blockIdx.x;
    const uint4 *src;
    float *dst;
    int blk;
    long long bh;
    int i;
    if (item < nq) {
        bh = item / Cq;
        i = static_cast<int>(item % Cq);
        blk = bq;
        src = q;
        dst = qc + item * D;
    } else {
        item -= nq;
        bh = item / Ck;
        i = static_cast<int>(item % Ck);
        blk = bk;
        src = k;
        dst = kc + item * D;
    }
    const int n = min(blk, S - i * blk);
    const uint4 *base = src + ((bh * S_pad + static_cast<long long>(i) * blk) * D) / 8;
    const int c = threadIdx.x % CH, r0 = threadIdx.x / CH;

    uint4 v[PASSES];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int r = r0 + p * RPI;
        v[p] = (r < n) ? __ldg(base + r * CH + c) : make_uint4(0, 0, 0, 0);
    }
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int p = 0; p < PASSES; ++p) bf16x8_add(v[p], acc);
#pragma unroll
    for (int e = 0; e < 8; ++e) red[r0][c * 8 + e] = acc[e];
    __syncthreads();
    for (int d = threadIdx.x; d < D; d += 256) {
        float s = 0.f;
#pragma unroll
        for (int r = 0; r < RPI; ++r) s += red[r][d];
        dst[d] = s / static_cast<float>(n);
    }
}

// CTA = (head, TM query rows) x all C_k key blocks.  Thread (ty, tx) owns
// rows ty*RPT .. +RPT-1 and columns tx + 32c (c < 4) of each 128-column tile.
template <int TM, int D>
__global__ void __launch_bounds__(256) score_kernel(const float *__restrict__ qc,
                                                    const float *__restrict__ kc,
                                                    float *__restrict__ probs, int S, int bk,
                                                    int Cq, int Ck, float inv_sqrt_d) {
    constexpr int TN = 128;
    constexpr int RPT = TM / 8;
    constexpr int KS = D + 4;  // padded k row stride (floats): conflict-free float4 reads
    extern __shared__ __align__(16) float smem[];
    float *ks = smem;              // [TN][KS]
    float *qs = ks + TN * KS;      // [TM][D]
    float *logit = qs + TM * D;    // [TM][Ck]

    const int tid = threadIdx.x, ty = tid / 32, tx = tid % 32;
    const int tiles_per_head = (Cq + TM - 1) / TM;
    const long long bh = blockIdx.x / tiles_per_head;
    const int i0 = (blockIdx.x % tiles_per_head) * TM;
    const int rows = min(TM, Cq - i0);

    const float4 *qsrc = reinterpret_cast<const float4 *>(qc + (bh * Cq + i0) * D);
    for (int e = tid; e < TM * D / 4; e += 256) {
        const int r = e / (D / 4);
        reinterpret_cast<float4 *>(qs)[e] = (r < rows) ? __ldg(qsrc + e) : make_float4(0, 0, 0, 0);
    }
    const float4 *kbase = reinterpret_cast<const float4 *>(kc + bh * Ck * D);

    for (int j0 = 0; j0 < Ck; j0 += TN) {
        __syncthreads();  // previous tile fully consumed (and qs visible on the first pass)
        const int ncols = min(TN, Ck - j0);
        for (int e = tid; e < TN * D / 4; e += 256) {
            const int col = e / (D / 4), d4 = e % (D / 4);
            const float4 val = (col < ncols) ? __ldg(kbase + (j0 + col) * (D / 4) + d4)
                                             : make_float4(0, 0, 0, 0);
            *reinterpret_cast<float4 *>(ks + col * KS + d4 * 4) = val;
        }
        __syncthreads();
        float acc[RPT][4];
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#pragma unroll 4
        for (int d = 0; d < D; d += 4) {
            float4 a[RPT], b[4];
#pragma unroll
            for (int r = 0; r < RPT; ++r)
                a[r] = *reinterpret_cast<const float4 *>(qs + (ty * RPT + r) * D + d);
#pragma unroll
            for (int c = 0; c < 4; ++c)
                b[c] = *reinterpret_cast<const float4 *>(ks + (tx + 32 * c) * KS + d);
#pragma unroll
            for (int r = 0; r < RPT; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    acc[r][c] = fmaf(a[r].x, b[c].x, acc[r][c]);
                    acc[r][c] = fmaf(a[r].y, b[c].y, acc[r][c]);
                    acc[r][c] = fmaf(a[r].z, b[c].z, acc[r][c]);
                    acc[r][c] = fmaf(a[r].w, b[c].w, acc[r][c]);
                }
        }
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int col = tx + 32 * c;
                if (col < ncols) logit[(ty * RPT + r) * Ck + j0 + col] = acc[r][c] * inv_sqrt_d;
            }
    }
    __syncthreads();

    // Row softmax weighted by the key-block sizes n_j: P'_j = n_j e^{s_j - m} / Z.
    const int warp = tid / 32, lane = tid % 32;
    for (int r = warp; r < rows; r += 8) {
        float *lr = logit + r * Ck;
        float m = -INFINITY;
        for (int j = lane; j < Ck; j += 32) m = fmaxf(m, lr[j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float z = 0.f;
        for (int j = lane; j < Ck; j += 32) {
            const int nj = min(bk, S - j * bk);
            const float w = static_cast<float>(nj) * expf(lr[j] - m);
            lr[j] = w;
            z += w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        float *dst = probs + (bh * Cq + i0 + r) * static_cast<long long>(Ck);
        for (int j = lane; j < Ck; j += 32) dst[j] = lr[j] / z;
    }
}

template <int TM, int D>
size_t score_smem_bytes(int Ck) {
    return sizeof(float) * (static_cast<size_t>(128) * (D + 4) + TM * D + static_cast<size_t>(TM) * Ck);
}

template <int TM, int D>
cudaError_t launch_scores_t(const Geometry &g, const float *qc, const float *kc, float *probs,
                            cudaStream_t st) {
    const size_t smem = score_smem_bytes<TM, D>(g.Ck);
    cudaError_t e = cudaFuncSetAttribute(score_kernel<TM, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const long long grid = static_cast<long long>(g.B) * g.H * ((g.Cq + TM - 1) / TM);
    score_kernel<TM, D><<<static_cast<unsigned>(grid), 256, smem, st>>>(
        qc, kc, probs, g.S, g.bk, g.Cq, g.Ck, 1.0f / sqrtf(static_cast<float>(g.D)));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(const Geometry &g, const void *q, const void *k, float *qc, float *kc,
                        cudaStream_t st) {
    const long long nq = static_cast<long long>(g.B) * g.H * g.Cq;
    const long long nk = static_cast<long long>(g.B) * g.H * g.Ck;
    const auto *q4 = static_cast<const uint4 *>(q);
    const auto *k4 = static_cast<const uint4 *>(k);
    if (g.D == 128)
        pool_kernel<128><<<static_cast<unsigned>(nq + nk), 256, 0, st>>>(
            q4, k4, qc, kc, g.S, g.S_pad, g.bq, g.bk, g.Cq, g.Ck, nq);
    else
        pool_kernel<64><<<static_cast<unsigned>(nq + nk), 256, 0, st>>>(
            q4, k4, qc, kc, g.S, g.S_pad, g.bq, g.bk, g.Cq, g.Ck, nq);
    return cudaGetLastError();
}

cudaError_t launch_scores(const Geometry &g, const float *qc, const float *kc, float *probs,
                          cudaStream_t st) {
    if (g.Ck <= 1024) {
        return g.D == 128 ? launch_scores_t<32, 128>(g, qc, kc, probs, st)
                          : launch_scores_t<32, 64>(g, qc, kc, probs, st);
    }
    return g.D == 128 ? launch_scores_t<16, 128>(g, qc, kc, probs, st)
                      : launch_scores_t<16, 64>(g, qc, kc, probs, st);
}

}  // namespace bsa
