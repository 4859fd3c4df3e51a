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
// Launches: pool_kernel (key centroids only); subcluster_kernel (one CTA per
// query block, the block's tokens in shared memory, each k-means round two
// tcgen05 products); score_kernel of scores.cu on the C_q * n_sub sub-centroid
// rows (split-tf32 tcgen05 GEMM with the fused row softmax; the logits go to a
// workspace and its last pass writes each block's size-weighted mixture).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace bsa {

namespace {

constexpr int kClusterThreads = 128;

constexpr int kPanel = 128 * 128;   // one 128-byte swizzle panel: 128 rows x 64 bf16
constexpr int kOhPanel = 16 * 128;  // one-hot operand panel: 16 rows x 64 tokens
constexpr uint32_t kTmemCols = 64;  // one accumulator, reused by the two products

// Byte offset of bf16 element (row r, column c < 64) in a 128-byte-swizzled
// panel: row r at r * 128, its 16-byte chunk c / 8 stored at chunk (c / 8) ^ (r % 8)
// (the layout TMA's 128-byte swizzle writes, read by the tensor core).
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
    return static_cast<uint32_t>(r * 128 + ((((c >> 3) ^ r) & 7) << 4) + (c & 7) * 2);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// x = hi + mid + lo with each part a bf16 (round to nearest; x - hi and the
// next remainder are exact in fp32), so the three parts carry 24 bits of x.
__device__ __forceinline__ void split3(float x, uint32_t &hi, uint32_t &mid, uint32_t &lo) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(h);
    const __nv_bfloat16 m = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(m);
    const __nv_bfloat16 l = __float2bfloat16_rn(r2);
    hi = __bfloat16_as_ushort(h);
    mid = __bfloat16_as_ushort(m);
    lo = __bfloat16_as_ushort(l);
}

// k-means of one query block on the tensor cores, one CTA of 128 threads per
// block.  The block's tokens X (bf16, exact) sit in shared memory once,
// 128 x 128 (dimensions past D and tokens past n zero); thread t owns token t
// for the assignment and dimension t of every centroid (in registers) for the
// update.  Each round is two tcgen05 products into one TMEM accumulator:
//   distances   X (128 tokens x D) . [C_hi; C_mid; C_lo]^T, the centroids split
//               into three bf16 parts, so x . c_k is the sum of three columns
//               to fp32 accuracy; thread t takes argmin_k ||c_k||^2 - 2 x_t . c_k
//               (ties to the lower k);
//   sums        X^T (D x 128 tokens, the same tile read dimension-major) .
//               OneHot (128 tokens x 16), OneHot[t][k] = 1 iff token t joined
//               cluster k; thread d reads the 16 cluster sums of dimension d,
//               moves its coordinate of every non-empty centroid, and writes the
//               three parts of it and its share of ||c_k||^2 for the next round.
// One thread issues the MMAs; every wait on their completion is bounded, and a
// CTA whose wait gives up writes NaN centroids and zero sizes.
template <int D, int NSUB>
__global__ void __launch_bounds__(kClusterThreads, 3) subcluster_kernel(
    const uint16_t *__restrict__ q, float *__restrict__ cent, int32_t *__restrict__ size, int S,
    int S_pad, int bq, int Cq, int iters) {
    constexpr int kWarps = kClusterThreads / 32;
    constexpr int ND = (3 * NSUB + 15) / 16 * 16;  // distance product N: hi, mid, lo rows
    constexpr uint32_t kIdescDist = idesc_bf16_f32(128, ND, false);
    constexpr uint32_t kIdescSum = idesc_bf16_f32(128, 16, false) | (1u << 15);  // A = X^T, MN-major
    static_assert(NSUB <= 16, "one-hot operand holds 16 clusters");
    static_assert(D <= kClusterThreads, "one thread per dimension");
    extern __shared__ uint8_t dyn[];
    __shared__ float cnp[kWarps][NSUB];  // per-warp shares of ||c_k||^2
    __shared__ int wcnt[kWarps][NSUB];
    __shared__ __align__(8) uint64_t bar, drain;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_v;

    uint8_t *sX = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
    uint8_t *sOH = sX + 2 * kPanel;     // 2 panels (tokens 0-63, 64-127) x 16 rows
    uint8_t *sBD = sOH + 2 * kOhPanel;  // 2 panels (dimensions 0-63, 64-127) x ND rows

    const long long blk = blockIdx.x;
    const long long bh = blk / Cq;
    const int i = static_cast<int>(blk % Cq);
    const int n = max(0, min(bq, S - i * bq));
    const int tid = threadIdx.x, lane = tid % 32, wid = tid / 32;
    const bool owns_dim = tid < D;

    if (tid == 0) {
        mbar_init(&bar, 1);
        mbar_init(&drain, 1);
        abort_v = 0;
        fence_mbar_init();
    }
    if (wid == 0) {
        tmem_alloc(&tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    // the one-hot and split operands start zero (their rows past the live ones stay so)
    for (int e = tid * 16; e < 2 * kOhPanel + 2 * ND * 128; e += kClusterThreads * 16)
        *reinterpret_cast<uint4 *>(sOH + e) = make_uint4(0u, 0u, 0u, 0u);
    {  // tokens -> X: warp w copies tokens 32w .. 32w + 31, each load 32 consecutive 16-byte
       // chunks of their rows (coalesced); chunks of tokens past n are zero
        constexpr int CH = D / 8;  // 16-byte chunks per token row
        const uint4 *src = reinterpret_cast<const uint4 *>(q + (bh * S_pad + static_cast<long long>(i) * bq) * D);
#pragma unroll
        for (int it2 = 0; it2 < CH; ++it2) {
            const int idx = it2 * 32 + lane;
            const int t = 32 * wid + idx / CH, j = idx % CH;
            const uint4 v = t < n ? __ldg(src + t * CH + j) : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4 *>(sX + (j / 8) * kPanel + t * 128 + (((j & 7) ^ (t & 7)) << 4)) = v;
        }
        if (D < 128)  // dimensions past D: the second panel is zero
            for (int e = tid * 16; e < kPanel; e += kClusterThreads * 16)
                *reinterpret_cast<uint4 *>(sX + kPanel + e) = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();

    // Coordinate tid of every centroid, its three bf16 parts into the distance
    // operand (rows k, NSUB + k, 2 NSUB + k) and the warp's share of ||c_k||^2.
    float cd[NSUB];
    auto publish = [&]() {
#pragma unroll
        for (int k = 0; k < NSUB; ++k) {
            float sq = 0.f;
            if (owns_dim) {
                uint32_t h, m, l;
                split3(cd[k], h, m, l);
                uint8_t *pb = sBD + (tid / 64) * (ND * 128);
                *reinterpret_cast<uint16_t *>(pb + sw128_off(k, tid % 64)) = static_cast<uint16_t>(h);
                *reinterpret_cast<uint16_t *>(pb + sw128_off(NSUB + k, tid % 64)) = static_cast<uint16_t>(m);
                *reinterpret_cast<uint16_t *>(pb + sw128_off(2 * NSUB + k, tid % 64)) = static_cast<uint16_t>(l);
                sq = cd[k] * cd[k];
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
            if (lane == 0) cnp[wid][k] = sq;
        }
        fence_proxy_async_smem();
    };
    // seeds: the tokens at floor(k * n / NSUB)
#pragma unroll
    for (int k = 0; k < NSUB; ++k) {
        const int t0 = n > 0 ? static_cast<int>((static_cast<long long>(k) * n) / NSUB) : 0;
        cd[k] = 0.f;
        if (owns_dim && n > 0)
            cd[k] = bf16_bits_to_float(
                *reinterpret_cast<const uint16_t *>(sX + (tid / 64) * kPanel + sw128_off(t0, tid % 64)));
    }
    publish();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wid * 32) << 16);

    uint32_t phase = 0;
    bool ok = true;
    int sz[NSUB];
#pragma unroll
    for (int k = 0; k < NSUB; ++k) sz[k] = 0;
    for (int it = 0; it < iters; ++it) {
        int best = 0;
        if (NSUB > 1) {
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t a_off = (kk / 4) * kPanel + (kk % 4) * 32;
                    const uint32_t b_off = (kk / 4) * (ND * 128) + (kk % 4) * 32;
                    mma_ss(tmem, sw128_desc(smem_u32(sX) + a_off, 16, 1024),
                           sw128_desc(smem_u32(sBD) + b_off, 16, 1024), kIdescDist, kk > 0 ? 1u : 0u);
                }
                mma_commit(&bar);
            }
            ok = mbar_wait(&bar, phase, &abort_v);
            phase ^= 1u;
            if (!__syncthreads_and(ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t r[ND];
#pragma unroll
            for (int q16 = 0; q16 < ND / 16; ++q16) {
                uint32_t part[16];
                tmem_ld16(t_lane + static_cast<uint32_t>(q16 * 16), part);
                tmem_ld_wait();
                reg_fence(part);
#pragma unroll
                for (int e = 0; e < 16; ++e) r[q16 * 16 + e] = part[e];
            }
            if (tid < n) {
                float bd = INFINITY;
#pragma unroll
                for (int k = 0; k < NSUB; ++k) {
                    float cn = cnp[0][k];
#pragma unroll
                    for (int w = 1; w < kWarps; ++w) cn += cnp[w][k];
                    const float dot = (__uint_as_float(r[k]) + __uint_as_float(r[NSUB + k])) +
                                      __uint_as_float(r[2 * NSUB + k]);
                    const float dist = fmaf(-2.f, dot, cn);
                    if (dist < bd) {
                        bd = dist;
                        best = k;
                    }
                }
            }
        }
        // cluster sizes by ballots; column tid of the one-hot operand
        const bool live = tid < n;
#pragma unroll
        for (int k = 0; k < NSUB; ++k) {
            const unsigned bal = __ballot_sync(0xffffffffu, live && best == k);
            if (lane == 0) wcnt[wid][k] = __popc(bal);
            *reinterpret_cast<uint16_t *>(sOH + (tid / 64) * kOhPanel + sw128_off(k, tid % 64)) =
                (live && best == k) ? static_cast<uint16_t>(0x3F80u) : static_cast<uint16_t>(0u);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t a_off = kk * 2048;  // tokens 16 kk .. 16 kk + 15 of X^T
                const uint32_t b_off = (kk / 4) * kOhPanel + (kk % 4) * 32;
                mma_ss(tmem, sw128_desc(smem_u32(sX) + a_off, kPanel, 1024),
                       sw128_desc(smem_u32(sOH) + b_off, 16, 1024), kIdescSum, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bar);
        }
#pragma unroll
        for (int k = 0; k < NSUB; ++k) {
            int s2 = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) s2 += wcnt[w][k];
            sz[k] = s2;
        }
        ok = mbar_wait(&bar, phase, &abort_v);
        phase ^= 1u;
        if (!__syncthreads_and(ok)) {
            ok = false;
            break;
        }
        tc_fence_after();
        {  // move the centroids: thread d reads the 16 cluster sums of dimension d
            uint32_t u[16];
            tmem_ld16(t_lane, u);
            tmem_ld_wait();
            reg_fence(u);
#pragma unroll
            for (int k = 0; k < NSUB; ++k)
                if (sz[k] > 0) cd[k] = __uint_as_float(u[k]) / static_cast<float>(sz[k]);
        }
        publish();
        tc_fence_before();
        __syncthreads();
    }
    if (!ok) {  // let whatever was issued finish before TMEM is freed
        if (tid == 0) {
            mma_commit(&drain);
            volatile int no_abort = 0;
            mbar_wait(&drain, 0, &no_abort);
        }
    }
    __syncthreads();
    if (owns_dim) {
#pragma unroll
        for (int k = 0; k < NSUB; ++k) cent[(blk * NSUB + k) * D + tid] = ok ? cd[k] : NAN;
    }
    if (tid == 0) {
#pragma unroll
        for (int k = 0; k < NSUB; ++k) size[blk * NSUB + k] = ok ? sz[k] : 0;
    }
    if (wid == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D, int NSUB>
cudaError_t launch_sub_t(const uint16_t *q, float *cent, int32_t *size, const Geometry &g,
                         long long blocks, int iters, cudaStream_t st) {
    constexpr int ND = (3 * NSUB + 15) / 16 * 16;
    const size_t smem = 1024 + 2 * kPanel + 2 * kOhPanel + 2 * ND * 128;
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
    // the sub-centroid rows as C_q * nsub query rows of the score kernel, which mixes
    // each block's rows into its P' row
    Geometry gs = g;
    gs.Cq = g.Cq * nsub;
    float *psub = static_cast<float *>(workspace);
    return launch_scores(gs, cent, kc, psub, st, size, nsub, probs);
}

}  // namespace bsa
