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
// score_kernel  the centroid GEMM (C_q x C_k x D per head) on the tensor
//               cores in split-tf32 (three kind::tf32 MMAs per K step), with
//               the n_j-weighted row softmax fused into the TMEM epilogue.
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

// One CTA per key block: the value centroid (mean of V over the block's valid
// tokens, as for the key centroid) and its L2 norm ||c^V_{h,j}||, the weight of
// the value-aware score ("Competition Domains Matter ..." s4).
template <int D>
__global__ void __launch_bounds__(256) vnorm_kernel(const uint4 *__restrict__ v,
                                                    float *__restrict__ vnorm, int S, int S_pad,
                                                    int bk, int Ck) {
    constexpr int CH = D / 8;      // 16-byte chunks per token row
    constexpr int RPI = 256 / CH;  // rows covered per pass of the CTA
    constexpr int PASSES = 128 / RPI;
    __shared__ float red[RPI][D];
    __shared__ float sq[8];
    const long long item = blockIdx.x;
    const long long bh = item / Ck;
    const int j = static_cast<int>(item % Ck);
    const int n = min(bk, S - j * bk);
    const uint4 *base = v + ((bh * S_pad + static_cast<long long>(j) * bk) * D) / 8;
    const int c = threadIdx.x % CH, r0 = threadIdx.x / CH;
    uint4 x[PASSES];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int r = r0 + p * RPI;
        x[p] = (r < n) ? __ldg(base + r * CH + c) : make_uint4(0, 0, 0, 0);
    }
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int p = 0; p < PASSES; ++p) bf16x8_add(x[p], acc);
#pragma unroll
    for (int e = 0; e < 8; ++e) red[r0][c * 8 + e] = acc[e];
    __syncthreads();
    float part = 0.f;
    for (int d = threadIdx.x; d < D; d += 256) {
        float sum = 0.f;
#pragma unroll
        for (int r = 0; r < RPI; ++r) sum += red[r][d];
        const float m = sum / static_cast<float>(n);
        part = fmaf(m, m, part);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (threadIdx.x % 32 == 0) sq[threadIdx.x / 32] = part;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += sq[w];
        vnorm[item] = sqrtf(t);
    }
}

// ---------------------------------------------------------------------------
// score_kernel: the centroid GEMM on the tensor cores, row softmax fused.
//
// Work item = (b*h, 128 query-block rows).  For each chunk of 128 key-block
// columns the item's logits accumulate in TMEM (four chunk buffers of 128
// columns, so the products run ahead while the epilogue normalises the
// previous item), fed by 2 shared-memory stages that each hold one 32-wide slice of
// D ("panel") of q-bar (128 x 32 fp32) and k-bar (128 x 32 fp32).
//
// Precision: plain tf32 keeps ~11 significant bits, far too coarse for logits
// of magnitude ~50 (P' must stay within 1e-4).  Each operand x is split
// exactly into hi = x with the low 13 mantissa bits cleared (a tf32 value)
// and lo = x - hi, and the product is hi_a hi_b + hi_a lo_b + lo_a hi_b
// (three tf32 MMAs), which leaves an error near 2^-21 relative.  The kind::tf32
// MMA reads only the upper 19 bits of each 32-bit operand, so the fp32 panel as
// loaded serves as hi and only lo is written.  q-bar is the same for all chunks of
// an item: its lo panels are made once per item into a resident region; per
// stage only k-bar's lo is made.
//
// Warp roles (384 threads):
//   warp 0      TMA producer: q-bar and k-bar panels into the stage
//   warp 1      TMEM owner; lane 0 issues the tcgen05.mma (kind::tf32)
//   warps 2-3   split workers: k-bar lo for each landed stage, and at an item's
//               first chunk also the q-bar lo panels of the item
//   warps 4-11  epilogue, two groups of four: thread = query-block row (TMEM
//               lane); group g takes 32-column slices 2g, 2g+1 of every chunk:
//               s2 = acc * log2(e)/sqrt(D) + log2(n_j/k_block), a running row max m2 and
//               sum z of 2^(s2 - m2); each warp transposes its own 32 x 32 slice
//               through shared memory so it writes one row's 32 values
//               contiguously.  After the last chunk the groups' (m2, z) are
//               merged and the eight warps rewrite 16 rows each,
//               s2 -> 2^(s2 - m2) / z, a row at a time across the warp.
namespace sc {

constexpr int kThreads = 384;
constexpr int kSplitThreads = 64;                    // warps 2-3
constexpr int kRows = 128;                           // MMA M
constexpr int kCols = 128;                           // MMA N: key-block columns per chunk
constexpr int kAPanelBytes = kRows * 128;            // 128 rows x 32 fp32
constexpr int kBPanelBytes = kCols * 128;            // 128 rows x 32 fp32
constexpr int kStageBytes = kAPanelBytes + 2 * kBPanelBytes;  // A, B, B_lo
constexpr int kMaxPanels = 4;                        // D / 32 for D <= 128
constexpr int kStages = 2;
constexpr int kAccBufs = 4;                          // chunk accumulators in TMEM
constexpr int kTmemCols = kAccBufs * kCols;
// Staging row pitch (floats): a multiple of 4, so a lane writes its row with
// 16-byte stores (conflict-free per quarter-warp), and 4i + lane keeps the
// column reads of one row conflict-free.
constexpr int kPitch = 36;

struct Header {
    uint64_t full[kStages];    // TMA landed (expect_tx)
    uint64_t split[kStages];   // hi / lo written (kSplitThreads arrivals)
    uint64_t empty[kStages];   // MMAs done with the stage (commit)
    uint64_t acc_full[kAccBufs];   // chunk accumulated (commit)
    uint64_t acc_empty[kAccBufs];  // epilogue read the chunk (256 arrivals)
    uint64_t mma_done;         // every issued MMA finished (commit)
    uint32_t tmem_base;
    int abort;
    float m2[2][kRows], z[2][kRows];  // per epilogue group: running max and sum of each row
};
constexpr int kHeaderBytes = 3072;
static_assert(sizeof(Header) <= kHeaderBytes, "header");
constexpr int kOffStaging = kHeaderBytes;
constexpr int kEpiWarps = 8;
constexpr int kOffStages = ((kOffStaging + kEpiWarps * 32 * kPitch * 4) + 1023) / 1024 * 1024;
constexpr int kOffALo = kOffStages + kStages * kStageBytes;  // the item's q-bar lo panels
constexpr int kSmemBytes = kOffALo + kMaxPanels * kAPanelBytes;
constexpr int kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 227 * 1024, "shared memory");

struct Params {
    float *probs;
    int Cq, Ck, S, bk, n_rt, n_items;
    float scale2;  // log2(e) / sqrt(D)
    float last_log2n;  // log2(n / k_block) of the last key block (the others hold k_block tokens)
    // Mixing (the rows are nsub sub-centroid rows per query block): instead of
    // normalising its rows in place, the last pass writes each block's row
    // sum_c (n_c / n) P'_c into mix_out; nullptr = plain rows.
    const int32_t *mix_size;  // [blocks, nsub] cluster sizes
    float *mix_out;           // [blocks, C_k]
    int nsub;
};

// Clear the low 13 mantissa bits: an exact tf32 value, and x - hi is exact.
__device__ __forceinline__ void split4(uint4 &x, uint4 &lo) {
    const uint32_t m = 0xFFFFE000u;
    const uint4 hi = make_uint4(x.x & m, x.y & m, x.z & m, x.w & m);
    lo = make_uint4(__float_as_uint(__uint_as_float(x.x) - __uint_as_float(hi.x)),
                    __float_as_uint(__uint_as_float(x.y) - __uint_as_float(hi.y)),
                    __float_as_uint(__uint_as_float(x.z) - __uint_as_float(hi.z)),
                    __float_as_uint(__uint_as_float(x.w) - __uint_as_float(hi.w)));
    x = hi;
}

}  // namespace sc

template <int D>
__global__ void __launch_bounds__(sc::kThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                 sc::Params p) {
    using namespace sc;
    constexpr int NP = D / 32;  // panels per chunk
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Header &hd = *reinterpret_cast<Header *>(smem);
    float *stg = reinterpret_cast<float *>(smem + kOffStaging);
    uint8_t *stages = smem + kOffStages;
    uint8_t *a_lo_res = smem + kOffALo;
    static_assert(NP <= kMaxPanels, "resident q-bar lo panels");
    volatile int *abort_flag = &hd.abort;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nch = (p.Ck + kCols - 1) / kCols;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&hd.full[s], 1);
            mbar_init(&hd.split[s], kSplitThreads);
            mbar_init(&hd.empty[s], 1);
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(&hd.acc_full[b], 1);
            mbar_init(&hd.acc_empty[b], 256);
        }
        mbar_init(&hd.mma_done, 1);
        hd.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&hd.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = hd.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&mq);
            prefetch_tmap(&mk);
            int it = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
                const int bh = item / p.n_rt, r0 = (item % p.n_rt) * kRows;
                for (int c = 0; ok && c < nch; ++c) {
                    for (int pn = 0; pn < NP; ++pn, ++it) {
                        const int st = it % kStages;
                        if (it >= kStages &&
                            !mbar_wait(&hd.empty[st], ((it / kStages) - 1) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        uint8_t *sb = stages + st * kStageBytes;
                        mbar_arrive_expect_tx(&hd.full[st], kAPanelBytes + kBPanelBytes);
                        tma_load_3d(sb, &mq, &hd.full[st], pn * 32, r0, bh);
                        tma_load_3d(sb + kAPanelBytes, &mk, &hd.full[st], pn * 32, c * kCols, bh);
                    }
                }
            }
            // the last loads must land before the CTA may exit
            volatile int no_abort = 0;
            for (int k = it > kStages ? it - kStages : 0; k < it; ++k)
                mbar_wait(&hd.full[k % kStages], (k / kStages) & 1, &no_abort);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_tf32_f32(kRows, kCols);
            int it = 0, ch = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
                for (int c = 0; ok && c < nch; ++c, ++ch) {
                    const int buf = ch % kAccBufs;
                    if (ch >= kAccBufs &&
                        !mbar_wait(&hd.acc_empty[buf], ((ch / kAccBufs) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d = tmem + static_cast<uint32_t>(buf * kCols);
                    for (int pn = 0; pn < NP; ++pn, ++it) {
                        const int st = it % kStages;
                        if (!mbar_wait(&hd.split[st], (it / kStages) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sb = smem_u32(stages + st * kStageBytes);
                        const uint64_t a_hi = sw128_desc(sb, 16, 1024);
                        const uint64_t a_lo =
                            sw128_desc(smem_u32(a_lo_res + pn * kAPanelBytes), 16, 1024);
                        const uint64_t b_hi = sw128_desc(sb + kAPanelBytes, 16, 1024);
                        const uint64_t b_lo = sw128_desc(sb + kAPanelBytes + kBPanelBytes, 16, 1024);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {  // K = 8 tf32 = 32 bytes per MMA
                            const uint64_t o = static_cast<uint64_t>(k * 2);
                            mma_tf32_ss(d, a_hi + o, b_hi + o, idesc, (pn | k) ? 1u : 0u);
                            mma_tf32_ss(d, a_hi + o, b_lo + o, idesc, 1u);
                            mma_tf32_ss(d, a_lo + o, b_hi + o, idesc, 1u);
                        }
                        mma_commit(&hd.empty[st]);
                    }
                    if (!ok) break;
                    mma_commit(&hd.acc_full[buf]);
                }
            }
            // every issued MMA completes before TMEM is released
            mma_commit(&hd.mma_done);
            volatile int no_abort = 0;
            mbar_wait(&hd.mma_done, 0, &no_abort);
        }
    } else if (warp == 2 || warp == 3) {
        // ------------------------------------------------------------ split workers
        const int tid = threadIdx.x - 64;
        int it = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
            for (int c = 0; ok && c < nch; ++c) {
                for (int pn = 0; pn < NP; ++pn, ++it) {
                    const int st = it % kStages;
                    if (!mbar_wait(&hd.full[st], (it / kStages) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint4 *a = reinterpret_cast<uint4 *>(stages + st * kStageBytes);
                    uint4 *b = a + kAPanelBytes / 16;
                    uint4 *b_lo = b + kBPanelBytes / 16;
                    // lo at the same byte offset as its source: the 128-byte swizzle depends
                    // only on the address bits inside the 1024-byte-aligned atom.  Eight
                    // 16-byte loads are in flight per thread before any is split.
                    auto split_panel = [&](const uint4 *src, uint4 *lo_out) {
                        constexpr int kPer = kAPanelBytes / 16 / kSplitThreads;
                        static_assert(kAPanelBytes == kBPanelBytes && kPer % 8 == 0, "split batches");
#pragma unroll
                        for (int b0 = 0; b0 < kPer; b0 += 8) {
                            uint4 x[8];
#pragma unroll
                            for (int u = 0; u < 8; ++u) x[u] = src[tid + (b0 + u) * kSplitThreads];
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                uint4 lo;
                                split4(x[u], lo);
                                lo_out[tid + (b0 + u) * kSplitThreads] = lo;
                            }
                        }
                    };
                    if (c == 0) {
                        // The item's q-bar lo panel pn is made from its first chunk.  Before
                        // the first one is overwritten, every product of the previous item
                        // (the last readers of the region) must have completed: the commit
                        // after stage use it-1 covers them all.
                        if (pn == 0 && it > 0 &&
                            !mbar_wait(&hd.empty[(it - 1) % kStages], ((it - 1) / kStages) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        split_panel(a, reinterpret_cast<uint4 *>(a_lo_res + pn * kAPanelBytes));
                    }
                    split_panel(b, b_lo);
                    fence_proxy_async_smem();
                    mbar_arrive(&hd.split[st]);
                }
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        // Two warpgroups: group eg takes slices 4*eg .. 4*eg+3 (32 columns each) of
        // every 256-column chunk; warp quarter ew of a group owns TMEM lanes
        // 32*ew .. 32*ew+31, i.e. tile rows, and keeps their running max m2 and sum z
        // over its own slices.  Each warp transposes its own 32 x 32 slices in a
        // private staging block, so the warps never wait for one another inside a
        // chunk.  At the end of an item the two groups' (m2, z) are merged through
        // shared memory and the eight warps rewrite 16 rows each:
        // s2 -> 2^(s2 - m2) / z.  The two named-barrier steps are votes
        // (bar.red.and), so an aborted wait makes all eight warps stop together.
        const int eg = (warp - 4) >> 2;
        const int ew = warp & 3;
        const int ewarp = warp - 4;        // 0 .. 7
        const int rl = ew * 32 + lane;     // row within the tile = TMEM lane
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(ew * 32) << 16);
        float *wst = stg + ewarp * 32 * kPitch;  // this warp's 32 x kPitch staging block
        int ch = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
            const int bh = item / p.n_rt, r0 = (item % p.n_rt) * kRows;
            const int nrows = min(kRows, p.Cq - r0);
            const int my_rows = max(0, min(32, nrows - ew * 32));  // rows of this warp's quarter
            float *wtile = p.probs + (static_cast<long long>(bh) * p.Cq + r0 + ew * 32) * p.Ck;
            float m2 = -INFINITY, z = 0.f;
            for (int c = 0; c < nch; ++c, ++ch) {
                const int buf = ch % kAccBufs;
                if (!__all_sync(0xffffffffu,
                                mbar_wait(&hd.acc_full[buf], (ch / kAccBufs) & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int n_sl = min(kCols / 32, (p.Ck - c * kCols + 31) / 32);
                const int s_lo = 2 * eg, s_hi = min(s_lo + 2, n_sl);
                uint32_t nxt[32];
                if (s_lo < s_hi) {
                    tmem_ld32(t_lane + static_cast<uint32_t>(buf * kCols + s_lo * 32), nxt);
                    tmem_ld_wait();
                    reg_fence(nxt);  // no read of nxt may move above the wait
                }
                for (int s = s_lo; s < s_hi; ++s) {
                    const int col0 = c * kCols + s * 32;
                    uint32_t r[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = nxt[j];
                    reg_fence(r);
                    // the next slice's TMEM load runs while this one is processed
                    if (s + 1 < s_hi)
                        tmem_ld32(t_lane + static_cast<uint32_t>(buf * kCols + (s + 1) * 32), nxt);
                    // s2 = acc * log2(e)/sqrt(D) + log2(n_j / k_block): every key block but
                    // the last holds k_block tokens, so the offset is 0 except in the last
                    // column (a common shift of a row leaves its softmax unchanged)
                    float mx = -INFINITY;
                    if (col0 + 32 < p.Ck) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float t = __uint_as_float(r[j]) * p.scale2;
                            r[j] = __float_as_uint(t);
                            mx = fmaxf(mx, t);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int col = col0 + j;
                            const float t = col < p.Ck ? fmaf(__uint_as_float(r[j]), p.scale2,
                                                              col == p.Ck - 1 ? p.last_log2n : 0.f)
                                                       : -INFINITY;
                            r[j] = __float_as_uint(t);
                            mx = fmaxf(mx, t);
                        }
                    }
                    const float mn = fmaxf(m2, mx);
                    float sum = 0.f;
#pragma unroll
                    for (int j = 0; j < 32; ++j) sum += ex2(__uint_as_float(r[j]) - mn);
                    z = z * ex2(m2 - mn) + sum;
                    m2 = mn;
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<uint4 *>(wst + lane * kPitch + j) =
                            make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]);
                    __syncwarp();
                    // row i of this warp: 32 consecutive columns, one 128-byte store
                    const int col = col0 + lane;
                    if (col < p.Ck) {
                        float v[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = wst[i * kPitch + lane];
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i < my_rows) wtile[static_cast<long long>(i) * p.Ck + col] = v[i];
                    }
                    __syncwarp();
                    if (s + 1 < s_hi) {
                        tmem_ld_wait();  // the prefetched slice has landed
                        reg_fence(nxt);
                    }
                }
                tc_fence_before();
                mbar_arrive(&hd.acc_empty[buf]);
            }
            // merge the two groups' statistics of every row (all eight warps vote, so an
            // abort in any of them ends the item in all of them)
            hd.m2[eg][rl] = m2;
            hd.z[eg][rl] = z;
            ok = bar_and(1, 256, ok);
            if (!ok) break;
            // P' = 2^(s2 - m2) / z for 16 rows per warp, one row at a time across the
            // warp (coalesced), two rows in flight
            const int w0 = ewarp * 16;                                  // first tile row
            const int w_rows = max(0, min(16, nrows - w0));
            float *wrows = p.probs + (static_cast<long long>(bh) * p.Cq + r0 + w0) * p.Ck;
            auto merged = [&](int tr, float &m, float &iz) {
                const float ma = hd.m2[0][tr], mb = hd.m2[1][tr];
                m = fmaxf(ma, mb);
                const float za = ma == -INFINITY ? 0.f : hd.z[0][tr] * ex2(ma - m);
                const float zb = mb == -INFINITY ? 0.f : hd.z[1][tr] * ex2(mb - m);
                iz = 1.0f / (za + zb);
            };
            if (p.mix_out) {
                // A block's nsub rows are consecutive and never straddle a warp's 16 rows
                // (nsub divides 16): its P' row is sum_c w_c 2^(s2_c - m2_c) / z_c with
                // w_c = n_c / n, the terms added in ascending c (fused multiply-add), the
                // same arithmetic as normalising the rows and then mixing them.
                const int ns = p.nsub;
                for (int i = 0; i < w_rows; i += ns) {
                    const long long brow = (static_cast<long long>(bh) * p.Cq + r0 + w0 + i) / ns;
                    int ntot = 0;
                    for (int c = 0; c < ns; ++c) ntot += __ldg(p.mix_size + brow * ns + c);
                    const float inv = ntot > 0 ? 1.f / static_cast<float>(ntot) : 0.f;
                    float *out = p.mix_out + brow * p.Ck;
                    for (int c0 = 0; c0 < p.Ck; c0 += 1024) {
                        float acc[32];
#pragma unroll
                        for (int k = 0; k < 32; ++k) acc[k] = 0.f;
                        for (int c = 0; c < ns; ++c) {
                            const float wc = static_cast<float>(__ldg(p.mix_size + brow * ns + c)) * inv;
                            if (!(wc > 0.f)) continue;
                            float mc, izc;
                            merged(w0 + i + c, mc, izc);
                            const float *rc = wrows + static_cast<long long>(i + c) * p.Ck;
                            float v[32];
#pragma unroll
                            for (int k = 0; k < 32; ++k) {
                                const int col = c0 + lane + 32 * k;
                                v[k] = col < p.Ck ? rc[col] : 0.f;
                            }
#pragma unroll
                            for (int k = 0; k < 32; ++k) acc[k] = fmaf(wc, ex2(v[k] - mc) * izc, acc[k]);
                        }
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const int col = c0 + lane + 32 * k;
                            if (col < p.Ck) out[col] = acc[k];
                        }
                    }
                }
            } else {
                for (int i = 0; i < w_rows; i += 2) {
                    const bool two = i + 1 < w_rows;
                    float ma, iza, mb = 0.f, izb = 0.f;
                    merged(w0 + i, ma, iza);
                    if (two) merged(w0 + i + 1, mb, izb);
                    float *ra = wrows + static_cast<long long>(i) * p.Ck;
                    float *rb = ra + p.Ck;
                    for (int c0 = 0; c0 < p.Ck; c0 += 1024) {
                        float va[32], vb[32];
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const int col = c0 + lane + 32 * k;
                            va[k] = col < p.Ck ? ra[col] : 0.f;
                            vb[k] = (two && col < p.Ck) ? rb[col] : 0.f;
                        }
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const int col = c0 + lane + 32 * k;
                            if (col < p.Ck) {
                                ra[col] = ex2(va[k] - ma) * iza;
                                if (two) rb[col] = ex2(vb[k] - mb) * izb;
                            }
                        }
                    }
                }
            }
            // the statistics are reused by the next item; its first-pass stores must
            // also come after this pass's reads of the same rows
            ok = bar_and(1, 256, ok);
        }
    }
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// [B*H, rows, D] fp32 view, box = 32 x box_rows x 1 with the 128-byte swizzle;
// rows past `rows` read as zeros.
bool make_f32_map(CUtensorMap *m, const float *base, long long BH, int rows, int D, int box_rows) {
    TensorMapEncoder enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                                static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 4,
                                   static_cast<cuuint64_t>(rows) * D * 4};
    const cuuint32_t box[3] = {32, static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_scores_t(const Geometry &g, const float *qc, const float *kc, float *probs,
                            cudaStream_t st, const int32_t *mix_size, int nsub, float *mix_out) {
    const long long BH = static_cast<long long>(g.B) * g.H;
    CUtensorMap mq, mk;
    if (!make_f32_map(&mq, qc, BH, g.Cq, D, sc::kRows) || !make_f32_map(&mk, kc, BH, g.Ck, D, sc::kCols))
        return cudaErrorInvalidValue;
    sc::Params p;
    p.probs = probs;
    p.Cq = g.Cq;
    p.Ck = g.Ck;
    p.S = g.S;
    p.bk = g.bk;
    p.n_rt = (g.Cq + sc::kRows - 1) / sc::kRows;
    const long long items = BH * p.n_rt;
    if (items > 0x7FFFFFFFll) return cudaErrorInvalidValue;
    p.n_items = static_cast<int>(items);
    p.scale2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
    p.last_log2n = log2f(static_cast<float>(g.S - (g.Ck - 1) * g.bk) / static_cast<float>(g.bk));
    p.mix_size = mix_size;
    p.mix_out = mix_out;
    p.nsub = nsub;
    if (mix_out && (!mix_size || nsub < 1 || 16 % nsub != 0 || g.Cq % nsub != 0)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         sc::kSmemAlloc);
    if (e != cudaSuccess) return e;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidValue;
    const int grid = p.n_items < sms ? p.n_items : sms;
    score_kernel<D><<<grid, sc::kThreads, sc::kSmemAlloc, st>>>(mq, mk, p);
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

cudaError_t launch_pool_keys(const Geometry &g, const void *k, float *kc, cudaStream_t st) {
    const long long nk = static_cast<long long>(g.B) * g.H * g.Ck;
    const uint4 *k4 = static_cast<const uint4 *>(k);
    if (g.D == 128)
        pool_kernel<128><<<static_cast<unsigned>(nk), 256, 0, st>>>(
            nullptr, k4, nullptr, kc, g.S, g.S_pad, g.bq, g.bk, g.Cq, g.Ck, 0);
    else
        pool_kernel<64><<<static_cast<unsigned>(nk), 256, 0, st>>>(
            nullptr, k4, nullptr, kc, g.S, g.S_pad, g.bq, g.bk, g.Cq, g.Ck, 0);
    return cudaGetLastError();
}

cudaError_t launch_value_norms(const Geometry &g, const void *v, float *vnorm, cudaStream_t st) {
    const long long nk = static_cast<long long>(g.B) * g.H * g.Ck;
    const auto *v4 = static_cast<const uint4 *>(v);
    if (g.D == 128)
        vnorm_kernel<128><<<static_cast<unsigned>(nk), 256, 0, st>>>(v4, vnorm, g.S, g.S_pad, g.bk, g.Ck);
    else
        vnorm_kernel<64><<<static_cast<unsigned>(nk), 256, 0, st>>>(v4, vnorm, g.S, g.S_pad, g.bk, g.Ck);
    return cudaGetLastError();
}

cudaError_t launch_scores(const Geometry &g, const float *qc, const float *kc, float *probs,
                          cudaStream_t st, const int32_t *mix_size, int nsub, float *mix_out) {
    return g.D == 128 ? launch_scores_t<128>(g, qc, kc, probs, st, mix_size, nsub, mix_out)
                      : launch_scores_t<64>(g, qc, kc, probs, st, mix_size, nsub, mix_out);
}

}  // namespace bsa
