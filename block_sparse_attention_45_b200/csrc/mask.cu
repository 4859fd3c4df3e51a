// mask.cu -- per-row top-p selection, overrides, per-head entropy, lists.
//
// "Competition Domains Matter ..." s3, domain 1 ("per-row local"): every
// query row (h, i) keeps the top-p portion of P'[h, i, :]; the per-head
// entropy H_h averages the row entropies -sum_j P' log(P' + eps) (Eq. 3) and
// is normalised by log C_k.  "Attention matrix view: make only frame-0 query
// rows dense" s4/s6: query blocks that overlap frame 0 keep every key block;
// s7: text/global key blocks are always kept.
//
// One warp per row; element j of the row lives in lane j % 32, slot j / 32.
// Top-p without sorting: P' >= 0, so the fp32 bit patterns order like the
// values.  With f(u) = sum of the values whose pattern is >= u (a step
// function, non-increasing in u), the cut value v* is the largest pattern u*
// with f(u*) >= p, found by bisection on u; the row keeps every value above
// v* plus, among the entries equal to v*, the lowest-index ones needed for the
// running sum to reach p -- the same set as sorting by (P' desc, j asc) and
// taking the shortest prefix whose sum reaches p.  Row entropies go to a
// workspace; a second kernel sums them per head in a fixed order.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace bsa {

namespace {

struct MaskArgs {
    const float *probs;
    uint8_t *mask;
    int32_t *kv_index;
    int32_t *kv_count;
    float *row_entropy;
    long long rows;
    int H, Cq, Ck;
    uint32_t flags;
    float eps;
    int text_kblocks, f0_first, f0_last;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int VPL>
__global__ void __launch_bounds__(256) mask_kernel(MaskArgs a, TopP tp) {
    const int lane = threadIdx.x % 32;
    const long long row = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
    if (row >= a.rows) return;  // whole warp leaves together
    const int Ck = a.Ck;
    const int i = static_cast<int>(row % a.Cq);
    const int h = static_cast<int>((row / a.Cq) % a.H);
    const float p = tp.p[h];
    const float *src = a.probs + row * Ck;

    float v[VPL];
    uint32_t u[VPL];
    float ent = 0.f, total = 0.f;
    uint32_t umax = 0;
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int j = lane + 32 * s;
        float x = (j < Ck) ? __ldg(src + j) : 0.f;
        x = fmaxf(x, 0.f);
        v[s] = x;
        u[s] = __float_as_uint(x);
        umax = max(umax, u[s]);
        total += x;
        if (j < Ck) ent -= x * logf(x + a.eps);
    }
    total = warp_sum(total);
    if (a.row_entropy) {
        ent = warp_sum(ent);
        if (lane == 0) a.row_entropy[row] = ent;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) umax = max(umax, __shfl_xor_sync(0xffffffffu, umax, o));

    bool keep_all = !(total >= p);  // the row never reaches p: keep everything
    uint32_t ucut = 0;
    int ties_needed = 0;
    if (!keep_all) {
        uint32_t lo = 0, hi = umax;  // invariant: f(lo) >= p
        while (lo < hi) {
            const uint32_t mid = lo + ((hi - lo + 1) >> 1);
            float f = 0.f;
#pragma unroll
            for (int s = 0; s < VPL; ++s) f += (u[s] >= mid) ? v[s] : 0.f;
            f = warp_sum(f);
            if (f >= p) lo = mid;
            else hi = mid - 1;
        }
        ucut = lo;
        float above = 0.f;
        int ties = 0;
#pragma unroll
        for (int s = 0; s < VPL; ++s) {
            above += (u[s] > ucut) ? v[s] : 0.f;
            ties += (u[s] == ucut && lane + 32 * s < Ck) ? 1 : 0;
        }
        above = warp_sum(above);
        ties = warp_sum_i(ties);
        const float vcut = __uint_as_float(ucut);
        float run = above + vcut;
        ties_needed = 1;
        while (run < p && ties_needed < ties) {
            run += vcut;
            ++ties_needed;
        }
    }

    const bool dense_row = (a.flags & BSA_FRAME0_DENSE) && i >= a.f0_first && i <= a.f0_last;
    const bool text = (a.flags & BSA_TEXT_KEEP) != 0;
    uint8_t *mrow = a.mask ? a.mask + row * Ck : nullptr;
    int32_t *irow = a.kv_index + row * Ck;
    const uint32_t lt_mask = (1u << lane) - 1u;
    int base = 0, tie_base = 0;
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int j = lane + 32 * s;
        const bool valid = j < Ck;
        const bool is_tie = valid && !keep_all && u[s] == ucut;
        const uint32_t tie_bal = __ballot_sync(0xffffffffu, is_tie);
        const int tie_rank = tie_base + __popc(tie_bal & lt_mask);
        tie_base += __popc(tie_bal);
        bool sel = keep_all || u[s] > ucut || (is_tie && tie_rank < ties_needed);
        sel = valid && (sel || dense_row || (text && j < a.text_kblocks));
        if (mrow && valid) mrow[j] = sel ? 1 : 0;
        const uint32_t bal = __ballot_sync(0xffffffffu, sel);
        if (sel) irow[base + __popc(bal & lt_mask)] = j;
        base += __popc(bal);
    }
    if (lane == 0) a.kv_count[row] = base;
}

// One warp per (b, h): mean of its C_q row entropies, summed in a fixed order.
__global__ void __launch_bounds__(256) entropy_reduce_kernel(const float *__restrict__ row_entropy,
                                                             float *entropy, float *entropy_norm,
                                                             long long BH, int Cq, float inv_log_ck) {
    const int lane = threadIdx.x % 32;
    const long long bh = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
    if (bh >= BH) return;
    const float *src = row_entropy + bh * Cq;
    double s = 0.0;
    for (int i = lane; i < Cq; i += 32) s += static_cast<double>(src[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
        const float H = static_cast<float>(s / Cq);
        if (entropy) entropy[bh] = H;
        if (entropy_norm) entropy_norm[bh] = H * inv_log_ck;
    }
}

template <int VPL>
cudaError_t launch_mask_t(const MaskArgs &a, const TopP &tp, cudaStream_t st) {
    const unsigned grid = static_cast<unsigned>((a.rows + 7) / 8);
    mask_kernel<VPL><<<grid, 256, 0, st>>>(a, tp);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mask(const Geometry &g, const float *probs, const TopP &tp, uint32_t flags,
                        float eps, uint8_t *mask, int32_t *kv_index, int32_t *kv_count,
                        float *row_entropy, cudaStream_t st) {
    MaskArgs a;
    a.probs = probs;
    a.mask = mask;
    a.kv_index = kv_index;
    a.kv_count = kv_count;
    a.row_entropy = row_entropy;
    a.rows = static_cast<long long>(g.B) * g.H * g.Cq;
    a.H = g.H;
    a.Cq = g.Cq;
    a.Ck = g.Ck;
    a.flags = flags;
    a.eps = eps;
    a.text_kblocks = g.text_kblocks;
    a.f0_first = g.f0_first;
    a.f0_last = g.f0_last;
    const int vpl = (g.Ck + 31) / 32;
    if (vpl <= 4) return launch_mask_t<4>(a, tp, st);
    if (vpl <= 8) return launch_mask_t<8>(a, tp, st);
    if (vpl <= 16) return launch_mask_t<16>(a, tp, st);
    if (vpl <= 32) return launch_mask_t<32>(a, tp, st);
    return launch_mask_t<64>(a, tp, st);
}

cudaError_t launch_entropy_reduce(const Geometry &g, const float *row_entropy, float *entropy,
                                  float *entropy_norm, cudaStream_t st) {
    const long long BH = static_cast<long long>(g.B) * g.H;
    const unsigned grid = static_cast<unsigned>((BH + 7) / 8);
    entropy_reduce_kernel<<<grid, 256, 0, st>>>(row_entropy, entropy, entropy_norm, BH, g.Cq,
                                                g.Ck > 1 ? 1.0f / logf(static_cast<float>(g.Ck)) : 0.f);
    return cudaGetLastError();
}

}  // namespace bsa
