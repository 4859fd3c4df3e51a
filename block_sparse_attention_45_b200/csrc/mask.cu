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
// Top-p without sorting: P' >= 0, so fp32 bit patterns order like the values.
// Stage A bisects on the exponent field, with fp64 sums, for the binade that
// holds the cut (the largest e with mass(exponent >= e) >= p); Stage B gathers
// that binade's entries into shared memory and keeps entry m iff it is the
// first of the (P' desc, j asc) order or the fp64 mass strictly before it is
// below p -- the shortest prefix of the sorted row whose running sum reaches p
// (at least one entry, also for p <= 0).  Rows whose binade holds more than
// kCandMax entries fall back to an fp64 bisection on the full bit pattern
// inside that binade.  Row entropies go to a workspace; a second kernel sums them
// per head in a fixed order.
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

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ uint64_t warp_min_u64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t w = __shfl_xor_sync(0xffffffffu, v, o);
        v = w < v ? w : v;
    }
    return v;
}

// Candidates of the cut binade kept in shared memory per warp.
constexpr int kCandMax = 128;

// Row (b,h,i) keeps every entry whose key (P' bits, -j) is at least (ucut, -jcut):
// u > ucut, or u == ucut and j <= jcut -- the shortest prefix of the (P' desc,
// j asc) order whose running sum reaches p.
template <int VPL>
__device__ __forceinline__ void find_cut(const float (&v)[VPL], int Ck,
                                         float p, uint32_t umax, int lane, float *cv, int *cj,
                                         uint32_t &ucut, int &jcut) {
    // Stage A: the binade (fp32 exponent field) that holds the cut: the largest e
    // with mass(exponent >= e) >= p, by bisection on e with fp64 sums (fp32 sums
    // cannot tell 1 - 2^-30 from 1 when p is close to the row total).
#define U(s) __float_as_uint(v[s])
    const double pd = static_cast<double>(p);
    uint32_t lo = 0, hi = umax >> 23;
    while (lo < hi) {
        const uint32_t mid = lo + ((hi - lo + 1) >> 1);
        const uint32_t thr = mid << 23;
        double f = 0.0;
#pragma unroll
        for (int s = 0; s < VPL; ++s) f += (U(s) >= thr) ? static_cast<double>(v[s]) : 0.0;
        if (warp_sum_d(f) >= pd) lo = mid;
        else hi = mid - 1;
    }
    const uint32_t e = lo;
    double above = 0.0;
    {
        double a_l = 0.0;
#pragma unroll
        for (int s = 0; s < VPL; ++s) a_l += ((U(s) >> 23) > e) ? static_cast<double>(v[s]) : 0.0;
        above = warp_sum_d(a_l);
    }
    // Stage B: the binade's entries, compacted in ascending j.
    const uint32_t lt_mask = (1u << lane) - 1u;
    int c = 0;
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int j = lane + 32 * s;
        const bool is_c = j < Ck && (U(s) >> 23) == e;
        const uint32_t bal = __ballot_sync(0xffffffffu, is_c);
        const int pos = c + __popc(bal & lt_mask);
        if (is_c && pos < kCandMax) {
            cv[pos] = v[s];
            cj[pos] = j;
        }
        c += __popc(bal);
    }
    __syncwarp();
    if (c <= kCandMax) {
        // Candidate m is kept iff the fp64 mass strictly before it in
        // (P' desc, j asc) order is below p; the cut is the last kept one.
        // The first entry of the order is always kept (k* >= 1, also for p <= 0).
        uint64_t best = ~0ull;
        for (int m = lane; m < c; m += 32) {
            const float vm = cv[m];
            const int jm = cj[m];
            double before = above;
            bool first = above == 0.0;
            for (int n = 0; n < c; ++n) {
                const float vn = cv[n];
                if (vn > vm || (vn == vm && cj[n] < jm)) {
                    before += static_cast<double>(vn);
                    first = false;
                }
            }
            if (before < pd || first) {
                const uint64_t key = (static_cast<uint64_t>(__float_as_uint(vm)) << 32) |
                                     (0xFFFFFFFFu - static_cast<uint32_t>(jm));
                best = key < best ? key : best;
            }
        }
        best = warp_min_u64(best);
        ucut = static_cast<uint32_t>(best >> 32);
        jcut = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(best));
        return;
    }
    // A binade with more than kCandMax entries (nearly flat rows): bisection on
    // the full bit pattern, then ties at the cut value in ascending j.
    uint32_t lo2 = e << 23, hi2 = min(umax, (e << 23) | 0x7FFFFFu);
    while (lo2 < hi2) {
        const uint32_t mid = lo2 + ((hi2 - lo2 + 1) >> 1);
        double f = 0.0;
#pragma unroll
        for (int s = 0; s < VPL; ++s) f += (U(s) >= mid) ? static_cast<double>(v[s]) : 0.0;
        if (warp_sum_d(f) >= pd) lo2 = mid;
        else hi2 = mid - 1;
    }
    ucut = lo2;
    double abv = 0.0;
    int ties = 0;
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        abv += (U(s) > ucut) ? static_cast<double>(v[s]) : 0.0;
        ties += (U(s) == ucut && lane + 32 * s < Ck) ? 1 : 0;
    }
    abv = warp_sum_d(abv);
    ties = warp_sum_i(ties);
    const double vcut = static_cast<double>(__uint_as_float(ucut));
    int need = 1;
    double run = abv + vcut;
    while (run < pd && need < ties) {
        run += vcut;
        ++need;
    }
    // jcut = index of the need-th tie in ascending j
    int seen = 0;
    jcut = -1;
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int j = lane + 32 * s;
        const bool is_t = j < Ck && U(s) == ucut;
        const uint32_t bal = __ballot_sync(0xffffffffu, is_t);
        const int cnt = __popc(bal);
        if (jcut < 0 && seen + cnt >= need) {
            // the (need - seen)-th set bit of bal
            uint32_t b = bal;
            for (int k = 1; k < need - seen; ++k) b &= b - 1;
            jcut = 32 * s + __ffs(b) - 1;
        }
        seen += cnt;
    }
#undef U
}

template <int VPL>
__global__ void __launch_bounds__(256) mask_kernel(MaskArgs a, TopP tp) {
    __shared__ float s_cv[8][kCandMax];
    __shared__ int s_cj[8][kCandMax];
    const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
    const long long row = static_cast<long long>(blockIdx.x) * 8 + wid;
    if (row >= a.rows) return;  // whole warp leaves together
    const int Ck = a.Ck;
    const int i = static_cast<int>(row % a.Cq);
    const int h = static_cast<int>((row / a.Cq) % a.H);
    const float p = tp.p[h];
    const float *src = a.probs + row * Ck;

    float v[VPL];
    float ent = 0.f;
    double total = 0.0;
    uint32_t umax = 0;
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int j = lane + 32 * s;
        float x = (j < Ck) ? __ldg(src + j) : 0.f;
        x = fmaxf(x, 0.f);
        v[s] = x;
        umax = max(umax, __float_as_uint(x));
        total += static_cast<double>(x);
        if (j < Ck) ent -= x * __logf(x + a.eps);
    }
    total = warp_sum_d(total);
    if (a.row_entropy) {
        ent = warp_sum(ent);
        if (lane == 0) a.row_entropy[row] = ent;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) umax = max(umax, __shfl_xor_sync(0xffffffffu, umax, o));

    // fp64 totals, like the running sum of the rule: the row never reaches p -> keep it all
    const bool keep_all = !(total >= static_cast<double>(p));
    uint32_t ucut = 0;
    int jcut = 0x7FFFFFFF;
    if (!keep_all) find_cut<VPL>(v, Ck, p, umax, lane, s_cv[wid], s_cj[wid], ucut, jcut);

    const bool dense_row = (a.flags & BSA_FRAME0_DENSE) && i >= a.f0_first && i <= a.f0_last;
    const bool text = (a.flags & BSA_TEXT_KEEP) != 0;
    uint8_t *mrow = a.mask ? a.mask + row * Ck : nullptr;
    int32_t *irow = a.kv_index + row * Ck;
    const uint32_t lt_mask = (1u << lane) - 1u;
    int base = 0;
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int j = lane + 32 * s;
        const bool valid = j < Ck;
        const uint32_t us = __float_as_uint(v[s]);
        bool sel = keep_all || us > ucut || (us == ucut && j <= jcut);
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
