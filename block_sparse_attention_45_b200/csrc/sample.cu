// sample.cu -- importance sampling of key blocks with inverse-inclusion-
// probability weights.
//
// "AB-Attention: accurate block-sparse attention for video diffusion", TL;DR
// fix (2): blocks are sampled in proportion to their importance and every
// sampled block is reweighted by the inverse of its inclusion probability, so
// that one sparse pass is an unbiased estimate of dense attention (numerator
// and normaliser alike).  The page gives no sampling law; this file takes the
// plain one:
//   - pair (b, h, i, j) is included independently of every other pair with
//     probability pi = min(1, fp32(K * P')), K the per-row budget (rows of P'
//     sum to one, so a row keeps at most K blocks in expectation); negative or
//     NaN P' counts as 0;
//   - the draw of pair idx = ((b*H + h)*C_q + i)*C_k + j is u = (z >> 40)*2^-24,
//     z the idx-th output of SplitMix64 started from `seed`; the pair is
//     included iff u < pi;
//   - an included pair carries w = 1/pi (fp32, correctly rounded); text
//     columns and frame-0 rows are included with pi = 1, w = 1.
// One warp per row of P', the row in registers (VPL values per lane); the
// kept blocks are compacted in ascending j by ballot, weights beside them.
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace bsa {

namespace {

constexpr int kWarpsPerCta = 4;

// The idx-th output (from 0) of SplitMix64 started from state `seed` (Steele,
// Lea and Flood, "Fast splittable pseudorandom number generators", OOPSLA
// 2014): state seed + (idx + 1) * golden-ratio increment, then two
// xor-shift-multiply rounds and a final xor-shift.
__device__ __forceinline__ uint64_t splitmix64_at(uint64_t seed, uint64_t idx) {
    uint64_t z = seed + (idx + 1ull) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

struct SampleArgs {
    const float *probs;   // [B,H,C_q,C_k]
    uint8_t *mask;        // [B,H,C_q,C_k] or nullptr
    int32_t *kv_index;    // [B,H,C_q,C_k]
    float *kv_weight;     // [B,H,C_q,C_k]
    int32_t *kv_count;    // [B,H,C_q]
    long long rows;
    int Cq, Ck;
    int text_k;           // forced key columns (0 without the flag)
    int f0_first, f0_last;  // forced query blocks (empty without the flag)
    float budget;
    uint64_t seed;
};

template <int VPL>
__global__ void __launch_bounds__(kWarpsPerCta * 32) sample_kernel(SampleArgs a) {
    const int lane = threadIdx.x % 32;
    const long long row = static_cast<long long>(blockIdx.x) * kWarpsPerCta + threadIdx.x / 32;
    if (row >= a.rows) return;  // whole warp leaves together
    const int Ck = a.Ck;
    const int i = static_cast<int>(row % a.Cq);
    const float *src = a.probs + row * Ck;
    float y[VPL];
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int j = lane + 32 * s;
        y[s] = j < Ck ? __ldg(src + j) : 0.f;
    }
    const bool dense_row = i >= a.f0_first && i <= a.f0_last;
    const uint64_t base_idx = static_cast<uint64_t>(row) * static_cast<uint64_t>(Ck);
    uint8_t *mrow = a.mask ? a.mask + row * Ck : nullptr;
    int32_t *irow = a.kv_index + row * Ck;
    float *wrow = a.kv_weight + row * Ck;
    const uint32_t lt_mask = (1u << lane) - 1u;
    int n = 0;
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int j = lane + 32 * s;
        bool keep = false;
        float w = 0.f;
        if (j < Ck) {
            float pi;
            if (dense_row || j < a.text_k) {
                pi = 1.f;
            } else {
                const float x = y[s] > 0.f ? y[s] : 0.f;
                const float prod = __fmul_rn(a.budget, x);
                pi = prod < 1.f ? prod : 1.f;
                if (!(pi >= 0.f)) pi = 0.f;
            }
            const uint64_t z = splitmix64_at(a.seed, base_idx + static_cast<uint64_t>(j));
            const float u = static_cast<float>(static_cast<uint32_t>(z >> 40)) * 5.9604644775390625e-8f;  // 2^-24
            keep = u < pi;
            if (keep) w = __fdiv_rn(1.f, pi);
            if (mrow) mrow[j] = keep ? 1 : 0;
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (keep) {
            const int pos = n + __popc(bal & lt_mask);
            irow[pos] = j;
            wrow[pos] = w;
        }
        n += __popc(bal);
    }
    if (lane == 0) a.kv_count[row] = n;
}

template <int VPL>
cudaError_t launch_sample_t(const SampleArgs &a, cudaStream_t st) {
    const unsigned grid = static_cast<unsigned>((a.rows + kWarpsPerCta - 1) / kWarpsPerCta);
    sample_kernel<VPL><<<grid, kWarpsPerCta * 32, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sample(const Geometry &g, const float *probs, float budget, uint64_t seed,
                          uint32_t flags, uint8_t *mask, int32_t *kv_index, float *kv_weight,
                          int32_t *kv_count, cudaStream_t st) {
    SampleArgs a;
    a.probs = probs;
    a.mask = mask;
    a.kv_index = kv_index;
    a.kv_weight = kv_weight;
    a.kv_count = kv_count;
    a.rows = static_cast<long long>(g.B) * g.H * g.Cq;
    a.Cq = g.Cq;
    a.Ck = g.Ck;
    a.text_k = (flags & BSA_TEXT_KEEP) ? g.text_kblocks : 0;
    a.f0_first = (flags & BSA_FRAME0_DENSE) ? g.f0_first : 1;
    a.f0_last = (flags & BSA_FRAME0_DENSE) ? g.f0_last : 0;
    a.budget = budget;
    a.seed = seed;
    if (a.rows == 0) return cudaSuccess;
    const int vpl = (g.Ck + 31) / 32;
    if (vpl <= 4) return launch_sample_t<4>(a, st);
    if (vpl <= 8) return launch_sample_t<8>(a, st);
    if (vpl <= 16) return launch_sample_t<16>(a, st);
    if (vpl <= 32) return launch_sample_t<32>(a, st);
    return launch_sample_t<64>(a, st);
}

}  // namespace bsa
