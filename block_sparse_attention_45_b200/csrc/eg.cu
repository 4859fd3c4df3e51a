// eg.cu -- pooled top-p over a competition domain, up to the final pass.
//
// "Competition Domains Matter: Selective Head Globalization for Training-Free
// Sparse Attention in Video Diffusion Transformers", s3.3 domain 3 ("grouped
// cross-head": heads split by the median of their entropy H_h; low-entropy
// heads compete in one shared pool, the others keep per-row local top-p), the
// one-key-per-row safeguard, and s4 (the pool ranks pairs by the value-aware
// score P'_{h,i,j} * ||c^V_{h,j}||); s3's other domains route the heads of a
// batch entry into other pools: one per head, one per entropy half, one for
// all heads (BSA_DOMAIN_*), G pools per batch entry.
//
// Pool (b, g) holds every pair (h, i, j) of its heads, ordered by (score desc,
// h, i, j asc), and keeps the shortest prefix whose running sum reaches pool_p
// times the pool total.  The cut is found
// without sorting by an exact radix select over the fp32 bit patterns of the
// scores (scores >= 0 order like their bit patterns): a histogram of the
// exponent field, then of mantissa bits 22..11, then 10..0, each bin holding
// the count and the exact integer sum of its scores' significands (within one
// binade a score is an integer times one power of two).  The pair that reaches
// the target then lies in one bit pattern u*: every pair above u* is kept, and
// of the pairs equal to u* the first `need` in (h, i, j) order.
//
// Launches (all on the caller's stream; the last CTA of each launch to finish
// does that launch's serial step, so no launch waits on another's CTAs):
//   entropy_level1_kernel  -sum_j P' ln(P' + eps) per row and a per-head
//                          histogram of the scores' exponent fields; its last
//                          CTA takes the per-head means, routes the heads to
//                          the domain's pools and lists each pool's heads
//   pool_level_kernel x2   mantissa bits 22..11, then 10..0, over the pooled
//                          heads only, c2 CTAs per pool; each CTA of the first
//                          takes its pool's level-1 pick (the same in all of
//                          them), and the last CTA of each pool picks that
//                          pool's bin
//   tie_kernel             pairs equal to the cut pattern per pooled row; the
//                          last CTA of each pool finds the row and rank of the
//                          last kept tie
#include <cuda_runtime.h>
#include <limits.h>
#include <math.h>
#include <stdint.h>

#include "bits.cuh"
#include "internal.h"

namespace bsa {

namespace {

constexpr int kThreads = 256;                 // every launch of this file
constexpr int kWarps = kThreads / 32;
constexpr int kL1Bins = 256;                  // exponent field
constexpr int kL1Copies = 4;                  // level-1 histograms per warp
constexpr int kL1Stride = 2 * kL1Bins + 1;    // words between copies (lo, hi; bank offset 1)
constexpr size_t kL1Smem = static_cast<size_t>(kThreads / 32) * kL1Copies * kL1Stride * sizeof(uint32_t);
constexpr int kMaxBins = 4096;                // widest later level
constexpr int kLevelBits[2] = {12, 11};       // mantissa 22..11, 10..0
constexpr uint32_t kBinCap = (1u << 20) - 1;  // pairs one 32-bit shared bin may take (12-bit halves)

__device__ __forceinline__ uint32_t pos_bits(float y) { return __float_as_uint(y > 0.f ? y : 0.f); }

// Score of a pooled pair as a bit pattern: P' (negatives and NaN as +0) times
// ||c^V|| (vn), rounded to fp32; P' alone without value norms.
__device__ __forceinline__ uint32_t score_bits(float p, bool value_aware, float vn) {
    const float x = p > 0.f ? p : 0.f;
    return pos_bits(value_aware ? __fmul_rn(x, vn) : x);
}

// The value norms of head bh, lane + 32 s in slot s (0 past C_k).
template <int VPL>
__device__ __forceinline__ void load_vnorm(const float *vnorm, long long bh, int Ck, int lane, float (&vn)[VPL]) {
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int j = lane + 32 * s;
        vn[s] = (vnorm && j < Ck) ? __ldg(vnorm + bh * Ck + j) : 0.f;
    }
}

// A shared-memory bin: count, and the significand split into 12-bit halves so
// that 32-bit atomics stay exact for up to kBinCap pairs.
__device__ __forceinline__ void bin_add(uint32_t *c, uint32_t *lo, uint32_t *hi, uint32_t bin,
                                        uint32_t u) {
    const uint32_t s = significand(u);
    atomicAdd(c + bin, 1u);
    atomicAdd(lo + bin, s & 0xFFFu);
    atomicAdd(hi + bin, s >> 12);
}

// Unsigned key ordering floats like <, with -0 == +0 and NaN above everything.
__device__ __forceinline__ uint32_t order_key(float f) {
    if (f != f) return 0xFFFFFFFFu;
    const uint32_t u = __float_as_uint(f + 0.0f);  // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The same without the count, for levels whose pick only needs to know which
// bins are empty: a bin of scores >= 2^-149 is non-empty iff its sum is
// positive; zero scores are flagged separately.
__device__ __forceinline__ void bin_add_sum(uint32_t *lo, uint32_t *hi, uint32_t bin, uint32_t u) {
    const uint32_t s = significand(u);
    atomicAdd(lo + bin, s & 0xFFFu);
    atomicAdd(hi + bin, s >> 12);
}

// Called by every thread after its last global write: true in the one CTA of
// the `total` that share `counter` to finish last, which then sees the others' writes.
__device__ bool last_cta(unsigned int *counter, unsigned int total) {
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(counter, 1u) == total - 1 ? 1 : 0;
    __syncthreads();
    const bool last = s_last != 0;
    if (last) __threadfence();
    return last;
}

struct ScanScratch {
    double m[kThreads];
    unsigned long long c[kThreads];
    double wm[kWarps];
    unsigned long long wc[kWarps];
    int owner, last_ne;
};

// Inclusive scan of (m, c) over the threads of the CTA in thread order; every
// thread's result also lands in sc.m / sc.c.
__device__ void cta_scan(double &m, unsigned long long &c, ScanScratch &sc) {
    const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double mo = __shfl_up_sync(0xffffffffu, m, o);
        const unsigned long long co = __shfl_up_sync(0xffffffffu, c, o);
        if (lane >= o) {
            m += mo;
            c += co;
        }
    }
    if (lane == 31) {
        sc.wm[wid] = m;
        sc.wc[wid] = c;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kWarps; ++w) {
            sc.wm[w] += sc.wm[w - 1];
            sc.wc[w] += sc.wc[w - 1];
        }
    }
    __syncthreads();
    if (wid > 0) {
        m += sc.wm[wid - 1];
        c += sc.wc[wid - 1];
    }
    sc.m[threadIdx.x] = m;
    sc.c[threadIdx.x] = c;
    __syncthreads();
}

// One radix level of one pool, by the whole CTA, on its histogram in
// shared memory (sum[k] = significand sum of bin k; cnt[k] = its count at the
// last level, before it only zero or not as the bin is empty or not).  The
// level's bin holding the cut: scanning bins from the largest value down, the
// first non-empty bin whose inclusive mass (plus the mass above the range)
// reaches the target; if rounding leaves the range short of it, its last
// non-empty bin.  Level 1 also fixes the target pool_p * total, and keep_all
// when the pool never reaches it.  The last level fixes the cut pattern and
// how many pairs equal to it are kept.  Thread t owns a run of bins from the
// top; the thread whose run holds the cut walks it.
__device__ void cta_pick(const uint32_t *cnt, const unsigned long long *sum, int nbits,
                         bool first_level, float pool_p, PoolState &st, ScanScratch &sc) {
    const int t = threadIdx.x;
    const int nb = 1 << nbits;
    const int per = nb / kThreads;
    const int lo = st.shift - nbits;
    const uint32_t range_e = first_level ? 0u : (st.pre << st.shift) >> 23;  // later levels: one binade
    auto unit_of = [&](int k) -> double {
        return unit_of_binade(first_level ? static_cast<uint32_t>(k) : range_e);
    };
    const int top = nb - 1 - t * per;
    double m_run = 0.0;
    unsigned long long c_run = 0;
    for (int s = 0; s < per; ++s) {
        const int k = top - s;
        if (cnt[k]) {
            m_run += static_cast<double>(sum[k]) * unit_of(k);
            c_run += cnt[k];
        }
    }
    double m_in = m_run;
    unsigned long long c_in = c_run;
    if (t == 0) {
        sc.owner = INT_MAX;
        sc.last_ne = -1;
    }
    cta_scan(m_in, c_in, sc);
    const double m_before = t ? sc.m[t - 1] : 0.0;
    double target = st.target;
    if (first_level) {
        const double total = sc.m[kThreads - 1];
        target = static_cast<double>(pool_p) * total;
        if (!(total >= target)) {  // every thread takes this branch
            __syncthreads();
            if (t == 0) st.keep_all = 1;
            __syncthreads();
            return;
        }
    }
    const bool reaches = c_run > 0 && st.above + m_before + m_run >= target;
    if (reaches) atomicMin(&sc.owner, t);
    if (c_run > 0) atomicMax(&sc.last_ne, t);
    __syncthreads();
    const bool hit = sc.owner != INT_MAX;
    const int owner = hit ? sc.owner : max(sc.last_ne, 0);
    if (t == owner) {
        double m = st.above + m_before;
        int pick = -1, last_ne = -1;
        for (int s = 0; s < per; ++s) {
            const int k = top - s;
            if (!cnt[k]) continue;
            const double mk = static_cast<double>(sum[k]) * unit_of(k);
            if (hit && m + mk >= target) {
                pick = k;
                break;
            }
            last_ne = k;
            m += mk;
        }
        if (pick < 0 && last_ne >= 0) {  // the range ends short of the target: its last bin
            pick = last_ne;
            m -= static_cast<double>(sum[pick]) * unit_of(pick);
        }
        if (first_level) st.target = target;
        if (pick < 0) {
            st.keep_all = 1;  // an empty range (not reachable from a non-empty pool)
        } else {
            st.above = m;
            st.pre = (st.pre << nbits) | static_cast<uint32_t>(pick);
            st.shift = lo;
            if (lo == 0) {
                // the cut bit pattern; keep its first `need` pairs in (h, i, j) order
                st.ucut = st.pre;
                const double v = static_cast<double>(__uint_as_float(st.ucut));
                const unsigned long long ties = cnt[pick];
                unsigned long long need = 1;
                if (v > 0.0 && st.above < target) {
                    const double n = ceil((target - st.above) / v);
                    need = n < 1.0 ? 1ull : static_cast<unsigned long long>(n);
                    // the closed form against the running sum of the rule
                    while (need > 1 && st.above + static_cast<double>(need - 1) * v >= target) --need;
                    while (need < ties && st.above + static_cast<double>(need) * v < target) ++need;
                }
                st.need = need < ties ? need : ties;
                // every tie kept: no row search needed
                st.cut_row = st.need == ties ? LLONG_MAX : -1;
                st.cut_rank = 0;
            }
        }
    }
    __syncthreads();
}

struct EgArgs {
    const float *probs;     // [B,H,C_q,C_k]
    const float *vnorm;     // [B,H,C_k] or nullptr
    double *ent_part;       // [B,H,ctas]: row-entropy sums of one CTA of level 1
    float *heads_h;         // [B,H]
    float *entropy;         // [B,H] or nullptr (caller's)
    float *entropy_norm;    // [B,H] or nullptr (caller's)
    int8_t *pool_of;        // [B,H]: the head's pool, -1 = per-row
    uint8_t *low_out;       // [B,H] or nullptr (caller's): 1 for pooled heads
    int8_t *pool_out;       // [B,H] or nullptr (caller's): copy of pool_of
    int *pool_heads;        // [B,G,H]: the heads of pool (b, g) in ascending order
    int *pool_nh;           // [B,G]: their number
    int G, domain;          // pools per batch entry, competition domain
    unsigned long long *hist1;  // [B,H,256,2]
    unsigned long long *hist;   // [B,G,4096,2]
    int *tiecnt;            // [B,H,C_q]
    PoolState *state;       // [B,G]
    unsigned int *counter;  // this launch's finish counter
    int B, H, Cq, Ck;
    int ctas;               // CTAs per head (level 1) or per pool (later passes)
    float eps, inv_log_ck, pool_p;
};

__device__ __forceinline__ bool pool_active(const PoolState &st) { return !st.empty && !st.keep_all; }

// Rows [r0, r1) of n rows split into contiguous runs, one per warp of the grid slice.
__device__ __forceinline__ void warp_rows(long long n, long long warp, long long warps, long long &r0,
                                          long long &r1) {
    const long long per = (n + warps - 1) / warps;
    r0 = min(n, warp * per);
    r1 = min(n, r0 + per);
}

// Row entropies of every head and the level-1 histogram (exponent field of the
// score) per head.  CTA blockIdx.x % ctas of head blockIdx.x / ctas takes a
// contiguous run of rows, each warp a run of that; a warp holds a whole row in
// registers (VPL values per lane) and bins into its own shared histogram.
template <int VPL>
__global__ void __launch_bounds__(kThreads) entropy_level1_kernel(EgArgs a) {
    // per warp kL1Copies histograms (count, lo, hi), lane l bins into copy l % kL1Copies;
    // copies kL1Stride words apart so that one bin's copies sit in different banks
    extern __shared__ __align__(16) uint32_t sh[];
    __shared__ double s_wsum[kWarps];
    __shared__ float s_h[kMaxHeads];
    __shared__ int s_pool[kMaxHeads];
    const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
    __shared__ int s_zero;
    {
        uint32_t *wbase = sh + wid * kL1Copies * kL1Stride;
        for (int k = lane; k < kL1Copies * kL1Stride; k += 32) wbase[k] = 0u;
        if (threadIdx.x == 0) s_zero = 0;
        __syncthreads();
        uint32_t *wl = wbase + (lane % kL1Copies) * kL1Stride, *wh = wl + kL1Bins;
        bool zero = false;
        const long long bh = blockIdx.x / a.ctas;
        const int part = blockIdx.x % a.ctas;
        const int Ck = a.Ck;
        const bool va = a.vnorm != nullptr;
        float vn[VPL];
        load_vnorm<VPL>(a.vnorm, bh, Ck, lane, vn);
        long long i0, i1;
        warp_rows(a.Cq, static_cast<long long>(part) * kWarps + wid, static_cast<long long>(a.ctas) * kWarps,
                  i0, i1);
        double wsum = 0.0;  // lane 0: this warp's rows, in row order
        for (long long i = i0; i < i1; ++i) {
            const float *prow = a.probs + (bh * a.Cq + i) * Ck;
            float y[VPL];
#pragma unroll
            for (int s = 0; s < VPL; ++s) {
                const int j = lane + 32 * s;
                y[s] = j < Ck ? __ldg(prow + j) : 0.f;
            }
            float ent = 0.f;
#pragma unroll
            for (int s = 0; s < VPL; ++s) {
                const int j = lane + 32 * s;
                if (j < Ck) {
                    const float x = y[s] > 0.f ? y[s] : 0.f;
                    ent = fmaf(x, lg2_approx(x + a.eps), ent);
                    const uint32_t u = score_bits(x, va, vn[s]);
                    bin_add_sum(wl, wh, u >> 23, u);
                    zero |= u == 0u;
                }
            }
            ent = warp_sum(ent);
            wsum += static_cast<double>(-ent * 0.6931471805599453f);  // ln 2
        }
        if (lane == 0) s_wsum[wid] = wsum;
        if (__any_sync(0xffffffffu, zero) && lane == 0) atomicOr(&s_zero, 1);
        __syncthreads();
        const int t = threadIdx.x;  // bin t
        unsigned long long s = 0;
        for (int w = 0; w < kWarps * kL1Copies; ++w) {
            const uint32_t *h = sh + w * kL1Stride;
            s += h[t] + (static_cast<unsigned long long>(h[kL1Bins + t]) << 12);
        }
        if (s || (t == 0 && s_zero)) {  // the count slot only marks non-empty bins
            atomicAdd(&a.hist1[(bh * kL1Bins + t) * 2], 1ull);
            atomicAdd(&a.hist1[(bh * kL1Bins + t) * 2 + 1], s);
        }
        if (t == 0) {
            double cs = 0.0;
            for (int w = 0; w < kWarps; ++w) cs += s_wsum[w];
            a.ent_part[bh * a.ctas + part] = cs;
        }
    }
    if (!last_cta(a.counter, gridDim.x)) return;

    // ---- the last CTA: per-head means, the domain's pools and their heads
    const long long BH = static_cast<long long>(a.B) * a.H;
    for (long long bh = wid; bh < BH; bh += kWarps) {
        double s = 0.0;  // fixed order: part-strided per lane, then a butterfly; lane 0's sum
        for (int q = lane; q < a.ctas; q += 32) s += __ldcg(a.ent_part + bh * a.ctas + q);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) {
            const float Hh = static_cast<float>(s / a.Cq);
            a.heads_h[bh] = Hh;
            if (a.entropy) a.entropy[bh] = Hh;
            if (a.entropy_norm) a.entropy_norm[bh] = Hh * a.inv_log_ck;
        }
    }
    __syncthreads();
    const int H = a.H, G = a.G;
    for (int b = 0; b < a.B; ++b) {
        for (int h = threadIdx.x; h < H; h += kThreads) s_h[h] = a.heads_h[static_cast<long long>(b) * H + h];
        __syncthreads();
        // The domain's pool of every head.  The grouped and entropy-guided domains split at
        // the median: heads ordered by (H_h asc, h asc), the first floor(H/2) are the
        // low-entropy ones; the ranks form a permutation even for NaN entropies.
        for (int h = threadIdx.x; h < H; h += kThreads) {
            const uint32_t x = order_key(s_h[h]);
            int rank = 0;
            for (int o = 0; o < H; ++o) {
                const uint32_t y = order_key(s_h[o]);
                rank += (y < x || (y == x && o < h)) ? 1 : 0;
            }
            const bool lowh = rank < H / 2;
            int pool;
            switch (a.domain) {
                case BSA_DOMAIN_HEAD: pool = h; break;
                case BSA_DOMAIN_GROUPED: pool = lowh ? 0 : 1; break;
                case BSA_DOMAIN_ALL: pool = 0; break;
                case BSA_DOMAIN_EG: pool = lowh ? 0 : -1; break;
                default: pool = -1; break;
            }
            const long long bh = static_cast<long long>(b) * H + h;
            s_pool[h] = pool;
            a.pool_of[bh] = static_cast<int8_t>(pool);
            if (a.low_out) a.low_out[bh] = pool >= 0 ? 1 : 0;
            if (a.pool_out) a.pool_out[bh] = static_cast<int8_t>(pool);
        }
        __syncthreads();
        // each pool's heads in ascending order, one thread per pool
        for (int g = threadIdx.x; g < G; g += kThreads) {
            const long long bp = static_cast<long long>(b) * G + g;
            int k = 0;
            for (int h = 0; h < H; ++h)
                if (s_pool[h] == g) a.pool_heads[bp * H + k++] = h;
            a.pool_nh[bp] = k;
        }
        __syncthreads();
    }
}

// The level-1 pick of a pool of batch entry b (its np heads in `heads`) into
// `st`, by the whole CTA: the pool's exponent histogram is the sum of its
// heads' histograms.  Every CTA
// of the pool takes it from the same complete histograms, so all agree.
__device__ __noinline__ void level1_pick(const EgArgs &a, int b, int np, const int *heads, uint32_t *cnt,
                            unsigned long long *sum, PoolState &st, ScanScratch &sc) {
    if (threadIdx.x == 0) {
        PoolState z;
        z.target = 0.0;
        z.above = 0.0;
        z.pad2 = 0;
        z.pre = 0;
        z.shift = 31;  // level 1 bins bits 30..23 of scores >= 0 (bit 31 is 0)
        z.keep_all = 0;
        z.empty = np == 0;
        z.ucut = 0;
        z.pad0 = 0;
        z.need = 0;
        z.cut_row = -1;
        z.cut_rank = 0;
        z.pad1 = 0;
        st = z;
    }
    __syncthreads();
    if (np == 0) return;
    const int t = threadIdx.x;  // bin t over the pool's heads, loads 8 heads at a time
    unsigned long long c = 0, s = 0;
    for (int k0 = 0; k0 < np; k0 += 8) {
        unsigned long long cc[8], ss[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            cc[q] = ss[q] = 0ull;
            if (k0 + q < np) {
                const unsigned long long *gp =
                    a.hist1 + ((static_cast<long long>(b) * a.H + heads[k0 + q]) * kL1Bins + t) * 2;
                cc[q] = __ldcg(gp);
                ss[q] = __ldcg(gp + 1);
            }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            c += cc[q];
            s += ss[q];
        }
    }
    cnt[t] = static_cast<uint32_t>(c);
    sum[t] = s;
    __syncthreads();
    cta_pick(cnt, sum, 8, true, a.pool_p, st, sc);
}

// Rows of a pool of batch entry b in (h, i) order: row r is row r % C_q of the
// (r / C_q)-th head of the pool.
__device__ __forceinline__ long long pooled_row(const EgArgs &a, const int *heads, int b, long long r) {
    const long long kk = r / a.Cq;
    return (static_cast<long long>(b) * a.H + heads[kk]) * a.Cq + (r - kk * a.Cq);
}

// One later radix level over the rows of pool blockIdx.x / ctas:
// every score in the current range (bits above `shift` equal to `pre`) adds
// (1, significand) to bin (u >> (shift - NBITS)) & (2^NBITS - 1).  The first
// of them (no counts) starts from the level-1 pick, which each of its CTAs
// takes itself; the second from the state the first one's last CTA wrote.
template <int VPL, int NBITS, bool COUNTS>
__global__ void __launch_bounds__(kThreads) pool_level_kernel(EgArgs a) {
    constexpr int nb = 1 << NBITS;
    constexpr int per = nb / kThreads;
    constexpr bool kFirst = !COUNTS;
    __shared__ int s_zero;
    extern __shared__ __align__(16) uint32_t sh[];  // [3 * nb]: count, lo, hi; then count + u64 sum
    __shared__ ScanScratch sc;
    __shared__ PoolState s_st;
    __shared__ int s_heads[kMaxHeads];
    const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
    const int bp = blockIdx.x / a.ctas, part = blockIdx.x % a.ctas;
    const int b = bp / a.G;
    const int np = a.pool_nh[bp];
    for (int k = threadIdx.x; k < np; k += kThreads) s_heads[k] = a.pool_heads[static_cast<long long>(bp) * a.H + k];
    if (kFirst) {
        __syncthreads();
        level1_pick(a, b, np, s_heads, sh, reinterpret_cast<unsigned long long *>(sh + 2 * kL1Bins), s_st, sc);
    } else {
        if (threadIdx.x == 0) s_st = a.state[bp];
        __syncthreads();
    }
    {
        const PoolState st = s_st;
        if (pool_active(st) && st.shift >= NBITS) {
            uint32_t *c = sh, *lo = sh + nb, *hi = sh + 2 * nb;
            for (int k = threadIdx.x; k < 3 * nb; k += kThreads) sh[k] = 0u;
            if (threadIdx.x == 0) s_zero = 0;
            bool zero = false;
            __syncthreads();
            const int shift = st.shift, low_bits = st.shift - NBITS;
            const uint32_t pre = st.pre;
            const int Ck = a.Ck;
            long long r0, r1;
            warp_rows(static_cast<long long>(np) * a.Cq, static_cast<long long>(part) * kWarps + wid,
                      static_cast<long long>(a.ctas) * kWarps, r0, r1);
            const bool va = a.vnorm != nullptr;
            float vn[VPL];
            long long cur_bh = -1;
            for (long long r = r0; r < r1; ++r) {
                const long long row = pooled_row(a, s_heads, b, r);
                const long long bh = row / a.Cq;
                if (va && bh != cur_bh) {
                    load_vnorm<VPL>(a.vnorm, bh, Ck, lane, vn);
                    cur_bh = bh;
                }
                const float *prow = a.probs + row * Ck;
                float y[VPL];
#pragma unroll
                for (int s = 0; s < VPL; ++s) {
                    const int j = lane + 32 * s;
                    y[s] = j < Ck ? __ldg(prow + j) : 0.f;
                }
#pragma unroll
                for (int s = 0; s < VPL; ++s) {
                    const int j = lane + 32 * s;
                    if (j < Ck) {
                        const uint32_t u = score_bits(y[s], va, vn[s]);
                        if ((u >> shift) == pre) {
                            if (COUNTS) {
                                bin_add(c, lo, hi, (u >> low_bits) & (nb - 1), u);
                            } else {
                                bin_add_sum(lo, hi, (u >> low_bits) & (nb - 1), u);
                                zero |= u == 0u;
                            }
                        }
                    }
                }
            }
            if (!COUNTS && __any_sync(0xffffffffu, zero) && lane == 0) atomicOr(&s_zero, 1);
            __syncthreads();
            unsigned long long *g = a.hist + static_cast<long long>(bp) * 2 * kMaxBins;
            for (int k = threadIdx.x; k < nb; k += kThreads) {
                const unsigned long long sk = lo[k] + (static_cast<unsigned long long>(hi[k]) << 12);
                const unsigned long long ck = COUNTS ? c[k] : ((sk || (k == 0 && s_zero)) ? 1ull : 0ull);
                if (ck) {
                    atomicAdd(&g[2 * k], ck);
                    atomicAdd(&g[2 * k + 1], sk);
                }
            }
        }
    }
    // ---- the last CTA of pool bp: its pick (s_st still holds the state this launch started from)
    if (!last_cta(a.counter + bp, static_cast<unsigned>(a.ctas))) return;
    uint32_t *cnt = sh;
    unsigned long long *sum = reinterpret_cast<unsigned long long *>(sh + nb);
    if (pool_active(s_st) && s_st.shift >= NBITS) {
        unsigned long long *g = a.hist + static_cast<long long>(bp) * 2 * kMaxBins;
        unsigned long long cc[per], ss[per];
#pragma unroll
        for (int q = 0; q < per; ++q) {
            const int k = threadIdx.x + q * kThreads;
            cc[q] = __ldcg(&g[2 * k]);
            ss[q] = __ldcg(&g[2 * k + 1]);
        }
#pragma unroll
        for (int q = 0; q < per; ++q) {
            const int k = threadIdx.x + q * kThreads;
            cnt[k] = static_cast<uint32_t>(cc[q]);
            sum[k] = ss[q];
            g[2 * k] = 0ull;  // ready for the next level
            g[2 * k + 1] = 0ull;
        }
        __syncthreads();
        cta_pick(cnt, sum, NBITS, false, a.pool_p, s_st, sc);
    }
    if (threadIdx.x == 0) a.state[bp] = s_st;
}

// Needed only when some but not all pairs equal to the cut pattern are kept:
// ties per pooled row, then (last CTA) the row, in (h, i) order, where their
// running count reaches `need` and how many of that row's ties are kept.
template <int VPL>
__global__ void __launch_bounds__(kThreads) tie_kernel(EgArgs a) {
    __shared__ ScanScratch sc;
    __shared__ int s_heads[kMaxHeads];
    const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
    {
        const int bp = blockIdx.x / a.ctas, part = blockIdx.x % a.ctas;
        const int b = bp / a.G;
        const PoolState st = a.state[bp];
        const int np = a.pool_nh[bp];
        const long long rows = static_cast<long long>(np) * a.Cq;
        if (pool_active(st) && st.cut_row == -1) {
            for (int k = threadIdx.x; k < np; k += kThreads)
                s_heads[k] = a.pool_heads[static_cast<long long>(bp) * a.H + k];
            __syncthreads();
            const int Ck = a.Ck;
            long long r0, r1;
            warp_rows(rows, static_cast<long long>(part) * kWarps + wid, static_cast<long long>(a.ctas) * kWarps,
                      r0, r1);
            const bool va = a.vnorm != nullptr;
            float vn[VPL];
            long long cur_bh = -1;
            for (long long r = r0; r < r1; ++r) {
                const long long row = pooled_row(a, s_heads, b, r);
                const long long bh = row / a.Cq;
                if (va && bh != cur_bh) {
                    load_vnorm<VPL>(a.vnorm, bh, Ck, lane, vn);
                    cur_bh = bh;
                }
                const float *prow = a.probs + row * Ck;
                float y[VPL];
#pragma unroll
                for (int s = 0; s < VPL; ++s) {
                    const int j = lane + 32 * s;
                    y[s] = j < Ck ? __ldg(prow + j) : 0.f;
                }
                int n = 0;
#pragma unroll
                for (int s = 0; s < VPL; ++s) {
                    const int j = lane + 32 * s;
                    n += __popc(__ballot_sync(0xffffffffu, j < Ck && score_bits(y[s], va, vn[s]) == st.ucut));
                }
                if (lane == 0) a.tiecnt[row] = n;
            }
        }
    }
    // ---- the last CTA of pool bp: a scan over its rows when it needs one
    const int bp = blockIdx.x / a.ctas;
    if (!last_cta(a.counter + bp, static_cast<unsigned>(a.ctas))) return;
    const int t = threadIdx.x;
    const int b = bp / a.G;
    const PoolState st = a.state[bp];
    if (!pool_active(st) || st.cut_row != -1) return;  // uniform over the CTA
    const int np = a.pool_nh[bp];
    const long long rows = static_cast<long long>(np) * a.Cq;
    for (int k = t; k < np; k += kThreads) s_heads[k] = a.pool_heads[static_cast<long long>(bp) * a.H + k];
    if (t == 0) sc.owner = INT_MAX;
    __syncthreads();
    const long long per = (rows + kThreads - 1) / kThreads;
    const long long r0 = min(rows, t * per), r1 = min(rows, r0 + per);
    unsigned long long n = 0;
    for (long long r = r0; r < r1; r += 8) {  // 8 loads in flight
        int v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = r + q < r1 ? __ldcg(a.tiecnt + pooled_row(a, s_heads, b, r + q)) : 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) n += static_cast<unsigned long long>(v[q]);
    }
    double dm = 0.0;
    unsigned long long run = n;
    cta_scan(dm, run, sc);  // inclusive tie counts in thread order
    if (n > 0 && run >= st.need) atomicMin(&sc.owner, t);
    __syncthreads();
    if (t == sc.owner) {
        unsigned long long acc = run - n;
        long long cut_row = -1;
        int cut_rank = 0;
        for (long long r = r0; r < r1 && cut_row < 0; r += 8) {
            int v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = r + q < r1 ? __ldcg(a.tiecnt + pooled_row(a, s_heads, b, r + q)) : 0;
            for (int q = 0; q < 8 && r + q < r1; ++q) {
                const unsigned long long c = static_cast<unsigned long long>(v[q]);
                if (acc + c >= st.need) {
                    cut_row = pooled_row(a, s_heads, b, r + q);
                    cut_rank = static_cast<int>(st.need - acc);
                    break;
                }
                acc += c;
            }
        }
        a.state[bp].cut_row = cut_row;
        a.state[bp].cut_rank = cut_rank;
    }
}

template <int VPL>
cudaError_t launch_eg_passes(const EgArgs &base, long long c1, long long c2, long long pools, long long BH,
                             cudaStream_t st) {
    unsigned int *counters = base.counter;
    EgArgs a = base;
    a.ctas = static_cast<int>(c1);
    a.counter = counters + 0;
    cudaError_t e = cudaFuncSetAttribute(entropy_level1_kernel<VPL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kL1Smem));
    if (e != cudaSuccess) return e;
    entropy_level1_kernel<VPL><<<static_cast<unsigned>(BH * c1), kThreads, kL1Smem, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (pools == 0) return cudaSuccess;  // every row per-row: no pool passes
    a.ctas = static_cast<int>(c2);
    const unsigned grid2 = static_cast<unsigned>(pools * c2);
    const size_t smem12 = 3 * (1 << kLevelBits[0]) * sizeof(uint32_t);
    const size_t smem11 = 3 * (1 << kLevelBits[1]) * sizeof(uint32_t);
    if ((e = cudaFuncSetAttribute(pool_level_kernel<VPL, kLevelBits[0], false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(smem12))) != cudaSuccess)
        return e;
    a.counter = counters + 1;  // then one counter per pool and pass
    pool_level_kernel<VPL, kLevelBits[0], false><<<grid2, kThreads, smem12, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    a.counter = counters + 1 + pools;
    pool_level_kernel<VPL, kLevelBits[1], true><<<grid2, kThreads, smem11, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    a.counter = counters + 1 + 2 * pools;
    tie_kernel<VPL><<<grid2, kThreads, 0, st>>>(a);
    return cudaGetLastError();
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Level-1 CTAs per head: at most one per kWarps rows.
long long eg_level1_ctas_max(int Cq) { return max(1ll, (static_cast<long long>(Cq) + kWarps - 1) / kWarps); }

static_assert(kL1Bins == kThreads, "the level-1 fold and pick take one bin per thread");
static_assert(kMaxBins % kThreads == 0 && (1 << kLevelBits[1]) % kThreads == 0, "bins per thread");

}  // namespace

int eg_pools(int H, int domain) {
    switch (domain) {
        case BSA_DOMAIN_HEAD: return H;
        case BSA_DOMAIN_GROUPED: return 2;
        case BSA_DOMAIN_ALL: return 1;
        case BSA_DOMAIN_EG: return 1;
        default: return 0;
    }
}

// Heads in the largest pool of the domain.
static int eg_max_pool_heads(int H, int domain) {
    switch (domain) {
        case BSA_DOMAIN_HEAD: return 1;
        case BSA_DOMAIN_GROUPED: return H - H / 2;
        case BSA_DOMAIN_ALL: return H;
        case BSA_DOMAIN_EG: return H / 2;
        default: return 0;
    }
}

EgWorkspace eg_workspace(const Geometry &g, int domain) {
    const size_t rows = static_cast<size_t>(g.B) * g.H * g.Cq;
    const size_t bh = static_cast<size_t>(g.B) * g.H;
    const size_t pools = static_cast<size_t>(g.B) * eg_pools(g.H, domain);
    EgWorkspace w;
    size_t off = 0;
    w.ent_part = off;
    off += round256(bh * static_cast<size_t>(eg_level1_ctas_max(g.Cq)) * sizeof(double));
    w.heads_h = off;
    off += round256(bh * sizeof(float));
    w.pool_of = off;
    off += round256(bh);
    w.pool_heads = off;
    off += round256(pools * g.H * sizeof(int));
    w.pool_nh = off;
    off += round256(pools * sizeof(int));
    w.state = off;
    off += round256(pools * sizeof(PoolState));
    // zeroed once per call: histograms, tie counts, finish counters
    w.zero_begin = off;
    w.hist1 = off;
    off += round256(bh * kL1Bins * 2 * sizeof(unsigned long long));
    w.hist = off;
    off += round256(pools * 2 * kMaxBins * sizeof(unsigned long long));
    w.tiecnt = off;
    off += round256(rows * sizeof(int));
    w.counters = off;
    off += round256((1 + 3 * pools) * sizeof(unsigned int));
    w.zero_bytes = off - w.zero_begin;
    w.bytes = off;
    return w;
}

cudaError_t launch_eg_prepare(const Geometry &g, int domain, const float *probs, const float *vnorm,
                              float pool_p, float eps, float *entropy, float *entropy_norm,
                              uint8_t *low_heads, int8_t *pool_out, uint8_t *workspace, cudaStream_t st) {
    const EgWorkspace w = eg_workspace(g, domain);
    cudaError_t e = cudaMemsetAsync(workspace + w.zero_begin, 0, w.zero_bytes, st);
    if (e != cudaSuccess) return e;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidValue;
    const int G = eg_pools(g.H, domain);

    EgArgs a;
    a.probs = probs;
    a.vnorm = vnorm;
    a.ent_part = reinterpret_cast<double *>(workspace + w.ent_part);
    a.heads_h = reinterpret_cast<float *>(workspace + w.heads_h);
    a.entropy = entropy;
    a.entropy_norm = entropy_norm;
    a.pool_of = reinterpret_cast<int8_t *>(workspace + w.pool_of);
    a.low_out = low_heads;
    a.pool_out = pool_out;
    a.pool_heads = reinterpret_cast<int *>(workspace + w.pool_heads);
    a.pool_nh = reinterpret_cast<int *>(workspace + w.pool_nh);
    a.G = G;
    a.domain = domain;
    a.hist1 = reinterpret_cast<unsigned long long *>(workspace + w.hist1);
    a.hist = reinterpret_cast<unsigned long long *>(workspace + w.hist);
    a.tiecnt = reinterpret_cast<int *>(workspace + w.tiecnt);
    a.state = reinterpret_cast<PoolState *>(workspace + w.state);
    a.counter = reinterpret_cast<unsigned int *>(workspace + w.counters);
    a.B = g.B;
    a.H = g.H;
    a.Cq = g.Cq;
    a.Ck = g.Ck;
    a.ctas = 0;
    a.eps = eps;
    a.inv_log_ck = g.Ck > 1 ? 1.0f / logf(static_cast<float>(g.Ck)) : 0.f;
    a.pool_p = pool_p;

    // level 1 with the row entropies: about two CTAs per SM, at least one row per
    // warp, and few enough rows per warp that its 32-bit bins stay exact
    const long long BH = static_cast<long long>(g.B) * g.H;
    const long long rows_cap = static_cast<long long>(kBinCap / static_cast<uint32_t>(g.Ck)) * kWarps;
    const long long c1 = max((static_cast<long long>(g.Cq) + rows_cap - 1) / rows_cap,
                             min((2ll * sms + BH - 1) / BH, eg_level1_ctas_max(g.Cq)));
    // later passes, c2 CTAs per pool: about two CTAs per SM in all, and at most
    // kBinCap pairs per CTA (its warps share one histogram)
    const long long pools = static_cast<long long>(g.B) * G;
    const long long prow = static_cast<long long>(eg_max_pool_heads(g.H, domain)) * g.Cq;
    const long long prow_cap =
        static_cast<long long>(kBinCap / (static_cast<uint32_t>(g.Ck) * kWarps)) * kWarps;
    const long long c2 =
        pools == 0 ? 0
                   : max(max(1ll, (prow + prow_cap - 1) / prow_cap),
                         min((2ll * sms + pools - 1) / pools, max(1ll, (prow + kWarps - 1) / kWarps)));
    if (BH * c1 > 0x7FFFFFFFll || pools * c2 > 0x7FFFFFFFll) return cudaErrorInvalidValue;
    const int vpl = (g.Ck + 31) / 32;
    if (vpl <= 4) return launch_eg_passes<4>(a, c1, c2, pools, BH, st);
    if (vpl <= 8) return launch_eg_passes<8>(a, c1, c2, pools, BH, st);
    if (vpl <= 16) return launch_eg_passes<16>(a, c1, c2, pools, BH, st);
    if (vpl <= 32) return launch_eg_passes<32>(a, c1, c2, pools, BH, st);
    return launch_eg_passes<64>(a, c1, c2, pools, BH, st);
}

}  // namespace bsa
