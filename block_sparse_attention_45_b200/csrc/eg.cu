// eg.cu -- entropy-guided grouped cross-head selection, up to the final pass.
//
// "Competition Domains Matter: Selective Head Globalization for Training-Free
// Sparse Attention in Video Diffusion Transformers", s3.3 domain 3 ("grouped
// cross-head": heads split by the median of their entropy H_h; low-entropy
// heads compete in one shared pool, the others keep per-row local top-p), the
// one-key-per-row safeguard, and s4 (the pool ranks pairs by the value-aware
// score P'_{h,i,j} * ||c^V_{h,j}||).
//
// Per batch entry b the pool holds every pair (h, i, j) of its low-entropy
// heads, ordered by (score desc, h, i, j asc), and keeps the shortest prefix
// whose running sum reaches pool_p times the pool total.  The cut is found
// without sorting by an exact radix select over the fp32 bit patterns of the
// scores (scores >= 0 order like their bit patterns): a histogram of the
// exponent field, then of mantissa bits 22..11, then 10..0, each bin holding
// the count and the exact integer sum of its scores' significands (within one
// binade a score is an integer times one power of two).  The pair that reaches
// the target then lies in one bit pattern u*: every pair above u* is kept, and
// of the pairs equal to u* the first `need` in (h, i, j) order.
//
// Kernels (all on the caller's stream):
//   row_entropy_kernel   -sum_j P' ln(P' + eps) per row (warp per row)
//   (entropy_reduce of mask.cu: per-head mean)
//   route_kernel         median split per batch entry, pool state reset
//   pool_hist_kernel     one radix level: shared-memory histogram, flushed
//                        with 64-bit atomics (persistent CTAs per batch entry)
//   pool_pick_kernel     one warp per batch entry: the bin that reaches target
//   tie_count_kernel     pairs equal to u* per pool row
//   tie_scan_kernel      the row and rank of the last kept tie
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace bsa {

namespace {

constexpr int kMaxBins = 4096;
constexpr int kLevelBits[3] = {8, 12, 11};  // exponent, mantissa 22..11, mantissa 10..0

__device__ __forceinline__ float lg2_fast(float y) {
    float r;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}

__device__ __forceinline__ uint32_t pos_bits(float y) { return __float_as_uint(y > 0.f ? y : 0.f); }

__device__ __forceinline__ uint32_t significand(uint32_t u) {
    return (u & 0x7FFFFFu) | ((u >> 23) ? 0x800000u : 0u);
}

// 2^(max(e, 1) - 150): the weight of one significand unit in binade e.
__device__ __forceinline__ double unit_of_binade(uint32_t e) {
    const int k = static_cast<int>(e > 1u ? e : 1u) - 150;
    return __longlong_as_double(static_cast<long long>(k + 1023) << 52);
}

// Score of pair (row, j) of a pooled head, as a bit pattern: P' * ||c^V|| rounded
// to fp32 (P' alone without value norms); -0 and NaN count as +0.
__device__ __forceinline__ uint32_t pool_score(const float *__restrict__ prow,
                                               const float *__restrict__ vrow, int j) {
    const float p = __ldg(prow + j);
    const float s = vrow ? __fmul_rn(p, __ldg(vrow + j)) : p;
    return pos_bits(s);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// -sum_j P' ln(P' + eps) of every row, one warp per row.
__global__ void __launch_bounds__(256) row_entropy_kernel(const float *__restrict__ probs,
                                                          float *__restrict__ row_ent,
                                                          long long rows, int Ck, float eps) {
    const int lane = threadIdx.x % 32;
    const long long row = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
    if (row >= rows) return;
    const float *src = probs + row * Ck;
    float ent = 0.f;
#pragma unroll 4
    for (int j = lane; j < Ck; j += 32) {
        const float y = __ldg(src + j);
        const float x = y > 0.f ? y : 0.f;
        ent = fmaf(x, lg2_fast(x + eps), ent);
    }
    ent = warp_sum(ent);
    if (lane == 0) row_ent[row] = -ent * 0.6931471805599453f;  // ln 2
}

// Median split: heads of batch entry b ordered by (H_h asc, h asc); the first
// floor(H/2) are pooled.  Also resets the pool state of b.
__global__ void __launch_bounds__(256) route_kernel(const float *__restrict__ heads_h, int H,
                                                    uint8_t *low, uint8_t *low_out,
                                                    PoolState *state) {
    const int b = blockIdx.x, h = threadIdx.x;
    const float *hb = heads_h + static_cast<long long>(b) * H;
    if (h < H) {
        const float x = hb[h];
        int rank = 0;
        for (int o = 0; o < H; ++o) {
            const float y = hb[o];
            rank += (y < x || (y == x && o < h)) ? 1 : 0;
        }
        const uint8_t l = rank < H / 2 ? 1 : 0;
        low[static_cast<long long>(b) * H + h] = l;
        if (low_out) low_out[static_cast<long long>(b) * H + h] = l;
    }
    if (h == 0) {
        PoolState s;
        s.target = 0.0;
        s.above = 0.0;
        s.cnt_above = 0;
        s.pre = 0;
        s.shift = 31;  // level 1 bins bits 30..23 of scores >= 0 (bit 31 is 0)
        s.keep_all = 0;
        s.empty = H / 2 == 0;
        s.ucut = 0;
        s.pad0 = 0;
        s.need = 0;
        s.cut_row = -1;
        s.cut_rank = 0;
        s.pad1 = 0;
        state[b] = s;
    }
}

// One radix level of batch entry blockIdx.y: every score in the current range
// (bits above `shift` equal to `pre`) adds (1, significand) to bin
// (u >> (shift - nbits)) & (2^nbits - 1) of a shared histogram, flushed at exit.
__global__ void __launch_bounds__(256) pool_hist_kernel(const float *__restrict__ probs,
                                                        const float *__restrict__ vnorm,
                                                        const uint8_t *__restrict__ low,
                                                        const PoolState *__restrict__ state,
                                                        unsigned long long *__restrict__ hist,
                                                        int H, int Cq, int Ck, int nbits) {
    extern __shared__ unsigned long long sh[];  // [2^nbits][2]: count, significand sum
    const int b = blockIdx.y;
    const PoolState st = state[b];
    if (st.empty || st.keep_all || st.shift < nbits) return;
    const int nb = 1 << nbits;
    for (int k = threadIdx.x; k < 2 * nb; k += blockDim.x) sh[k] = 0ull;
    __syncthreads();
    const int lo = st.shift - nbits;
    const uint32_t pre = st.pre;
    const uint32_t bmask = static_cast<uint32_t>(nb - 1);
    const int lane = threadIdx.x % 32;
    const long long rows_b = static_cast<long long>(H) * Cq;
    const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
    for (long long w = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
         w < rows_b; w += warps) {
        const int h = static_cast<int>(w / Cq);
        if (!low[static_cast<long long>(b) * H + h]) continue;  // warp-uniform
        const long long bh = static_cast<long long>(b) * H + h;
        const float *prow = probs + (bh * Cq + (w % Cq)) * Ck;
        const float *vrow = vnorm ? vnorm + bh * Ck : nullptr;
        for (int j = lane; j < Ck; j += 32) {
            const uint32_t u = pool_score(prow, vrow, j);
            if ((u >> st.shift) == pre) {  // shift 31: every score (bit 31 clear)
                const uint32_t bin = (u >> lo) & bmask;
                atomicAdd(&sh[2 * bin], 1ull);
                atomicAdd(&sh[2 * bin + 1], static_cast<unsigned long long>(significand(u)));
            }
        }
    }
    __syncthreads();
    unsigned long long *g = hist + static_cast<long long>(b) * 2 * kMaxBins;
    for (int k = threadIdx.x; k < nb; k += blockDim.x) {
        if (sh[2 * k]) {
            atomicAdd(&g[2 * k], sh[2 * k]);
            atomicAdd(&g[2 * k + 1], sh[2 * k + 1]);
        }
    }
}

// The bin of the current level that holds the cut: scanning bins from the
// largest value down, the first non-empty bin whose inclusive mass (plus the
// mass above the range) reaches the target; if rounding leaves the whole range
// short of it, the last non-empty bin.  Level 1 also fixes the target
// pool_p * total, and keep_all when the pool never reaches it.  One warp per
// batch entry; lane l owns a contiguous run of bins from the top.
__global__ void __launch_bounds__(32) pool_pick_kernel(const unsigned long long *__restrict__ hist,
                                                       PoolState *state, float pool_p, int nbits,
                                                       int first_level) {
    const int b = blockIdx.x, lane = threadIdx.x;
    PoolState st = state[b];
    if (st.empty || st.keep_all || st.shift < nbits) return;
    const int nb = 1 << nbits;
    const int per = nb / 32;
    const unsigned long long *g = hist + static_cast<long long>(b) * 2 * kMaxBins;
    const int lo = st.shift - nbits;
    // bin k (value order) -> its mass unit: level 1 bins are binades, later
    // levels lie inside the binade fixed by level 1 (the top 8 bits of pre)
    auto unit_of = [&](int k) -> double {
        if (first_level) return unit_of_binade(static_cast<uint32_t>(k));
        const uint32_t e = (st.pre << st.shift) >> 23;  // exponent of the range
        return unit_of_binade(e);
    };
    // lane l: bins top - l*per - t, t = 0..per-1 (descending value)
    double m_run = 0.0;
    unsigned long long c_run = 0;
    const int top = nb - 1 - lane * per;
    for (int t = 0; t < per; ++t) {
        const int k = top - t;
        const unsigned long long c = g[2 * k];
        if (c) {
            m_run += static_cast<double>(g[2 * k + 1]) * unit_of(k);
            c_run += c;
        }
    }
    // exclusive prefix over lanes (value order)
    double m_ex = m_run;
    unsigned long long c_ex = c_run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double mo = __shfl_up_sync(0xffffffffu, m_ex, o);
        const unsigned long long co = __shfl_up_sync(0xffffffffu, c_ex, o);
        if (lane >= o) {
            m_ex += mo;
            c_ex += co;
        }
    }
    const double m_before = m_ex - m_run;   // mass of the lanes above this one
    const unsigned long long c_before = c_ex - c_run;
    if (first_level) {
        const double total = __shfl_sync(0xffffffffu, m_ex, 31);
        st.target = static_cast<double>(pool_p) * total;
        if (!(total >= st.target)) {
            if (lane == 0) {
                st.keep_all = 1;
                state[b] = st;
            }
            return;
        }
    }
    const double target = st.target;
    const bool reaches = c_run > 0 && st.above + m_before + m_run >= target;
    const uint32_t hit = __ballot_sync(0xffffffffu, reaches);
    int owner;
    if (hit) {
        owner = __ffs(hit) - 1;
    } else {
        const uint32_t ne = __ballot_sync(0xffffffffu, c_run > 0);
        owner = ne ? 31 - __clz(ne) : 0;
    }
    if (lane == owner) {
        double m = st.above + m_before;
        unsigned long long c = st.cnt_above + c_before;
        int pick = -1, last_ne = -1;
        for (int t = 0; t < per; ++t) {
            const int k = top - t;
            const unsigned long long ck = g[2 * k];
            if (!ck) continue;
            const double mk = static_cast<double>(g[2 * k + 1]) * unit_of(k);
            if (hit && m + mk >= target) {
                pick = k;
                break;
            }
            last_ne = k;
            m += mk;
            c += ck;
        }
        if (pick < 0) {  // the range ends short of the target: its last bin
            pick = last_ne;
            // undo the last bin's mass: it is the cut bin itself
            const double mk = static_cast<double>(g[2 * pick + 1]) * unit_of(pick);
            m -= mk;
            c -= g[2 * pick];
        }
        st.above = m;
        st.cnt_above = c;
        st.pre = (st.pre << nbits) | static_cast<uint32_t>(pick);
        st.shift = lo;
        if (lo == 0) {
            // the cut bit pattern; keep its first `need` pairs in (h, i, j) order
            st.ucut = st.pre;
            const double v = static_cast<double>(__uint_as_float(st.ucut));
            const unsigned long long ties = g[2 * pick];
            unsigned long long need = 1;
            if (v > 0.0 && st.above < target) {
                const double n = ceil((target - st.above) / v);
                need = n < 1.0 ? 1ull : static_cast<unsigned long long>(n);
                // the closed form against the running sum of the rule
                while (need > 1 && st.above + static_cast<double>(need - 1) * v >= target) --need;
                while (need < ties && st.above + static_cast<double>(need) * v < target) ++need;
            }
            st.need = need < ties ? need : ties;
        }
        state[b] = st;
    }
}

// Pairs equal to the cut pattern in each pooled row.
__global__ void __launch_bounds__(256) tie_count_kernel(const float *__restrict__ probs,
                                                        const float *__restrict__ vnorm,
                                                        const uint8_t *__restrict__ low,
                                                        const PoolState *__restrict__ state,
                                                        int *__restrict__ tiecnt, long long rows,
                                                        int H, int Cq, int Ck) {
    const int lane = threadIdx.x % 32;
    const long long row = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
    if (row >= rows) return;
    const long long bh = row / Cq;
    const int b = static_cast<int>(bh / H);
    const PoolState st = state[b];
    int n = 0;
    if (!st.empty && !st.keep_all && low[bh]) {
        const float *prow = probs + row * Ck;
        const float *vrow = vnorm ? vnorm + bh * Ck : nullptr;
        for (int j = lane; j < Ck; j += 32) n += pool_score(prow, vrow, j) == st.ucut ? 1 : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
    }
    if (lane == 0) tiecnt[row] = n;
}

// The row (in (h, i) order) where the running count of ties reaches `need`,
// and how many ties of that row are kept.  One block per batch entry.
__global__ void __launch_bounds__(1024) tie_scan_kernel(const int *__restrict__ tiecnt,
                                                        PoolState *state, int H, int Cq) {
    __shared__ unsigned long long part[1024];
    const int b = blockIdx.x;
    const PoolState st = state[b];
    if (st.empty || st.keep_all) return;
    const long long rows_b = static_cast<long long>(H) * Cq;
    const long long base = static_cast<long long>(b) * rows_b;
    const long long per = (rows_b + blockDim.x - 1) / blockDim.x;
    const long long r0 = threadIdx.x * per, r1 = min(rows_b, r0 + per);
    unsigned long long s = 0;
    for (long long r = r0; r < r1; ++r) s += static_cast<unsigned long long>(tiecnt[base + r]);
    part[threadIdx.x] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long run = 0;
        int owner = -1;
        for (int t = 0; t < static_cast<int>(blockDim.x); ++t) {
            if (run + part[t] >= st.need) {
                owner = t;
                break;
            }
            run += part[t];
        }
        PoolState s2 = st;
        s2.cut_row = -1;
        s2.cut_rank = 0;
        if (owner >= 0) {
            const long long a = owner * per, e = min(rows_b, a + per);
            for (long long r = a; r < e; ++r) {
                const unsigned long long c = static_cast<unsigned long long>(tiecnt[base + r]);
                if (run + c >= st.need) {
                    s2.cut_row = base + r;
                    s2.cut_rank = static_cast<int>(st.need - run);
                    break;
                }
                run += c;
            }
        }
        state[b] = s2;
    }
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

EgWorkspace eg_workspace(const Geometry &g) {
    const size_t rows = static_cast<size_t>(g.B) * g.H * g.Cq;
    const size_t bh = static_cast<size_t>(g.B) * g.H;
    EgWorkspace w;
    size_t off = 0;
    w.row_entropy = off;
    off += round256(rows * sizeof(float));
    w.heads_h = off;
    off += round256(bh * sizeof(float));
    w.low = off;
    off += round256(bh);
    w.hist = off;
    off += round256(static_cast<size_t>(g.B) * 2 * kMaxBins * sizeof(unsigned long long));
    w.state = off;
    off += round256(static_cast<size_t>(g.B) * sizeof(PoolState));
    w.tiecnt = off;
    off += round256(rows * sizeof(int));
    w.bytes = off;
    return w;
}

cudaError_t launch_eg_prepare(const Geometry &g, const float *probs, const float *vnorm,
                              float pool_p, float eps, float *entropy, float *entropy_norm,
                              uint8_t *low_heads, uint8_t *workspace, cudaStream_t st) {
    const EgWorkspace w = eg_workspace(g);
    float *row_ent = reinterpret_cast<float *>(workspace + w.row_entropy);
    float *heads_h = reinterpret_cast<float *>(workspace + w.heads_h);
    uint8_t *low = workspace + w.low;
    unsigned long long *hist = reinterpret_cast<unsigned long long *>(workspace + w.hist);
    PoolState *state = reinterpret_cast<PoolState *>(workspace + w.state);
    int *tiecnt = reinterpret_cast<int *>(workspace + w.tiecnt);
    const long long rows = static_cast<long long>(g.B) * g.H * g.Cq;
    const unsigned rgrid = static_cast<unsigned>((rows + 7) / 8);

    row_entropy_kernel<<<rgrid, 256, 0, st>>>(probs, row_ent, rows, g.Ck, eps);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = launch_entropy_reduce(g, row_ent, heads_h, entropy_norm, st);
    if (e != cudaSuccess) return e;
    if (entropy) {
        e = cudaMemcpyAsync(entropy, heads_h, static_cast<size_t>(g.B) * g.H * sizeof(float),
                            cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return e;
    }
    route_kernel<<<g.B, 256, 0, st>>>(heads_h, g.H, low, low_heads, state);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidValue;
    const long long pool_rows = static_cast<long long>(g.H / 2) * g.Cq;
    const unsigned hx = static_cast<unsigned>(
        max(1ll, min(static_cast<long long>(2 * sms) / max(g.B, 1), (pool_rows + 7) / 8)));
    for (int level = 0; level < 3; ++level) {
        const int nbits = kLevelBits[level];
        const size_t smem = static_cast<size_t>(2) << nbits << 3;  // 2^nbits x 2 x 8 bytes
        if ((e = cudaMemsetAsync(hist, 0,
                                 static_cast<size_t>(g.B) * 2 * kMaxBins * sizeof(unsigned long long),
                                 st)) != cudaSuccess)
            return e;
        if (smem > 48 * 1024 &&
            (e = cudaFuncSetAttribute(pool_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(smem))) != cudaSuccess)
            return e;
        pool_hist_kernel<<<dim3(hx, g.B), 256, smem, st>>>(probs, vnorm, low, state, hist, g.H,
                                                          g.Cq, g.Ck, nbits);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        pool_pick_kernel<<<g.B, 32, 0, st>>>(hist, state, pool_p, nbits, level == 0 ? 1 : 0);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    tie_count_kernel<<<rgrid, 256, 0, st>>>(probs, vnorm, low, state, tiecnt, rows, g.H, g.Cq, g.Ck);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    tie_scan_kernel<<<g.B, 1024, 0, st>>>(tiecnt, state, g.H, g.Cq);
    return cudaGetLastError();
}

}  // namespace bsa
