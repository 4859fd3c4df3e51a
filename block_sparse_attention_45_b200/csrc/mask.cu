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
// Top-p without sorting: P' >= 0, so fp32 bit patterns order like the values,
// and the kept set is every entry whose key (bits, -j) is at least the cut's.
// The cut is found by an exact radix selection: histograms of integer
// significand sums pick the binade, then mantissa digits, until at most 32
// candidates remain; candidate m is kept iff it is the first of the
// (P' desc, j asc) order or the mass strictly before it is below p -- the
// shortest prefix of the sorted row whose running sum reaches p (at least one
// entry, also for p <= 0).  Masses inside one binade are exact integers; the
// binades above it are summed in fp64.  Row entropies go to a workspace; a
// second kernel sums them per head in a fixed order.
//
// Two kernels: topp_kernel (per-row top-p for every head: bsa_build_mask) and
// mask_kernel<VPL, true> (the pooled domains of bsa_build_mask_eg /
// bsa_build_mask_domain, whose per-row heads take find_cut).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "bits.cuh"
#include "internal.h"
#include "ptx.cuh"  // red_add_shared

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
    // pooled mode: pooled heads take their pool's cut
    const float *vnorm;           // value-centroid norms [B,H,C_k], or nullptr
    const int8_t *pool_of;        // [B,H]: the head's pool, -1 = per-row
    const PoolState *state;       // [B,G]
    int G;                        // pools per batch entry
};

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

// ---------------------------------------------------------------------------
// Exact radix selection of the cut.
//
// Keys order like (P' desc, j asc).  Level 1 histograms the fp32 exponent
// field over the 27 binades from the row's largest one down (binade r holds the
// entries whose exponent is emax - r; everything further down lands in row
// kUnder, the underflow bin); the later levels histogram 4 mantissa bits at a
// time inside the chosen range, until at most 32 entries remain.  Each lane
// owns one column of a kRowsTab x 32 table in shared memory (28 rows keep a
// 4-warp CTA at 30 KB, so 7 CTAs fit an SM) and adds (1 << 40 | mantissa) of
// its own entries to it; the implicit leading bits are added per bin from the
// count, so a bin holds the exact integer sum of its entries' significands.
// Within one binade masses are integers times one power of two, so every
// prefix below the level-1 split is exact.  Row r of the table is the r-th bin
// in descending order; lane r sums row r and the warp scans the rows.
//
// Padding slots (j >= Ck) hold +0.0, which has exponent field 0 and mantissa 0:
// they add no mass, and their count is taken off the one bin they fall in.
constexpr int kLanes = 32;
constexpr int kRowsTab = 28;          // table rows
constexpr int kUnder = kRowsTab - 1;  // level-1 row of everything below the binade window
constexpr int kDigitBits = 4;         // mantissa bits per later level (16 rows)
constexpr uint64_t kCountOne = 1ull << 40;
constexpr uint64_t kSigMask = kCountOne - 1;
constexpr uint64_t kImplicit = 1ull << 23;

struct WarpScratch {
    unsigned long long bins[kRowsTab][kLanes];  // [row][lane]
    uint32_t cand_u[32];
    int cand_j[32];
};

// Lane r < kRowsTab returns the sum of row r and clears it (other lanes 0).
// Quarter-warps read 8 distinct bank groups thanks to the rotation.
__device__ __forceinline__ unsigned long long bin_row_sum(unsigned long long (*bins)[kLanes],
                                                         int lane) {
    unsigned long long acc = 0;
    if (lane < kRowsTab) {
        ulonglong2 *row = reinterpret_cast<ulonglong2 *>(bins[lane]);
#pragma unroll
        for (int k = 0; k < kLanes / 2; ++k) {
            const int kk = (k + lane) & (kLanes / 2 - 1);
            const ulonglong2 x = row[kk];
            acc += x.x + x.y;
            row[kk] = make_ulonglong2(0ull, 0ull);
        }
    }
    return acc;
}

__device__ __forceinline__ unsigned long long scan_incl_u64(unsigned long long x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long t = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += t;
    }
    return x;
}

__device__ __forceinline__ double scan_incl_d(double x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += t;
    }
    return x;
}

// The row of the cut: the first non-empty row whose inclusive mass reaches p,
// else (rounding left the whole range short of p) the last non-empty row.
__device__ __forceinline__ int pick_row(bool nonempty, bool reaches) {
    const uint32_t hit = __ballot_sync(0xffffffffu, nonempty && reaches);
    if (hit) return __ffs(hit) - 1;
    const uint32_t ne = __ballot_sync(0xffffffffu, nonempty);
    return ne ? 31 - __clz(ne) : 0;
}

// j of the n-th (1-based) entry with bit pattern uc, in ascending j.
template <int VPL>
__device__ __forceinline__ int nth_tie(const float (&v)[VPL], int Ck, uint32_t uc, int n, int lane) {
    int seen = 0, jc = -1;
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const bool is_t = lane + 32 * s < Ck && __float_as_uint(v[s]) == uc;
        const uint32_t bal = __ballot_sync(0xffffffffu, is_t);
        const int cnt = __popc(bal);
        if (jc < 0 && seen + cnt >= n) {
            uint32_t b = bal;
            for (int k = 1; k < n - seen; ++k) b &= b - 1;
            jc = 32 * s + __ffs(b) - 1;
        }
        seen += cnt;
    }
    return jc;
}

// Bit pattern of max(y, +0.0), NaN -> +0.0: the value every pass works on.
__device__ __forceinline__ uint32_t pos_bits(float y) { return __float_as_uint(y > 0.f ? y : 0.f); }

// fp64 mass of the row's entries with bit pattern in [lo_u, hi_u].
__device__ __noinline__ double mass_between(const float *__restrict__ src, int Ck, uint32_t lo_u,
                                            uint32_t hi_u, int lane) {
    double f = 0.0;
    for (int j = lane; j < Ck; j += 32) {
        const float y = __ldg(src + j);
        const float x = y > 0.f ? y : 0.f;
        const uint32_t u = __float_as_uint(x);
        if (u >= lo_u && u <= hi_u) f += static_cast<double>(x);
    }
    return warp_sum_d(f);
}

// Cut inside the underflow range u <= hi (entries kUnder or more binades below the
// row maximum), given that the row reaches p only there: fp64 bisection on the
// bit pattern, then ties in ascending j.  Reached only when p lies within about
// 2^-30 of the row total, so it re-reads the row from global memory instead of
// holding fp64 copies in registers.
__device__ __noinline__ void cut_in_underflow(const float *__restrict__ src, int Ck, double pd,
                                              double above, uint32_t hi, int lane,
                                              uint32_t *ucut_out, int *jcut_out) {
    uint32_t lo = 0, top = hi;
    while (lo < top) {
        const uint32_t mid = lo + ((top - lo + 1) >> 1);
        if (above + mass_between(src, Ck, mid, hi, lane) >= pd) lo = mid;
        else top = mid - 1;
    }
    const uint32_t uc = lo;
    const double abv = uc < hi ? above + mass_between(src, Ck, uc + 1, hi, lane) : above;
    int ties = 0;
    for (int j = lane; j < Ck; j += 32) ties += pos_bits(__ldg(src + j)) == uc;
    ties = warp_sum_i(ties);
    const double vc = static_cast<double>(__uint_as_float(uc));
    int need = 1;
    double run = abv + vc;
    while (run < pd && need < ties) {
        run += vc;
        ++need;
    }
    int seen = 0, jc = -1;
    for (int j0 = 0; j0 < Ck; j0 += 32) {
        const int j = j0 + lane;
        const bool is_t = j < Ck && pos_bits(__ldg(src + j)) == uc;
        const uint32_t bal = __ballot_sync(0xffffffffu, is_t);
        const int cnt = __popc(bal);
        if (jc < 0 && seen + cnt >= need) {
            uint32_t b = bal;
            for (int k = 1; k < need - seen; ++k) b &= b - 1;
            jc = j0 + __ffs(b) - 1;
        }
        seen += cnt;
    }
    *ucut_out = uc;
    *jcut_out = jc;
}

// Sets (ucut, jcut) so that the row keeps exactly the entries with u > ucut,
// or u == ucut and j <= jcut; (0, INT_MAX) keeps the whole row (it never
// reaches p).
template <int VPL>
__device__ __forceinline__ void find_cut(const float (&v)[VPL], const float *__restrict__ src,
                                         int Ck, float p, uint32_t umax, int lane,
                                         WarpScratch &ws, uint32_t &ucut, int &jcut) {
    const double pd = static_cast<double>(p);
    const uint32_t emax = umax >> 23;
    const int npad = 32 * VPL - Ck;
    // ---- level 1: binades emax .. emax-(kUnder-1) in rows 0..kUnder-1, the rest in kUnder
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const uint32_t u = __float_as_uint(v[s]);
        const uint32_t r = min(emax - (u >> 23), static_cast<uint32_t>(kUnder));
        ws.bins[r][lane] += kCountOne | (u & 0x7FFFFFu);
    }
    __syncwarp();
    const unsigned long long acc1 = bin_row_sum(ws.bins, lane);
    __syncwarp();
    const uint32_t pad_row = min(emax, static_cast<uint32_t>(kUnder));
    const int cnt_r = static_cast<int>(acc1 >> 40) - (lane == static_cast<int>(pad_row) ? npad : 0);
    const uint32_t ex_r = emax - static_cast<uint32_t>(lane);  // exponent field of row `lane`
    double mass_r = 0.0;
    if (lane < kUnder && lane <= static_cast<int>(emax)) {
        const unsigned long long sig = (acc1 & kSigMask) +
            (ex_r > 0u ? kImplicit * static_cast<unsigned long long>(cnt_r) : 0ull);
        mass_r = static_cast<double>(sig) * unit_of_binade(ex_r);
    }
    const double incl = scan_incl_d(mass_r, lane);  // rows kUnder.. add nothing here
    const int cincl = static_cast<int>(scan_incl_u64(static_cast<unsigned long long>(cnt_r), lane));
    double excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.0;
    const uint32_t hit = __ballot_sync(0xffffffffu, lane < kUnder && cnt_r > 0 && incl >= pd);
    if (!hit) {
        // Binades emax..emax-30 do not reach p: the row total decides.
        const double head = __shfl_sync(0xffffffffu, incl, kUnder);
        const int n_under = __shfl_sync(0xffffffffu, cnt_r, kUnder);
        const double tail = n_under > 0 ? mass_between(src, Ck, 0u, ((emax - static_cast<uint32_t>(kUnder - 1)) << 23) - 1u, lane)
                                        : 0.0;
        if (!(head + tail >= pd)) {
            ucut = 0u;
            jcut = 0x7FFFFFFF;
            return;
        }
        // Reaching p needs the underflow entries (tail > 0 here).
        cut_in_underflow(src, Ck, pd, head, ((emax - static_cast<uint32_t>(kUnder - 1)) << 23) - 1u, lane, &ucut, &jcut);
        return;
    }
    const int b = __ffs(hit) - 1;
    const double above = __shfl_sync(0xffffffffu, excl, b);
    int cnt_above = __shfl_sync(0xffffffffu, cincl - cnt_r, b);
    int cnt = __shfl_sync(0xffffffffu, cnt_r, b);
    // ---- mantissa levels inside binade e: candidates share (u >> sh) == pre
    const uint32_t e = emax - static_cast<uint32_t>(b);
    const double unit = unit_of_binade(e);
    const unsigned long long implicit = e > 0u ? kImplicit : 0ull;
    bool pad_in = e == 0u;           // padding (+0.0) still inside the range
    unsigned long long s_above = 0;  // significands of the binade's entries above the range
    uint32_t pre = e;
    int sh = 23;
    while (cnt > 32 && sh > 0) {
        const int w = sh >= kDigitBits ? kDigitBits : sh;
        sh -= w;
        const uint32_t top = (1u << w) - 1u;
#pragma unroll
        for (int s = 0; s < VPL; ++s) {
            const uint32_t u = __float_as_uint(v[s]);
            if ((u >> (sh + w)) == pre)
                ws.bins[top - ((u >> sh) & top)][lane] += kCountOne | (u & 0x7FFFFFu);
        }
        __syncwarp();
        const unsigned long long acc = bin_row_sum(ws.bins, lane);
        __syncwarp();
        const int c_r = static_cast<int>(acc >> 40) -
                        (pad_in && lane == static_cast<int>(top) ? npad : 0);
        const unsigned long long sg_r = (acc & kSigMask) +
                                        implicit * static_cast<unsigned long long>(c_r);
        const unsigned long long sg_incl = scan_incl_u64(sg_r, lane);
        const int c_incl = static_cast<int>(scan_incl_u64(static_cast<unsigned long long>(c_r), lane));
        const bool reaches = above + static_cast<double>(s_above + sg_incl) * unit >= pd;
        const int r = pick_row(c_r > 0, reaches);
        s_above += __shfl_sync(0xffffffffu, sg_incl - sg_r, r);
        cnt_above += __shfl_sync(0xffffffffu, c_incl - c_r, r);
        cnt = __shfl_sync(0xffffffffu, c_r, r);
        pad_in = pad_in && r == static_cast<int>(top);
        pre = (pre << w) | (top - static_cast<uint32_t>(r));
    }
    if (cnt <= 32) {
        // ---- at most 32 candidates: each one knows the exact mass before it
        const uint32_t lt_mask = (1u << lane) - 1u;
        int c = 0;
#pragma unroll
        for (int s = 0; s < VPL; ++s) {
            const uint32_t u = __float_as_uint(v[s]);
            const int j = lane + 32 * s;
            const bool is_c = (u >> sh) == pre && j < Ck;
            const uint32_t bal = __ballot_sync(0xffffffffu, is_c);
            if (is_c) {
                const int pos = c + __popc(bal & lt_mask);
                ws.cand_u[pos] = u;
                ws.cand_j[pos] = j;
            }
            c += __popc(bal);
        }
        __syncwarp();
        const bool mine = lane < cnt;
        const uint32_t um = mine ? ws.cand_u[lane] : 0u;
        const int jm = mine ? ws.cand_j[lane] : 0;
        unsigned long long s_before = 0;
        int n_before = 0;
#pragma unroll 4
        for (int n = 0; n < cnt; ++n) {
            const uint32_t un = ws.cand_u[n];
            if (un > um || (un == um && n < lane)) {
                s_before += significand(un);
                ++n_before;
            }
        }
        __syncwarp();
        const double before = above + static_cast<double>(s_above + s_before) * unit;
        const bool kept = mine && (before < pd || (cnt_above == 0 && n_before == 0));
        const uint64_t key = kept ? ((static_cast<uint64_t>(um) << 32) |
                                     (0xFFFFFFFFu - static_cast<uint32_t>(jm)))
                                  : ~0ull;
        const uint64_t best = warp_min_u64(key);
        if (best == ~0ull) {  // the range starts past p (rounding): keep only what is above it
            uint32_t mx = mine ? um : 0u;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            ucut = mx;
            jcut = -1;
        } else {
            ucut = static_cast<uint32_t>(best >> 32);
            jcut = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(best));
        }
        return;
    }
    // ---- more than 32 entries with one bit pattern: ties in ascending j
    const uint32_t uc = pre;
    const unsigned long long sg = significand(uc);
    int n_keep = 0;
    for (int k = lane; k < cnt; k += 32)
        n_keep += (above + static_cast<double>(s_above + sg * static_cast<unsigned long long>(k)) *
                               unit < pd) ? 1 : 0;
    n_keep = warp_sum_i(n_keep);
    if (n_keep == 0 && cnt_above == 0) n_keep = 1;
    ucut = uc;
    jcut = n_keep == 0 ? -1 : nth_tie<VPL>(v, Ck, uc, n_keep, lane);
}

// ---------------------------------------------------------------------------
// Per-row top-p, the path of bsa_build_mask.
//
// The same selection as find_cut above, organised for throughput:
//   * each warp walks rows blockIdx*4+warp, + 4*gridDim, ... (7 CTAs of 4 warps
//     per SM at 72 registers up to C_k = 1024, 3 beyond), so its tables are
//     cleared once, not per row;
//   * level 1 bins the binades below the row maximum in windows of kWin
//     binades (per-lane columns, fire-and-forget shared reductions), moving the
//     window down only when the cut lies deeper;
//   * inside the cut binade, 5-bit digit levels (shared reductions into 32
//     bins) narrow the range until at most 32 entries remain;
//   * those candidates are resolved by a warp loop over register shuffles: each
//     knows the exact significand sum of the candidates before it in (P' desc,
//     j asc) order.
// Masses inside one binade are exact integers; binades are summed in fp64,
// exactly while the cut is within ~2^-29 of the row total (as in the oracle's
// own fp64 running sum).  Zero entries (and padding) carry no mass and are
// never the cut except in an all-zero row, so they are left out of the bins.
constexpr int kTpWarps = 4;              // warps per CTA, one row at a time each
constexpr int kL1Rows = 16;              // level-1 table rows
constexpr int kWin = kL1Rows - 1;        // binades per level-1 window; row kWin: deeper

struct alignas(16) TpWarp {
    unsigned long long l1[kL1Rows][kLanes];  // level-1 bins, one column per lane
    unsigned long long dig[32];              // digit bins (shared by the lanes)
    uint32_t cand_u[32];
    int cand_j[32];
};

// Level-1 pass over one window: ranks [off, off + kWin) below the maximum's
// binade go to rows 0 .. kWin-1, deeper ones to row kWin; ranks above the
// window are skipped (their mass is already known).  NONZERO: leave out zero
// entries (needed once the window reaches exponent field 0).
template <int VPL, bool NONZERO>
__device__ __forceinline__ void tp_bin_window(const float (&v)[VPL], uint32_t emax, int off,
                                              unsigned long long *col) {
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const uint32_t u = __float_as_uint(v[s]);
        const int r = static_cast<int>(emax - (u >> 23)) - off;
        const bool in = r >= 0 && (!NONZERO || u != 0u);
        if (in) red_add_shared(col + min(r, kWin) * kLanes, kCountOne | (u & 0x7FFFFFu));
    }
}

// The cut of one row held as v[s] = max(P'[lane + 32 s], 0) (padding 0):
// the row keeps the entries with pattern > ucut, or == ucut and j <= jcut.
template <int VPL>
__device__ __forceinline__ void tp_cut(const float (&v)[VPL], int Ck, float p, uint32_t umax,
                                       int lane, TpWarp &ws, uint32_t &ucut, int &jcut) {
    const double pd = static_cast<double>(p);
    if (umax == 0u) {  // every entry is zero: nothing ever reaches p > 0
        ucut = 0u;
        jcut = pd <= 0.0 ? 0 : 0x7FFFFFFF;
        return;
    }
    const uint32_t emax = umax >> 23;
    double above = 0.0;  // mass of the binades above the current range
    int cnt_above = 0;
    int cnt = 0;
    uint32_t e = 0;
    unsigned long long *col = &ws.l1[0][lane];
    // lane L sums half (L & 1) of level-1 row L >> 1
    const int prow = lane >> 1, phalf = lane & 1;
    for (int off = 0;; off += kWin) {
        if (static_cast<int>(emax) < off + kWin) tp_bin_window<VPL, true>(v, emax, off, col);
        else tp_bin_window<VPL, false>(v, emax, off, col);
        __syncwarp();
        unsigned long long half = 0;
        {
            ulonglong2 *rw = reinterpret_cast<ulonglong2 *>(&ws.l1[prow][16 * phalf]);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int kk = (k + lane) & 7;
                const ulonglong2 x = rw[kk];
                half += x.x + x.y;
                rw[kk] = make_ulonglong2(0ull, 0ull);
            }
        }
        __syncwarp();
        const unsigned long long tot2 = half + __shfl_xor_sync(0xffffffffu, half, 1);
        const unsigned long long tot = __shfl_sync(0xffffffffu, tot2, (2 * lane) & 31);
        const int e_r = static_cast<int>(emax) - off - lane;  // exponent field of row `lane`
        const bool real = lane < kWin && e_r >= 0;
        const int cnt_r = real ? static_cast<int>(tot >> 40) : 0;
        double mass_r = 0.0;
        if (real) {
            const unsigned long long sig = (tot & kSigMask) +
                (e_r > 0 ? kImplicit * static_cast<unsigned long long>(cnt_r) : 0ull);
            mass_r = static_cast<double>(sig) * unit_of_binade(static_cast<uint32_t>(e_r));
        }
        const double incl = scan_incl_d(mass_r, lane);
        const int cincl = static_cast<int>(scan_incl_u64(static_cast<unsigned long long>(cnt_r), lane));
        const uint32_t hit = __ballot_sync(0xffffffffu, cnt_r > 0 && above + incl >= pd);
        if (hit) {
            const int b = __ffs(hit) - 1;
            above += __shfl_sync(0xffffffffu, incl - mass_r, b);
            cnt_above += __shfl_sync(0xffffffffu, cincl - cnt_r, b);
            cnt = __shfl_sync(0xffffffffu, cnt_r, b);
            e = emax - static_cast<uint32_t>(off + b);
            break;
        }
        // Not in this window: move below it, or keep the whole row if nothing is left.
        above += __shfl_sync(0xffffffffu, incl, kWin - 1);
        cnt_above += __shfl_sync(0xffffffffu, cincl, kWin - 1);
        const int deeper = static_cast<int>(__shfl_sync(0xffffffffu, tot2, 2 * kWin) >> 40);
        if (deeper == 0 || static_cast<int>(emax) < off + kWin) {
            ucut = 0u;
            jcut = 0x7FFFFFFF;
            return;
        }
    }
    // ---- digit levels inside binade e: the range is [lo, hi] = prefix `pre` above bit sh
    const double unit = unit_of_binade(e);
    const unsigned long long implicit = e > 0u ? kImplicit : 0ull;
    unsigned long long s_above = 0;  // significands of the binade's entries above the range
    uint32_t pre = e;
    int sh = 23;
    uint32_t lo = e > 0u ? (e << 23) : 1u, span = (e << 23 | 0x7FFFFFu) - lo;
    while (cnt > 32 && sh > 0) {
        const int w = sh >= 5 ? 5 : sh;
        sh -= w;
        const uint32_t top = (1u << w) - 1u;
#pragma unroll
        for (int s = 0; s < VPL; ++s) {
            const uint32_t u = __float_as_uint(v[s]);
            if (u - lo <= span)
                red_add_shared(&ws.dig[top - ((u >> sh) & top)], kCountOne | (u & 0x7FFFFFu));
        }
        __syncwarp();
        unsigned long long acc = 0;
        if (lane <= static_cast<int>(top)) {
            acc = ws.dig[lane];
            ws.dig[lane] = 0ull;
        }
        __syncwarp();
        const int c_r = static_cast<int>(acc >> 40);
        const unsigned long long sg_r = (acc & kSigMask) + implicit * static_cast<unsigned long long>(c_r);
        const unsigned long long sg_incl = scan_incl_u64(sg_r, lane);
        const int c_incl = static_cast<int>(scan_incl_u64(static_cast<unsigned long long>(c_r), lane));
        const bool reaches = above + static_cast<double>(s_above + sg_incl) * unit >= pd;
        const int r = pick_row(c_r > 0, reaches);
        s_above += __shfl_sync(0xffffffffu, sg_incl - sg_r, r);
        cnt_above += __shfl_sync(0xffffffffu, c_incl - c_r, r);
        cnt = __shfl_sync(0xffffffffu, c_r, r);
        pre = (pre << w) | (top - static_cast<uint32_t>(r));
        const uint32_t lo_new = pre << sh;
        lo = lo_new > 0u ? lo_new : 1u;
        span = (lo_new | ((1u << sh) - 1u)) - lo;
    }
    if (cnt <= 32) {
        // ---- at most 32 candidates: compact them, then each learns the exact mass before it
        const uint32_t lt_mask = (1u << lane) - 1u;
        int c = 0;
#pragma unroll
        for (int s = 0; s < VPL; ++s) {
            const uint32_t u = __float_as_uint(v[s]);
            const bool is_c = u - lo <= span;
            const uint32_t bal = __ballot_sync(0xffffffffu, is_c);
            if (is_c) {
                const int pos = c + __popc(bal & lt_mask);
                ws.cand_u[pos] = u;
                ws.cand_j[pos] = lane + 32 * s;
            }
            c += __popc(bal);
        }
        __syncwarp();
        const bool mine = lane < cnt;
        const uint32_t um = mine ? ws.cand_u[lane] : 0u;
        const int jm = mine ? ws.cand_j[lane] : 0;
        __syncwarp();
        const uint32_t imp32 = e > 0u ? 0x800000u : 0u;
        uint32_t s_before = 0;  // < 32 * 2^24
        int n_before = 0;
        for (int n = 0; n < cnt; ++n) {
            const uint32_t un = __shfl_sync(0xffffffffu, um, n);
            const int jn = __shfl_sync(0xffffffffu, jm, n);
            if (un > um || (un == um && jn < jm)) {
                s_before += (un & 0x7FFFFFu) | imp32;
                ++n_before;
            }
        }
        const double before = above + static_cast<double>(s_above + s_before) * unit;
        const bool kept = mine && (before < pd || (cnt_above == 0 && n_before == 0));
        const uint64_t key = kept ? ((static_cast<uint64_t>(um) << 32) |
                                     (0xFFFFFFFFu - static_cast<uint32_t>(jm)))
                                  : ~0ull;
        const uint64_t best = warp_min_u64(key);
        if (best == ~0ull) {  // the range starts past p (rounding): keep only what is above it
            uint32_t mx = mine ? um : 0u;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            ucut = mx;
            jcut = -1;
        } else {
            ucut = static_cast<uint32_t>(best >> 32);
            jcut = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(best));
        }
        return;
    }
    // ---- more than 32 entries with one bit pattern: ties in ascending j
    const uint32_t uc = pre;
    const unsigned long long sg = significand(uc);
    int n_keep = 0;
    for (int k = lane; k < cnt; k += 32)
        n_keep += (above + static_cast<double>(s_above + sg * static_cast<unsigned long long>(k)) *
                               unit < pd) ? 1 : 0;
    n_keep = warp_sum_i(n_keep);
    if (n_keep == 0 && cnt_above == 0) n_keep = 1;
    ucut = uc;
    jcut = n_keep == 0 ? -1 : nth_tie<VPL>(v, Ck, uc, n_keep, lane);
}

// One warp per row at a time; rows blockIdx.x * 4 + warp, then + 4 * gridDim.x.
// KFULL: slots that are never padding (the launcher guarantees Ck > 32 * KFULL).
template <int VPL, int KFULL>
__global__ void __launch_bounds__(128, VPL <= 32 ? 7 : 3) topp_kernel(MaskArgs a, TopP tp) {
    __shared__ TpWarp s_tp[kTpWarps];
    const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
    TpWarp &ws = s_tp[wid];
    {
        ulonglong2 *t = reinterpret_cast<ulonglong2 *>(&ws.l1[0][0]);
        for (int k = lane; k < kL1Rows * kLanes / 2; k += 32) t[k] = make_ulonglong2(0ull, 0ull);
        ws.dig[lane] = 0ull;
        __syncwarp();
    }
    const int Ck = a.Ck;
    const long long stride = static_cast<long long>(gridDim.x) * kTpWarps;
    for (long long row = static_cast<long long>(blockIdx.x) * kTpWarps + wid; row < a.rows; row += stride) {
        const float *src = a.probs + row * Ck;
        float v[VPL];
#pragma unroll
        for (int s = 0; s < VPL; ++s) {
            const int j = lane + 32 * s;
            v[s] = (s < KFULL || j < Ck) ? __ldg(src + j) : 0.f;
        }
        const int row32 = static_cast<int>(row);  // rows < 2^31 (checked on the host)
        const int i = row32 % a.Cq;
        const int h = (row32 / a.Cq) % a.H;
        float ent = 0.f;
        uint32_t umax = 0;
        const bool want_ent = a.row_entropy != nullptr;
#pragma unroll
        for (int s = 0; s < VPL; ++s) {
            const float x = v[s] > 0.f ? v[s] : 0.f;  // -0.0 and NaN become +0.0
            if (want_ent && (s < KFULL || lane + 32 * s < Ck)) ent = fmaf(x, lg2_approx(x + a.eps), ent);
            v[s] = x;
            umax = max(umax, __float_as_uint(x));
        }
        if (want_ent) {
            ent = -warp_sum(ent) * 0.6931471805599453f;  // ln 2
            if (lane == 0) a.row_entropy[row] = ent;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) umax = max(umax, __shfl_xor_sync(0xffffffffu, umax, o));

        const bool dense_row = (a.flags & BSA_FRAME0_DENSE) && i >= a.f0_first && i <= a.f0_last;
        uint32_t ucut = 0;
        int jcut = 0x7FFFFFFF;  // keep every entry
        if (!dense_row) tp_cut<VPL>(v, Ck, tp.p[h], umax, lane, ws, ucut, jcut);

        const int text_k = (a.flags & BSA_TEXT_KEEP) ? a.text_kblocks : 0;
        uint8_t *mrow = a.mask ? a.mask + row * Ck : nullptr;
        int32_t *irow = a.kv_index + row * Ck;
        const uint32_t lt_mask = (1u << lane) - 1u;
        int base = 0;
#pragma unroll
        for (int s = 0; s < VPL; ++s) {
            const int j = lane + 32 * s;
            const bool real = s < KFULL || j < Ck;
            const uint32_t us = __float_as_uint(v[s]);
            const bool sel = real && (us > ucut || (us == ucut && j <= jcut) || j < text_k);
            if (mrow && real) mrow[j] = sel ? 1 : 0;
            const uint32_t bal = __ballot_sync(0xffffffffu, sel);
            if (sel) irow[base + __popc(bal & lt_mask)] = j;
            base += __popc(bal);
        }
        if (lane == 0) a.kv_count[row] = base;
    }
}

template <int VPL>
cudaError_t launch_topp_t(const MaskArgs &a, const TopP &tp, cudaStream_t st) {
    constexpr int kStep = VPL <= 32 ? 2 : 8;  // the dispatcher's VPL granularity
    constexpr int kFull = VPL - kStep;         // so Ck > 32 * kFull
    auto kern = topp_kernel<VPL, kFull>;
    static int blocks_per_sm = 0;  // the same on every device this library runs on
    if (blocks_per_sm == 0) {
        int nb = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, 128, 0) != cudaSuccess)
            return cudaErrorInvalidValue;
        blocks_per_sm = nb > 0 ? nb : 1;
    }
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidValue;
    const long long want = (a.rows + kTpWarps - 1) / kTpWarps;
    const long long cap = static_cast<long long>(sms) * blocks_per_sm;
    const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
    kern<<<grid, 128, 0, st>>>(a, tp);
    return cudaGetLastError();
}

template <int VPL>
cudaError_t launch_topp_upto(const MaskArgs &a, const TopP &tp, int vpl, cudaStream_t st) {
    if constexpr (VPL < 64) {
        if (vpl > VPL) return launch_topp_upto<VPL < 32 ? VPL + 2 : VPL + 8>(a, tp, vpl, st);
    }
    return launch_topp_t<VPL>(a, tp, st);
}

// Hardware base-2 logarithm (MUFU approximation, relative error ~2^-22).
// EG = false: every row takes its per-row top-p.  EG = true ("Competition
// Domains Matter ..." s3.3 domain 3 and s3's other pooled domains): rows of
// pooled heads keep the pairs of their pool's cut (scores P' * ||c^V|| above the cut pattern, ties at
// it up to the cut row's rank) and, if that leaves them empty, their single
// best key block (the one-key-per-row safeguard); the other rows keep their
// per-row top-p.  Entropies are not computed in that mode.
template <int VPL, bool EG>
__global__ void __launch_bounds__(128, VPL <= 32 ? 7 : 3)
mask_kernel(MaskArgs a, TopP tp) {
    __shared__ __align__(16) WarpScratch s_ws[4];
    const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
    WarpScratch &ws = s_ws[wid];
    {   // clear this warp's table once; every level leaves it cleared
        ulonglong2 *t = reinterpret_cast<ulonglong2 *>(&ws.bins[0][0]);
#pragma unroll
        for (int k = lane; k < kRowsTab * kLanes / 2; k += 32) t[k] = make_ulonglong2(0ull, 0ull);
        __syncwarp();
    }
    const long long row = static_cast<long long>(blockIdx.x) * 4 + wid;
    if (row >= a.rows) return;  // whole warp leaves together
    const int Ck = a.Ck;
    const int i = static_cast<int>(row % a.Cq);
    const int h = static_cast<int>((row / a.Cq) % a.H);
    const float p = tp.p[h];
    const float *src = a.probs + row * Ck;

    // Issue every load before any arithmetic on them.
    float v[VPL];
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int j = lane + 32 * s;
        v[s] = (j < Ck) ? __ldg(src + j) : 0.f;
    }
    const long long bh = row / a.Cq;
    const int pool = EG ? a.pool_of[bh] : -1;
    const bool pooled = pool >= 0;
    float ent = 0.f;
    uint32_t umax = 0;
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const float x = v[s] > 0.f ? v[s] : 0.f;  // -0.0 and NaN become +0.0
        if (!EG && lane + 32 * s < Ck) ent = fmaf(x, lg2_approx(x + a.eps), ent);
        float y = x;
        if (pooled && a.vnorm) {  // the pool's value-aware score, rounded to fp32
            const int j = lane + 32 * s;
            y = (j < Ck) ? __fmul_rn(x, __ldg(a.vnorm + bh * Ck + j)) : 0.f;
            y = y > 0.f ? y : 0.f;
        }
        v[s] = y;
        umax = max(umax, __float_as_uint(y));
    }
    if (!EG && a.row_entropy) {
        ent = -warp_sum(ent) * 0.6931471805599453f;  // ln 2
        if (lane == 0) a.row_entropy[row] = ent;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) umax = max(umax, __shfl_xor_sync(0xffffffffu, umax, o));

    const bool dense_row = (a.flags & BSA_FRAME0_DENSE) && i >= a.f0_first && i <= a.f0_last;
    uint32_t ucut = 0;
    int jcut = 0x7FFFFFFF;  // keep every entry
    if (!dense_row) {
        if (!pooled) {
            find_cut<VPL>(v, src, Ck, p, umax, lane, ws, ucut, jcut);
        } else {
            const PoolState st = a.state[(bh / a.H) * a.G + pool];
            if (!st.keep_all) {
                ucut = st.ucut;
                jcut = row < st.cut_row ? 0x7FFFFFFF
                       : row == st.cut_row ? nth_tie<VPL>(v, Ck, ucut, st.cut_rank, lane)
                                           : -1;
                // safeguard: an empty row keeps its best key block (lowest j on ties)
                bool any = false;
#pragma unroll
                for (int s = 0; s < VPL; ++s) {
                    const int j = lane + 32 * s;
                    const uint32_t us = __float_as_uint(v[s]);
                    any |= j < Ck && (us > ucut || (us == ucut && j <= jcut));
                }
                if (!__any_sync(0xffffffffu, any)) {
                    ucut = umax;
                    jcut = nth_tie<VPL>(v, Ck, umax, 1, lane);
                }
            }
        }
    }

    const int text_k = (a.flags & BSA_TEXT_KEEP) ? a.text_kblocks : 0;
    uint8_t *mrow = a.mask ? a.mask + row * Ck : nullptr;
    int32_t *irow = a.kv_index + row * Ck;
    const uint32_t lt_mask = (1u << lane) - 1u;
    int base = 0;
#pragma unroll
    for (int s = 0; s < VPL; ++s) {
        const int j = lane + 32 * s;
        const uint32_t us = __float_as_uint(v[s]);
        const bool sel = j < Ck && (us > ucut || (us == ucut && j <= jcut) || j < text_k);
        if (mrow && j < Ck) mrow[j] = sel ? 1 : 0;
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

template <int VPL, bool EG>
cudaError_t launch_mask_t(const MaskArgs &a, const TopP &tp, cudaStream_t st) {
    const unsigned grid = static_cast<unsigned>((a.rows + 3) / 4);
    mask_kernel<VPL, EG><<<grid, 128, 0, st>>>(a, tp);
    return cudaGetLastError();
}

template <bool EG>
cudaError_t launch_mask_vpl(const MaskArgs &a, const TopP &tp, int Ck, cudaStream_t st) {
    const int vpl = (Ck + 31) / 32;
    if (vpl <= 4) return launch_mask_t<4, EG>(a, tp, st);
    if (vpl <= 8) return launch_mask_t<8, EG>(a, tp, st);
    if (vpl <= 16) return launch_mask_t<16, EG>(a, tp, st);
    if (vpl <= 32) return launch_mask_t<32, EG>(a, tp, st);
    return launch_mask_t<64, EG>(a, tp, st);
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
    a.vnorm = nullptr;
    a.pool_of = nullptr;
    a.state = nullptr;
    a.G = 0;
    return launch_topp_upto<2>(a, tp, (g.Ck + 31) / 32, st);
}

cudaError_t launch_mask_eg(const Geometry &g, const float *probs, const float *vnorm,
                           const TopP &tp, uint32_t flags, uint8_t *mask, int32_t *kv_index,
                           int32_t *kv_count, const int8_t *pool_of, int G, const PoolState *state,
                           cudaStream_t st) {
    MaskArgs a;
    a.probs = probs;
    a.mask = mask;
    a.kv_index = kv_index;
    a.kv_count = kv_count;
    a.row_entropy = nullptr;
    a.rows = static_cast<long long>(g.B) * g.H * g.Cq;
    a.H = g.H;
    a.Cq = g.Cq;
    a.Ck = g.Ck;
    a.flags = flags;
    a.eps = 0.f;
    a.text_kblocks = g.text_kblocks;
    a.f0_first = g.f0_first;
    a.f0_last = g.f0_last;
    a.vnorm = vnorm;
    a.pool_of = pool_of;
    a.state = state;
    a.G = G;
    return launch_mask_vpl<true>(a, tp, g.Ck, st);
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
