// attention.cu -- block-sparse exact attention on sm_100a (TMA + tcgen05 + TMEM).
//
// "Attention matrix view: make only frame-0 query rows dense" s2: a query row
// attends either to every K/V token (dense) or to the selected K/V only
// (sparse); "AB-Attention: accurate block-sparse attention for video
// diffusion" TL;DR: exact attention is computed only on the selected key
// blocks, and key blocks smaller than a tensor-core tile are gathered into
// full tiles.  The output is the exact softmax over the selected keys,
// renormalised over them alone.
//
// Work item = one 128-row query tile (a query block of 128, or a block of 64
// in the upper half of the tile) of one (batch, head).  It walks that block's
// compacted key-block list; skipped blocks cost nothing.  Every list position
// t is one 128-key tile: one key block of 128, or (k_block = 64) the blocks at
// list positions 2t and 2t+1 gathered into the two halves of the tile.
//
// Persistent: one CTA per SM.  Its producer thread claims the next item from a
// global counter (items are ordered head-major, so the CTAs in flight share one
// head's K/V in L2, and a CTA that drew a dense frame-0 row simply claims fewer
// items) and hands it to the other roles through a 4-slot ring in shared
// memory.  Without a counter the CTAs take items blockIdx.x, +gridDim.x, ...
// Barriers, TMEM and tensor-map prefetches are set up once; every pipeline
// phase is carried across items, so item n+1's Q/K/V loads and first QK^T
// products overlap item n's epilogue.  Every wait is bounded (see mbar_wait).
//
// Warp roles (12 warps):
//   warp 0      TMA producer: Q per item, K into a 2-stage ring, V into a 3-stage ring
//   warp 1      tcgen05 issuer (one thread) and TMEM owner (512 columns)
//   warps 4-7   softmax stream 0: list positions 0, 2, 4, ...
//   warps 8-11  softmax stream 1: list positions 1, 3, 5, ...
// Each stream s has S_s (128 fp32 columns; its first 64 are reused for the
// bf16 P of the same tile) and O_s (D fp32 columns) in TMEM, so the tensor
// core computes one stream's QK^T or PV while the other stream's softmax
// runs.  The two partial (O_s, m_s, l_s) are merged in the epilogue.  Each
// softmax thread owns one query row (TMEM lane): row max and row sum need no
// shuffles.  The running max is raised lazily (O_s is rescaled only when it
// grows by more than 2^8), which keeps every P below 256.  Every exponential
// runs on the MUFU unit: moving a share of them to a polynomial on the FMA pipe
// measured slower (the softmax is bound by instruction issue, not by MUFU).
//
// Tensor-core issue order per item: S(0) S(1) | PV(0) S(2) | PV(1) S(3) | ...
// tcgen05 operations of one thread complete in issue order, so
//   * S_s(t+2) may overwrite P_s(t): it is issued after PV(t);
//   * when S_s(t) is complete, the previous PV into O_s is too, so the softmax
//     may rescale O_s as soon as it sees S_s(t).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace bsa {

namespace {

constexpr int kThreads = 384;
// Launch: 168 registers x 384 threads.  Warps 0-3 (producer, MMA issuer, two
// idle warps) give back to kRegsControl; the two softmax warpgroups take the
// rest (56 -> 224 by default): kRegsControl*128 + kRegsSoftmax*256 = 168*384.
#ifndef BSA_REGS_CONTROL
#define BSA_REGS_CONTROL 56
#endif
constexpr uint32_t kRegsControl = BSA_REGS_CONTROL;
constexpr uint32_t kRegsSoftmax = (168 * kThreads - kRegsControl * 128) / 256;
static_assert(kRegsControl * 128 + kRegsSoftmax * 256 == 168 * kThreads, "register split");
static_assert(kRegsControl % 8 == 0 && kRegsSoftmax % 8 == 0, "setmaxnreg takes multiples of 8");
constexpr uint32_t kTmemCols = 512;
// O is rescaled only when a row's max grows by more than 2^8 (P stays below 256).
constexpr float kRescaleLog2 = 8.0f;
constexpr int kPanelBytes = 128 * 128;  // 128 rows x 64 bf16 (one 128-byte swizzle panel)

template <int D>
struct Cfg {
    static constexpr int kPanels = D / 64;
    static constexpr int kTileBytes = kPanels * kPanelBytes;  // 128 rows x D bf16
    // K is released as soon as its QK^T product is done; V only after the PV product
    // that follows the softmax, so V gets the deeper ring.
    static constexpr int kStagesK = (D == 128) ? 2 : 4;
    static constexpr int kStagesV = (D == 128) ? 3 : 4;
    static constexpr int kHeader = 1024;
    static constexpr int kOffStats = kHeader;  // [item parity][m, l][stream][row] floats: 4 KB
    static constexpr int kOffQ = kOffStats + 4096;
    static constexpr int kOffK = kOffQ + kTileBytes;
    static constexpr int kOffV = kOffK + kStagesK * kTileBytes;
    static constexpr int kBytes = kOffV + kStagesV * kTileBytes;
    static constexpr int kSmemAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

struct AttnParams {
    const int32_t *kv_index;  // nullptr: dense (every key block)
    const float *kv_weight;   // with W: the weight of every list entry (exp terms scaled by it)
    const int32_t *kv_count;
    __nv_bfloat16 *out;
    float *lse;
    int32_t *err;
    int *sched;               // work-queue counter (zeroed before launch), or nullptr: static
    long long n_items;
    unsigned long long wait_ns;  // limit of every pipeline wait (the drains keep kWaitTimeoutNs)
    int S, S_pad, Cq, Ck, bq;
    float scale_log2;
};

template <int D>
struct Header {
    uint64_t q_full, q_empty;
    uint64_t k_full[Cfg<D>::kStagesK], k_empty[Cfg<D>::kStagesK];
    uint64_t v_full[Cfg<D>::kStagesV], v_empty[Cfg<D>::kStagesV];
    uint64_t s_full[2], p_full[2];
    uint64_t o_full, o_free;
    uint64_t item_full[4], item_empty[4];  // work-item ring: producer -> MMA + softmax warps
    uint64_t stats_full;                   // both streams' (m, l) of an item are in smem
    uint64_t mma_drain;                    // every product issued has completed (at exit)
    int item_ring[4];
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Header<64>) <= Cfg<64>::kHeader && sizeof(Header<128>) <= Cfg<128>::kHeader,
              "barrier header fits its slot");
constexpr int kItemConsumers = 1 + 8;  // the MMA thread + one arrival per softmax warp

// List entries of a work item, clamped to [0, C_k], and its number of tiles.
template <int BK>
__device__ __forceinline__ void item_lists(const AttnParams &p, long long item,
                                           const int32_t *&entries, int &n_entries, int &n_tiles,
                                           bool &bad_count) {
    entries = p.kv_index ? p.kv_index + item * p.Ck : nullptr;
    n_entries = p.Ck;
    bad_count = false;
    if (p.kv_index) {
        const int c = p.kv_count[item];
        bad_count = c < 0 || c > p.Ck;
        n_entries = min(max(c, 0), p.Ck);
    }
    n_tiles = (BK == 128) ? n_entries : (n_entries + 1) / 2;
}

// Key block of half `hf` of list tile t, and how many of its key columns are
// real (0 for a missing or invalid entry).
template <int BK>
__device__ __forceinline__ void tile_block(const AttnParams &p, const int32_t *entries,
                                           int n_entries, int t, int hf, int &j_load,
                                           int &valid, bool &bad) {
    const int e = (BK == 128) ? t : 2 * t + hf;
    bad = false;
    int j;
    if (e >= n_entries) {  // odd tail of a gathered tile: reuse the first half's block, masked
        const int e0 = 2 * t;
        j = entries ? entries[e0] : e0;
        valid = 0;
    } else {
        j = entries ? entries[e] : e;
        valid = 1;
    }
    if (j < 0 || j >= p.Ck) {
        bad = valid != 0;
        j = 0;
        valid = 0;
    }
    j_load = j;
    if (valid) valid = min(BK, p.S - j * BK);
}

template <int D, int BK, bool W>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using C = Cfg<D>;
    constexpr int NK = C::kStagesK, NV = C::kStagesV;
    constexpr int kHalves = 128 / BK;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Header<D> &hd = *reinterpret_cast<Header<D> *>(smem);
    float *stats = reinterpret_cast<float *>(smem + C::kOffStats);
    uint8_t *sQ = smem + C::kOffQ;
    uint8_t *sK = smem + C::kOffK;
    uint8_t *sV = smem + C::kOffV;
    volatile int *abort_flag = &hd.abort;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        mbar_init(&hd.q_full, 1);
        mbar_init(&hd.q_empty, 1);
        for (int s = 0; s < NK; ++s) {
            mbar_init(&hd.k_full[s], 1);
            mbar_init(&hd.k_empty[s], 1);
        }
        for (int s = 0; s < NV; ++s) {
            mbar_init(&hd.v_full[s], 1);
            mbar_init(&hd.v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&hd.s_full[s], 1);
            mbar_init(&hd.p_full[s], 128);
        }
        mbar_init(&hd.o_full, 1);
        mbar_init(&hd.o_free, 256);
        for (int s = 0; s < 4; ++s) {
            mbar_init(&hd.item_full[s], 1);
            mbar_init(&hd.item_empty[s], kItemConsumers);
        }
        mbar_init(&hd.stats_full, 256);
        mbar_init(&hd.mma_drain, 1);
        hd.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&hd.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (p.bq < 128) {  // rows bq..127 of the Q tile are never loaded: make them zero
        const int per_panel = (128 - p.bq) * 128;
        for (int e = threadIdx.x * 16; e < C::kPanels * per_panel; e += kThreads * 16) {
            const int panel = e / per_panel, off = e % per_panel;
            *reinterpret_cast<uint4 *>(sQ + panel * kPanelBytes + p.bq * 128 + off) =
                make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = hd.tmem_base;
    if (warp < 4) {
    regs_dec<kRegsControl>();
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            // Q tiles and O rows are used once: evict them first, so that L2 keeps the K and
            // V blocks that the head's other query blocks fetch again
            const uint64_t pol_q = policy_evict_first(), pol_kv = policy_evict_last();
            int kt = 0, vt = 0, qn = 0, q_loads = 0;
            bool any_bad = false, any_bad_count = false, stop = false;
            for (;; ++qn) {
                // Claim the next item and publish it (an index >= n_items ends the loop).
                const int slot = qn & 3;
                if (!mbar_wait(&hd.item_empty[slot], ((qn >> 2) & 1) ^ 1, abort_flag, p.wait_ns)) break;
                long long item = p.sched ? static_cast<long long>(atomicAdd(p.sched, 1))
                                         : blockIdx.x + static_cast<long long>(qn) * gridDim.x;
                if (stop || item > p.n_items) item = p.n_items;
                hd.item_ring[slot] = static_cast<int>(item);
                mbar_arrive(&hd.item_full[slot]);
                if (item >= p.n_items || stop) break;
                const int bh = static_cast<int>(item / p.Cq), qi = static_cast<int>(item % p.Cq);
                const int32_t *entries;
                int n_entries, n_tiles;
                bool bad_count;
                item_lists<BK>(p, item, entries, n_entries, n_tiles, bad_count);
                any_bad_count |= bad_count;
                if (!mbar_wait(&hd.q_empty, (qn & 1) ^ 1, abort_flag, p.wait_ns)) {
                    stop = true;
                    continue;   // publishes the end marker next
                }
                mbar_arrive_expect_tx(&hd.q_full, static_cast<uint32_t>(p.bq * D * 2));
                for (int pn = 0; pn < C::kPanels; ++pn)
                    tma_load_3d_hint(sQ + pn * kPanelBytes, &tmQ, &hd.q_full, pn * 64, qi * p.bq, bh, pol_q);
                ++q_loads;
                for (int t = 0; t < n_tiles; ++t) {
                    int jl[kHalves];
#pragma unroll
                    for (int hf = 0; hf < kHalves; ++hf) {
                        int valid;
                        bool bad;
                        tile_block<BK>(p, entries, n_entries, t, hf, jl[hf], valid, bad);
                        any_bad |= bad;
                    }
                    const int ks = kt % NK;
                    if (!mbar_wait(&hd.k_empty[ks], ((kt / NK) & 1) ^ 1, abort_flag, p.wait_ns)) {
                        stop = true;
                        break;
                    }
                    // (an item cut short by an abort still publishes the end marker next)
                    mbar_arrive_expect_tx(&hd.k_full[ks], static_cast<uint32_t>(C::kTileBytes));
#pragma unroll
                    for (int hf = 0; hf < kHalves; ++hf)
                        for (int pn = 0; pn < C::kPanels; ++pn)
                            tma_load_3d_hint(sK + ks * C::kTileBytes + pn * kPanelBytes + hf * BK * 128,
                                             &tmK, &hd.k_full[ks], pn * 64, jl[hf] * BK, bh, pol_kv);
                    ++kt;
                    const int vs = vt % NV;
                    if (!mbar_wait(&hd.v_empty[vs], ((vt / NV) & 1) ^ 1, abort_flag, p.wait_ns)) {
                        stop = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&hd.v_full[vs], static_cast<uint32_t>(C::kTileBytes));
#pragma unroll
                    for (int hf = 0; hf < kHalves; ++hf)
                        for (int pn = 0; pn < C::kPanels; ++pn)
                            tma_load_3d_hint(sV + vs * C::kTileBytes + pn * kPanelBytes + hf * BK * 128,
                                             &tmV, &hd.v_full[vs], pn * 64, jl[hf] * BK, bh, pol_kv);
                    ++vt;
                }
            }
            if (any_bad && p.err) atomicOr(p.err, BSA_DEVERR_BAD_INDEX);
            if (any_bad_count && p.err) atomicOr(p.err, BSA_DEVERR_BAD_COUNT);
            // Drain: every copy this thread started must land before the CTA ends.
            volatile int no_abort = 0;
            if (q_loads > 0) mbar_wait(&hd.q_full, (q_loads - 1) & 1, &no_abort);
            for (int s = 0; s < NK; ++s) {
                const int f = kt / NK + (s < kt % NK ? 1 : 0);
                if (f > 0) mbar_wait(&hd.k_full[s], (f - 1) & 1, &no_abort);
            }
            for (int s = 0; s < NV; ++s) {
                const int f = vt / NV + (s < vt % NV ? 1 : 0);
                if (f > 0) mbar_wait(&hd.v_full[s], (f - 1) & 1, &no_abort);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
            // Descriptor halves: the start address (>> 4) is in the low word, so every
            // K-step below is a compile-time offset added to it.
            const uint64_t q_desc = sw128_desc(smem_u32(sQ), 16, 1024);
            const uint64_t k_desc0 = sw128_desc(smem_u32(sK), 16, 1024);
            const uint64_t v_desc0 = sw128_desc(smem_u32(sV), kPanelBytes, 1024);
            const uint32_t q_lo = static_cast<uint32_t>(q_desc);
            const uint32_t kv_hi_k = static_cast<uint32_t>(k_desc0 >> 32);
            const uint32_t kv_hi_v = static_cast<uint32_t>(v_desc0 >> 32);
            const uint32_t q_hi = static_cast<uint32_t>(q_desc >> 32);
            int kt = 0, vt = 0, qn = 0, pc[2] = {0, 0};
            bool ok = true;
            for (; ok; ++qn) {
                const int slot = qn & 3;
                if (!mbar_wait(&hd.item_full[slot], (qn >> 2) & 1, abort_flag, p.wait_ns)) {
                    ok = false;
                    break;
                }
                const long long item = *reinterpret_cast<volatile int *>(&hd.item_ring[slot]);
                mbar_arrive(&hd.item_empty[slot]);
                if (item >= p.n_items) break;
                const int32_t *entries;
                int n_entries, n_tiles;
                bool bad_count;
                item_lists<BK>(p, item, entries, n_entries, n_tiles, bad_count);
                // S_s(t) = Q K_t^T; frees the K stage, and Q once t is the item's last tile.
                auto issue_s = [&](int t, bool k_ready) -> bool {
                    const int ks = kt % NK;
                    if (!k_ready && !mbar_wait(&hd.k_full[ks], (kt / NK) & 1, abort_flag, p.wait_ns))
                        return false;
                    tc_fence_after();
                    const uint32_t k_lo = static_cast<uint32_t>(k_desc0) +
                                          static_cast<uint32_t>(ks * (C::kTileBytes >> 4));
                    const uint32_t d_tmem = tmem + static_cast<uint32_t>((t & 1) * 128);
                    mma_ss_c<0>(d_tmem, q_lo, q_hi, k_lo, kv_hi_k, idesc_qk);
#pragma unroll
                    for (int kk = 1; kk < D / 16; ++kk) {
                        const uint32_t off = ((kk / 4) * kPanelBytes + (kk % 4) * 32) >> 4;
                        mma_ss_c<1>(d_tmem, q_lo + off, q_hi, k_lo + off, kv_hi_k, idesc_qk);
                    }
                    mma_commit(&hd.k_empty[ks]);
                    mma_commit(&hd.s_full[t & 1]);
                    if (t == n_tiles - 1) mma_commit(&hd.q_empty);
                    ++kt;
                    return true;
                };
                ok = mbar_wait(&hd.q_full, qn & 1, abort_flag, p.wait_ns);
                if (ok && n_tiles == 0) mma_commit(&hd.q_empty);
                if (ok && n_tiles > 0) ok = issue_s(0, false);
                if (ok && n_tiles > 1) ok = issue_s(1, false);
                // O_a / O_b still hold the previous item until its epilogue has read them.
                // Waited for every item (even one without tiles) so that the wait never
                // runs two phases ahead of the epilogues.
                if (ok && qn > 0) ok = mbar_wait(&hd.o_free, (qn - 1) & 1, abort_flag, p.wait_ns);
                for (int t = 0; ok && t < n_tiles; ++t) {
                    const int s = t & 1;
                    // V(t) and K(t+2) normally landed long ago; checking them before P(t)
                    // keeps those barrier round trips off the softmax -> PV path.
                    const int vs = vt % NV;
                    if (!mbar_wait(&hd.v_full[vs], (vt / NV) & 1, abort_flag, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    if (t + 2 < n_tiles &&
                        !mbar_wait(&hd.k_full[kt % NK], (kt / NK) & 1, abort_flag, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(&hd.p_full[s], pc[s] & 1, abort_flag, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    ++pc[s];
                    tc_fence_after();
                    const uint32_t v_lo = static_cast<uint32_t>(v_desc0) +
                                          static_cast<uint32_t>(vs * (C::kTileBytes >> 4));
                    const uint32_t o_tmem = tmem + 256u + static_cast<uint32_t>(s * 128);
                    const uint32_t p_tmem = tmem + static_cast<uint32_t>(s * 128);
                    mma_ts_r(o_tmem, p_tmem, v_lo, kv_hi_v, idesc_pv, t >= 2 ? 1u : 0u);
#pragma unroll
                    for (int kk = 1; kk < 8; ++kk)
                        mma_ts_r(o_tmem, p_tmem + kk * 8, v_lo + ((kk * 2048) >> 4), kv_hi_v,
                                 idesc_pv, 1u);
                    mma_commit(&hd.v_empty[vs]);
                    ++vt;
                    if (t + 2 < n_tiles && !issue_s(t + 2, true)) {
                        ok = false;
                        break;
                    }
                }
                mma_commit(&hd.o_full);
            }
            // Let whatever was issued finish before TMEM is freed, on every exit: after an
            // abort the epilogue may have skipped its wait for the last item's products.
            // A barrier of its own, so that no role waiting on o_full sees an extra phase.
            mma_commit(&hd.mma_drain);
            volatile int no_abort = 0;
            mbar_wait(&hd.mma_drain, 0, &no_abort);
        }
    }
    } else {
        regs_inc<kRegsSoftmax>();
        // ------------------------------------------------------------ softmax streams
        const int s = (warp >> 2) - 1;  // stream
        const int rw = warp & 3;        // TMEM lane quarter
        const int r = rw * 32 + lane;   // query row within the tile
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(rw * 32) << 16);
        const uint32_t t_s = t_lane + static_cast<uint32_t>(s * 128);
        const uint32_t t_o = t_lane + 256u + static_cast<uint32_t>(s * 128);
        int sc = 0, qn = 0;
        bool ok = true;
        for (;; ++qn) {
            const int slot = qn & 3;
            if (!__all_sync(0xffffffffu, mbar_wait(&hd.item_full[slot], (qn >> 2) & 1, abort_flag, p.wait_ns)))
                break;
            const long long item = *reinterpret_cast<volatile int *>(&hd.item_ring[slot]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&hd.item_empty[slot]);
            if (item >= p.n_items) break;
            const int bh = static_cast<int>(item / p.Cq), qi = static_cast<int>(item % p.Cq);
            const int32_t *entries;
            int n_entries, n_tiles;
            bool bad_count;
            item_lists<BK>(p, item, entries, n_entries, n_tiles, bad_count);
            const float *weights = (W && entries) ? p.kv_weight + item * p.Ck : nullptr;
            const int n_s = (n_tiles > s) ? (n_tiles - s + 1) / 2 : 0;
            float m_run = -INFINITY, l_run = 0.f;
            // The list entries (and weights) of this stream's next tile are read one
            // tile ahead (raw block indices; -1 = no block) so their latency is hidden.
            int j_next0 = -1, j_next1 = -1;
            float w_next0 = 1.f, w_next1 = 1.f;
            if (n_s > 0) {
                const int e0 = (BK == 128) ? s : 2 * s;
                j_next0 = entries ? __ldg(entries + e0) : e0;
                if (W && weights) w_next0 = __ldg(weights + e0);
                if (BK != 128 && e0 + 1 < n_entries) {
                    j_next1 = entries ? __ldg(entries + e0 + 1) : e0 + 1;
                    if (W && weights) w_next1 = __ldg(weights + e0 + 1);
                }
            }
            for (int it = 0; ok && it < n_s; ++it) {
                const int t = 2 * it + s;
                const int j0 = j_next0, j1 = j_next1;
                const float w0 = w_next0, w1 = w_next1;
                if (t + 2 < n_tiles) {
                    const int e0 = (BK == 128) ? t + 2 : 2 * (t + 2);
                    j_next0 = entries ? __ldg(entries + e0) : e0;
                    if (W && weights) w_next0 = __ldg(weights + e0);
                    j_next1 = -1;
                    w_next1 = 1.f;
                    if (BK != 128 && e0 + 1 < n_entries) {
                        j_next1 = entries ? __ldg(entries + e0 + 1) : e0 + 1;
                        if (W && weights) w_next1 = __ldg(weights + e0 + 1);
                    }
                }
                // tcgen05.ld/st below are warp-collective: leave together or not at all.
                if (!__all_sync(0xffffffffu, mbar_wait(&hd.s_full[s], sc & 1, abort_flag, p.wait_ns))) {
                    ok = false;
                    break;
                }
                ++sc;
                tc_fence_after();
                uint32_t raw[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(t_s + c * 32, raw[c]);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 4; ++c) reg_fence(raw[c]);
#define X(i) (*reinterpret_cast<float *>(&raw[(i) >> 5][(i) & 31]))
                // Mask key columns past seq_len, and missing / invalid halves.
                int vc[kHalves];
                vc[0] = (j0 >= 0 && j0 < p.Ck) ? min(BK, p.S - j0 * BK) : 0;
                if (kHalves > 1) vc[kHalves - 1] = (j1 >= 0 && j1 < p.Ck) ? min(BK, p.S - j1 * BK) : 0;
                bool partial = false;
#pragma unroll
                for (int hf = 0; hf < kHalves; ++hf) partial |= vc[hf] < BK;
                if (partial) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if ((c % BK) >= vc[c / BK]) X(c) = -INFINITY;
                }
                float mx;
                {
                    float pm[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        pm[k] = fmaxf(X(32 * k), X(32 * k + 1));
#pragma unroll
                        for (int e = 2; e < 32; e += 2) pm[k] = max3(pm[k], X(32 * k + e), X(32 * k + e + 1));
                    }
                    mx = fmaxf(max3(pm[0], pm[1], pm[2]), pm[3]);
                }
                const float m_new = fmaxf(m_run, mx * p.scale_log2);
                // Raise the row's max lazily; O_s is rescaled below, after P is written
                // (the S values are dead by then, so the O round trip has registers).
                float alpha = 1.0f;
                bool rescale = false;
                if (it == 0) {
                    m_run = m_new;
                } else {
                    const bool need = m_new > m_run + kRescaleLog2;
                    rescale = __any_sync(0xffffffffu, need);
                    if (need) {
                        alpha = ex2(m_run - m_new);
                        m_run = m_new;
                    }
                }
                const float nm = (m_run == -INFINITY) ? 0.f : -m_run;
                const float sl = p.scale_log2;
                // Reweighting: w * 2^(s*sl - m) = 2^(s*sl - m + log2 w), one offset per half.
                float nmh0 = nm, nmh1 = nm;
                if (W) {
                    nmh0 = nm + __log2f(w0);
                    nmh1 = (kHalves > 1) ? nm + __log2f(w1) : nmh0;
                }
                float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t pk[16];
                    const float off = (W && kHalves > 1 && c >= 2) ? nmh1 : nmh0;
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float t0, t1, p0, p1;
                        fma2(t0, t1, X(c * 32 + 2 * e), X(c * 32 + 2 * e + 1), sl, sl, off, off);
                        p0 = ex2(t0);
                        p1 = ex2(t1);
                        pk[e] = pack_bf16x2(p0, p1);
                        if (e & 1) add2(b0, b1, b0, b1, p0, p1);
                        else add2(a0, a1, a0, a1, p0, p1);
                    }
                    tmem_st16(t_s + c * 16, pk);
                }
                l_run = l_run * alpha + ((a0 + a1) + (b0 + b1));
#undef X
                if (rescale) {  // O_s *= alpha; PV(t) waits for p_full below, so no race
                    uint32_t o[D / 32][32];
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) tmem_ld32(t_o + c * 32, o[c]);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        reg_fence(o[c]);
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float y0, y1;
                            fma2(y0, y1, __uint_as_float(o[c][e]), __uint_as_float(o[c][e + 1]), alpha,
                                 alpha, 0.f, 0.f);
                            o[c][e] = __float_as_uint(y0);
                            o[c][e + 1] = __float_as_uint(y1);
                        }
                        tmem_st32(t_o + c * 32, o[c]);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&hd.p_full[s]);
            }

            // -------------------------------------------------------- epilogue
            ok = ok && !*abort_flag && mbar_wait(&hd.o_full, qn & 1, abort_flag, p.wait_ns);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            // Exchange (m, l) between the streams.  Double-buffered by item parity: a
            // stream cannot write item n+2's stats before the other stream has read
            // item n's, because item n+2's PV waits for both streams' o_free of n+1.
            float *st = stats + (qn & 1) * 512;
            st[s * 128 + r] = m_run;
            st[256 + s * 128 + r] = l_run;
            mbar_arrive(&hd.stats_full);
            ok = __all_sync(0xffffffffu, mbar_wait(&hd.stats_full, qn & 1, abort_flag, p.wait_ns) && ok);
            const float ma = st[r], mb = st[128 + r];
            const float la = st[256 + r], lb = st[384 + r];
            const float m = fmaxf(ma, mb);
            const float sa = (ma == -INFINITY) ? 0.f : ex2(ma - m);
            const float sb = (mb == -INFINITY) ? 0.f : ex2(mb - m);
            const float L = la * sa + lb * sb;
            const float inv = (L > 0.f) ? 1.0f / L : 0.f;
            const bool has_a = n_tiles > 0, has_b = n_tiles > 1;
            const long long t_abs = static_cast<long long>(qi) * p.bq + r;
            const bool row_out = r < p.bq && t_abs < p.S_pad;
            const bool row_valid = t_abs < p.S;
            const long long grow = static_cast<long long>(bh) * p.S_pad + t_abs;
            // Stream s writes output columns [s*D/2, (s+1)*D/2) of its row.
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                const int col = s * (D / 2) + c * 32;
                uint32_t oa[32], ob[32];
                if (ok && has_a) tmem_ld32(t_lane + 256u + col, oa);
                if (ok && has_b) tmem_ld32(t_lane + 384u + col, ob);
                tmem_ld_wait();
                reg_fence(oa);
                reg_fence(ob);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float v0 = 0.f, v1 = 0.f;
                    if (ok && has_a && row_valid) {
                        v0 = __uint_as_float(oa[2 * e]) * sa;
                        v1 = __uint_as_float(oa[2 * e + 1]) * sa;
                    }
                    if (ok && has_b && row_valid) {
                        v0 = fmaf(__uint_as_float(ob[2 * e]), sb, v0);
                        v1 = fmaf(__uint_as_float(ob[2 * e + 1]), sb, v1);
                    }
                    pk[e] = pack_bf16x2(v0 * inv, v1 * inv);
                }
                if (row_out && ok) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.out + grow * D + col);
                    const uint64_t pol_o = policy_evict_first();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        st_v4_hint(dst + q4, make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]), pol_o);
                }
            }
            tc_fence_before();
            mbar_arrive(&hd.o_free);
            if (s == 0 && row_out && p.lse)
                p.lse[grow] = !row_valid ? -INFINITY
                              : ok       ? (m + __log2f(L)) * 0.69314718055994531f
                                         : NAN;
        }
    }

    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0 && hd.abort && p.err) atomicOr(p.err, BSA_DEVERR_TIMEOUT);
}

// ------------------------------------------------------------------ host side

std::atomic<unsigned long long> g_wait_limit_ns{kWaitTimeoutNs};

unsigned long long attention_wait_limit_ns() { return g_wait_limit_ns.load(); }

// [B*H, S, D] bf16 view with rows >= S out of bounds (loads read zero).
bool make_map(CUtensorMap *m, const void *base, const Geometry &g, int box_rows) {
    TensorMapEncoder enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(g.D), static_cast<cuuint64_t>(g.S),
                                static_cast<cuuint64_t>(g.B) * g.H};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(g.D) * 2,
                                   static_cast<cuuint64_t>(g.S_pad) * g.D * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int BK, bool W>
int launch_t(const Geometry &g, const void *q, const void *k, const void *v,
             const int32_t *kv_index, const float *kv_weight, const int32_t *kv_count,
             float softmax_scale, void *out, float *lse, int32_t *err, void *workspace,
             cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, g, g.bq) || !make_map(&mk, k, g, BK) || !make_map(&mv, v, g, BK))
        return BSA_ERR_DRIVER;
    AttnParams p;
    p.kv_index = kv_index;
    p.kv_weight = kv_weight;
    p.kv_count = kv_count;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.err = err;
    p.sched = static_cast<int *>(workspace);
    p.n_items = static_cast<long long>(g.B) * g.H * g.Cq;
    p.wait_ns = attention_wait_limit_ns();
    p.S = g.S;
    p.S_pad = g.S_pad;
    p.Cq = g.Cq;
    p.Ck = g.Ck;
    p.bq = g.bq;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    const int smem = Cfg<D>::kSmemAlloc;
    if (cudaFuncSetAttribute(attn_kernel<D, BK, W>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
        return BSA_ERR_LAUNCH;
    const int sms = sm_count();
    if (sms <= 0) return BSA_ERR_LAUNCH;
    const long long grid = p.n_items < sms ? p.n_items : sms;
    if (workspace && cudaMemsetAsync(workspace, 0, sizeof(int), st) != cudaSuccess)
        return BSA_ERR_LAUNCH;
    attn_kernel<D, BK, W><<<static_cast<unsigned>(grid), kThreads, smem, st>>>(mq, mk, mv, p);
    return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_LAUNCH;
}

}  // namespace

template <bool W>
int launch_attention_w(const Geometry &g, const void *q, const void *k, const void *v,
                       const int32_t *kv_index, const float *kv_weight, const int32_t *kv_count,
                       float softmax_scale, void *out, float *lse, int32_t *err_flag,
                       void *workspace, cudaStream_t st) {
    if (g.D == 128) {
        return g.bk == 128 ? launch_t<128, 128, W>(g, q, k, v, kv_index, kv_weight, kv_count,
                                                   softmax_scale, out, lse, err_flag, workspace, st)
                           : launch_t<128, 64, W>(g, q, k, v, kv_index, kv_weight, kv_count,
                                                  softmax_scale, out, lse, err_flag, workspace, st);
    }
    return g.bk == 128 ? launch_t<64, 128, W>(g, q, k, v, kv_index, kv_weight, kv_count,
                                              softmax_scale, out, lse, err_flag, workspace, st)
                       : launch_t<64, 64, W>(g, q, k, v, kv_index, kv_weight, kv_count,
                                             softmax_scale, out, lse, err_flag, workspace, st);
}

int launch_attention(const Geometry &g, const void *q, const void *k, const void *v,
                     const int32_t *kv_index, const float *kv_weight, const int32_t *kv_count,
                     float softmax_scale, void *out, float *lse, int32_t *err_flag,
                     void *workspace, cudaStream_t st) {
    if (kv_weight)
        return launch_attention_w<true>(g, q, k, v, kv_index, kv_weight, kv_count, softmax_scale,
                                        out, lse, err_flag, workspace, st);
    return launch_attention_w<false>(g, q, k, v, kv_index, nullptr, kv_count, softmax_scale, out,
                                     lse, err_flag, workspace, st);
}

}  // namespace bsa

extern "C" int bsa_set_wait_limit_ns(unsigned long long ns) {
    bsa::g_wait_limit_ns.store(ns == 0 ? bsa::kWaitTimeoutNs : ns);
    return BSA_OK;
}
