// pipeline.cu -- bsa_sparse_attention_host: the whole path for host-resident
// Q, K, V and O, with the PCIe copies overlapped with the kernels.
//
// The path is independent per (b, h) ("Competition Domains Matter ..." s3
// domain 1 selects per head and per query row; attention is per head), so the
// heads are cut into groups of `heads_per_group`.  Group c goes through three
// streams:
//
//   h2d stream:      Q, K, V of group c  -> device slot c % 2
//   compute stream:  bsa_block_scores, bsa_build_mask, bsa_attention_fwd on
//                    the slot
//   d2h stream:      O (and per-head entropy, list counts) -> host
//
// with two device slots, so the copy-in of group c+1 and the copy-out of
// group c-1 run while group c computes.  Events order the streams: a slot is
// refilled only after the kernels that read it finished, and recomputed only
// after its previous output left for the host.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "bsa.h"
#include "internal.h"

namespace {

constexpr size_t kAlign = 256;
constexpr int kSlots = 2;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Byte offsets of one slot's buffers for a group of g heads.
struct SlotPlan {
    size_t q, k, v, out, qc, kc, probs, idx, cnt, ent, entn, mask_ws, attn_ws, bytes;
};

SlotPlan plan_slot(const bsa_layout &L, int g) {
    const size_t tok = static_cast<size_t>(g) * L.seq_pad * L.head_dim * 2;  // bf16
    const size_t cq = static_cast<size_t>(L.seq_pad / L.q_block);
    const size_t ck = static_cast<size_t>(L.seq_pad / L.k_block);
    bsa_layout Lg = L;
    Lg.batch = 1;
    Lg.heads = g;
    SlotPlan s;
    size_t off = 0;
    auto take = [&](size_t n) {
        const size_t o = off;
        off += round_up(n);
        return o;
    };
    s.q = take(tok);
    s.k = take(tok);
    s.v = take(tok);
    s.out = take(tok);
    s.qc = take(static_cast<size_t>(g) * cq * L.head_dim * sizeof(float));
    s.kc = take(static_cast<size_t>(g) * ck * L.head_dim * sizeof(float));
    s.probs = take(static_cast<size_t>(g) * cq * ck * sizeof(float));
    s.idx = take(static_cast<size_t>(g) * cq * ck * sizeof(int32_t));
    s.cnt = take(static_cast<size_t>(g) * cq * sizeof(int32_t));
    s.ent = take(static_cast<size_t>(g) * sizeof(float));
    s.entn = take(static_cast<size_t>(g) * sizeof(float));
    s.mask_ws = take(bsa_build_mask_workspace_bytes(&Lg));
    s.attn_ws = take(bsa_attention_workspace_bytes(&Lg));
    s.bytes = off;
    return s;
}

int group_size(const bsa_layout &L, int heads_per_group) {
    return heads_per_group < L.heads ? heads_per_group : L.heads;
}

int check_group(const bsa_layout *L, int heads_per_group) {
    int rc = bsa::check_layout(L);
    if (rc != BSA_OK) return rc;
    if (heads_per_group < 1) return BSA_ERR_INVALID_ARG;
    const bsa::Geometry g = bsa::make_geometry(*L);
    if (g.Ck > bsa::kMaxScoreCk || g.Ck > bsa::kMaxMaskCk) return BSA_ERR_UNSUPPORTED;
    return BSA_OK;
}

struct Events {
    cudaEvent_t start = nullptr, in_ready[kSlots] = {}, done[kSlots] = {}, out_sent[kSlots] = {};
    bool ok = true;
    Events() {
        ok = cudaEventCreateWithFlags(&start, cudaEventDisableTiming) == cudaSuccess;
        for (int s = 0; s < kSlots; ++s) {
            ok = ok && cudaEventCreateWithFlags(&in_ready[s], cudaEventDisableTiming) == cudaSuccess;
            ok = ok && cudaEventCreateWithFlags(&done[s], cudaEventDisableTiming) == cudaSuccess;
            ok = ok && cudaEventCreateWithFlags(&out_sent[s], cudaEventDisableTiming) == cudaSuccess;
        }
    }
    ~Events() {  // pending records are released by the runtime once they complete
        if (start) cudaEventDestroy(start);
        for (int s = 0; s < kSlots; ++s) {
            if (in_ready[s]) cudaEventDestroy(in_ready[s]);
            if (done[s]) cudaEventDestroy(done[s]);
            if (out_sent[s]) cudaEventDestroy(out_sent[s]);
        }
    }
};

}  // namespace

extern "C" {

size_t bsa_pipeline_workspace_bytes(const bsa_layout *layout, int heads_per_group) {
    if (check_group(layout, heads_per_group) != BSA_OK) return 0;
    const SlotPlan s = plan_slot(*layout, group_size(*layout, heads_per_group));
    return kAlign + kSlots * s.bytes;
}

int bsa_sparse_attention_host(const bsa_layout *layout, int heads_per_group, const void *q,
                              const void *k, const void *v, const float *top_p, uint32_t flags,
                              float eps, float softmax_scale, void *out, float *entropy,
                              float *entropy_norm, int32_t *kv_count, int32_t *err_flag,
                              void *workspace, size_t workspace_bytes, void *compute_stream,
                              void *h2d_stream, void *d2h_stream) {
    int rc = check_group(layout, heads_per_group);
    if (rc != BSA_OK) return rc;
    if (!q || !k || !v || !out || !top_p || !workspace) return BSA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign != 0) return BSA_ERR_INVALID_ARG;
    if (workspace_bytes < bsa_pipeline_workspace_bytes(layout, heads_per_group))
        return BSA_ERR_INVALID_ARG;
    if (flags & ~static_cast<uint32_t>(BSA_TEXT_KEEP | BSA_FRAME0_DENSE)) return BSA_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !(eps < 1e30f)) return BSA_ERR_INVALID_ARG;
    if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f)) return BSA_ERR_INVALID_ARG;
    for (int h = 0; h < layout->heads; ++h)
        if (top_p[h] != top_p[h]) return BSA_ERR_INVALID_ARG;  // NaN

    const bsa_layout &L = *layout;
    const int G = group_size(L, heads_per_group);
    const int groups_per_batch = (L.heads + G - 1) / G;
    const int n_groups = L.batch * groups_per_batch;
    const SlotPlan plan = plan_slot(L, G);
    const int cq = L.seq_pad / L.q_block;
    const size_t head_bytes = static_cast<size_t>(L.seq_pad) * L.head_dim * 2;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int32_t *d_err = reinterpret_cast<int32_t *>(ws);
    auto slot_base = [&](int s) { return ws + kAlign + static_cast<size_t>(s) * plan.bytes; };

    cudaStream_t cs = static_cast<cudaStream_t>(compute_stream);
    cudaStream_t hs = static_cast<cudaStream_t>(h2d_stream);
    cudaStream_t ds = static_cast<cudaStream_t>(d2h_stream);
    Events ev;
    if (!ev.ok) return BSA_ERR_LAUNCH;
    auto ck = [](cudaError_t e) { return e == cudaSuccess; };
    // Everything below runs after what the caller queued on the compute stream.
    if (!ck(cudaMemsetAsync(d_err, 0, sizeof(int32_t), cs)) || !ck(cudaEventRecord(ev.start, cs)) ||
        !ck(cudaStreamWaitEvent(hs, ev.start, 0)) || !ck(cudaStreamWaitEvent(ds, ev.start, 0)))
        return BSA_ERR_LAUNCH;

    for (int c = 0; c < n_groups; ++c) {
        const int b = c / groups_per_batch;
        const int h0 = (c % groups_per_batch) * G;
        const int g = (L.heads - h0) < G ? (L.heads - h0) : G;
        const int s = c % kSlots;
        uint8_t *base = slot_base(s);
        const size_t first_head = static_cast<size_t>(b) * L.heads + h0;
        const size_t off = first_head * head_bytes;
        const size_t bytes = static_cast<size_t>(g) * head_bytes;
        bsa_layout Lg = L;
        Lg.batch = 1;
        Lg.heads = g;

        // copy in, once the kernels that last read this slot are done
        if (c >= kSlots && !ck(cudaStreamWaitEvent(hs, ev.done[s], 0))) return BSA_ERR_LAUNCH;
        if (!ck(cudaMemcpyAsync(base + plan.q, static_cast<const uint8_t *>(q) + off, bytes,
                                cudaMemcpyHostToDevice, hs)) ||
            !ck(cudaMemcpyAsync(base + plan.k, static_cast<const uint8_t *>(k) + off, bytes,
                                cudaMemcpyHostToDevice, hs)) ||
            !ck(cudaMemcpyAsync(base + plan.v, static_cast<const uint8_t *>(v) + off, bytes,
                                cudaMemcpyHostToDevice, hs)) ||
            !ck(cudaEventRecord(ev.in_ready[s], hs)))
            return BSA_ERR_LAUNCH;

        // compute, once the inputs landed and the slot's previous output left
        if (!ck(cudaStreamWaitEvent(cs, ev.in_ready[s], 0))) return BSA_ERR_LAUNCH;
        if (c >= kSlots && !ck(cudaStreamWaitEvent(cs, ev.out_sent[s], 0))) return BSA_ERR_LAUNCH;
        float *qc = reinterpret_cast<float *>(base + plan.qc);
        float *kc = reinterpret_cast<float *>(base + plan.kc);
        float *probs = reinterpret_cast<float *>(base + plan.probs);
        int32_t *idx = reinterpret_cast<int32_t *>(base + plan.idx);
        int32_t *cnt = reinterpret_cast<int32_t *>(base + plan.cnt);
        float *ent = reinterpret_cast<float *>(base + plan.ent);
        float *entn = reinterpret_cast<float *>(base + plan.entn);
        rc = bsa_block_scores(&Lg, base + plan.q, base + plan.k, qc, kc, probs, cs);
        if (rc != BSA_OK) return rc;
        rc = bsa_build_mask(&Lg, probs, top_p + h0, flags, eps, nullptr, idx, cnt, ent, entn,
                            base + plan.mask_ws, cs);
        if (rc != BSA_OK) return rc;
        rc = bsa_attention_fwd(&Lg, base + plan.q, base + plan.k, base + plan.v, idx, cnt,
                               softmax_scale, base + plan.out, nullptr, d_err, base + plan.attn_ws,
                               cs);
        if (rc != BSA_OK) return rc;
        if (!ck(cudaEventRecord(ev.done[s], cs))) return BSA_ERR_LAUNCH;

        // copy out
        if (!ck(cudaStreamWaitEvent(ds, ev.done[s], 0)) ||
            !ck(cudaMemcpyAsync(static_cast<uint8_t *>(out) + off, base + plan.out, bytes,
                                cudaMemcpyDeviceToHost, ds)))
            return BSA_ERR_LAUNCH;
        if (entropy && !ck(cudaMemcpyAsync(entropy + first_head, ent, g * sizeof(float),
                                           cudaMemcpyDeviceToHost, ds)))
            return BSA_ERR_LAUNCH;
        if (entropy_norm && !ck(cudaMemcpyAsync(entropy_norm + first_head, entn, g * sizeof(float),
                                                cudaMemcpyDeviceToHost, ds)))
            return BSA_ERR_LAUNCH;
        if (kv_count && !ck(cudaMemcpyAsync(kv_count + first_head * cq, cnt,
                                            static_cast<size_t>(g) * cq * sizeof(int32_t),
                                            cudaMemcpyDeviceToHost, ds)))
            return BSA_ERR_LAUNCH;
        if (!ck(cudaEventRecord(ev.out_sent[s], ds))) return BSA_ERR_LAUNCH;
    }
    // The compute stream ends after the last copy-out, so waiting on it (or on
    // an event recorded on it) covers the whole call.
    for (int s = 0; s < kSlots && s < n_groups; ++s)
        if (!ck(cudaStreamWaitEvent(cs, ev.out_sent[s], 0))) return BSA_ERR_LAUNCH;
    if (err_flag && !ck(cudaMemcpyAsync(err_flag, d_err, sizeof(int32_t), cudaMemcpyDeviceToHost, cs)))
        return BSA_ERR_LAUNCH;
    return BSA_OK;
}

}  // extern "C"
