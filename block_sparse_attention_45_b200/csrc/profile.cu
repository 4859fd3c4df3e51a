// profile.cu -- per-head frame attention scores for autoregressive generation.
//
// "Efficient Autoregressive Video Diffusion with Dummy Head", Step 0: for every
// head, how the current frame's queries spread their attention over (a) the
// sink frame, (b) the neighbor window and (c) the current frame, as a triple
// [alpha_sink, alpha_neighbor, alpha_current] that sums to one.  The key
// window is the layout's num_frames frames (frame 0 the sink, frames
// 1 .. F-2 the neighbors, frame F-1 the current one); the queries are every
// query_stride-th token of the current frame.
//
// The group masses are an attention output: with V_u the one-hot vector of
// key u's group, O_t = sum_u softmax_u(scale q_t . k_u) V_u holds query t's
// three masses in its first three columns.  So the profile runs the block-
// sparse attention kernel (tcgen05, bf16 products, fp32 softmax) with a
// one-hot V, lists that give the current frame's query blocks every key block
// and every other query block none, and then averages the three columns over
// the profiled queries.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace bsa {

namespace {

// V[bh, u, d] = 1 if d is key u's group (0 sink, 1 neighbor, 2 current), else 0;
// rows past the window are zero.  Eight bf16 (16 bytes) per thread.
__global__ void __launch_bounds__(256) onehot_v_kernel(uint4 *__restrict__ v, long long n16, int D,
                                                       int S_pad, int T, int F) {
    const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e >= n16) return;
    const int per_row = D / 8;
    const long long row = e / per_row;
    const int d0 = static_cast<int>(e % per_row) * 8;
    const int u = static_cast<int>(row % S_pad);
    int grp = -1;
    if (u < F * T) {
        const int f = u / T;
        grp = f == 0 ? 0 : (f == F - 1 ? 2 : 1);
    }
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (grp >= d0 && grp < d0 + 8) {
        const int slot = grp - d0;  // bf16 1.0 = 0x3F80
        w[slot / 2] = (slot & 1) ? 0x3F800000u : 0x00003F80u;
    }
    v[e] = make_uint4(w[0], w[1], w[2], w[3]);
}

// Query blocks that hold a profiled query get every key block, the rest none.
__global__ void __launch_bounds__(256) profile_lists_kernel(int32_t *__restrict__ kv_index,
                                                            int32_t *__restrict__ kv_count,
                                                            long long items, int Cq, int Ck,
                                                            int i_first, int i_last) {
    const long long item = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
    if (item >= items) return;
    const int lane = threadIdx.x % 32;
    const int i = static_cast<int>(item % Cq);
    const bool on = i >= i_first && i <= i_last;
    if (on)
        for (int j = lane; j < Ck; j += 32) kv_index[item * Ck + j] = j;
    if (lane == 0) kv_count[item] = on ? Ck : 0;
}

// alpha[bh, g] = mean over the profiled queries of O[bh, t, g], one CTA per (b, h),
// summed per thread in query order and then in thread order.
__global__ void __launch_bounds__(256) alpha_reduce_kernel(const __nv_bfloat16 *__restrict__ out,
                                                           float *__restrict__ alpha, int S_pad,
                                                           int D, int t0, int t1, int stride) {
    __shared__ double part[3][256];
    const long long bh = blockIdx.x;
    double acc[3] = {0.0, 0.0, 0.0};
    int nq = 0;
    for (int t = t0 + threadIdx.x * stride; t < t1; t += blockDim.x * stride) {
        const __nv_bfloat16 *o = out + (bh * S_pad + t) * D;
#pragma unroll
        for (int g = 0; g < 3; ++g) acc[g] += static_cast<double>(__bfloat162float(o[g]));
        ++nq;
    }
#pragma unroll
    for (int g = 0; g < 3; ++g) part[g][threadIdx.x] = acc[g];
    __syncthreads();
    if (threadIdx.x < 3) {
        double s = 0.0;
        for (int k = 0; k < static_cast<int>(blockDim.x); ++k) s += part[threadIdx.x][k];
        const int n = (t1 - t0 + stride - 1) / stride;
        alpha[bh * 3 + threadIdx.x] = n > 0 ? static_cast<float>(s / n) : 0.f;
    }
    (void)nq;
}

size_t al256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

ProfileWorkspace profile_workspace(const Geometry &g) {
    const size_t bh = static_cast<size_t>(g.B) * g.H;
    ProfileWorkspace w;
    size_t off = 0;
    w.v = off;
    off += al256(bh * g.S_pad * g.D * 2);
    w.out = off;
    off += al256(bh * g.S_pad * g.D * 2);
    w.kv_index = off;
    off += al256(bh * g.Cq * g.Ck * sizeof(int32_t));
    w.kv_count = off;
    off += al256(bh * g.Cq * sizeof(int32_t));
    w.sched = off;
    off += al256(kAttnWorkspaceBytes);
    w.bytes = off;
    return w;
}

int launch_frame_scores(const Geometry &g, int T, int F, const void *q, const void *k,
                        float softmax_scale, int query_stride, float *alpha, uint8_t *workspace,
                        cudaStream_t st) {
    const ProfileWorkspace w = profile_workspace(g);
    const long long bh = static_cast<long long>(g.B) * g.H;
    const long long n16 = bh * g.S_pad * (g.D / 8);
    onehot_v_kernel<<<static_cast<unsigned>((n16 + 255) / 256), 256, 0, st>>>(
        reinterpret_cast<uint4 *>(workspace + w.v), n16, g.D, g.S_pad, T, F);
    if (cudaGetLastError() != cudaSuccess) return BSA_ERR_LAUNCH;
    const int t0 = (F - 1) * T, t1 = F * T;
    const long long items = bh * g.Cq;
    int32_t *kv_index = reinterpret_cast<int32_t *>(workspace + w.kv_index);
    int32_t *kv_count = reinterpret_cast<int32_t *>(workspace + w.kv_count);
    profile_lists_kernel<<<static_cast<unsigned>((items + 7) / 8), 256, 0, st>>>(
        kv_index, kv_count, items, g.Cq, g.Ck, t0 / g.bq, (t1 - 1) / g.bq);
    if (cudaGetLastError() != cudaSuccess) return BSA_ERR_LAUNCH;
    void *out = workspace + w.out;
    const int rc = launch_attention(g, q, k, workspace + w.v, kv_index, nullptr, kv_count,
                                    softmax_scale, out, nullptr, nullptr, workspace + w.sched, st);
    if (rc != BSA_OK) return rc;
    alpha_reduce_kernel<<<static_cast<unsigned>(bh), 256, 0, st>>>(
        static_cast<const __nv_bfloat16 *>(out), alpha, g.S_pad, g.D, t0, t1, query_stride);
    return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_LAUNCH;
}

}  // namespace bsa
