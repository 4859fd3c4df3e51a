// internal.h -- launchers shared between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bsa.h"

namespace bsa {

constexpr int kMaxHeads = 256;
constexpr int kMaxScoreCk = 2048;  // bsa_block_scores
constexpr int kMaxMaskCk = 2048;   // bsa_build_mask

struct Geometry {
    int B, H, S, S_pad, D, bq, bk, Cq, Ck;
    int text_kblocks;       // key blocks holding text tokens
    int f0_first, f0_last;  // frame-0 query-block range, f0_last < f0_first when empty
};

Geometry make_geometry(const bsa_layout &L);

// cuTensorMapEncodeTiled, looked up once through the runtime (nullptr if the
// driver lacks it), and the current device's SM count (0 on error).
typedef CUresult (*TensorMapEncoder)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                     const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                     const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
TensorMapEncoder tensor_map_encoder();
int sm_count();

// Host-side validation of a layout shared by every entry point: BSA_OK,
// BSA_ERR_INVALID_ARG or BSA_ERR_UNSUPPORTED.
int check_layout(const bsa_layout *L);

cudaError_t launch_pool(const Geometry &g, const void *q, const void *k, float *qc, float *kc,
                        cudaStream_t st);
cudaError_t launch_scores(const Geometry &g, const float *qc, const float *kc, float *probs,
                          cudaStream_t st);

struct TopP {
    float p[kMaxHeads];
};

cudaError_t launch_mask(const Geometry &g, const float *probs, const TopP &tp, uint32_t flags,
                        float eps, uint8_t *mask, int32_t *kv_index, int32_t *kv_count,
                        float *row_entropy, cudaStream_t st);
cudaError_t launch_entropy_reduce(const Geometry &g, const float *row_entropy, float *entropy,
                                  float *entropy_norm, cudaStream_t st);

// Returns BSA_* status.
int launch_attention(const Geometry &g, const void *q, const void *k, const void *v,
                     const int32_t *kv_index, const int32_t *kv_count, float softmax_scale,
                     void *out, float *lse, int32_t *err_flag, void *workspace, cudaStream_t st);

constexpr size_t kAttnWorkspaceBytes = 256;

}  // namespace bsa
