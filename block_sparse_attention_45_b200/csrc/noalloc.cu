// noalloc.cu -- bsa_build_mask_noalloc: bsa_build_mask for callers that cannot
// allocate device memory.
//
// bsa_build_mask needs a device workspace (one fp32 entropy per query-block
// row, summed per head by a second kernel).  Some callers cannot provide one:
// code that runs where cudaMalloc is not allowed or not wanted -- inside a
// framework's custom allocator or memory-planning pass, in a process whose
// device memory is fully reserved up front, or in a plugin whose host owns
// every allocation -- and they have no buffer to lend either.  This variant
// takes the workspace from a fixed array compiled into the library instead,
// so the call allocates nothing.
//
// The array lives in device memory of every GPU that loads the library, for as
// long as the process runs.  Its size caps the problem when entropies are
// requested: batch * heads * (seq_pad / q_block) must not exceed
// BSA_NOALLOC_MAX_MASK_ROWS.  A call that asks for neither entropy nor
// entropy_norm needs no workspace at all, so it neither touches the array nor
// is capped by it.  All calls on one device share the array and it keeps the
// last call's row entropies; every row is written before it is read, so nothing
// needs clearing between calls, but two calls that overlap on the GPU (e.g. on
// two streams without ordering) race on it.
//
// The first call on a device that asks for entropies looks up the array's
// device address with cudaGetSymbolAddress while that device is current, and
// caches it per device together with the id of the current context.  Under
// CUDA's lazy module loading (the default), that lookup is also what loads the
// module holding the array onto the device, so that first call is the one that
// reserves the array's memory: make it before reserving the rest of device
// memory and before capturing a stream into a CUDA graph.  If the context
// changes (a device reset destroys it), the next call repeats the lookup.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "bsa.h"

namespace {

static __device__ __align__(256) float g_mask_row_scratch[BSA_NOALLOC_MAX_MASK_ROWS];

constexpr int kMaxDevices = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

struct DriverFns {
    CtxGetCurrentFn get_current = nullptr;
    CtxGetIdFn get_id = nullptr;
};

const DriverFns &driver_fns() {
    static DriverFns fns;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fns.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fns.get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    return fns;
}

// Id of the calling thread's current context (0 if it cannot be read).
unsigned long long current_context_id() {
    const DriverFns &f = driver_fns();
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!f.get_current || !f.get_id || f.get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

std::mutex g_lock;
void *g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

// Device address of g_mask_row_scratch on the current device (nullptr on error).
void *scratch_for_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    // 0 when no context is current yet; the lookup below makes the device's
    // primary context current, and its id is read again after it.
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> guard(g_lock);
    if (!g_scratch_addr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_mask_row_scratch) != cudaSuccess || !p) return nullptr;
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = current_context_id();
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" int bsa_build_mask_noalloc(const bsa_layout *layout, const float *probs,
                                      const float *top_p, uint32_t flags, float eps,
                                      uint8_t *mask, int32_t *kv_index, int32_t *kv_count,
                                      float *entropy, float *entropy_norm, void *stream) {
    const size_t need = bsa_build_mask_workspace_bytes(layout);  // 0 for an invalid layout
    if (need == 0) return BSA_ERR_INVALID_ARG;
    void *scratch = nullptr;
    if (entropy || entropy_norm) {  // only the entropies use the workspace
        const size_t rows = static_cast<size_t>(layout->batch) * layout->heads *
                            (layout->seq_pad / layout->q_block);
        if (rows > static_cast<size_t>(BSA_NOALLOC_MAX_MASK_ROWS)) return BSA_ERR_UNSUPPORTED;
        scratch = scratch_for_current_device();
        if (!scratch) return BSA_ERR_LAUNCH;
    }
    return bsa_build_mask(layout, probs, top_p, flags, eps, mask, kv_index, kv_count, entropy,
                          entropy_norm, scratch, stream);
}
