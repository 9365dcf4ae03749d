// stepq_decode_step_static: the whole decode step without any device
// allocation, for callers that cannot call cudaMalloc -- code that runs where
// a caching allocator owns all device memory, code inside a process that must
// not grow its device footprint after start-up, or plain C callers with no
// allocator of their own.  The delta vector the readout kernel hands to the
// fit kernel lives in a fixed array in the library's device memory instead of
// a caller-supplied workspace.
//
// The array below is loaded with the library and stays resident on every GPU
// that loads it until the process exits: 4 MiB per device.  Calls are limited
// to n * n_heads * d_v <= STEPQ_STATIC_DELTA_FLOATS.
#include <cuda.h>

#include <mutex>

#include "stepq_internal.cuh"

namespace {

constexpr size_t kDeltaFloats = STEPQ_STATIC_DELTA_FLOATS;
constexpr size_t kDeltaBytes = kDeltaFloats * sizeof(float);
constexpr int kMaxDevices = 64;

// One delta vector shared by every call on a device.  Each call's readout
// kernel writes every entry its fit kernel reads (a head whose slot index is
// out of range is skipped by both), so nothing has to start at zero.
static __device__ __align__(256) float g_delta[kDeltaFloats];

// In host code g_delta names a host-side stand-in, not device memory: the
// device address comes from the runtime, with the device current.  It is
// looked up once per device and context: a device reset (cudaDeviceReset)
// ends the context the address belonged to, and the next call looks it up
// again in the new one.
struct DeltaAddr {
    unsigned long long ctx_id;
    void *ptr;
};
std::mutex g_mu;
DeltaAddr g_delta_addr[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// The current context's unique id (driver entry points obtained through the
// runtime, so the library links no driver library); false if no context is
// current or the driver lacks the call.
bool current_context_id(unsigned long long *id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
    });
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

int delta_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return stepq::set_error(STEPQ_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return stepq::set_error(STEPQ_ERR_UNSUPPORTED, "device index beyond the static scratch table");
    unsigned long long id = 0;
    const bool have_ctx = current_context_id(&id);
    std::lock_guard<std::mutex> lock(g_mu);
    DeltaAddr &slot = g_delta_addr[dev];
    if (!(have_ctx && slot.ptr && slot.ctx_id == id)) {
        // (this call makes the device's primary context current if none is)
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_delta);
        if (e != cudaSuccess || !p)
            return stepq::set_error(STEPQ_ERR_CUDA, "cudaGetSymbolAddress of the static delta array failed");
        if (!current_context_id(&id))
            return stepq::set_error(STEPQ_ERR_CUDA, "no current CUDA context after the symbol lookup");
        slot.ctx_id = id;
        slot.ptr = p;
    }
    *out = slot.ptr;
    return STEPQ_OK;
}

}  // namespace

extern "C" int stepq_decode_step_static(const stepq_plan *plan, stepq_pool *pool,
                                        const int32_t *slot_idx, int64_t n, int32_t qkv_dtype,
                                        const void *q, const void *k, const void *v,
                                        const float *beta, const float *gate, float *y,
                                        void *main_stream, void *side_stream) {
    size_t need = 0;
    int rc = stepq_workspace_bytes(plan, n, &need);
    if (rc) return rc;
    if (need > kDeltaBytes)
        return stepq::set_error(STEPQ_ERR_INVALID,
                                "n * n_heads * d_v exceeds the static delta array "
                                "(STEPQ_STATIC_DELTA_FLOATS = 1048576 floats); use stepq_decode_step");
    void *delta = nullptr;
    if ((rc = delta_address(&delta))) return rc;
    return stepq_decode_step(plan, pool, slot_idx, n, qkv_dtype, q, k, v, beta, gate, y, delta,
                             kDeltaBytes, main_stream, side_stream);
}
