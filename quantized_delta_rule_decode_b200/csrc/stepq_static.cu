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

std::mutex g_mu;
void *g_delta_addr[kMaxDevices];  // device address of g_delta, looked up once per device

// In host code g_delta names a host-side stand-in, not device memory: the
// device address comes from the runtime, once per device, with that device
// current.
int delta_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return stepq::set_error(STEPQ_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return stepq::set_error(STEPQ_ERR_UNSUPPORTED, "device index beyond the static scratch table");
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_delta_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_delta);
        if (e != cudaSuccess || !p)
            return stepq::set_error(STEPQ_ERR_CUDA, "cudaGetSymbolAddress of the static delta array failed");
        g_delta_addr[dev] = p;
    }
    *out = g_delta_addr[dev];
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
