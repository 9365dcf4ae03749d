// Internal definitions shared by the host API and the kernels of libstepq.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/stepq.h"

namespace stepq {

// How a head is stored.
enum : uint8_t {
    HK_UNIFORM = 0,  // every key row quantised at one width (head units)
    HK_MIXED = 1,    // per-key-row widths, possibly with FP16 pivot rows (row units)
    HK_PIVOT = 2,    // the whole head is an FP16 pivot: d_k*d_v raw halves
};

// Device-side view of a plan; passed by value to every kernel.
struct PlanDev {
    int dk, dv, H, gate_kind, unit_kind, mode;
    uint32_t slot_bytes;
    uint32_t max_head_bytes;
    const uint32_t *head_off;    // [H] byte offset of the head blob in a slot
    const uint32_t *head_bytes;  // [H] blob size (multiple of 16)
    const uint32_t *scale_off;   // [H] offset of rho[dk]; c[dv] follows
    const uint8_t *head_kind;    // [H] HK_*
    const uint8_t *head_bits;    // [H] width of a HK_UNIFORM head
    const uint8_t *row_bits;     // [H*dk] 4/6/8/16
    const uint16_t *row_off;     // [H*dk] offset of the row inside the blob
    const float *w;              // [H*dk] row-impact weights
    const float *kappa;          // [H*dk] qmax_hi / qmax_i (1 for one-width heads)
    const float *qmax_hi;        // [H] largest qmax over the head's quantised rows
    int n_qheads, n_pheads;      // quantised heads, FP16 pivot heads
    uint32_t max_qhead_bytes;    // largest blob of a quantised (non-pivot) head
    const int16_t *qheads;       // [n_qheads] indices of the quantised heads
    const int16_t *pheads;       // [n_pheads] indices of the FP16 pivot heads
    const uint8_t *chunk_rows;   // [H] rows per staged chunk of the readout (readout_chunk_rows)
};

// The readout stages a head's packed rows into shared memory in chunks of
// whole rows, at most 32 * d bytes each (4 KB at d = 128): the largest power
// of two of rows, at most d, whose widest row fits that many times.
__host__ __device__ constexpr int readout_chunk_rows(int d, int max_row_bytes) {
    int r = d;
    while (r > 1 && r * max_row_bytes > 32 * d) r >>= 1;
    return r;
}

// Everything a decode / pack launch needs besides the plan.
struct StepArgs {
    const uint8_t *pool_ro;
    uint8_t *pool;
    int64_t num_slots;
    const int32_t *slot_idx;
    int64_t n;
    const void *q, *k, *v;
    const float *beta, *gate;
    float *y;
    float *delta;      // workspace [n][H][dv]
    const float *X;    // pack input [n][H][dk][dv]
    float *S_out;      // unpack output
    double *dist;      // per-unit distortion output [n][units], or [units] summed (dist_accumulate)
    int dist_accumulate;
    uint32_t *status;
    uint32_t test_faults;   // STEPQ_TEST_* bits (0 in normal operation)
    uint64_t wait_limit_ns; // bound on each device wait
};

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s

// ---- launchers (stepq_kernels.cu) ------------------------------------------
cudaError_t launch_readout(const PlanDev &P, const StepArgs &a, int qkv_dtype, cudaStream_t s);
cudaError_t launch_fitpack(const PlanDev &P, const StepArgs &a, int qkv_dtype, cudaStream_t s);
cudaError_t launch_pack(const PlanDev &P, const StepArgs &a, cudaStream_t s);
cudaError_t launch_unpack(const PlanDev &P, const StepArgs &a, cudaStream_t s);
cudaError_t launch_distortion(const PlanDev &P, const StepArgs &a, cudaStream_t s);
cudaError_t launch_row_impact(int d, int H, int gate_kind, int qkv, int64_t n, const void *q,
                              const void *k, const float *beta, const float *gate, double *score,
                              cudaStream_t s);
cudaError_t launch_fp32_step(int d, int H, int gate_kind, int qkv_dtype, float *S, int64_t num_slots,
                             const int32_t *slot_idx, int64_t n, const void *q, const void *k,
                             const void *v, const float *beta, const float *gate, float *y,
                             uint32_t *status, cudaStream_t s);


// Record an error message for stepq_last_error(); returns code.
int set_error(int code, const char *msg);
size_t quant_smem_bytes(int d);

}  // namespace stepq
