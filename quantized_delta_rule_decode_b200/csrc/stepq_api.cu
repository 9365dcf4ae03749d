// C ABI of libstepq: plan and pool objects, argument checks, stream/event
// plumbing of the two-kernel decode step, and launches.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>

#include <string>
#include <vector>

#include "stepq_internal.cuh"

struct stepq_plan {
    int device = -1;
    int dk = 0, dv = 0, H = 0, gate_kind = 0, unit_kind = 0, mode = 0;
    size_t slot_bytes = 0;
    uint32_t max_head_bytes = 0;
    std::vector<uint32_t> head_off, head_bytes, scale_off;
    std::vector<uint8_t> head_kind, head_bits, row_bits;
    std::vector<uint16_t> row_off;
    std::vector<float> w, kappa, qmax_hi;
    std::vector<int16_t> qheads, pheads;
    std::vector<uint8_t> chunk_rows;
    uint32_t max_qhead_bytes = 0;
    void *dev_tables = nullptr;
    stepq::PlanDev dev{};
};

struct stepq_pool {
    const stepq_plan *plan = nullptr;
    int device = -1;
    int64_t num_slots = 0;
    uint8_t *base = nullptr;
    uint32_t *status = nullptr;
    cudaEvent_t readout_done = nullptr;
    cudaEvent_t fit_done = nullptr;
    bool fit_pending = false;
    uint32_t test_faults = 0;
    uint64_t wait_limit_ns = stepq::kDefaultWaitLimitNs;
    // the host-buffer entry's copy streams and events, created on its first call
    cudaStream_t copy_in = nullptr, copy_out = nullptr;
    cudaEvent_t in_done = nullptr, y_ready = nullptr, y_done = nullptr;
};

namespace {

thread_local std::string g_err;

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(STEPQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int check_device(int want) {
    int cur = -1;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (cur != want)
        return fail(STEPQ_ERR_INVALID, "object belongs to device %d but device %d is current", want, cur);
    return STEPQ_OK;
}

int check_pool(const stepq_plan *plan, const stepq_pool *pool) {
    if (!plan || !pool) return fail(STEPQ_ERR_INVALID, "plan and pool must be non-NULL");
    if (pool->plan != plan) return fail(STEPQ_ERR_INVALID, "pool was created for another plan");
    return check_device(plan->device);
}

int check_rows(const stepq_plan *plan, const int32_t *slot_idx, int64_t n) {
    if (n < 0) return fail(STEPQ_ERR_INVALID, "n must be >= 0");
    if (n > 0 && !slot_idx) return fail(STEPQ_ERR_INVALID, "slot_idx is NULL");
    if (n * (int64_t)plan->H > (int64_t)0x7fffffff)
        return fail(STEPQ_ERR_INVALID, "n * n_heads exceeds the grid limit");
    return STEPQ_OK;
}

int check_inputs(const void *p, const char *name) {
    if (!p) return fail(STEPQ_ERR_INVALID, "%s is NULL", name);
    if (!aligned16(p)) return fail(STEPQ_ERR_INVALID, "%s is not 16-byte aligned", name);
    return STEPQ_OK;
}

stepq::StepArgs base_args(const stepq_plan *plan, stepq_pool *pool, const int32_t *slot_idx,
                          int64_t n) {
    stepq::StepArgs a{};
    a.pool_ro = pool->base;
    a.pool = pool->base;
    a.num_slots = pool->num_slots;
    a.slot_idx = slot_idx;
    a.n = n;
    a.status = pool->status;
    a.test_faults = pool->test_faults;
    a.wait_limit_ns = pool->wait_limit_ns;
    (void)plan;
    return a;
}

// The host-buffer entry's two copy streams and three events, created with
// the pool on its device (the entry checks again, in case creation failed).
int host_streams(stepq_pool *pool) {
    if (pool->y_done) return STEPQ_OK;
    cudaError_t e = cudaSuccess;
    if (!pool->copy_in) e = cudaStreamCreateWithFlags(&pool->copy_in, cudaStreamNonBlocking);
    if (e == cudaSuccess && !pool->copy_out) e = cudaStreamCreateWithFlags(&pool->copy_out, cudaStreamNonBlocking);
    if (e == cudaSuccess && !pool->in_done) e = cudaEventCreateWithFlags(&pool->in_done, cudaEventDisableTiming);
    if (e == cudaSuccess && !pool->y_ready) e = cudaEventCreateWithFlags(&pool->y_ready, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&pool->y_done, cudaEventDisableTiming);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "copy streams");
}

// Make `stream` wait for a fit still pending on the pool's slots.
int wait_pending_fit(stepq_pool *pool, cudaStream_t s) {
    if (!pool->fit_pending) return STEPQ_OK;
    cudaError_t e = cudaStreamWaitEvent(s, pool->fit_done, 0);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
    return STEPQ_OK;
}

}  // namespace

namespace stepq {
int set_error(int code, const char *msg) { return fail(code, "%s", msg); }
}  // namespace stepq

extern "C" {

const char *stepq_last_error(void) { return g_err.c_str(); }

int stepq_plan_create(const stepq_plan_desc *desc, stepq_plan **out) {
    g_err.clear();
    if (!out) return fail(STEPQ_ERR_INVALID, "out is NULL");
    *out = nullptr;
    if (!desc) return fail(STEPQ_ERR_INVALID, "desc is NULL");
    const stepq_plan_desc &d = *desc;
    if (d.d_k <= 0 || d.d_v <= 0 || d.n_heads <= 0)
        return fail(STEPQ_ERR_INVALID, "d_k, d_v, n_heads must be positive");
    if (d.gate_kind != STEPQ_GATE_SCALAR && d.gate_kind != STEPQ_GATE_DIAG)
        return fail(STEPQ_ERR_INVALID, "gate_kind %d unknown", d.gate_kind);
    if (d.unit_kind != STEPQ_UNIT_HEAD && d.unit_kind != STEPQ_UNIT_ROW)
        return fail(STEPQ_ERR_INVALID, "unit_kind %d unknown", d.unit_kind);
    if (d.mode != STEPQ_MODE_STEPQUANT && d.mode != STEPQ_MODE_UNIFORM)
        return fail(STEPQ_ERR_INVALID, "mode %d unknown", d.mode);
    if (!d.bits || !d.w) return fail(STEPQ_ERR_INVALID, "bits and w must be non-NULL");
    const int H = d.n_heads, dk = d.d_k, dv = d.d_v;
    const size_t units = d.unit_kind == STEPQ_UNIT_HEAD ? (size_t)H : (size_t)H * dk;
    for (size_t u = 0; u < units; ++u) {
        const int b = d.bits[u];
        if (b != 4 && b != 6 && b != 8 && b != 16)
            return fail(STEPQ_ERR_INVALID, "bits[%zu] = %d, expected 4, 6, 8 or 16", u, b);
    }
    for (size_t i = 0; i < (size_t)H * dk; ++i)
        if (!(d.w[i] > 0.0f) || isinf(d.w[i]))
            return fail(STEPQ_ERR_INVALID, "w[%zu] must be finite and > 0", i);
    if (dk != dv || (dk != 64 && dk != 128))
        return fail(STEPQ_ERR_UNSUPPORTED, "the library runs d_k == d_v in {64, 128} (got %d x %d)", dk, dv);

    stepq_plan *p = new stepq_plan();
    p->dk = dk; p->dv = dv; p->H = H;
    p->gate_kind = d.gate_kind; p->unit_kind = d.unit_kind; p->mode = d.mode;
    p->head_off.resize(H); p->head_bytes.resize(H); p->scale_off.resize(H);
    p->head_kind.resize(H); p->head_bits.resize(H); p->qmax_hi.resize(H);
    p->row_bits.resize((size_t)H * dk); p->row_off.resize((size_t)H * dk);
    p->w.assign(d.w, d.w + (size_t)H * dk);
    p->kappa.resize((size_t)H * dk);
    p->chunk_rows.resize(H);
    size_t off = 0;
    for (int h = 0; h < H; ++h) {
        bool all_same = true, any_pivot = false;
        int qhi = 0;
        for (int i = 0; i < dk; ++i) {
            const int b = d.unit_kind == STEPQ_UNIT_HEAD ? d.bits[h] : d.bits[(size_t)h * dk + i];
            p->row_bits[(size_t)h * dk + i] = (uint8_t)b;
            if (b != p->row_bits[(size_t)h * dk]) all_same = false;
            if (b == 16) any_pivot = true;
            else qhi = std::max(qhi, (1 << (b - 1)) - 1);
        }
        const bool pivot_head = d.unit_kind == STEPQ_UNIT_HEAD && d.bits[h] == 16;
        p->head_kind[h] = pivot_head ? stepq::HK_PIVOT
                          : (all_same && !any_pivot) ? stepq::HK_UNIFORM : stepq::HK_MIXED;
        p->head_bits[h] = p->row_bits[(size_t)h * dk];
        p->qmax_hi[h] = (float)qhi;
        size_t hb = 0;
        for (int i = 0; i < dk; ++i) {
            const int b = p->row_bits[(size_t)h * dk + i];
            p->row_off[(size_t)h * dk + i] = (uint16_t)hb;
            hb += b == 16 ? (size_t)dv * 2 : (size_t)dv * b / 8;
            p->kappa[(size_t)h * dk + i] =
                b == 16 ? 0.0f : (float)qhi / (float)((1 << (b - 1)) - 1);
        }
        p->scale_off[h] = (uint32_t)hb;
        int widest = 0;
        for (int i = 0; i < dk; ++i) {
            const int b = p->row_bits[(size_t)h * dk + i];
            widest = std::max(widest, b == 16 ? 2 * dv : dv * b / 8);
        }
        p->chunk_rows[h] = (uint8_t)stepq::readout_chunk_rows(dk, widest);
        if (pivot_head) {
            p->pheads.push_back((int16_t)h);
        } else {
            hb += (size_t)dk * 2 + (size_t)dv * 2;
            p->qheads.push_back((int16_t)h);
            p->max_qhead_bytes = std::max<uint32_t>(p->max_qhead_bytes, (uint32_t)round_up(hb, 16));
        }
        hb = round_up(hb, 16);
        p->head_off[h] = (uint32_t)off;
        p->head_bytes[h] = (uint32_t)hb;
        p->max_head_bytes = std::max<uint32_t>(p->max_head_bytes, (uint32_t)hb);
        off += hb;
    }
    p->slot_bytes = round_up(off, 256);
    if (p->slot_bytes > 0xffffffffu) {
        delete p;
        return fail(STEPQ_ERR_UNSUPPORTED, "slot of %zu bytes is too large", off);
    }

    // one device allocation holds every table
    const size_t HD = (size_t)H * dk;
    size_t o_head_off = 0, o_head_bytes = o_head_off + 4 * H, o_scale_off = o_head_bytes + 4 * H;
    size_t o_kind = o_scale_off + 4 * H, o_hbits = o_kind + H, o_rbits = o_hbits + H;
    size_t o_roff = round_up(o_rbits + HD, 16), o_w = round_up(o_roff + 2 * HD, 16);
    size_t o_kap = o_w + 4 * HD, o_qhi = o_kap + 4 * HD;
    size_t o_qh = round_up(o_qhi + 4 * H, 16), o_ph = round_up(o_qh + 2 * H, 16);
    size_t o_chunk = round_up(o_ph + 2 * H, 16);
    size_t total = o_chunk + H;
    std::vector<uint8_t> host(total, 0);
    memcpy(&host[o_head_off], p->head_off.data(), 4 * H);
    memcpy(&host[o_head_bytes], p->head_bytes.data(), 4 * H);
    memcpy(&host[o_scale_off], p->scale_off.data(), 4 * H);
    memcpy(&host[o_kind], p->head_kind.data(), H);
    memcpy(&host[o_hbits], p->head_bits.data(), H);
    memcpy(&host[o_rbits], p->row_bits.data(), HD);
    memcpy(&host[o_roff], p->row_off.data(), 2 * HD);
    memcpy(&host[o_w], p->w.data(), 4 * HD);
    memcpy(&host[o_kap], p->kappa.data(), 4 * HD);
    memcpy(&host[o_qhi], p->qmax_hi.data(), 4 * H);
    if (!p->qheads.empty()) memcpy(&host[o_qh], p->qheads.data(), 2 * p->qheads.size());
    if (!p->pheads.empty()) memcpy(&host[o_ph], p->pheads.data(), 2 * p->pheads.size());
    memcpy(&host[o_chunk], p->chunk_rows.data(), H);
    cudaError_t e = cudaGetDevice(&p->device);
    if (e == cudaSuccess) e = cudaMalloc(&p->dev_tables, total);
    if (e == cudaSuccess) e = cudaMemcpy(p->dev_tables, host.data(), total, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        if (p->dev_tables) cudaFree(p->dev_tables);
        delete p;
        return cuda_fail(e, "plan tables");
    }
    uint8_t *t = static_cast<uint8_t *>(p->dev_tables);
    stepq::PlanDev &v = p->dev;
    v.dk = dk; v.dv = dv; v.H = H; v.gate_kind = d.gate_kind; v.unit_kind = d.unit_kind;
    v.mode = d.mode;
    v.slot_bytes = (uint32_t)p->slot_bytes;
    v.max_head_bytes = p->max_head_bytes;
    v.head_off = reinterpret_cast<const uint32_t *>(t + o_head_off);
    v.head_bytes = reinterpret_cast<const uint32_t *>(t + o_head_bytes);
    v.scale_off = reinterpret_cast<const uint32_t *>(t + o_scale_off);
    v.head_kind = t + o_kind;
    v.head_bits = t + o_hbits;
    v.row_bits = t + o_rbits;
    v.row_off = reinterpret_cast<const uint16_t *>(t + o_roff);
    v.w = reinterpret_cast<const float *>(t + o_w);
    v.kappa = reinterpret_cast<const float *>(t + o_kap);
    v.qmax_hi = reinterpret_cast<const float *>(t + o_qhi);
    v.n_qheads = (int)p->qheads.size();
    v.n_pheads = (int)p->pheads.size();
    v.max_qhead_bytes = p->max_qhead_bytes;
    v.qheads = reinterpret_cast<const int16_t *>(t + o_qh);
    v.pheads = reinterpret_cast<const int16_t *>(t + o_ph);
    v.chunk_rows = t + o_chunk;
    *out = p;
    return STEPQ_OK;
}

int stepq_plan_destroy(stepq_plan *plan) {
    g_err.clear();
    if (!plan) return STEPQ_OK;
    if (plan->dev_tables) cudaFree(plan->dev_tables);
    delete plan;
    return STEPQ_OK;
}

int stepq_plan_slot_bytes(const stepq_plan *plan, size_t *out) {
    if (!plan || !out) return fail(STEPQ_ERR_INVALID, "plan and out must be non-NULL");
    *out = plan->slot_bytes;
    return STEPQ_OK;
}

int stepq_plan_head_layout(const stepq_plan *plan, int32_t head, size_t *offset, size_t *bytes) {
    if (!plan || !offset || !bytes) return fail(STEPQ_ERR_INVALID, "NULL argument");
    if (head < 0 || head >= plan->H) return fail(STEPQ_ERR_INVALID, "head %d out of range", head);
    *offset = plan->head_off[head];
    *bytes = plan->head_bytes[head];
    return STEPQ_OK;
}

int stepq_pool_alloc(const stepq_plan *plan, int64_t num_slots, void *dev_buf, size_t buf_bytes,
                     stepq_pool **out) {
    g_err.clear();
    if (!out) return fail(STEPQ_ERR_INVALID, "out is NULL");
    *out = nullptr;
    if (!plan) return fail(STEPQ_ERR_INVALID, "plan is NULL");
    if (num_slots <= 0) return fail(STEPQ_ERR_INVALID, "num_slots must be positive");
    if (num_slots > 0x7fffffff) return fail(STEPQ_ERR_INVALID, "num_slots exceeds int32 slot indices");
    if (!dev_buf) return fail(STEPQ_ERR_INVALID, "dev_buf is NULL");
    if (reinterpret_cast<uintptr_t>(dev_buf) & 255u)
        return fail(STEPQ_ERR_INVALID, "dev_buf must be 256-byte aligned");
    if ((size_t)num_slots > buf_bytes / plan->slot_bytes)
        return fail(STEPQ_ERR_INVALID, "buffer of %zu bytes holds fewer than %lld slots of %zu bytes",
                    buf_bytes, (long long)num_slots, plan->slot_bytes);
    int rc = check_device(plan->device);
    if (rc) return rc;
    stepq_pool *p = new stepq_pool();
    p->plan = plan;
    p->device = plan->device;
    p->num_slots = num_slots;
    p->base = static_cast<uint8_t *>(dev_buf);
    cudaError_t e = cudaMalloc(&p->status, 256);
    if (e == cudaSuccess) e = cudaMemset(p->status, 0, 256);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->readout_done, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->fit_done, cudaEventDisableTiming);
    if (e != cudaSuccess) {
        if (p->status) cudaFree(p->status);
        if (p->readout_done) cudaEventDestroy(p->readout_done);
        delete p;
        return cuda_fail(e, "pool status/events");
    }
    // the host-buffer entry's copy streams, made here so that no call of it
    // pays for their creation
    int rc2 = host_streams(p);
    if (rc2) {
        const std::string msg = g_err;   // stepq_pool_free clears the message
        stepq_pool_free(p);
        g_err = msg;
        return rc2;
    }
    *out = p;
    return STEPQ_OK;
}

int stepq_pool_free(stepq_pool *pool) {
    g_err.clear();
    if (!pool) return STEPQ_OK;
    if (pool->status) cudaFree(pool->status);
    if (pool->readout_done) cudaEventDestroy(pool->readout_done);
    if (pool->fit_done) cudaEventDestroy(pool->fit_done);
    if (pool->copy_in) cudaStreamDestroy(pool->copy_in);
    if (pool->copy_out) cudaStreamDestroy(pool->copy_out);
    if (pool->in_done) cudaEventDestroy(pool->in_done);
    if (pool->y_ready) cudaEventDestroy(pool->y_ready);
    if (pool->y_done) cudaEventDestroy(pool->y_done);
    delete pool;
    return STEPQ_OK;
}

int stepq_workspace_bytes(const stepq_plan *plan, int64_t n, size_t *out) {
    if (!plan || !out) return fail(STEPQ_ERR_INVALID, "plan and out must be non-NULL");
    if (n < 0) return fail(STEPQ_ERR_INVALID, "n must be >= 0");
    *out = round_up((size_t)n * plan->H * plan->dv * sizeof(float), 256);
    return STEPQ_OK;
}

int stepq_pack(const stepq_plan *plan, stepq_pool *pool, const int32_t *slot_idx, int64_t n,
               const float *X, void *stream) {
    g_err.clear();
    int rc = check_pool(plan, pool);
    if (!rc) rc = check_rows(plan, slot_idx, n);
    if (rc) return rc;
    if (n == 0) return STEPQ_OK;
    if ((rc = check_inputs(X, "X"))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((rc = wait_pending_fit(pool, s))) return rc;
    stepq::StepArgs a = base_args(plan, pool, slot_idx, n);
    a.X = X;
    cudaError_t e = stepq::launch_pack(plan->dev, a, s);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "pack launch");
}

int stepq_unpack(const stepq_plan *plan, stepq_pool *pool, const int32_t *slot_idx, int64_t n,
                 float *S_out, void *stream) {
    g_err.clear();
    int rc = check_pool(plan, pool);
    if (!rc) rc = check_rows(plan, slot_idx, n);
    if (rc) return rc;
    if (n == 0) return STEPQ_OK;
    if ((rc = check_inputs(S_out, "S_out"))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((rc = wait_pending_fit(pool, s))) return rc;
    stepq::StepArgs a = base_args(plan, pool, slot_idx, n);
    a.S_out = S_out;
    cudaError_t e = stepq::launch_unpack(plan->dev, a, s);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "unpack launch");
}

static int unit_distortion(const stepq_plan *plan, stepq_pool *pool, const int32_t *slot_idx,
                           int64_t n, const float *X, double *dist, void *stream, bool accumulate);

int stepq_unit_distortion(const stepq_plan *plan, stepq_pool *pool, const int32_t *slot_idx,
                          int64_t n, const float *X, double *dist, void *stream) {
    return unit_distortion(plan, pool, slot_idx, n, X, dist, stream, false);
}

int stepq_unit_distortion_accumulate(const stepq_plan *plan, stepq_pool *pool, const int32_t *slot_idx,
                                     int64_t n, const float *X, double *dist_sum, void *stream) {
    return unit_distortion(plan, pool, slot_idx, n, X, dist_sum, stream, true);
}

static int unit_distortion(const stepq_plan *plan, stepq_pool *pool, const int32_t *slot_idx,
                           int64_t n, const float *X, double *dist, void *stream, bool accumulate) {
    g_err.clear();
    int rc = check_pool(plan, pool);
    if (!rc) rc = check_rows(plan, slot_idx, n);
    if (rc) return rc;
    if (n == 0) return STEPQ_OK;
    if ((rc = check_inputs(X, "X")) || (rc = check_inputs(dist, "dist"))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((rc = wait_pending_fit(pool, s))) return rc;
    stepq::StepArgs a = base_args(plan, pool, slot_idx, n);
    a.X = X;
    a.dist = dist;
    a.dist_accumulate = accumulate ? 1 : 0;
    cudaError_t e = stepq::launch_distortion(plan->dev, a, s);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "distortion launch");
}

static int check_step_inputs(const stepq_plan *plan, int64_t n, int32_t qkv_dtype, const void *q,
                             const void *k, const void *v, const float *beta, const float *gate,
                             const float *y, const void *ws, size_t ws_bytes, bool readout) {
    int rc;
    if (qkv_dtype != STEPQ_DTYPE_F32 && qkv_dtype != STEPQ_DTYPE_BF16)
        return fail(STEPQ_ERR_INVALID, "qkv_dtype %d unknown", qkv_dtype);
    if ((rc = check_inputs(k, "k")) || (rc = check_inputs(gate, "gate"))) return rc;
    if (readout && ((rc = check_inputs(q, "q")) || (rc = check_inputs(v, "v")) ||
                    (rc = check_inputs(beta, "beta")) || (rc = check_inputs(y, "y"))))
        return rc;
    if ((rc = check_inputs(ws, "workspace"))) return rc;
    size_t need = 0;
    stepq_workspace_bytes(plan, n, &need);
    if (ws_bytes < need)
        return fail(STEPQ_ERR_INVALID, "workspace of %zu bytes, %zu needed", ws_bytes, need);
    return STEPQ_OK;
}

int stepq_decode_readout(const stepq_plan *plan, stepq_pool *pool, const int32_t *slot_idx,
                         int64_t n, int32_t qkv_dtype, const void *q, const void *k, const void *v,
                         const float *beta, const float *gate, float *y, void *workspace,
                         size_t ws_bytes, void *stream) {
    g_err.clear();
    int rc = check_pool(plan, pool);
    if (!rc) rc = check_rows(plan, slot_idx, n);
    if (rc) return rc;
    if (n == 0) return STEPQ_OK;
    if ((rc = check_step_inputs(plan, n, qkv_dtype, q, k, v, beta, gate, y, workspace, ws_bytes, true)))
        return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((rc = wait_pending_fit(pool, s))) return rc;
    stepq::StepArgs a = base_args(plan, pool, slot_idx, n);
    a.q = q; a.k = k; a.v = v; a.beta = beta; a.gate = gate; a.y = y;
    a.delta = static_cast<float *>(workspace);
    cudaError_t e = stepq::launch_readout(plan->dev, a, qkv_dtype, s);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "readout launch");
}

int stepq_decode_fitpack(const stepq_plan *plan, stepq_pool *pool, const int32_t *slot_idx,
                         int64_t n, int32_t qkv_dtype, const void *k, const float *gate,
                         void *workspace, size_t ws_bytes, void *stream) {
    g_err.clear();
    int rc = check_pool(plan, pool);
    if (!rc) rc = check_rows(plan, slot_idx, n);
    if (rc) return rc;
    if (n == 0) return STEPQ_OK;
    if ((rc = check_step_inputs(plan, n, qkv_dtype, nullptr, k, nullptr, nullptr, gate, nullptr,
                                workspace, ws_bytes, false)))
        return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    stepq::StepArgs a = base_args(plan, pool, slot_idx, n);
    a.k = k; a.gate = gate;
    a.delta = static_cast<float *>(workspace);
    cudaError_t e = stepq::launch_fitpack(plan->dev, a, qkv_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "fitpack launch");
    e = cudaEventRecord(pool->fit_done, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    pool->fit_pending = true;
    return STEPQ_OK;
}

// A batch whose packed state is larger than a share of L2 is stepped in
// chunks of requests: each chunk's readout (main stream) is followed, after
// an event, by that chunk's fit + pack (side stream), so the fit re-reads the
// blobs while the readout has just brought them into L2 and the next chunk's
// readout overlaps it.  Every head is computed exactly as in one launch.
constexpr size_t kChunkStateBytes = 48ull << 20;

int stepq_decode_step(const stepq_plan *plan, stepq_pool *pool, const int32_t *slot_idx, int64_t n,
                      int32_t qkv_dtype, const void *q, const void *k, const void *v,
                      const float *beta, const float *gate, float *y, void *workspace,
                      size_t ws_bytes, void *main_stream, void *side_stream) {
    // the whole batch's arguments are checked (and the previous step's fit
    // waited for) by the readout of the first chunk, called on all of them
    g_err.clear();
    int rc = check_pool(plan, pool);
    if (!rc) rc = check_rows(plan, slot_idx, n);
    if (rc) return rc;
    if (n == 0) return STEPQ_OK;
    if ((rc = check_step_inputs(plan, n, qkv_dtype, q, k, v, beta, gate, y, workspace, ws_bytes, true)))
        return rc;
    cudaStream_t m = static_cast<cudaStream_t>(main_stream);
    cudaStream_t s = side_stream ? static_cast<cudaStream_t>(side_stream) : m;
    if ((rc = wait_pending_fit(pool, m))) return rc;
    // requests per chunk: a multiple of 16 (every per-request input offset
    // stays 16-byte aligned), chunks of near-equal size
    int64_t most = std::max<int64_t>(16, (int64_t)(kChunkStateBytes / std::max<size_t>(plan->slot_bytes, 1)));
    const int64_t nch = (n + most - 1) / most;
    int64_t chunk = (n + nch - 1) / nch;
    chunk = (chunk + 15) / 16 * 16;
    const size_t H = (size_t)plan->H;
    const size_t es = qkv_dtype == STEPQ_DTYPE_BF16 ? 2 : 4;
    const size_t gate_per_req = plan->gate_kind == STEPQ_GATE_DIAG ? H * plan->dk : H;
    for (int64_t r0 = 0; r0 < n; r0 += chunk) {
        const int64_t nn = std::min(chunk, n - r0);
        const uint8_t *qb = static_cast<const uint8_t *>(q), *kb = static_cast<const uint8_t *>(k);
        const uint8_t *vb = static_cast<const uint8_t *>(v);
        const size_t qkv_off = (size_t)r0 * H * plan->dk * es;
        stepq::StepArgs a = base_args(plan, pool, slot_idx + r0, nn);
        a.q = qb + qkv_off; a.k = kb + qkv_off; a.v = vb + qkv_off;
        a.beta = beta + (size_t)r0 * H;
        a.gate = gate + (size_t)r0 * gate_per_req;
        a.y = y + (size_t)r0 * H * plan->dv;
        a.delta = static_cast<float *>(workspace) + (size_t)r0 * H * plan->dv;
        cudaError_t e = stepq::launch_readout(plan->dev, a, qkv_dtype, m);
        if (e != cudaSuccess) return cuda_fail(e, "readout launch");
        if (s != m) {
            e = cudaEventRecord(pool->readout_done, m);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(s, pool->readout_done, 0);
            if (e != cudaSuccess) return cuda_fail(e, "stream handoff");
        }
        e = stepq::launch_fitpack(plan->dev, a, qkv_dtype, s);
        if (e != cudaSuccess) return cuda_fail(e, "fitpack launch");
    }
    cudaError_t e = cudaEventRecord(pool->fit_done, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    pool->fit_pending = true;
    return STEPQ_OK;
}

namespace {
struct HostLayout {
    size_t delta, q, k, v, beta, gate, y, total, qkv_bytes, gate_bytes, y_bytes, beta_bytes;
};
HostLayout host_layout(const stepq_plan *plan, int64_t n, int32_t qkv_dtype) {
    HostLayout L{};
    const size_t nh = (size_t)n * plan->H;
    const size_t es = qkv_dtype == STEPQ_DTYPE_BF16 ? 2 : 4;
    L.qkv_bytes = nh * plan->dk * es;
    L.beta_bytes = nh * 4;
    L.gate_bytes = plan->gate_kind == STEPQ_GATE_DIAG ? nh * plan->dk * 4 : nh * 4;
    L.y_bytes = nh * plan->dv * 4;
    L.delta = 0;
    L.q = round_up(nh * plan->dv * 4, 256);
    L.k = L.q + round_up(L.qkv_bytes, 256);
    L.v = L.k + round_up(L.qkv_bytes, 256);
    L.beta = L.v + round_up(L.qkv_bytes, 256);
    L.gate = L.beta + round_up(L.beta_bytes, 256);
    L.y = L.gate + round_up(L.gate_bytes, 256);
    L.total = L.y + round_up(L.y_bytes, 256);
    return L;
}
}  // namespace

int stepq_host_workspace_bytes(const stepq_plan *plan, int64_t n, int32_t qkv_dtype, size_t *out) {
    if (!plan || !out) return fail(STEPQ_ERR_INVALID, "plan and out must be non-NULL");
    if (n < 0) return fail(STEPQ_ERR_INVALID, "n must be >= 0");
    if (qkv_dtype != STEPQ_DTYPE_F32 && qkv_dtype != STEPQ_DTYPE_BF16)
        return fail(STEPQ_ERR_INVALID, "qkv_dtype %d unknown", qkv_dtype);
    *out = host_layout(plan, n, qkv_dtype).total;
    return STEPQ_OK;
}

int stepq_decode_step_host(const stepq_plan *plan, stepq_pool *pool, const int32_t *slot_idx,
                           int64_t n, int32_t qkv_dtype, const void *q_host, const void *k_host,
                           const void *v_host, const float *beta_host, const float *gate_host,
                           float *y_host, void *workspace, size_t ws_bytes, void *main_stream,
                           void *side_stream) {
    g_err.clear();
    int rc = check_pool(plan, pool);
    if (!rc) rc = check_rows(plan, slot_idx, n);
    if (rc) return rc;
    if (n == 0) return STEPQ_OK;
    if (qkv_dtype != STEPQ_DTYPE_F32 && qkv_dtype != STEPQ_DTYPE_BF16)
        return fail(STEPQ_ERR_INVALID, "qkv_dtype %d unknown", qkv_dtype);
    if (!q_host || !k_host || !v_host || !beta_host || !gate_host || !y_host)
        return fail(STEPQ_ERR_INVALID, "host buffers must be non-NULL");
    if ((rc = check_inputs(workspace, "workspace"))) return rc;
    const HostLayout L = host_layout(plan, n, qkv_dtype);
    if (ws_bytes < L.total)
        return fail(STEPQ_ERR_INVALID, "workspace of %zu bytes, %zu needed", ws_bytes, L.total);
    uint8_t *w = static_cast<uint8_t *>(workspace);
    cudaStream_t m = static_cast<cudaStream_t>(main_stream);
    if ((rc = host_streams(pool))) return rc;
    // The inputs' copies run on the pool's copy-in stream.  They wait for
    // this pool's previous fit (which reads k and gate from the staging area,
    // after its readout read q, k and v), not for earlier work on main_stream,
    // so they overlap the readouts and copies of the layers before this one.
    if ((rc = wait_pending_fit(pool, pool->copy_in))) return rc;
    cudaStream_t ci = pool->copy_in, co = pool->copy_out;
    cudaError_t e = cudaMemcpyAsync(w + L.q, q_host, L.qkv_bytes, cudaMemcpyHostToDevice, ci);
    if (e == cudaSuccess) e = cudaMemcpyAsync(w + L.k, k_host, L.qkv_bytes, cudaMemcpyHostToDevice, ci);
    if (e == cudaSuccess) e = cudaMemcpyAsync(w + L.v, v_host, L.qkv_bytes, cudaMemcpyHostToDevice, ci);
    if (e == cudaSuccess) e = cudaMemcpyAsync(w + L.beta, beta_host, L.beta_bytes, cudaMemcpyHostToDevice, ci);
    if (e == cudaSuccess) e = cudaMemcpyAsync(w + L.gate, gate_host, L.gate_bytes, cudaMemcpyHostToDevice, ci);
    if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
    e = cudaEventRecord(pool->in_done, ci);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(m, pool->in_done, 0);
    if (e != cudaSuccess) return cuda_fail(e, "copy-in event");
    rc = stepq_decode_step(plan, pool, slot_idx, n, qkv_dtype, w + L.q, w + L.k, w + L.v,
                           reinterpret_cast<const float *>(w + L.beta),
                           reinterpret_cast<const float *>(w + L.gate),
                           reinterpret_cast<float *>(w + L.y), w + L.delta, L.q, main_stream,
                           side_stream);
    if (rc) return rc;
    // y goes back on the copy-out stream; main_stream then waits for it, so
    // y_host is valid once main_stream has reached this point and the next
    // readout on main_stream cannot overwrite the staged y before it is read
    e = cudaEventRecord(pool->y_ready, m);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(co, pool->y_ready, 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(y_host, w + L.y, L.y_bytes, cudaMemcpyDeviceToHost, co);
    if (e == cudaSuccess) e = cudaEventRecord(pool->y_done, co);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(m, pool->y_done, 0);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "device-to-host copy");
}

int stepq_row_impact(int32_t d_k, int32_t n_heads, int32_t gate_kind, int32_t qkv_dtype, int64_t n,
                     const void *q, const void *k, const float *beta, const float *gate,
                     double *score_sum, void *stream) {
    g_err.clear();
    if (d_k != 64 && d_k != 128) return fail(STEPQ_ERR_UNSUPPORTED, "the library runs d_k in {64, 128}");
    if (n_heads <= 0 || n_heads > 65535) return fail(STEPQ_ERR_INVALID, "n_heads must be in [1, 65535]");
    if (gate_kind != STEPQ_GATE_SCALAR && gate_kind != STEPQ_GATE_DIAG)
        return fail(STEPQ_ERR_INVALID, "gate_kind %d unknown", gate_kind);
    if (qkv_dtype != STEPQ_DTYPE_F32 && qkv_dtype != STEPQ_DTYPE_BF16)
        return fail(STEPQ_ERR_INVALID, "qkv_dtype %d unknown", qkv_dtype);
    if (n < 0) return fail(STEPQ_ERR_INVALID, "n must be >= 0");
    int rc;
    if ((rc = check_inputs(score_sum, "score_sum"))) return rc;
    if (n == 0) return STEPQ_OK;
    if ((rc = check_inputs(q, "q")) || (rc = check_inputs(k, "k")) || (rc = check_inputs(beta, "beta")) ||
        (rc = check_inputs(gate, "gate")))
        return rc;
    cudaError_t e = stepq::launch_row_impact(d_k, n_heads, gate_kind, qkv_dtype, n, q, k, beta, gate,
                                             score_sum, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "row impact launch");
}

int stepq_fp32_step(int32_t d_k, int32_t d_v, int32_t n_heads, int32_t gate_kind,
                    int32_t qkv_dtype, float *S, int64_t num_slots, const int32_t *slot_idx,
                    int64_t n, const void *q, const void *k, const void *v, const float *beta,
                    const float *gate, float *y, uint32_t *dev_status, void *stream) {
    g_err.clear();
    if (d_k != d_v || (d_k != 64 && d_k != 128))
        return fail(STEPQ_ERR_UNSUPPORTED, "the library runs d_k == d_v in {64, 128}");
    if (n_heads <= 0 || num_slots <= 0) return fail(STEPQ_ERR_INVALID, "n_heads, num_slots must be positive");
    if (gate_kind != STEPQ_GATE_SCALAR && gate_kind != STEPQ_GATE_DIAG)
        return fail(STEPQ_ERR_INVALID, "gate_kind %d unknown", gate_kind);
    if (qkv_dtype != STEPQ_DTYPE_F32 && qkv_dtype != STEPQ_DTYPE_BF16)
        return fail(STEPQ_ERR_INVALID, "qkv_dtype %d unknown", qkv_dtype);
    if (n < 0) return fail(STEPQ_ERR_INVALID, "n must be >= 0");
    if (n * (int64_t)n_heads * (d_k / 32) > (int64_t)0x7fffffff)
        return fail(STEPQ_ERR_INVALID, "n * n_heads exceeds the grid limit");
    if (n == 0) return STEPQ_OK;
    int rc;
    if (!slot_idx) return fail(STEPQ_ERR_INVALID, "slot_idx is NULL");
    if ((rc = check_inputs(S, "S")) || (rc = check_inputs(q, "q")) || (rc = check_inputs(k, "k")) ||
        (rc = check_inputs(v, "v")) || (rc = check_inputs(beta, "beta")) ||
        (rc = check_inputs(gate, "gate")) || (rc = check_inputs(y, "y")))
        return rc;
    cudaError_t e = stepq::launch_fp32_step(d_k, n_heads, gate_kind, qkv_dtype, S, num_slots,
                                            slot_idx, n, q, k, v, beta, gate, y, dev_status,
                                            static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "fp32 step launch");
}

int stepq_get_status(stepq_pool *pool, uint32_t *out) {
    g_err.clear();
    if (!pool || !out) return fail(STEPQ_ERR_INVALID, "pool and out must be non-NULL");
    int rc = check_device(pool->device);
    if (rc) return rc;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(out, pool->status, 4, cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "status read");
}

int stepq_pool_set_test_faults(stepq_pool *pool, uint32_t flags, uint32_t wait_limit_us) {
    g_err.clear();
    if (!pool) return fail(STEPQ_ERR_INVALID, "pool is NULL");
    if (flags & ~STEPQ_TEST_NO_STAGING_COPY) return fail(STEPQ_ERR_INVALID, "unknown test flags %#x", flags);
    if (flags && (wait_limit_us < 1 || wait_limit_us > 1000000))
        return fail(STEPQ_ERR_INVALID, "wait_limit_us %u outside 1 .. 1000000", wait_limit_us);
    pool->test_faults = flags;
    pool->wait_limit_ns = flags ? (uint64_t)wait_limit_us * 1000ull : stepq::kDefaultWaitLimitNs;
    return STEPQ_OK;
}

int stepq_clear_status(stepq_pool *pool, void *stream) {
    g_err.clear();
    if (!pool) return fail(STEPQ_ERR_INVALID, "pool is NULL");
    cudaError_t e = cudaMemsetAsync(pool->status, 0, 4, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "status clear");
}

}  // extern "C"
