"""ctypes marshalling for libstepq (argument checks and pointer passing only)."""

from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libstepq.so")

OK, ERR_INVALID, ERR_CUDA, ERR_UNSUPPORTED = 0, 1, 2, 3
DEV_BAD_SLOT, DEV_NONFINITE, DEV_TIMEOUT = 1, 2, 4
TEST_NO_STAGING_COPY = 1
GATE_SCALAR, GATE_DIAG = 0, 1
UNIT_HEAD, UNIT_ROW = 0, 1
MODE_STEPQUANT, MODE_UNIFORM = 0, 1
DTYPE_F32, DTYPE_BF16 = 0, 1

# every entry point the header declares, with its ctypes signature
_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_SIGS = {
    "stepq_plan_create": [_P, _P],
    "stepq_plan_destroy": [_P],
    "stepq_plan_slot_bytes": [_P, ctypes.POINTER(_SZ)],
    "stepq_plan_head_layout": [_P, _I32, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)],
    "stepq_pool_alloc": [_P, _I64, _P, _SZ, _P],
    "stepq_pool_free": [_P],
    "stepq_pack": [_P, _P, _P, _I64, _P, _P],
    "stepq_unpack": [_P, _P, _P, _I64, _P, _P],
    "stepq_workspace_bytes": [_P, _I64, ctypes.POINTER(_SZ)],
    "stepq_decode_readout": [_P, _P, _P, _I64, _I32, _P, _P, _P, _P, _P, _P, _P, _SZ, _P],
    "stepq_decode_fitpack": [_P, _P, _P, _I64, _I32, _P, _P, _P, _SZ, _P],
    "stepq_decode_step": [_P, _P, _P, _I64, _I32, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _P],
    "stepq_fp32_step": [_I32, _I32, _I32, _I32, _I32, _P, _I64, _P, _I64, _P, _P, _P, _P, _P, _P,
                        _P, _P],
    "stepq_host_workspace_bytes": [_P, _I64, _I32, ctypes.POINTER(_SZ)],
    "stepq_decode_step_host": [_P, _P, _P, _I64, _I32, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _P],
    "stepq_decode_step_static": [_P, _P, _P, _I64, _I32, _P, _P, _P, _P, _P, _P, _P, _P],
    "stepq_unit_distortion": [_P, _P, _P, _I64, _P, _P, _P],
    "stepq_unit_distortion_accumulate": [_P, _P, _P, _I64, _P, _P, _P],
    "stepq_lifetime_weight": [_I64, _I64, _I32, _P, _P],
    "stepq_allocate_bits": [_I64, _P, _P, _I32, _I64, _P],
    "stepq_row_impact": [_I32, _I32, _I32, _I32, _I64, _P, _P, _P, _P, _P, _P],
    "stepq_impact_weights": [_I64, _I64, _P, _P],
    "stepq_get_status": [_P, ctypes.POINTER(ctypes.c_uint32)],
    "stepq_clear_status": [_P, _P],
    "stepq_pool_set_test_faults": [_P, ctypes.c_uint32, ctypes.c_uint32],
    "stepq_last_error": [],
}


class StepqError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"stepq error {code}: {msg}")
        self.code = code


class _Desc(ctypes.Structure):
    _fields_ = [("d_k", _I32), ("d_v", _I32), ("n_heads", _I32), ("gate_kind", _I32),
                ("unit_kind", _I32), ("mode", _I32), ("bits", _P), ("w", _P)]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load the in-tree libstepq.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"libstepq.so not built at {_LIB_PATH}; run "
                              "`python -m quantized_delta_rule_decode_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_char_p if name == "stepq_last_error" else ctypes.c_int
        _lib = L
    return _lib


def _call(name, *args):
    L = load_library()
    rc = getattr(L, name)(*args)
    if rc != OK:
        raise StepqError(rc, L.stepq_last_error().decode())


def _stream(s):
    if s is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(s, int):
        return ctypes.c_void_p(s)
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t, dtype=None, name="tensor"):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _qkv_dtype(t):
    import torch
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    if t.dtype == torch.float32:
        return DTYPE_F32
    raise ValueError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


class Plan:
    """Owns a stepq_plan handle."""

    def __init__(self, handle, d_k, d_v, n_heads, gate_kind, unit_kind, mode):
        self.handle = handle
        self.d_k, self.d_v, self.n_heads = d_k, d_v, n_heads
        self.gate_kind, self.unit_kind, self.mode = gate_kind, unit_kind, mode

    def __del__(self):
        if getattr(self, "handle", None) and _lib is not None:
            _lib.stepq_plan_destroy(self.handle)
            self.handle = None


class Pool:
    """Owns a stepq_pool handle; keeps the plan and the device buffer alive."""

    def __init__(self, handle, plan, buf, num_slots):
        self.handle, self.plan, self.buf, self.num_slots = handle, plan, buf, num_slots

    def __del__(self):
        if getattr(self, "handle", None) and _lib is not None:
            _lib.stepq_pool_free(self.handle)
            self.handle = None


def stepq_plan_create(d_k, d_v, n_heads, gate_kind, unit_kind, mode, bits, w) -> Plan:
    bits = np.ascontiguousarray(bits, dtype=np.uint8)
    w = np.ascontiguousarray(w, dtype=np.float32)
    need = n_heads if unit_kind == UNIT_HEAD else n_heads * d_k
    if bits.size != need or w.size != n_heads * d_k:
        raise ValueError("bits / w have the wrong number of entries")
    d = _Desc(d_k, d_v, n_heads, gate_kind, unit_kind, mode,
              bits.ctypes.data_as(_P), w.ctypes.data_as(_P))
    h = ctypes.c_void_p()
    _call("stepq_plan_create", ctypes.byref(d), ctypes.byref(h))
    return Plan(h, d_k, d_v, n_heads, gate_kind, unit_kind, mode)


def stepq_plan_destroy(plan: Plan):
    if plan.handle:
        _call("stepq_plan_destroy", plan.handle)
        plan.handle = None


def stepq_plan_slot_bytes(plan: Plan) -> int:
    out = _SZ()
    _call("stepq_plan_slot_bytes", plan.handle, ctypes.byref(out))
    return out.value


def stepq_plan_head_layout(plan: Plan, head: int):
    off, nb = _SZ(), _SZ()
    _call("stepq_plan_head_layout", plan.handle, head, ctypes.byref(off), ctypes.byref(nb))
    return off.value, nb.value


def stepq_pool_alloc(plan: Plan, num_slots: int, buf) -> Pool:
    import torch
    if buf.dtype != torch.uint8:
        raise ValueError("pool buffer must be uint8")
    h = ctypes.c_void_p()
    _call("stepq_pool_alloc", plan.handle, num_slots, _ptr(buf, name="buf"), buf.numel(),
          ctypes.byref(h))
    return Pool(h, plan, buf, num_slots)


def stepq_pool_free(pool: Pool):
    if pool.handle:
        _call("stepq_pool_free", pool.handle)
        pool.handle = None


def stepq_workspace_bytes(plan: Plan, n: int) -> int:
    out = _SZ()
    _call("stepq_workspace_bytes", plan.handle, n, ctypes.byref(out))
    return out.value


def _slots(slot_idx):
    import torch
    return _ptr(slot_idx, torch.int32, "slot_idx"), slot_idx.numel()


def stepq_pack(plan: Plan, pool: Pool, slot_idx, X, stream=None):
    import torch
    s, n = _slots(slot_idx)
    _call("stepq_pack", plan.handle, pool.handle, s, n, _ptr(X, torch.float32, "X"), _stream(stream))


def stepq_unpack(plan: Plan, pool: Pool, slot_idx, S_out, stream=None):
    import torch
    s, n = _slots(slot_idx)
    _call("stepq_unpack", plan.handle, pool.handle, s, n, _ptr(S_out, torch.float32, "S_out"),
          _stream(stream))


def stepq_decode_readout(plan, pool, slot_idx, q, k, v, beta, gate, y, workspace, stream=None):
    import torch
    s, n = _slots(slot_idx)
    _call("stepq_decode_readout", plan.handle, pool.handle, s, n, _qkv_dtype(q), _ptr(q, q.dtype, "q"),
          _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"), _ptr(beta, torch.float32, "beta"),
          _ptr(gate, torch.float32, "gate"), _ptr(y, torch.float32, "y"),
          _ptr(workspace, name="workspace"), workspace.numel() * workspace.element_size(),
          _stream(stream))


def stepq_decode_fitpack(plan, pool, slot_idx, k, gate, workspace, stream=None):
    import torch
    s, n = _slots(slot_idx)
    _call("stepq_decode_fitpack", plan.handle, pool.handle, s, n, _qkv_dtype(k), _ptr(k, k.dtype, "k"),
          _ptr(gate, torch.float32, "gate"), _ptr(workspace, name="workspace"),
          workspace.numel() * workspace.element_size(), _stream(stream))


def stepq_decode_step(plan, pool, slot_idx, q, k, v, beta, gate, y, workspace, main_stream=None,
                      side_stream=None):
    import torch
    s, n = _slots(slot_idx)
    m = _stream(main_stream)
    sd = _stream(side_stream) if side_stream is not None else m
    _call("stepq_decode_step", plan.handle, pool.handle, s, n, _qkv_dtype(q), _ptr(q, q.dtype, "q"),
          _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"), _ptr(beta, torch.float32, "beta"),
          _ptr(gate, torch.float32, "gate"), _ptr(y, torch.float32, "y"),
          _ptr(workspace, name="workspace"), workspace.numel() * workspace.element_size(), m, sd)


def stepq_host_workspace_bytes(plan: Plan, n: int, qkv_dtype: int) -> int:
    out = _SZ()
    _call("stepq_host_workspace_bytes", plan.handle, n, qkv_dtype, ctypes.byref(out))
    return out.value


def _hptr(t, name):
    if t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous host tensor")
    return ctypes.c_void_p(t.data_ptr())


def stepq_decode_step_host(plan, pool, slot_idx, q, k, v, beta, gate, y, workspace,
                           main_stream=None, side_stream=None):
    """q..gate and y are host (ideally pinned) tensors; workspace is on the device."""
    s, n = _slots(slot_idx)
    m = _stream(main_stream)
    sd = _stream(side_stream) if side_stream is not None else m
    _call("stepq_decode_step_host", plan.handle, pool.handle, s, n, _qkv_dtype(q), _hptr(q, "q"),
          _hptr(k, "k"), _hptr(v, "v"), _hptr(beta, "beta"), _hptr(gate, "gate"), _hptr(y, "y"),
          _ptr(workspace, name="workspace"), workspace.numel() * workspace.element_size(), m, sd)


STATIC_DELTA_FLOATS = 1048576


def stepq_decode_step_static(plan, pool, slot_idx, q, k, v, beta, gate, y, main_stream=None,
                             side_stream=None):
    """stepq_decode_step without a workspace (no device allocation anywhere)."""
    import torch
    s, n = _slots(slot_idx)
    m = _stream(main_stream)
    sd = _stream(side_stream) if side_stream is not None else m
    _call("stepq_decode_step_static", plan.handle, pool.handle, s, n, _qkv_dtype(q),
          _ptr(q, q.dtype, "q"), _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"),
          _ptr(beta, torch.float32, "beta"), _ptr(gate, torch.float32, "gate"),
          _ptr(y, torch.float32, "y"), m, sd)


def stepq_fp32_step(S, slot_idx, q, k, v, beta, gate, y, gate_kind, dev_status=None, stream=None):
    import torch
    num_slots, H, dk, dv = S.shape
    s, n = _slots(slot_idx)
    _call("stepq_fp32_step", dk, dv, H, gate_kind, _qkv_dtype(q), _ptr(S, torch.float32, "S"),
          num_slots, s, n, _ptr(q, q.dtype, "q"), _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"),
          _ptr(beta, torch.float32, "beta"), _ptr(gate, torch.float32, "gate"),
          _ptr(y, torch.float32, "y"), _ptr(dev_status, name="dev_status"), _stream(stream))


def stepq_unit_distortion(plan: Plan, pool: Pool, slot_idx, X, dist=None, stream=None):
    """Per-unit squared reconstruction error [n][units] (float64, on the device)."""
    import torch
    s, n = _slots(slot_idx)
    units = plan.n_heads * plan.d_k if plan.unit_kind == UNIT_ROW else plan.n_heads
    if dist is None:
        dist = torch.empty((n, units), dtype=torch.float64, device=X.device)
    _call("stepq_unit_distortion", plan.handle, pool.handle, s, n, _ptr(X, torch.float32, "X"),
          _ptr(dist, torch.float64, "dist"), _stream(stream))
    return dist


def stepq_unit_distortion_accumulate(plan: Plan, pool: Pool, slot_idx, X, dist_sum, stream=None):
    """dist_sum [units] (float64, on the device) += the per-unit squared
    reconstruction error summed over the requests."""
    import torch
    s, n = _slots(slot_idx)
    _call("stepq_unit_distortion_accumulate", plan.handle, pool.handle, s, n,
          _ptr(X, torch.float32, "X"), _ptr(dist_sum, torch.float64, "dist_sum"), _stream(stream))
    return dist_sum


def stepq_lifetime_weight(gate) -> np.ndarray:
    """gate: host float32 [n_steps][n_units][gates_per_unit] (or [n_steps][n_units])."""
    g = np.ascontiguousarray(gate, np.float32)
    if g.ndim == 2:
        g = g[:, :, None]
    steps, units, per = g.shape
    out = np.zeros(units, np.float64)
    _call("stepq_lifetime_weight", units, steps, per, g.ctypes.data_as(_P), out.ctypes.data_as(_P))
    return out


def stepq_allocate_bits(weight, dist, budget_bits: int, n_pivots: int) -> np.ndarray:
    """weight [n_units] float64, dist [n_units][3] float64 (4, 6, 8 bits) -> uint8 widths."""
    w = np.ascontiguousarray(weight, np.float64)
    d = np.ascontiguousarray(dist, np.float64)
    if d.shape != (w.size, 3):
        raise ValueError("dist must be [n_units][3]")
    bits = np.zeros(w.size, np.uint8)
    _call("stepq_allocate_bits", w.size, w.ctypes.data_as(_P), d.ctypes.data_as(_P), int(budget_bits),
          int(n_pivots), bits.ctypes.data_as(_P))
    return bits


def stepq_row_impact(gate_kind, q, k, beta, gate, score_sum, stream=None):
    """score_sum [n_heads][d_k] float64 (device) += squared readout weighting factors of q, k."""
    import torch
    n, H, dk = q.shape
    _call("stepq_row_impact", dk, H, gate_kind, _qkv_dtype(q), n, _ptr(q, q.dtype, "q"),
          _ptr(k, q.dtype, "k"), _ptr(beta, torch.float32, "beta"), _ptr(gate, torch.float32, "gate"),
          _ptr(score_sum, torch.float64, "score_sum"), _stream(stream))
    return score_sum


def stepq_impact_weights(score_sum, count: int) -> np.ndarray:
    """Host float64 sums [n_rows] -> fp32 weights sqrt(sum / count)."""
    s = np.ascontiguousarray(score_sum, np.float64).reshape(-1)
    w = np.zeros(s.size, np.float32)
    _call("stepq_impact_weights", s.size, int(count), s.ctypes.data_as(_P), w.ctypes.data_as(_P))
    return w


def stepq_get_status(pool: Pool) -> int:
    out = ctypes.c_uint32()
    _call("stepq_get_status", pool.handle, ctypes.byref(out))
    return out.value


def stepq_clear_status(pool: Pool, stream=None):
    _call("stepq_clear_status", pool.handle, _stream(stream))


def stepq_pool_set_test_faults(pool: Pool, flags: int, wait_limit_us: int = 0):
    """Test hook: with TEST_NO_STAGING_COPY the pool's readout and fit kernels
    issue no staging copy and give up each wait after wait_limit_us (0 flags:
    normal operation)."""
    _call("stepq_pool_set_test_faults", pool.handle, int(flags), int(wait_limit_us))
