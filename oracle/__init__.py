"""CPU oracle for the quantised Delta-rule decode step -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never loads it.

The arithmetic lives in ``stepq_oracle.c`` (plain single-threaded C, binary32,
no fused multiply-add); this module only marshals numpy arrays to it.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# STEPQ_ORACLE_SRC / STEPQ_ORACLE_LIB: build and load another copy of the
# source instead (the mutation test plants mistakes in copies to check that
# the pins catch them)
_SRC = os.environ.get("STEPQ_ORACLE_SRC", os.path.join(_HERE, "stepq_oracle.c"))
_LIB = os.environ.get("STEPQ_ORACLE_LIB", os.path.join(_HERE, "liboracle_stepq.so"))
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        I64 = ctypes.c_int64
        L.orc_half_to_float.argtypes = [ctypes.c_uint16]
        L.orc_half_to_float.restype = F
        L.orc_float_to_half.argtypes = [F]
        L.orc_float_to_half.restype = ctypes.c_uint16
        L.orc_plan_new.argtypes = [I, I, I, I, I, I, P, P, ctypes.POINTER(P)]
        L.orc_plan_new.restype = I
        L.orc_plan_free.argtypes = [P]
        L.orc_slot_bytes.argtypes = [P]
        L.orc_slot_bytes.restype = Z
        L.orc_head_layout.argtypes = [P, I, ctypes.POINTER(Z), ctypes.POINTER(Z)]
        L.orc_pack_codes.argtypes = [P, I, P, P, P, P, P]
        L.orc_unpack_codes.argtypes = [P, I, P, P, P, P, P]
        L.orc_dequantize_head.argtypes = [P, I, P, P]
        L.orc_column_codes.argtypes = [P, I, P, P, I, ctypes.c_uint16, P]
        L.orc_quantize_head.argtypes = [P, I, P, P, P, P, P]
        L.orc_quantize_head.restype = I
        L.orc_delta_update.argtypes = [I, I, P, P, P, P, F, P, I, P, P]
        L.orc_delta_update_d.argtypes = [I, I, P, P, P, P, F, P, I, P, P, P]
        L.orc_step_head.argtypes = [P, I, P, P, P, P, F, P, P, P]
        L.orc_step_head.restype = I
        L.orc_pack.argtypes = [P, P, I64, P, I64, P]
        L.orc_pack.restype = I
        L.orc_unpack.argtypes = [P, P, I64, P, I64, P]
        L.orc_unpack.restype = I
        L.orc_decode_step.argtypes = [P, P, I64, P, I64, P, P, P, P, P, P]
        L.orc_decode_step.restype = I
        L.orc_fp32_step_head.argtypes = [I, I, P, P, P, P, F, P, I, P]
        L.orc_fp32_step.argtypes = [I, I, I, I, P, I64, P, I64, P, P, P, P, P, P]
        L.orc_fp32_step.restype = I
        L.orc_unit_distortion.argtypes = [P, P, I64, P, I64, P, P]
        L.orc_unit_distortion.restype = I
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def half_to_float(h: int) -> float:
    return lib().orc_half_to_float(int(h))


def float_to_half(x: float) -> int:
    return lib().orc_float_to_half(float(x))


STATUS_BAD_SLOT = 1
STATUS_NONFINITE = 2


class Plan:
    """The oracle's own view of a quantisation plan and its byte layout."""

    def __init__(self, dk, dv, H, gate_kind, unit_kind, mode, bits, w):
        self.dk, self.dv, self.H = dk, dv, H
        self.gate_kind, self.unit_kind, self.mode = gate_kind, unit_kind, mode
        self._bits = np.ascontiguousarray(bits, dtype=np.uint8)
        self._w = _f32(w).reshape(H * dk).copy()
        h = ctypes.c_void_p()
        rc = lib().orc_plan_new(dk, dv, H, gate_kind, unit_kind, mode, _p(self._bits), _p(self._w),
                                ctypes.byref(h))
        if rc != 0:
            raise ValueError("oracle rejected the plan")
        self.h = h

    def __del__(self):
        if getattr(self, "h", None) and _lib is not None:
            _lib.orc_plan_free(self.h)
            self.h = None

    @property
    def slot_bytes(self) -> int:
        return lib().orc_slot_bytes(self.h)

    def head_layout(self, h):
        off, nb = ctypes.c_size_t(), ctypes.c_size_t()
        lib().orc_head_layout(self.h, h, ctypes.byref(off), ctypes.byref(nb))
        return off.value, nb.value

    # ---- one head -------------------------------------------------------
    def pack_codes(self, h, codes, piv, rho, c):
        _, nb = self.head_layout(h)
        blob = np.zeros(nb, np.uint8)
        lib().orc_pack_codes(self.h, h, _p(np.ascontiguousarray(codes, np.int16)),
                             _p(np.ascontiguousarray(piv, np.uint16)),
                             _p(np.ascontiguousarray(rho, np.uint16)),
                             _p(np.ascontiguousarray(c, np.uint16)), _p(blob))
        return blob

    def unpack_codes(self, h, blob):
        codes = np.zeros((self.dk, self.dv), np.int16)
        piv = np.zeros((self.dk, self.dv), np.uint16)
        rho = np.zeros(self.dk, np.uint16)
        c = np.zeros(self.dv, np.uint16)
        lib().orc_unpack_codes(self.h, h, _p(np.ascontiguousarray(blob, np.uint8)), _p(codes),
                               _p(piv), _p(rho), _p(c))
        return codes, piv, rho, c

    def dequantize_head(self, h, blob):
        S = np.zeros((self.dk, self.dv), np.float32)
        lib().orc_dequantize_head(self.h, h, _p(np.ascontiguousarray(blob, np.uint8)), _p(S))
        return S

    def quantize_head(self, h, X, diag=False):
        _, nb = self.head_layout(h)
        blob = np.zeros(nb, np.uint8)
        X = _f32(X).reshape(self.dk, self.dv)
        if diag:
            E = np.zeros((self.dv, 8), np.float32)
            cand = np.zeros((self.dv, 8), np.uint16)
            best = np.zeros(self.dv, np.int8)
            st = lib().orc_quantize_head(self.h, h, _p(X), _p(blob), _p(E), _p(cand), _p(best))
            return blob, st, E, cand, best
        st = lib().orc_quantize_head(self.h, h, _p(X), _p(blob), None, None, None)
        return blob, st

    def column_codes(self, h, X, rho, j, c_bits):
        out = np.zeros(self.dk, np.int16)
        lib().orc_column_codes(self.h, h, _p(_f32(X)), _p(np.ascontiguousarray(rho, np.uint16)),
                               int(j), int(c_bits), _p(out))
        return out

    def step_head(self, h, blob, q, k, v, beta, gate):
        """One quantised step in place on ``blob``; returns (y, X, status)."""
        y = np.zeros(self.dv, np.float32)
        X = np.zeros((self.dk, self.dv), np.float32)
        g = _f32(np.atleast_1d(gate))
        st = lib().orc_step_head(self.h, h, _p(blob), _p(_f32(q)), _p(_f32(k)), _p(_f32(v)),
                                 float(beta), _p(g), _p(y), _p(X))
        return y, X, st

    # ---- pool level -----------------------------------------------------
    def new_pool(self, num_slots):
        return np.zeros(num_slots * self.slot_bytes, np.uint8)

    def pack(self, pool, slot_idx, X):
        sl = np.ascontiguousarray(slot_idx, np.int32)
        return lib().orc_pack(self.h, _p(pool), pool.size // self.slot_bytes, _p(sl), sl.size,
                              _p(_f32(X)))

    def unpack(self, pool, slot_idx):
        sl = np.ascontiguousarray(slot_idx, np.int32)
        S = np.zeros((sl.size, self.H, self.dk, self.dv), np.float32)
        st = lib().orc_unpack(self.h, _p(pool), pool.size // self.slot_bytes, _p(sl), sl.size, _p(S))
        return S, st

    def unit_distortion(self, pool, slot_idx, X):
        """Per-unit squared reconstruction error [n][units] (float64) and status."""
        sl = np.ascontiguousarray(slot_idx, np.int32)
        units = self.H * self.dk if self.unit_kind else self.H
        dist = np.zeros((sl.size, units), np.float64)
        st = lib().orc_unit_distortion(self.h, _p(pool), pool.size // self.slot_bytes, _p(sl), sl.size,
                                       _p(_f32(X)), _p(dist))
        return dist, st

    def decode_step(self, pool, slot_idx, q, k, v, beta, gate):
        sl = np.ascontiguousarray(slot_idx, np.int32)
        y = np.zeros((sl.size, self.H, self.dv), np.float32)
        st = lib().orc_decode_step(self.h, _p(pool), pool.size // self.slot_bytes, _p(sl), sl.size,
                                   _p(_f32(q)), _p(_f32(k)), _p(_f32(v)), _p(_f32(beta)),
                                   _p(_f32(gate)), _p(y))
        return y, st


def delta_update(S, q, k, v, beta, gate, gate_kind, with_delta=False):
    """X = D S + beta k (v^T - k^T D S) and y = X^T q on one head (float32);
    with ``with_delta`` also delta = beta (v - k^T D S) [dv]."""
    S = _f32(S)
    dk, dv = S.shape
    X = np.zeros((dk, dv), np.float32)
    y = np.zeros(dv, np.float32)
    delta = np.zeros(dv, np.float32)
    lib().orc_delta_update_d(dk, dv, _p(S), _p(_f32(q)), _p(_f32(k)), _p(_f32(v)), float(beta),
                             _p(_f32(np.atleast_1d(gate))), int(gate_kind), _p(X), _p(y), _p(delta))
    return (X, y, delta) if with_delta else (X, y)


def fp32_step(S, slot_idx, q, k, v, beta, gate, gate_kind):
    """Unquantised step in place on S [slots][H][dk][dv]; returns (y, status)."""
    num_slots, H, dk, dv = S.shape
    sl = np.ascontiguousarray(slot_idx, np.int32)
    y = np.zeros((sl.size, H, dv), np.float32)
    st = lib().orc_fp32_step(dk, dv, H, int(gate_kind), _p(S), num_slots, _p(sl), sl.size,
                             _p(_f32(q)), _p(_f32(k)), _p(_f32(v)), _p(_f32(beta)),
                             _p(_f32(gate)), _p(y))
    return y, st
