"""Helpers for the GPU-vs-oracle parity tests.

The GPU side is driven only through the C ABI (``quantized_delta_rule_decode_b200``,
ctypes over libstepq.so); the expected values come only from ``oracle/``;
both read their inputs from ``workload`` (seeded, synthetic).

Comparison rules:

* packing from an identical X is bit-exact, except that the column-scale
  argmin may pick another candidate when the two candidates' objectives are
  equal within the rounding bound of a binary32 evaluation; such a column is
  accepted only if its codes are exactly the oracle's codes under the GPU's
  chosen scale.
* after a full step (where X itself carries fp32 rounding differences),
  at most 0.1% of codes may differ, by 1 only, outside columns whose scale
  differs; at most 0.1% of row factors / column scales may differ, by one
  half-precision ulp, or (column scales) by a near-tie candidate switch.
"""

from __future__ import annotations

import numpy as np

import oracle
import workload as W

U = 2.0 ** -24
QMAX = {4: 7, 6: 31, 8: 127}


def torch_mod():
    import torch
    return torch


def lib():
    import quantized_delta_rule_decode_b200 as S
    return S


def h2f(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


class Pair:
    """A plan on both sides, from one workload config."""

    def __init__(self, cfg: W.Config, mode=W.MODE_STEPQUANT, uniform_bits=None, budget=None,
                 pivots=True, bits=None):
        self.cfg = cfg
        self.pin = W.make_plan(cfg, budget=budget, uniform_bits=uniform_bits, pivots=pivots)
        if bits is not None:
            # a hand-made width per unit instead of the synthetic plan's
            import dataclasses
            self.pin = dataclasses.replace(self.pin, bits=np.asarray(bits, np.uint8).reshape(-1))
        self.mode = mode
        d, H = cfg.d, cfg.heads
        S = lib()
        self.gpu = S.stepq_plan_create(d, d, H, cfg.gate_kind, cfg.unit_kind, mode, self.pin.bits,
                                       self.pin.w)
        self.ora = oracle.Plan(d, d, H, cfg.gate_kind, cfg.unit_kind, mode, self.pin.bits, self.pin.w)
        self.slot_bytes = S.stepq_plan_slot_bytes(self.gpu)
        assert self.slot_bytes == self.ora.slot_bytes
        self.row_bits = np.zeros((H, d), np.int64)
        for h in range(H):
            if cfg.unit_kind == W.UNIT_HEAD:
                self.row_bits[h] = self.pin.bits[h]
            else:
                self.row_bits[h] = self.pin.bits[h * d:(h + 1) * d]

    def gpu_pool(self, num_slots):
        torch = torch_mod()
        buf = torch.zeros(num_slots * self.slot_bytes, dtype=torch.uint8, device="cuda")
        return lib().stepq_pool_alloc(self.gpu, num_slots, buf)

    def head_blob(self, pool_bytes: np.ndarray, slot: int, h: int) -> np.ndarray:
        off, nb = self.ora.head_layout(h)
        base = slot * self.slot_bytes + off
        return pool_bytes[base:base + nb]


def pool_to_host(pool) -> np.ndarray:
    torch = torch_mod()
    torch.cuda.synchronize()
    return pool.buf.cpu().numpy()


def dev(a, dtype=None):
    torch = torch_mod()
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def step_tensors(cfg: W.Config, si: W.StepInputs):
    """Device tensors for one step; q/k/v as bf16 when the workload says so."""
    torch = torch_mod()
    dt = torch.bfloat16 if cfg.bf16_inputs else torch.float32
    return dict(q=dev(si.q, dt), k=dev(si.k, dt), v=dev(si.v, dt), beta=dev(si.beta),
                gate=dev(si.gate))


def candidate_objective(X_col, rho, w, c, qmax_rows):
    """float64 objective sum_i w^2 (X - rho c code)^2 and its binary32 error bound.

    Codes are taken from the oracle's rule (exact quotient, ties to even);
    the bound covers both sides' binary32 evaluations: the per-term
    cancellation 2|e| * (few u |X|) and (n + 10) u of summation.
    """
    X = X_col.astype(np.float64)
    act = (rho > 0) & (qmax_rows > 0)
    P = rho * c
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(act & (P > 0), X / np.where(P > 0, P, 1), 0.0)
    code = np.clip(np.rint(t), -qmax_rows, qmax_rows) * act
    e = (X - P * code) * act
    w2 = w.astype(np.float64) ** 2
    E = float(np.sum(w2 * e * e))
    n = int(np.sum(act))
    B = float(np.sum(w2 * 14 * U * np.abs(e) * np.abs(X))) + 2 * (n + 10) * U * E
    return E, B


def compare_pack(pair: Pair, h: int, g_blob, o_blob, X, stats, looser=1.0):
    """Pack parity of one head from an identical X (see module docstring)."""
    if np.array_equal(g_blob, o_blob):
        stats["exact_heads"] += 1
        return
    gc, gp, gr, gcc = pair.ora.unpack_codes(h, g_blob)
    oc, op_, orr, occ = pair.ora.unpack_codes(h, o_blob)
    rb = pair.row_bits[h]
    piv = rb == 16
    assert np.array_equal(gp[piv], op_[piv]), f"head {h}: pivot halves differ"
    assert np.array_equal(gr, orr), f"head {h}: row factors differ"
    _, _, E, cand, best = pair.ora.quantize_head(h, X, diag=True)
    rho = h2f(orr)
    w = pair.pin.w[h]
    qrows = np.array([QMAX.get(int(b), 0) for b in rb], np.float64)
    for j in np.flatnonzero(gcc != occ):
        stats["switched_cols"] += 1
        ag = np.flatnonzero(cand[j] == gcc[j])
        assert ag.size, f"head {h} col {j}: GPU scale {gcc[j]:#x} is not a candidate"
        ao = int(best[j])
        Eg, Bg = candidate_objective(X[:, j], rho, w, float(h2f(gcc[j])), qrows)
        Eo, Bo = candidate_objective(X[:, j], rho, w, float(h2f(occ[j])), qrows)
        assert Eg <= Eo + looser * (Bg + Bo), \
            f"head {h} col {j}: GPU candidate {ag} objective {Eg} vs oracle {ao} {Eo} (bound {Bg + Bo})"
        ref = pair.ora.column_codes(h, X, orr, j, int(gcc[j]))
        assert np.array_equal(gc[~piv, j], ref[~piv]), f"head {h} col {j}: codes under GPU scale differ"
    same = gcc == occ
    assert np.array_equal(gc[~piv][:, same], oc[~piv][:, same]), f"head {h}: codes differ"


def new_stats():
    return {"exact_heads": 0, "switched_cols": 0}


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def rel_l2_worst_head(a, b):
    """The largest relative L2 error of any one head's readout (last axis =
    d_v): one small-norm head cannot hide inside a batch-wide norm."""
    a = np.asarray(a, np.float64).reshape(-1, np.shape(a)[-1])
    b = np.asarray(b, np.float64).reshape(-1, np.shape(b)[-1])
    num = np.linalg.norm(a - b, axis=1)
    den = np.maximum(np.linalg.norm(b, axis=1), 1e-300)
    return float(np.max(num / den))


class StepDiff:
    """Accumulates full-step blob differences over many heads."""

    def __init__(self):
        self.codes = 0
        self.codes_diff = 0
        self.codes_big = 0
        self.rows = 0
        self.rho_diff = 0
        self.cols = 0
        self.c_diff = 0

    def add(self, pair: Pair, h, g_blob, o_blob, X_oracle):
        rb = pair.row_bits[h]
        if pair.ora.head_layout(h)[1] and np.all(rb == 16) and pair.cfg.unit_kind == W.UNIT_HEAD:
            gS = pair.ora.dequantize_head(h, g_blob)
            oS = pair.ora.dequantize_head(h, o_blob)
            d = np.abs(gS.astype(np.float64) - oS) <= np.abs(oS) * 2.0 ** -10 + 1e-30
            self.codes += d.size
            self.codes_diff += int(np.sum(~d))
            return
        gc, gp, gr, gcc = pair.ora.unpack_codes(h, g_blob)
        oc, op_, orr, occ = pair.ora.unpack_codes(h, o_blob)
        q = rb != 16
        self.rows += int(np.sum(q))
        rdiff = gr[q] != orr[q]
        self.rho_diff += int(np.sum(rdiff))
        assert np.all(np.abs(gr[q].astype(np.int64) - orr[q].astype(np.int64)) <= 1), "row factor off by > 1 ulp"
        self.cols += gcc.size
        cdiff = gcc != occ
        self.c_diff += int(np.sum(cdiff))
        dc = np.abs(gc.astype(np.int64) - oc.astype(np.int64))[q]
        self.codes += dc.size
        self.codes_diff += int(np.sum(dc > 0))
        big = dc > 1
        # a difference larger than one level is allowed only in a column whose
        # scale differs or in a row whose factor differs
        ok = cdiff[None, :] | rdiff[:, None]
        assert not np.any(big & ~ok), "code differs by more than 1 outside a re-scaled column/row"
        self.codes_big += int(np.sum(big))
        # piv rows: halves within one half-ulp-ish of each other
        if np.any(~q):
            a = h2f(gp[~q])
            b = h2f(op_[~q])
            assert np.all(np.abs(a - b) <= np.abs(b) * 2.0 ** -10 + 2.0 ** -24)

    def check(self, frac=1e-3):
        assert self.codes_diff <= frac * max(self.codes, 1), vars(self)
        assert self.rho_diff <= frac * max(self.rows, 1) + 1, vars(self)
        assert self.c_diff <= frac * max(self.cols, 1) + 1, vars(self)
