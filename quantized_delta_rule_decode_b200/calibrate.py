"""Offline calibration of a plan, driven through the C ABI.

hyper.ai summary of the paper, section "Method" (the paragraphs on
Lifetime-Aware Bit Allocation and on the spatial distribution of errors);
rcap.io post, "Temporal" part and the sentence placing calibration offline.
Before decoding, every key row gets its impact weight and every state unit
(a head, or one key row) its width:

0. the plan's row-impact weights from the calibration inputs
   (``stepq_row_impact``, ``stepq_impact_weights``; hyper.ai, the paragraph on
   the spatial distribution of errors);
1. quantise calibration states with a plan of one width b for every unit
   (b = 4, 6, 8; the full quantiser: row factors, dual-axis fit) and measure
   each unit's squared reconstruction error (``stepq_unit_distortion``);
2. the unit's lifetime weight from its retention gates
   (``stepq_lifetime_weight``);
3. FP16 pivots and the widths of the rest under the budget
   (``stepq_allocate_bits``).

Every measurement runs in the library's kernels (``stepq_pack``,
``stepq_unit_distortion``); this module only sums the per-request results
and passes arrays between the calls.
"""

from __future__ import annotations

import numpy as np

from ._ffi import (MODE_STEPQUANT, UNIT_ROW, stepq_allocate_bits, stepq_impact_weights,
                   stepq_lifetime_weight, stepq_pack, stepq_plan_create, stepq_pool_alloc,
                   stepq_plan_slot_bytes, stepq_row_impact, stepq_unit_distortion_accumulate)

WIDTHS = (4, 6, 8)


def impact_weights(gate_kind, d_k, n_heads, inputs, stream=None) -> np.ndarray:
    """The plan's row-impact weights w [n_heads][d_k] from calibration inputs.

    hyper.ai summary, section "Method" (the paragraph on the spatial
    distribution of errors): a key row's impact score is the mean square of
    the factor through which its error reaches the readout; the weight is its
    square root.  inputs: iterable of device (q, k, beta, gate) in the decode
    step's layouts ([n][n_heads][d_k], [n][n_heads], gate per head or row)."""
    import torch
    score = None
    count = 0
    for q, k, beta, gate in inputs:
        if score is None:
            score = torch.zeros((n_heads, d_k), dtype=torch.float64, device=q.device)
        stepq_row_impact(gate_kind, q, k, beta, gate, score, stream=stream)
        count += q.shape[0]
    if score is None:
        raise ValueError("no calibration inputs")
    return stepq_impact_weights(score.cpu().numpy(), count).reshape(n_heads, d_k)


def measure_distortion(d_k, d_v, n_heads, gate_kind, unit_kind, w, states, stream=None):
    """Distortion of every unit at 4, 6 and 8 bits, summed over the states.

    states: device fp32 tensors [n][n_heads][d_k][d_v] (any n per tensor).
    Returns float64 [units][3]: per unit, the squared reconstruction error
    summed over every request of every state tensor, on the device
    (stepq_unit_distortion_accumulate); this function only passes buffers."""
    import torch
    units = n_heads * d_k if unit_kind == UNIT_ROW else n_heads
    total = np.zeros((units, 3), np.float64)
    for col, b in enumerate(WIDTHS):
        plan = stepq_plan_create(d_k, d_v, n_heads, gate_kind, unit_kind, MODE_STEPQUANT,
                                 np.full(units, b, np.uint8), w)
        sb = stepq_plan_slot_bytes(plan)
        dist_sum = None
        for X in states:
            n = X.shape[0]
            if dist_sum is None:
                dist_sum = torch.zeros(units, dtype=torch.float64, device=X.device)
            buf = torch.zeros(n * sb, dtype=torch.uint8, device=X.device)
            pool = stepq_pool_alloc(plan, n, buf)
            slots = torch.arange(n, dtype=torch.int32, device=X.device)
            stepq_pack(plan, pool, slots, X, stream=stream)
            stepq_unit_distortion_accumulate(plan, pool, slots, X, dist_sum, stream=stream)
        if dist_sum is not None:
            total[:, col] = dist_sum.cpu().numpy()
    return total


def lifetime_weights(gates) -> np.ndarray:
    """gates: host [n_steps][units][gates_per_unit] in (0, 1) -> float64 [units]."""
    return stepq_lifetime_weight(gates)


def allocate(weight, dist, budget_bits: int, n_pivots: int) -> np.ndarray:
    """Per-unit widths (4, 6, 8; 16 = FP16 pivot)."""
    return stepq_allocate_bits(weight, dist, budget_bits, n_pivots)


def calibrate_bits(d_k, d_v, n_heads, gate_kind, unit_kind, w, states, gates, budget_bits: int,
                   n_pivots: int, stream=None):
    """The whole offline step: returns (bits, weight, dist)."""
    dist = measure_distortion(d_k, d_v, n_heads, gate_kind, unit_kind, w, states, stream)
    weight = lifetime_weights(gates)
    return allocate(weight, dist, budget_bits, n_pivots), weight, dist
