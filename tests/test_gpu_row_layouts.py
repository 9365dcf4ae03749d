"""Per-key-row widths that stress the fit kernel's staging, against the oracle.

In the fit kernel each warp stages its 16 packed rows inside the fp32 rows it
is about to write, and writes the new packed rows over the start of those
rows.  Which bytes overlap depends on the widths of the warp's rows: FP16
pivot rows are the widest (half an fp32 row), so blocks of pivot rows, a pivot
row at the start or end of a warp's block, and heads made almost or entirely
of pivot rows are the cases where an ordering mistake would show.  Plans with
such widths are packed and stepped on both sides; the bytes must be identical
(the KDA row-unit method of the rcap.io post, "Unit granularity" paragraph;
pivot rows kept in FP16, hyper.ai summary, "Method").
"""

import dataclasses

import numpy as np
import pytest

import workload as W
from gpu_harness import Pair, dev, lib, pool_to_host, rel_l2, step_tensors

pytestmark = pytest.mark.gpu


def _patterns(d: int) -> np.ndarray:
    """Row widths [heads][d]: one adversarial pattern per head."""
    rng = np.random.default_rng(20261202 + d)
    blocks = [
        [16] * 16,                                   # a warp of pivot rows (largest staged block)
        [4] * 16,                                    # narrowest block after the widest
        [16, 6] * 8,                                 # alternating
        [8] * 15 + [16],                             # pivot row last in its warp
        [16] + [6] * 15,                             # pivot row first in its warp
        [4, 6, 8, 16] * 4,                           # every width
        [16] * 12 + [4] * 4,
        [6] * 4 + [16] * 12,
    ]
    heads = []
    heads.append(np.concatenate([blocks[k % len(blocks)] for k in range(d // 16)]))
    heads.append(np.array([16] * (d - 1) + [4]))            # almost all pivot rows
    heads.append(rng.choice([4, 6, 8, 16], size=d))         # random widths
    heads.append(rng.choice([4, 16], size=d))               # half pivot rows
    heads.append(np.full(d, 6))                             # uniform rows in a row-unit plan
    heads.append(np.full(d, 16))                            # every row a pivot row
    return np.stack(heads).astype(np.uint8)


def _config(d: int) -> W.Config:
    base = W.CONFIGS["kda"]
    return dataclasses.replace(base, name=f"rowlayout{d}", seed=40 + d, requests=3, heads=6, d=d,
                               pool_slots=5, permute_slots=False, bf16_inputs=(d == 128))


@pytest.mark.parametrize("d", [64, 128])
def test_row_width_patterns_pack_and_step_match_oracle(d):
    import torch
    cfg = _config(d)
    bits = _patterns(d)
    pair = Pair(cfg, bits=bits)
    S = lib()
    R = cfg.requests
    slots = np.array([4, 0, 2], dtype=np.int32)
    X0 = W.initial_state(cfg, range(R))
    # admission: pack the same fp32 states on both sides
    o = pair.ora.new_pool(cfg.pool_slots)
    assert pair.ora.pack(o, slots, X0) == 0
    pool = pair.gpu_pool(cfg.pool_slots)
    S.stepq_pack(pair.gpu, pool, dev(slots), dev(X0))
    assert np.array_equal(pool_to_host(pool), o)
    ws = torch.empty(S.stepq_workspace_bytes(pair.gpu, R), dtype=torch.uint8, device="cuda")
    y = torch.empty((R, cfg.heads, d), dtype=torch.float32, device="cuda")
    side = torch.cuda.Stream()
    for step in range(3):
        si = W.step_inputs(cfg, step, pair.pin, range(R))
        t = step_tensors(cfg, si)
        S.stepq_decode_step(pair.gpu, pool, dev(slots), t["q"], t["k"], t["v"], t["beta"], t["gate"],
                            y, ws, None, side)
        torch.cuda.synchronize()
        yo = np.zeros((R, cfg.heads, d), np.float32)
        for r in range(R):
            for h in range(cfg.heads):
                off, nb = pair.ora.head_layout(h)
                base = int(slots[r]) * pair.slot_bytes + off
                blob = o[base:base + nb].copy()
                yy, _, _ = pair.ora.step_head(h, blob, si.q[r, h], si.k[r, h], si.v[r, h],
                                              si.beta[r, h], si.gate[r, h])
                o[base:base + nb] = blob
                yo[r, h] = yy
        assert rel_l2(y.cpu().numpy(), yo) <= 1e-5
        assert np.array_equal(pool_to_host(pool), o), f"state bytes differ after step {step}"
    assert S.stepq_get_status(pool) == 0
