"""The readout kernel alone, through the C ABI (stepq_decode_readout).

The readout forms u_j = sum_i k_i (g_i S_ij) in ascending i with the plain
definition's roundings, so the delta vector it leaves in the workspace
(delta = beta (v - u), hyper.ai summary, Method, last paragraph: the output
is produced before requantisation) must equal the oracle's bit for bit; the
readout y = X^T q must match within relative L2 1e-5, checked here for every
head on its own (not only over the whole batch).  Workloads: the gdn shape
with each one-width plan (4, 6, 8 bits) and with its mixed plan (one FP16
pivot head), kda (per-key-row widths with FP16 pivot rows, permuted slots)
and the tiny d = 64 head, all in the launch configuration the benchmark
uses (every request of the workload in one launch).
"""

import numpy as np
import pytest

import oracle
import workload as W
from gpu_harness import Pair, dev, lib, pool_to_host, rel_l2

pytestmark = pytest.mark.gpu


def _run(cfg, pair, picks, seeded_reqs):
    import torch
    S = lib()
    R, H, d = cfg.requests, cfg.heads, cfg.d
    slots_np = W.slot_indices(cfg)
    slots = dev(slots_np)
    X = torch.randn((R, H, d, d), dtype=torch.float32, device="cuda")
    X *= torch.exp(torch.randn((R, H, d, 1), device="cuda"))
    X0s = W.initial_state(cfg, seeded_reqs)
    for a, r in enumerate(seeded_reqs):
        X[r] = torch.from_numpy(X0s[a]).cuda()
    pool = pair.gpu_pool(cfg.pool_slots)
    S.stepq_pack(pair.gpu, pool, slots, X)
    del X
    g0 = pool_to_host(pool)
    si = W.step_inputs(cfg, 0, pair.pin)
    dt = torch.bfloat16 if cfg.bf16_inputs else torch.float32
    q, k, v = (torch.from_numpy(a).to(dt).cuda() for a in (si.q, si.k, si.v))
    beta, gate = torch.from_numpy(si.beta).cuda(), torch.from_numpy(si.gate).cuda()
    y = torch.full((R, H, d), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.full((S.stepq_workspace_bytes(pair.gpu, R) // 4,), float("nan"), dtype=torch.float32,
                    device="cuda")
    S.stepq_decode_readout(pair.gpu, pool, slots, q, k, v, beta, gate, y, ws)
    torch.cuda.synchronize()
    assert np.array_equal(pool_to_host(pool), g0), "the readout must not write the pool"
    assert S.stepq_get_status(pool) == 0
    yg = y.cpu().numpy()
    dg = ws.cpu().numpy()[:R * H * d].reshape(R, H, d)
    worst = 0.0
    ys, yos = [], []
    for r, h in picks:
        blob = pair.head_blob(g0, slots_np[r], h)
        ob, st = pair.ora.quantize_head(h, X0s[seeded_reqs.index(r), h])
        assert st == 0 and np.array_equal(blob, ob), (r, h)
        Sm = pair.ora.dequantize_head(h, blob)
        g = si.gate[r, h]
        _, yo, do = oracle.delta_update(Sm, si.q[r, h], si.k[r, h], si.v[r, h], si.beta[r, h],
                                        g, cfg.gate_kind, with_delta=True)
        assert np.array_equal(dg[r, h].view(np.uint32), do.view(np.uint32)), \
            f"delta of (request {r}, head {h}) differs from the oracle's"
        e = rel_l2(yg[r, h], yo)
        worst = max(worst, e)
        ys.append(yg[r, h])
        yos.append(yo)
    assert worst <= 1e-5, f"largest per-head readout rel-L2 {worst}"
    assert rel_l2(np.array(ys), np.array(yos)) <= 1e-5


@pytest.mark.parametrize("bits", [4, 6, 8, None])
def test_readout_gdn_every_head(bits):
    cfg = W.CONFIGS["gdn"]
    pair = Pair(cfg, uniform_bits=bits) if bits else Pair(cfg)
    R, H = 16, cfg.heads
    import dataclasses
    cfg = dataclasses.replace(cfg, requests=R, pool_slots=R)
    picks = [(r, h) for r in range(R) for h in range(H)]
    _run(cfg, pair, picks, list(range(R)))


def test_readout_gdn_fullsize_sampled():
    cfg = W.CONFIGS["gdn"]
    pair = Pair(cfg)
    rng = np.random.default_rng(7)
    picks = sorted({(int(rng.integers(cfg.requests)), int(rng.integers(cfg.heads))) for _ in range(96)})
    _run(cfg, pair, picks, sorted({r for r, _ in picks}))


def test_readout_kda_fullsize_sampled():
    cfg = W.CONFIGS["kda"]
    pair = Pair(cfg)
    rng = np.random.default_rng(8)
    picks = sorted({(int(rng.integers(cfg.requests)), int(rng.integers(cfg.heads))) for _ in range(128)})
    # every head of one request too: all row-width mixes of the plan
    picks = sorted(set(picks) | {(3, h) for h in range(cfg.heads)})
    _run(cfg, pair, picks, sorted({r for r, _ in picks}))


def test_readout_tiny_d64():
    cfg = W.CONFIGS["tiny"]
    for bits in (4, 6, 8):
        pair = Pair(cfg, uniform_bits=bits)
        _run(cfg, pair, [(0, h) for h in range(cfg.heads)], [0])
