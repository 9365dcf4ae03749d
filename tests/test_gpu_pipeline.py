"""The overlapped multi-layer schedule the benchmark times, against the oracle.

The pages run the scale fit and pack write-back on a second CUDA stream,
overlapped with the following computation (hyper.ai summary, Method, last
paragraph; rcap.io post, the sentence after the pseudocode).  The benchmark
does this over several layers: the readouts run on a high-priority main
stream, and layer l's fit + pack on one of two side streams taken in turn, so
that it runs beside layer l + 1's readout and beside the start of layer
l + 1's fit; each layer has its own pool and workspace, and the next step's
readout of a layer waits for that layer's previous fit.  This test runs that
schedule on the full gdn workload (64 requests x 32 heads per layer, three
layers, eight steps), alternating stepq_decode_step with the split calls
(stepq_decode_readout, an event, stepq_decode_fitpack on the side stream)
that the benchmark's instrumented pass uses.  After every step of every
layer, a copy of the pool taken on that layer's side stream and of y taken
on the main stream (so the steps still overlap)
are compared on sampled (request, head) pairs with the oracle continuing
from its own state: identical bytes, and y within relative L2 1e-5 per head.
A race (a missing event, a shared workspace) would show as a difference.
"""

import numpy as np
import pytest

import workload as W
from gpu_harness import Pair, dev, lib, rel_l2

pytestmark = pytest.mark.gpu

LAYERS, STEPS, SAMPLES = 3, 8, 10


def test_overlapped_layers_match_oracle():
    import torch
    cfg = W.CONFIGS["gdn"]
    pair = Pair(cfg)
    S = lib()
    R, H, d = cfg.requests, cfg.heads, cfg.d
    slots = dev(np.arange(R, dtype=np.int32))
    X0 = torch.from_numpy(W.initial_state(cfg)).cuda()
    pools, wss, ys = [], [], []
    for _ in range(LAYERS):
        p = pair.gpu_pool(R)
        S.stepq_pack(pair.gpu, p, slots, X0)
        pools.append(p)
        wss.append(torch.empty(S.stepq_workspace_bytes(pair.gpu, R), dtype=torch.uint8, device="cuda"))
        ys.append(torch.empty((R, H, d), dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    g0 = pools[0].buf.cpu().numpy()
    rng = np.random.default_rng(11)
    picks = [sorted({(int(rng.integers(R)), int(rng.integers(H))) for _ in range(SAMPLES)})
             for _ in range(LAYERS)]
    blobs = [{(r, h): pair.head_blob(g0, r, h).copy() for r, h in picks[l]} for l in range(LAYERS)]
    main = torch.cuda.Stream(priority=-5)
    sides = [torch.cuda.Stream(), torch.cuda.Stream()]
    main.wait_stream(torch.cuda.current_stream())   # the packs above
    keep, snaps = [], []
    dt = torch.bfloat16
    for s in range(STEPS):
        for l in range(LAYERS):
            si = W.step_inputs(cfg, s * LAYERS + l, pair.pin)
            q, k, v = (torch.from_numpy(a).to(dt).cuda() for a in (si.q, si.k, si.v))
            beta, gate = torch.from_numpy(si.beta).cuda(), torch.from_numpy(si.gate).cuda()
            keep.append((q, k, v, beta, gate))
            side = sides[l % 2]
            main.wait_stream(torch.cuda.current_stream())   # the inputs' copies
            if s % 2 == 0:
                S.stepq_decode_step(pair.gpu, pools[l], slots, q, k, v, beta, gate, ys[l], wss[l], main, side)
            else:
                S.stepq_decode_readout(pair.gpu, pools[l], slots, q, k, v, beta, gate, ys[l], wss[l], main)
                ev = torch.cuda.Event()
                ev.record(main)
                side.wait_event(ev)
                S.stepq_decode_fitpack(pair.gpu, pools[l], slots, k, gate, wss[l], side)
            with torch.cuda.stream(main):
                y_snap = ys[l].clone()              # on main, after this layer's readout
            with torch.cuda.stream(side):
                p_snap = pools[l].buf.clone()       # on the side stream, after this layer's fit
            snaps.append((s, l, si, y_snap, p_snap))
    for side in sides:
        main.wait_stream(side)
    torch.cuda.synchronize()
    worst = 0.0
    for s, l, si, y_snap, p_snap in snaps:
        gb = p_snap.cpu().numpy()
        yg = y_snap.cpu().numpy()
        for r, h in picks[l]:
            blob = blobs[l][(r, h)]
            yo, _, st = pair.ora.step_head(h, blob, si.q[r, h], si.k[r, h], si.v[r, h], si.beta[r, h],
                                           si.gate[r, h])
            assert st == 0
            assert np.array_equal(pair.head_blob(gb, r, h), blob), \
                f"step {s} layer {l} (request {r}, head {h}): packed state differs"
            worst = max(worst, rel_l2(yg[r, h], yo))
    assert worst <= 1e-5, f"largest per-head readout rel-L2 {worst}"
    for p in pools:
        assert S.stepq_get_status(p) == 0
