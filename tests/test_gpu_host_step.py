"""The host-buffer decode step over several layers, against the oracle.

stepq_decode_step_host copies a step's inputs host -> device on a stream of
the pool's own that waits only for that pool's previous fit (not for earlier
work on the main stream), runs the step, and copies y back on a second stream
of the pool's own that the main stream then waits for (the readout emits y
before the state is requantised: rcap.io post, decode-step pseudocode; the fit
runs on a separate stream: hyper.ai summary, Method, last paragraph).  This
test runs it the way a model would: three layers of the full gdn workload (64
requests x 32 heads, six steps) and two layers of the full kda workload (256
requests x 32 heads with per-row gates and widths, which the step takes in
chunks of requests; three steps), each layer with its own pool, staging
workspace and side stream, a high-priority main stream, fresh pinned inputs
and a pinned y buffer for every call and nothing synchronised between calls.  The
staging areas are reused every step, so a copy that overtook the previous
fit of its pool, or a y read back before its readout, would show: after
every step of every layer, sampled (request, head) blobs of a copy of the
pool taken on the layer's side stream must equal the oracle's bytes, and y
must be within relative L2 1e-5 of the oracle per head.
"""

import numpy as np
import pytest

import workload as W
from gpu_harness import Pair, dev, lib, rel_l2

pytestmark = pytest.mark.gpu

SAMPLES = 8


@pytest.mark.parametrize("name,layers,steps", [("gdn", 3, 6), ("kda", 2, 3)])
def test_host_step_layers_match_oracle(name, layers, steps):
    import torch
    cfg = W.CONFIGS[name]
    LAYERS, STEPS = layers, steps
    pair = Pair(cfg)
    S = lib()
    R, H, d = cfg.requests, cfg.heads, cfg.d
    slots = dev(np.arange(R, dtype=np.int32))
    X0 = torch.from_numpy(W.initial_state(cfg)).cuda()
    code = S.DTYPE_BF16
    pools, wss = [], []
    for _ in range(LAYERS):
        p = pair.gpu_pool(R)
        S.stepq_pack(pair.gpu, p, slots, X0)
        pools.append(p)
        wss.append(torch.empty(S.stepq_host_workspace_bytes(pair.gpu, R, code), dtype=torch.uint8,
                               device="cuda"))
    torch.cuda.synchronize()
    g0 = pools[0].buf.cpu().numpy()
    rng = np.random.default_rng(5)
    picks = [sorted({(int(rng.integers(R)), int(rng.integers(H))) for _ in range(SAMPLES)})
             for _ in range(LAYERS)]
    blobs = [{(r, h): pair.head_blob(g0, r, h).copy() for r, h in picks[l]} for l in range(LAYERS)]
    main = torch.cuda.Stream(priority=-5)
    sides = [torch.cuda.Stream() for _ in range(LAYERS)]
    keep, snaps = [], []
    for s in range(STEPS):
        for l in range(LAYERS):
            si = W.step_inputs(cfg, 100 + s * LAYERS + l, pair.pin)
            host = [torch.from_numpy(a).to(torch.bfloat16).pin_memory() for a in (si.q, si.k, si.v)]
            host += [torch.from_numpy(si.beta).pin_memory(), torch.from_numpy(si.gate).pin_memory()]
            y = torch.full((R, H, d), float("nan"), dtype=torch.float32).pin_memory()
            keep.append(host)
            S.stepq_decode_step_host(pair.gpu, pools[l], slots, *host, y, wss[l], main, sides[l])
            with torch.cuda.stream(sides[l]):
                p_snap = pools[l].buf.clone()       # after this layer's fit
            snaps.append((s, l, si, y, p_snap))
    for side in sides:
        main.wait_stream(side)
    main.synchronize()
    torch.cuda.synchronize()
    worst = 0.0
    for s, l, si, y, p_snap in snaps:
        gb = p_snap.cpu().numpy()
        yg = y.numpy()
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
