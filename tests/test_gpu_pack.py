"""GPU pack / unpack vs the oracle, through the C ABI (bit-exact contract).

Pack quantises a given X (the same quantiser the decode step applies to the
updated state: rcap.io post, decode-step pseudocode, its fit and quantise
steps; the key-row-aware dual-axis fit of the hyper.ai summary, "Method").
From an identical X the packed bytes must equal the oracle's.  compare_pack
would also accept an argmin that differs on a near tie (the general
contract), and the tests then require that no column needed it.
"""

import numpy as np
import pytest

import workload as W
from gpu_harness import Pair, compare_pack, dev, lib, new_stats, pool_to_host

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", W.MODE_STEPQUANT, None, 1),
    ("tiny", W.MODE_UNIFORM, 6, 1),
    ("gdn", W.MODE_STEPQUANT, None, 4),
    ("kda", W.MODE_STEPQUANT, None, 3),
    ("pool", W.MODE_STEPQUANT, None, 3),
    ("rollout", W.MODE_STEPQUANT, None, 3),
    ("rollout", W.MODE_UNIFORM, 8, 2),
    ("rollout", W.MODE_UNIFORM, 6, 2),
    ("gdn", W.MODE_STEPQUANT, 4, 2),     # every head 4-bit: the search moves most
    # ablations: lifetime-aware widths with per-row scales only (temporal),
    # the dual-axis fit on uniform widths of key rows (spatial)
    ("gdn", W.MODE_UNIFORM, None, 2),
    ("kda", W.MODE_UNIFORM, None, 2),
    ("kda", W.MODE_STEPQUANT, 6, 2),
]


@pytest.mark.parametrize("name,mode,ub,R", CASES, ids=lambda x: str(x))
def test_pack_matches_oracle(name, mode, ub, R):
    cfg = W.CONFIGS[name]
    pair = Pair(cfg, mode=mode, uniform_bits=ub)
    reqs = list(range(R))
    X = W.initial_state(cfg, reqs)
    slots = np.arange(R, dtype=np.int32)[::-1].copy()
    pool = pair.gpu_pool(R)
    S = lib()
    S.stepq_pack(pair.gpu, pool, dev(slots), dev(X))
    g = pool_to_host(pool)
    o = pair.ora.new_pool(R)
    assert pair.ora.pack(o, slots, X) == 0
    stats = new_stats()
    for r in range(R):
        for h in range(cfg.heads):
            compare_pack(pair, h, pair.head_blob(g, slots[r], h), pair.head_blob(o, slots[r], h),
                         X[r, h], stats)
    assert S.stepq_get_status(pool) == 0
    # the kernels evaluate the column objective in the oracle's stated order,
    # so even the argmin agrees: the bytes are identical
    assert stats["switched_cols"] == 0, stats
    assert np.array_equal(g, o)


def test_pack_degenerate_values():
    """Zero rows and columns, huge and tiny magnitudes, negative zero."""
    cfg = W.CONFIGS["gdn"]
    pair = Pair(cfg)
    rng = np.random.default_rng(9)
    X = W.initial_state(cfg, [0])
    X[0, 0, 5] = 0.0
    X[0, 1, :, 7] = 0.0
    X[0, 2] *= np.float32(1e-30)
    X[0, 3] *= np.float32(1e25)
    X[0, 4, 3] = -0.0
    X[0, 5] = 0.0
    X[0, 6, rng.integers(0, 128, 40), rng.integers(0, 128, 40)] = np.float32(3e4)
    X[0, 8] = np.float32(2.0 ** -140)        # fp32 subnormals
    pool = pair.gpu_pool(1)
    slots = np.zeros(1, np.int32)
    lib().stepq_pack(pair.gpu, pool, dev(slots), dev(X))
    g = pool_to_host(pool)
    o = pair.ora.new_pool(1)
    pair.ora.pack(o, slots, X)
    stats = new_stats()
    for h in range(cfg.heads):
        compare_pack(pair, h, pair.head_blob(g, 0, h), pair.head_blob(o, 0, h), X[0, h], stats)


def test_pack_nonfinite_sets_status():
    cfg = W.CONFIGS["tiny"]
    pair = Pair(cfg)
    X = W.initial_state(cfg)
    X[0, 1, 3, 4] = np.nan
    X[0, 2, 7, 0] = np.inf
    pool = pair.gpu_pool(1)
    slots = np.zeros(1, np.int32)
    S = lib()
    S.stepq_pack(pair.gpu, pool, dev(slots), dev(X))
    g = pool_to_host(pool)
    o = pair.ora.new_pool(1)
    st = pair.ora.pack(o, slots, X)
    assert st & 2
    assert S.stepq_get_status(pool) & S.DEV_NONFINITE
    assert np.array_equal(g, o)


@pytest.mark.parametrize("name,mode,ub", [("tiny", 0, None), ("gdn", 0, None), ("kda", 0, None),
                                          ("rollout", 1, 8)])
def test_unpack_bit_exact(name, mode, ub):
    """GPU reconstruction of oracle-packed slots equals the oracle's, bit for bit."""
    import torch
    cfg = W.CONFIGS[name]
    pair = Pair(cfg, mode=mode, uniform_bits=ub)
    R = 2 if cfg.requests > 1 else 1
    X = W.initial_state(cfg, range(R))
    slots = np.arange(R, dtype=np.int32)
    o = pair.ora.new_pool(R)
    pair.ora.pack(o, slots, X)
    pool = pair.gpu_pool(R)
    pool.buf.copy_(torch.from_numpy(o))
    out = torch.empty((R, cfg.heads, cfg.d, cfg.d), dtype=torch.float32, device="cuda")
    lib().stepq_unpack(pair.gpu, pool, dev(slots), out)
    ref, st = pair.ora.unpack(o, slots)
    assert st == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_bad_slot_flagged_and_skipped():
    import torch
    cfg = W.CONFIGS["tiny"]
    pair = Pair(cfg)
    S = lib()
    pool = pair.gpu_pool(2)
    X = W.initial_state(cfg)
    S.stepq_pack(pair.gpu, pool, dev(np.array([7], np.int32)), dev(X))
    assert S.stepq_get_status(pool) & S.DEV_BAD_SLOT
    assert int(pool.buf.sum().item()) == 0
    S.stepq_clear_status(pool)
    assert S.stepq_get_status(pool) == 0
    out = torch.zeros((1, cfg.heads, cfg.d, cfg.d), dtype=torch.float32, device="cuda")
    S.stepq_unpack(pair.gpu, pool, dev(np.array([-1], np.int32)), out)
    assert S.stepq_get_status(pool) & S.DEV_BAD_SLOT
