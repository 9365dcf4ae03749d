"""The seeded synthetic inputs: determinism, addressability and the plan recipe."""

import numpy as np

import workload as W


def test_plan_recipe_counts():
    def counts(name):
        b = W.make_plan(W.CONFIGS[name]).bits
        return {k: int(np.sum(b == k)) for k in (4, 6, 8, 16)}
    assert counts("tiny") == {4: 0, 6: 4, 8: 0, 16: 0}
    assert counts("gdn") == {4: 7, 6: 17, 8: 7, 16: 1}
    assert counts("kda") == {4: 1019, 6: 2038, 8: 1019, 16: 20}
    assert counts("pool") == {4: 31, 6: 0, 8: 0, 16: 1}
    assert counts("rollout") == {4: 4, 6: 8, 8: 4, 16: 0}


def test_plan_ranks_by_half_life():
    cfg = W.CONFIGS["gdn"]
    p = W.make_plan(cfg)
    order = np.argsort(-p.half_life, kind="stable")
    assert p.bits[order[0]] == 16                      # longest-lived head is the pivot
    assert np.all(p.bits[order[1:8]] == 8) and np.all(p.bits[order[-7:]] == 4)
    assert np.allclose(p.gate, np.exp(-1.0 / p.half_life).astype(np.float32))
    assert np.all((p.half_life >= 1) & (p.half_life <= 4096))


def test_inputs_are_addressable_and_deterministic():
    cfg = W.CONFIGS["kda"]
    p = W.make_plan(cfg)
    full = W.step_inputs(cfg, 3, p, requests=range(4))
    part = W.step_inputs(cfg, 3, p, requests=[2], heads=[5, 7])
    assert np.array_equal(part.q[0], full.q[2, [5, 7]])
    assert np.array_equal(part.gate[0], full.gate[2, [5, 7]])
    s_full = W.initial_state(cfg, requests=[1, 2], heads=range(3))
    s_part = W.initial_state(cfg, requests=[2], heads=[2])
    assert np.array_equal(s_part[0, 0], s_full[1, 2])
    again = W.step_inputs(cfg, 3, p, requests=range(4))
    assert np.array_equal(again.k, full.k)


def test_input_distributions():
    cfg = W.CONFIGS["gdn"]
    p = W.make_plan(cfg)
    si = W.step_inputs(cfg, 0, p, requests=range(8))
    assert np.allclose(np.linalg.norm(si.q, axis=-1), 1.0, atol=1e-2)
    assert np.allclose(np.linalg.norm(si.k, axis=-1), 1.0, atol=1e-2)
    # bf16-representable: the low 16 bits are zero
    assert np.all((si.v.view(np.uint32) & 0xFFFF) == 0)
    assert np.all((si.beta > 0) & (si.beta < 1))
    tiny = W.CONFIGS["tiny"]
    st = W.step_inputs(tiny, 0, W.make_plan(tiny))
    assert np.any((st.v.view(np.uint32) & 0xFFFF) != 0)   # fp32 inputs stay fp32


def test_slot_indices():
    kda = W.CONFIGS["kda"]
    s = W.slot_indices(kda)
    assert s.size == 256 and len(set(s.tolist())) == 256 and s.max() < 512
    assert np.array_equal(W.slot_indices(W.CONFIGS["gdn"]), np.arange(64))
