"""Seeded synthetic inputs for the quantised gated Delta-rule decode step.

This module is the only code shared by the CPU oracle (``oracle/``) and the CUDA
path (``quantized_delta_rule_decode_b200``).  It draws random numbers and lays
them out; it contains none of the method's arithmetic (no state update, no
readout, no scale fitting, no quantisation, no packing).

Every tensor is drawn from its own counter-addressed stream: the numpy
``SeedSequence`` entropy is ``(config seed, tensor tag, step, request, ...)``,
so any (request, head) can be regenerated on its own, which is what the
sampled full-size parity tests rely on.

Workloads (the five synthetic configurations the pages' serving scenario maps
to; the pages run on model traces that are not available, see the STEPQuant
rcap.io post, "Calibration" paragraph):

* ``tiny``   : 1 request x 4 heads, d=64, fp32 inputs, uniform 6-bit, 16 steps
* ``gdn``    : 64 requests x 32 heads, d=128, bf16 q/k/v, per-head {4,6,8}
               plan averaging 6 bits + 1% FP16 pivot heads
* ``kda``    : 256 requests x 32 heads, d=128, per-key-row gates and widths,
               0.5% pivot rows, slots a permutation of a 512-slot pool
* ``pool``   : 1024 requests x 32 heads, d=128, 4-bit budget + 1% pivot heads
* ``rollout``: 128 requests x 16 heads, d=128, 6-bit mix, 4096 steps

Input recipe (all configurations): q, k ~ N(0,1) then L2-normalised in fp32;
v ~ N(0,1); q, k, v rounded to bf16 (RNE) except for ``tiny``;
beta = sigmoid(N(0,1)); per-unit half-life h log-uniform in [1, h_max] and
gate g = exp(-1/h); S0 = diag(a) G diag(b) with G ~ N(0,1), a, b ~
lognormal(0,1); row-impact weights w ~ lognormal(0, 0.5) per (head, key row).

Synthetic plan (stands in for the offline lifetime-aware allocator): units
(heads, or key rows for KDA) ranked by half-life, longest first, ties by
index; the top max(1, round(p * units)) become FP16 pivots; of the rest, for
a 6-bit budget the top quarter get 8 bits, the bottom quarter 4 bits and the
middle 6 bits; for a 4-bit budget all get 4 bits.
"""

from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# tensor tags for the counter-addressed streams
_T_PLAN_HALF = 1
_T_PLAN_W = 2
_T_S0 = 3
_T_STEP = 4
_T_SLOTS = 5

GATE_SCALAR = 0
GATE_DIAG = 1
UNIT_HEAD = 0
UNIT_ROW = 1
MODE_STEPQUANT = 0
MODE_UNIFORM = 1


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    seed: int
    requests: int
    heads: int
    d: int
    steps: int
    gate_kind: int
    unit_kind: int
    budget: int            # 6 or 4: average bits of the non-pivot units
    pivot_frac: float      # fraction of units kept as FP16 pivots (0: none)
    half_life_max: float
    bf16_inputs: bool
    pool_slots: int        # slots in the pool (>= requests)
    permute_slots: bool    # slot indices a random permutation of the pool
    uniform_bits: int = 0  # >0: every unit gets this width, no pivots

    @property
    def units(self) -> int:
        return self.heads * (self.d if self.unit_kind == UNIT_ROW else 1)

    def head_updates_per_step(self) -> int:
        return self.requests * self.heads


CONFIGS = {
    "tiny": Config("tiny", 0, 1, 4, 64, 16, GATE_SCALAR, UNIT_HEAD, 6, 0.0,
                   256.0, False, 1, False, uniform_bits=6),
    "gdn": Config("gdn", 1, 64, 32, 128, 1000, GATE_SCALAR, UNIT_HEAD, 6,
                  0.01, 4096.0, True, 64, False),
    "kda": Config("kda", 2, 256, 32, 128, 1000, GATE_DIAG, UNIT_ROW, 6,
                  0.005, 4096.0, True, 512, True),
    "pool": Config("pool", 3, 1024, 32, 128, 1000, GATE_SCALAR, UNIT_HEAD, 4,
                   0.01, 4096.0, True, 1024, False),
    "rollout": Config("rollout", 4, 128, 16, 128, 4096, GATE_SCALAR, UNIT_HEAD,
                      6, 0.0, 4096.0, True, 128, False),
}
CONFIG_ORDER = ["tiny", "gdn", "kda", "pool", "rollout"]


def _rng(*entropy: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(entropy))))


@dataclasses.dataclass
class PlanInputs:
    """What the offline allocator hands the runtime, plus the gate half-lives."""
    bits: np.ndarray        # uint8 [units]: 4/6/8, or 16 for an FP16 pivot
    w: np.ndarray           # float32 [heads, d]: row-impact weights (> 0)
    half_life: np.ndarray   # float64 [heads] (scalar gate) or [heads, d] (diagonal)
    gate: np.ndarray        # float32, same shape: g = exp(-1/h)


def make_plan(cfg: Config, *, budget: int | None = None, uniform_bits: int | None = None,
              pivots: bool = True) -> PlanInputs:
    """Synthetic plan: half-lives, gates, row-impact weights and unit widths."""
    r = _rng(cfg.seed, _T_PLAN_HALF)
    shape = (cfg.heads, cfg.d) if cfg.gate_kind == GATE_DIAG else (cfg.heads,)
    half_life = np.exp(r.uniform(0.0, np.log(cfg.half_life_max), size=shape))
    gate = np.exp(-1.0 / half_life).astype(np.float32)
    w = _rng(cfg.seed, _T_PLAN_W).lognormal(0.0, 0.5, size=(cfg.heads, cfg.d)).astype(np.float32)

    ub = cfg.uniform_bits if uniform_bits is None else uniform_bits
    bud = cfg.budget if budget is None else budget
    n = cfg.units
    bits = np.zeros(n, dtype=np.uint8)
    if ub:
        bits[:] = ub
    else:
        # unit lifetime: per-head half-life (HEAD units) or per-row (ROW units)
        life = half_life.reshape(-1)
        if cfg.unit_kind == UNIT_ROW and cfg.gate_kind == GATE_SCALAR:
            life = np.repeat(half_life, cfg.d)
        order = np.lexsort((np.arange(n), -life))   # longest first, ties by index
        n_piv = max(1, int(round(cfg.pivot_frac * n))) if (pivots and cfg.pivot_frac > 0) else 0
        rest = order[n_piv:]
        bits[order[:n_piv]] = 16
        if bud == 6:
            q = len(rest) // 4
            bits[rest[:q]] = 8
            bits[rest[q:len(rest) - q]] = 6
            bits[rest[len(rest) - q:]] = 4
        elif bud == 4:
            bits[rest] = 4
        else:
            raise ValueError(f"budget {bud} not in (4, 6)")
    return PlanInputs(bits=bits, w=w, half_life=half_life, gate=gate)


def slot_indices(cfg: Config) -> np.ndarray:
    """int32 [requests]: the pool slot of each request."""
    if cfg.permute_slots:
        perm = _rng(cfg.seed, _T_SLOTS).permutation(cfg.pool_slots)
        return perm[: cfg.requests].astype(np.int32)
    return np.arange(cfg.requests, dtype=np.int32)


def _s0_one(cfg: Config, req: int, head: int) -> np.ndarray:
    r = _rng(cfg.seed, _T_S0, req, head)
    g = r.standard_normal((cfg.d, cfg.d))
    a = r.lognormal(0.0, 1.0, size=cfg.d)
    b = r.lognormal(0.0, 1.0, size=cfg.d)
    return ((a[:, None] * g) * b[None, :]).astype(np.float32)


def initial_state(cfg: Config, requests=None, heads=None, out: np.ndarray | None = None,
                  threads: int | None = None) -> np.ndarray:
    """float32 [len(requests), len(heads), d, d]: S0 = diag(a) G diag(b) per (request, head)."""
    requests = list(range(cfg.requests)) if requests is None else list(requests)
    heads = list(range(cfg.heads)) if heads is None else list(heads)
    if out is None:
        out = np.empty((len(requests), len(heads), cfg.d, cfg.d), dtype=np.float32)

    def fill(ri):
        for hi, h in enumerate(heads):
            out[ri, hi] = _s0_one(cfg, requests[ri], h)

    nt = threads or min(16, os.cpu_count() or 1)
    if len(requests) * len(heads) > 64 and nt > 1:
        with ThreadPoolExecutor(nt) as ex:
            list(ex.map(fill, range(len(requests))))
    else:
        for ri in range(len(requests)):
            fill(ri)
    return out


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returned as float32."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


@dataclasses.dataclass
class StepInputs:
    q: np.ndarray      # float32 [R, H, d] (values already bf16-representable when bf16_inputs)
    k: np.ndarray
    v: np.ndarray
    beta: np.ndarray   # float32 [R, H]
    gate: np.ndarray   # float32 [R, H] (scalar) or [R, H, d] (diagonal)


def step_inputs(cfg: Config, step: int, plan: PlanInputs, requests=None, heads=None) -> StepInputs:
    """Fresh q, k, v, beta for one decode step; gates from the plan's half-lives."""
    requests = list(range(cfg.requests)) if requests is None else list(requests)
    heads = list(range(cfg.heads)) if heads is None else list(heads)
    R, H, d = len(requests), len(heads), cfg.d
    q = np.empty((R, H, d), np.float32)
    k = np.empty((R, H, d), np.float32)
    v = np.empty((R, H, d), np.float32)
    beta = np.empty((R, H), np.float32)
    for ri, req in enumerate(requests):
        r = _rng(cfg.seed, _T_STEP, step, req)
        z = r.standard_normal((cfg.heads, 3, d)).astype(np.float32)
        bz = r.standard_normal(cfg.heads)
        z = z[heads]
        qq, kk = z[:, 0], z[:, 1]
        q[ri] = qq / np.sqrt(np.sum(qq * qq, axis=-1, keepdims=True, dtype=np.float32))
        k[ri] = kk / np.sqrt(np.sum(kk * kk, axis=-1, keepdims=True, dtype=np.float32))
        v[ri] = z[:, 2]
        beta[ri] = (1.0 / (1.0 + np.exp(-bz[heads]))).astype(np.float32)
    if cfg.bf16_inputs:
        q, k, v = bf16_round(q), bf16_round(k), bf16_round(v)
    g = plan.gate[heads]
    gate = np.broadcast_to(g, (R,) + g.shape).astype(np.float32).copy()
    return StepInputs(q=q, k=k, v=v, beta=beta, gate=gate)


def fp32_state_bytes(cfg: Config) -> int:
    return cfg.heads * cfg.d * cfg.d * 4
