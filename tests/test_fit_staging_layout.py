"""The slot format leaves room for the fit kernel's in-place staging.

The fit kernel gives each warp 16 consecutive key rows.  It copies their
packed bytes, which are contiguous in the slot, into the END of the warp's 16
fp32 rows of X in shared memory, rebuilds X row by row in ascending order, and
later writes the new packed rows from the START of the same region.  That is
safe when, for every width mix the format allows (4, 6, 8 bits or FP16 per
key row):

* the warp's packed rows start on a 16-byte boundary and span a multiple of
  16 bytes (one bulk copy each way), and fit in the region;
* writing X row r never reaches a packed row after r that is still unread;
* writing packed row r never reaches an X row after r that is still unread.

The row layout is the format's (key rows ascending, a b-bit row d_v * b / 8
bytes, an FP16 row 2 d_v bytes; STEPQuant rcap.io post, "Unit granularity"),
cross-checked against the oracle's head sizes.  No GPU is needed.
"""

import numpy as np
import pytest

import oracle
import workload as W


def _row_bytes(d, bits):
    return np.array([2 * d if int(b) == 16 else d * int(b) // 8 for b in bits], np.int64)


def _check_head(d, bits):
    rb = _row_bytes(d, bits)
    off = np.concatenate([[0], np.cumsum(rb)])
    RB = 4 * d                   # one fp32 row of X
    W_ = 16 * RB                 # a warp's 16 rows of X
    for w in range(d // 16):
        r0 = 16 * w
        p0, pb = off[r0], off[r0 + 16] - off[r0]
        assert p0 % 16 == 0 and pb % 16 == 0 and 0 < pb <= W_ // 2
        stage = W_ - pb          # packed rows staged at the end of the region
        for r in range(16):
            start_in = stage + off[r0 + r] - p0
            # X row r (bytes [r RB, (r + 1) RB)) ends before any later packed row
            if r + 1 < 16:
                assert (r + 1) * RB <= stage + off[r0 + r + 1] - p0
            # its own packed row lies within the region, a 4-byte over-read included
            assert 0 <= start_in and start_in + rb[r0 + r] <= W_
            # packed row r, written from the start, ends before X row r + 1
            assert off[r0 + r] - p0 + rb[r0 + r] <= (r + 1) * RB


@pytest.mark.parametrize("d", [64, 128])
def test_staging_invariants_hold_for_every_width_mix(d):
    rng = np.random.default_rng(7 + d)
    patterns = [np.full(d, b) for b in (4, 6, 8, 16)]
    patterns += [rng.choice([4, 6, 8, 16], size=d) for _ in range(300)]
    patterns += [rng.choice([4, 16], size=d, p=[0.2, 0.8]) for _ in range(100)]
    for bits in patterns:
        _check_head(d, bits)


@pytest.mark.parametrize("d", [64, 128])
def test_row_layout_matches_the_oracle_head_sizes(d):
    rng = np.random.default_rng(11 + d)
    H = 3
    bits = rng.choice([4, 6, 8, 16], size=(H, d)).astype(np.uint8)
    bits[2] = 6
    w = np.ones((H, d), np.float32)
    ora = oracle.Plan(d, d, H, W.GATE_DIAG, W.UNIT_ROW, W.MODE_STEPQUANT, bits.reshape(-1), w)
    for h in range(H):
        _, nb = ora.head_layout(h)
        codes = int(_row_bytes(d, bits[h]).sum())
        assert nb == -(-(codes + 4 * d) // 16) * 16   # rows, then rho and c as halves, 16-byte padded
