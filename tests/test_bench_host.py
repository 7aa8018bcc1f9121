"""Host-side logic of bench.py that needs no GPU: how many timed windows are
taken, and the check of the last timed step's codes against the oracle."""
import os
import sys

import numpy as np
import torch

import synthetic

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_windows_needed():
    assert bench.windows_needed(1.6, 0.5) == 313      # 20 steps of 80 us: 313 windows for 0.5 s
    assert bench.windows_needed(600.0, 0.5) == 1      # a long window is enough alone
    assert bench.windows_needed(0.0, 0.5) == 400      # capped
    assert bench.windows_needed(100.0, 0.25) == 3


def test_spot_check_accepts_the_oracle_and_rejects_a_wrong_code(orc):
    bits = synthetic.sweep(8, tokens=40, seed=11)
    signs = synthetic.sign_bits(256, 5)
    wl = dict(bits=bits, clip=0.9, signs=signs)
    packed, scales = orc.r4_rows(bits, 0.9, signs)
    q, s = torch.from_numpy(packed.copy()), torch.from_numpy(scales.copy())
    rep = bench.spot_check(orc, wl, packed, scales.astype(np.float64), q, s, 40)
    assert rep["ok"] and rep["rows_bit_identical"] == 40
    bad = packed.copy()
    bad[7, 3] ^= 0x40  # one code moved by 4 steps (bit 2 of the high nibble)
    rep = bench.spot_check(orc, wl, packed, scales.astype(np.float64), torch.from_numpy(bad), s, 40)
    assert not rep["ok"] and rep["codes_outside_tie_band"] == 1
    s_bad = s.clone()
    s_bad[3] *= 1.001
    rep = bench.spot_check(orc, wl, packed, scales.astype(np.float64), q, s_bad, 40)
    assert not rep["ok"]
