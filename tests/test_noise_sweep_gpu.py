"""The SNR sweep on the bf16 V1 decode kernel against the fp64 oracle, from 1k
to 256k keys ("差分注意力" tutorial, exercise 1).  Needs a B200.

Each instance's signal column (weight on key 0) and noise column (total weight
on keys 1..N-1) are compared with the oracle's explicit attention row, each to
2e-2 of its own magnitude.  Both columns are free of cancellation: for plain
softmax they are sums of positive weights, and the difference's noise mass is
about -lambda (1 - A2[0]).  So the output tolerance applies per column rather
than against the row's largest value, which for plain softmax would leave the
noise mass (1e-13 and below) unchecked.  V's other columns are zero, and so
must the output be there."""

import numpy as np
import pytest
import torch

import differential_attention_transformers_b200 as da
from differential_attention_transformers_b200 import inputs, noise
from oracle import diffattn as orc
from tests.test_parity_gpu import BF16_TOL, DEV

pytestmark = pytest.mark.gpu

LENGTHS = (1024, 16384, 262144)
N_INST = 8


def _oracle_columns(p, i, lam):
    r = orc.noise_probe(p["q1"][i:i + 1, 0], p["k1"][i:i + 1, 0], p["q2"][i:i + 1, 0], p["k2"][i:i + 1, 0], lam)
    row = r["diff"][0] if lam != 0.0 else r["plain"][0]
    return np.array([row[0], row[1:].sum()])


def test_sweep_columns_match_oracle():
    x = inputs.noise_sweep(n=N_INST, N=max(LENGTHS), device=DEV)
    for N in LENGTHS:
        p = inputs.sweep_prefix(x, N)
        for lam in (0.0, 0.5):
            lt = torch.full((1,), lam, dtype=torch.float32, device=DEV)
            out = da.decode_v1(p["q1"], p["k1"], p["q2"], p["k2"], p["v"], lt)
            torch.cuda.synchronize()
            assert da.last_status() == da.OK
            assert torch.all(out[:, :, 2:] == 0), (N, lam)
            got = out[:, 0, :2].double().cpu().numpy()
            for i in range(N_INST):
                ref = _oracle_columns(p, i, lam)
                assert np.all(np.abs(got[i] - ref) <= BF16_TOL * np.abs(ref)), (N, lam, i, got[i], ref)
                s_got, s_ref = got[i, 0] * (N - 1) / got[i, 1], ref[0] * (N - 1) / ref[1]
                assert abs(s_got - s_ref) <= 2 * BF16_TOL * abs(s_ref), (N, lam, i, s_got, s_ref)
        del p


def test_sweep_summary():
    rows = noise.sweep(lengths=(1024, 4096), n=4)
    assert [r["N"] for r in rows] == [1024, 4096]
    for r in rows:
        for key in ("snr_plain", "snr_diff", "noise_fraction_plain", "signal_plain", "signal_diff", "noise_mass_diff"):
            assert len(r[key]) == 3 and all(np.isfinite(r[key])), key
            assert r[key][0] <= r[key][1] <= r[key][2], key
        assert r["snr_plain"][0] > 0 and r["noise_fraction_plain"][2] < 1e-3
        # rows of A1 - lambda A2 sum to 1 - lambda: the difference's noise mass is near -0.5
        assert abs(r["signal_diff"][1] + r["noise_mass_diff"][1] - 0.5) <= BF16_TOL
