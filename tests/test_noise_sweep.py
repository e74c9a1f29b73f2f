"""The SNR-vs-context-length sweep ("差分注意力" tutorial, Step 1, Step 3 and
exercise 1): its construction and host arithmetic, on the CPU.

The GPU sweep reads the row's signal weight and total noise weight from two
indicator columns of V.  These tests pin that reading on the oracle (it must
equal the weights of the explicit attention row), the nesting of the
contexts (prefixes of one draw: the plain noise fraction can only grow with
N), and the ratio and summary arithmetic of ``noise``."""

import numpy as np
import pytest
import torch

from differential_attention_transformers_b200 import inputs
from differential_attention_transformers_b200 import noise
from oracle import diffattn as orc


def _rows(x, lam):
    """Explicit attention rows from the oracle's probe: (plain [n, N], diff [n, N])."""
    r = orc.noise_probe(x["q1"][:, 0], x["k1"][:, 0], x["q2"][:, 0], x["k2"][:, 0], lam)
    return r["plain"], r["diff"]


@pytest.mark.parametrize("lam", [0.0, 0.5, -0.3])
def test_indicator_columns_read_the_row_masses(lam):
    x = inputs.noise_sweep(n=3, N=300, seed=7)
    plain, diff = _rows(x, lam)
    row = diff if lam != 0.0 else plain
    # the decode is the one-row V1 forward over all keys
    q1, q2 = x["q1"][:, :, None], x["q2"][:, :, None]
    out = orc.diffattn_v1(q1, x["k1"], q2, x["k2"], x["v"], np.array([lam]), causal=True)[:, 0, 0]
    assert np.allclose(out[:, 0], row[:, 0], rtol=1e-12, atol=0)
    assert np.allclose(out[:, 1], row[:, 1:].sum(axis=1), rtol=1e-12, atol=1e-300)
    assert np.all(out[:, 2:] == 0.0)
    # rows of A1 - lambda A2 sum to 1 - lambda
    assert np.allclose(out[:, 0] + out[:, 1], 1.0 - lam, rtol=0, atol=1e-12)


def test_construction_layout():
    x = inputs.noise_sweep(n=2, N=40, seed=3)
    assert x["q1"].shape == (2, 1, 64) and x["k1"].shape == (2, 1, 40, 64) and x["v"].shape == (2, 1, 40, 128)
    assert all(t.dtype == torch.bfloat16 for t in x.values())
    # key 0 is the strong match 5q, formed in fp32 and rounded once: within
    # two bf16 roundings of 5 times the rounded q
    assert torch.allclose(x["k1"][:, 0, 0].float(), 5.0 * x["q1"][:, 0].float(), rtol=2 ** -7, atol=0)
    v = x["v"].float()
    assert torch.all(v[:, 0, 0, 0] == 1) and torch.all(v[:, 0, 1:, 0] == 0)
    assert torch.all(v[:, 0, 1:, 1] == 1) and torch.all(v[:, 0, 0, 1] == 0)
    assert torch.all(v[..., 2:] == 0)
    p = inputs.sweep_prefix(x, 16)
    assert p["k1"].is_contiguous() and p["v"].shape == (2, 1, 16, 128)
    assert torch.equal(p["k2"], x["k2"][:, :, :16])


def test_plain_noise_fraction_grows_along_nested_contexts():
    """Adding keys to the same instance adds positive weight to the noise and
    to the normaliser: the plain noise fraction strictly rises and the signal
    weight never rises (Step 1's noise floor; at d = 64 the signal weight is
    1 to fp64 precision)."""
    x = inputs.noise_sweep(n=4, N=2048, seed=11)
    prev_frac, prev_sig = None, None
    for N in (64, 256, 1024, 2048):
        plain, _ = _rows(inputs.sweep_prefix(x, N), 0.0)
        frac = plain[:, 1:].sum(axis=1)
        sig = plain[:, 0]
        if prev_frac is not None:
            assert np.all(frac > prev_frac) and np.all(sig <= prev_sig)
        prev_frac, prev_sig = frac, sig


def test_snr_and_summary_arithmetic():
    sig = torch.tensor([0.9, 0.6, 0.5, 0.99], dtype=torch.float64)
    nz = torch.tensor([0.1, 0.2, 0.5, 0.01], dtype=torch.float64)
    N = 101
    assert torch.allclose(noise.snr(sig, nz, N), sig * 100 / nz)
    r = noise.summarize(N, sig, nz, sig, -nz)
    assert r["N"] == N
    frac = (nz / (sig + nz)).numpy()
    assert r["noise_fraction_plain"] == pytest.approx(list(np.quantile(frac, [0.25, 0.5, 0.75])))
    assert r["snr_plain"] == pytest.approx(list(np.quantile((sig * 100 / nz).numpy(), [0.25, 0.5, 0.75])))
    assert r["snr_diff"][1] == pytest.approx(-r["snr_plain"][1])
    assert r["noise_mass_diff"] == pytest.approx(list(np.quantile(-nz.numpy(), [0.25, 0.5, 0.75])))


def test_sweep_lengths():
    assert inputs.SWEEP_LENGTHS[0] == 1024 and inputs.SWEEP_LENGTHS[-1] == 262144
    assert all(b == 2 * a for a, b in zip(inputs.SWEEP_LENGTHS, inputs.SWEEP_LENGTHS[1:]))
