"""The fp64 oracle against its pins (CPU only)."""

import numpy as np
import pytest
import torch

from oracle import diffattn as orc
from tests import pins
from differential_attention_transformers_b200 import inputs


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(orc)


def test_lambda_of_workloads_matches_brute():
    """The lambdas of every workload: oracle vs the loop twin, exact after fp32 rounding."""
    from oracle import brute
    for name, w in inputs.WORKLOADS.items():
        if w.explicit_lambda is not None:
            continue
        p = [t.double().numpy() for t in inputs.lambda_params(w)]
        init = orc.lambda_init(w.layer)
        got = orc.lambda_(*p, init)
        ref = np.array(brute.lam(*[x.tolist() for x in p], init), dtype=np.float64)
        assert np.all(np.abs(got.astype(np.float64) - ref) <= np.abs(ref) * 2 ** -24 + 1e-30), name


def test_empty_and_degenerate_shapes():
    rng = np.random.default_rng(3)
    # Lk = 0: no key visible anywhere -> zeros
    q = rng.normal(size=(1, 2, 3, 4))
    out = orc.diffattn_v2(q, np.zeros((1, 1, 0, 4)), np.zeros((1, 1, 0, 4)), np.ones(1), causal=True)
    assert out.shape == (1, 1, 3, 4) and np.all(out == 0.0)
    # Lq > Lk under the causal mask: the first Lq - Lk rows see nothing
    q = rng.normal(size=(1, 2, 5, 4)); k = rng.normal(size=(1, 1, 3, 4)); v = rng.normal(size=(1, 1, 3, 4))
    out = orc.diffattn_v2(q, k, v, np.array([0.3]), causal=True)
    assert np.all(out[0, 0, :2] == 0.0) and np.all(out[0, 0, 2:] != 0.0)
    # Lq = 0
    out = orc.diffattn_v2(np.zeros((1, 2, 0, 4)), k, v, np.array([0.3]))
    assert out.shape == (1, 1, 0, 4)


def test_noise_probe_identities_and_report():
    """Tutorial Step 1/3 construction: row sums = 1 - lambda, plain weights > 0.

    The SNR values are reported, not pinned (parity unpinned: the tutorial's
    claims are not met by the literal construction at d = 64).
    """
    w = inputs.WORKLOADS["noise_probe"]
    x = inputs.make(w)
    r = orc.noise_probe(x["q1"][:, 0, 0], x["k1"][:, 0], x["q2"][:, 0, 0], x["k2"][:, 0], 0.5)
    assert np.all(np.abs(r["diff"].sum(axis=1) - 0.5) < 1e-12)
    assert np.all(r["plain"] > 0.0)
    assert np.all(r["plain"][:, 0] > 0.99)           # the strong match dominates
    assert np.all(np.isfinite(r["snr_plain"])) and np.all(r["snr_plain"] > 1.0)
    # the oracle's V1 path with V = I returns the same rows
    sub = slice(0, 4)
    out = orc.diffattn_v1(x["q1"][sub], x["k1"][sub], x["q2"][sub], x["k2"][sub], x["v"][sub],
                          np.array([0.5]), causal=False)
    assert np.max(np.abs(out[:, 0, 0] - r["diff"][sub])) < 1e-14


def test_inputs_are_deterministic():
    w = inputs.with_shape(inputs.WORKLOADS["v2_prefill"], B=1, H=4, Hkv=2, Lq=16, Lk=16)
    a = inputs.make(w)
    b = inputs.make(w)
    for key in a:
        assert torch.equal(a[key], b[key])
    assert a["q"].dtype == torch.bfloat16
