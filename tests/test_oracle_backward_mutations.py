"""Plant plausible chain-rule mistakes in a copy of the backward oracle (CPU)
and check that at least one pin of tests/test_oracle_backward.py fails for
each: finite differences of the forward oracle, autograd of an independent
torch forward, and lambda's parameter gradients.

The mistakes go into a per-head backward rebuilt here with switches; with
every switch off it must pass all pins (checked below), so each failure is
the switch's doing."""

import importlib

import numpy as np
import pytest

from tests.test_oracle_backward import PINS


def _fresh():
    spec = importlib.util.find_spec("oracle.backward")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _head(m, drop_d=False, plus_lambda=False, dlam_sign=False, rms_no_projection=False, no_scale=False,
          dv_map1_only=False, dk_maps_crossed=False):
    def head_backward(q1, k1, q2, k2, v, lam, dout, causal, rms=False, eps=1e-5):
        q1, k1, q2, k2, v, dout = (m._f64(t) for t in (q1, k1, q2, k2, v, dout))
        lam = float(lam)
        Lq, d = q1.shape
        s = 1.0 if no_scale else 1.0 / np.sqrt(d)
        A1, A2 = m.maps(q1, k1, q2, k2, causal, 0, Lq)
        O1, O2 = A1 @ v, A2 @ v
        dx = dout
        if rms:
            x = O1 - lam * O2
            r = 1.0 / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + eps)
            dx = r * dx if rms_no_projection else r * dx - (r ** 3 / x.shape[1]) * x * np.sum(x * dx, axis=1,
                                                                                               keepdims=True)
        dv = (A1 if dv_map1_only else A1 - lam * A2).T @ dx
        dW = dx @ v.T
        D1 = 0.0 if drop_d else np.sum(dx * O1, axis=1, keepdims=True)
        D2 = 0.0 if drop_d else np.sum(dx * O2, axis=1, keepdims=True)
        dS1 = A1 * (dW - D1)
        dS2 = (lam if plus_lambda else -lam) * A2 * (dW - D2)
        dq1, dq2 = s * (dS1 @ k1), s * (dS2 @ k2)
        dk1, dk2 = s * (dS1.T @ q1), s * (dS2.T @ q2)
        if dk_maps_crossed:
            dk1, dk2 = s * (dS2.T @ q1), s * (dS1.T @ q2)
        dlam = float(np.sum(dx * O2)) if dlam_sign else -float(np.sum(dx * O2))
        return dq1, dk1, dq2, dk2, dv, dlam
    return head_backward


SWITCHES = ["drop_d", "plus_lambda", "dlam_sign", "rms_no_projection", "no_scale", "dv_map1_only",
            "dk_maps_crossed"]


def _failures(m):
    failed = []
    for pin, args in PINS:
        try:
            pin(m, *args)
        except Exception:
            failed.append(pin.__name__)
    return failed


def test_rebuilt_head_passes_every_pin():
    m = _fresh()
    m.head_backward = _head(m)
    assert _failures(m) == []


@pytest.mark.parametrize("switch", SWITCHES)
def test_mistake_is_caught(switch):
    m = _fresh()
    m.head_backward = _head(m, **{switch: True})
    assert _failures(m), f"no pin catches {switch}"


def test_lambda_parameter_mistake_is_caught():
    m = _fresh()
    orig = m.lambda_backward
    m.lambda_backward = lambda lq1, lk1, lq2, lk2, dlam: tuple(-t for t in orig(lq1, lk1, lq2, lk2, dlam))
    assert _failures(m)
