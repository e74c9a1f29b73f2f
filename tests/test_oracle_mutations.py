"""Plant plausible mistakes in a copy of the oracle (CPU) and check the pins catch each.

Every mutation below must make at least one pin of ``tests/pins.py`` fail;
otherwise the pins would not be able to vouch for the oracle.
"""

import importlib
import math
import sys

import numpy as np
import pytest

from tests import pins


def _fresh_oracle():
    spec = importlib.util.find_spec("oracle.diffattn")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mut_drop_scale(m):
    m._scale = lambda d: 1.0


def _mut_scale_by_d(m):
    m._scale = lambda d: 1.0 / d


def _mut_top_left_causal(m):
    def vis(rows, Lq, Lk, causal):
        cols = np.arange(Lk)[None, :]
        if not causal:
            return np.ones((rows.shape[0], Lk), dtype=bool)
        return cols <= rows[:, None]
    m._visible = vis


def _mut_strict_causal(m):
    def vis(rows, Lq, Lk, causal):
        cols = np.arange(Lk)[None, :]
        if not causal:
            return np.ones((rows.shape[0], Lk), dtype=bool)
        return cols < (rows[:, None] + (Lk - Lq))
    m._visible = vis


def _mut_plus_lambda(m):
    orig = m.diff_head

    def dh(q1, k1, q2, k2, v, lam, causal, rms=False, eps=1e-5):
        return orig(q1, k1, q2, k2, v, -lam, causal, rms, eps)
    m.diff_head = dh


def _mut_swap_pairs(m):
    m._pair_heads = lambda h: (2 * h + 1, 2 * h)


def _mut_second_map_uses_k1(m):
    orig = m.maps

    def mp(q1, k1, q2, k2, causal, row0=0, Lq=None):
        return orig(q1, k1, q2, k1, causal, row0, Lq)
    m.maps = mp


def _mut_lambda_init_no_shift(m):
    m.lambda_init = lambda layer: 0.8 - 0.6 * math.exp(-0.3 * layer)


def _mut_lambda_sign(m):
    orig = m.lambda_

    def lam(lq1, lk1, lq2, lk2, init):
        return orig(lq2, lk2, lq1, lk1, init)
    m.lambda_ = lam


def _mut_rms_no_eps(m):
    m.rmsnorm = lambda x, eps: x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True))


def _mut_softmax_no_max(m):
    # a sum over all columns including masked ones (forgets the mask in the normaliser)
    def sm(S, visible):
        E = np.exp(S - S.max(axis=-1, keepdims=True))
        return np.where(visible, E, 0.0) / E.sum(axis=-1, keepdims=True)
    m._softmax_masked = sm


MUTATIONS = [_mut_drop_scale, _mut_scale_by_d, _mut_top_left_causal, _mut_strict_causal,
             _mut_plus_lambda, _mut_swap_pairs, _mut_second_map_uses_k1,
             _mut_lambda_init_no_shift, _mut_lambda_sign, _mut_rms_no_eps, _mut_softmax_no_max]


def _mut_snr_sum_not_mean(m):
    orig = m.noise_probe

    def probe(q1, k1, q2, k2, lam):
        r = orig(q1, k1, q2, k2, lam)
        r["snr_plain"] = r["plain"][:, 0] / r["plain"][:, 1:].sum(axis=1)
        r["snr_diff"] = r["diff"][:, 0] / r["diff"][:, 1:].sum(axis=1)
        return r
    m.noise_probe = probe


def _mut_signal_counted_as_noise(m):
    orig = m.noise_probe

    def probe(q1, k1, q2, k2, lam):
        r = orig(q1, k1, q2, k2, lam)
        r["snr_plain"] = r["plain"][:, 0] / r["plain"].mean(axis=1)
        r["noise_fraction_plain"] = r["plain"].sum(axis=1)
        return r
    m.noise_probe = probe


MUTATIONS += [_mut_snr_sum_not_mean, _mut_signal_counted_as_noise]


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda f: f.__name__)
def test_mutation_is_caught(mutate):
    m = _fresh_oracle()
    mutate(m)
    failures = []
    for pin in pins.ALL_PINS:
        try:
            pin(m)
        except AssertionError as e:
            failures.append(f"{pin.__name__}: {e}")
    assert failures, f"no pin caught {mutate.__name__}"


def test_unmutated_copy_passes():
    m = _fresh_oracle()
    for pin in pins.ALL_PINS:
        pin(m)
