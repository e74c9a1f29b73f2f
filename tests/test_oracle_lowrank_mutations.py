"""Plant plausible mistakes in a copy of the low-rank oracle (CPU) and check
that at least one pin of tests/test_oracle_lowrank.py fails for each, so the
pins can vouch for oracle/lowrank.py."""

import importlib

import numpy as np
import pytest

from tests.test_oracle_lowrank import PINS


def _fresh():
    spec = importlib.util.find_spec("oracle.lowrank")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _map(m, weights, norm_axis=1, mask_in_norm=True, guard=True):
    """A noise_map variant built from the module's own helpers."""
    def noise_map(F, G, Lq, Lk, causal):
        F = np.asarray(F, dtype=np.float64)
        G = np.asarray(G, dtype=np.float64)
        if np.any(F < 0) or np.any(G < 0):
            raise ValueError("the factors must be non-negative")
        vis = m._visible(np.arange(Lq), Lq, Lk, causal)
        W_all = weights(F, G)
        W = np.where(vis, W_all, 0.0)
        z = (W if mask_in_norm else W_all).sum(axis=norm_axis, keepdims=True)
        if guard:
            return np.divide(W, z, out=np.zeros_like(W), where=z > 0)
        with np.errstate(divide="ignore", invalid="ignore"):
            return W / z
    return noise_map


def _mut_mask_ignored_in_normaliser(m):
    m.noise_map = _map(m, lambda F, G: F @ G.T, mask_in_norm=False)


def _mut_columns_normalised(m):
    m.noise_map = _map(m, lambda F, G: F @ G.T, norm_axis=0)


def _mut_no_zero_mass_guard(m):
    m.noise_map = _map(m, lambda F, G: F @ G.T, guard=False)


def _mut_query_factor_twice(m):
    m.noise_map = _map(m, lambda F, G: F @ (F if F.shape == G.shape else G).T)


def _mut_top_left_causal(m):
    def vis(rows, Lq, Lk, causal):
        cols = np.arange(Lk)[None, :]
        if not causal:
            return np.ones((rows.shape[0], Lk), dtype=bool)
        return cols <= rows[:, None]
    m._visible = vis


def _mut_plus_lambda(m):
    orig = m.lowrank_head
    m.lowrank_head = lambda q1, k1, v, F, G, lam, causal: orig(q1, k1, v, F, G, -lam, causal)


def _mut_no_score_scale(m):
    m._scale = lambda d: 1.0


def _mut_gqa_modulo(m):
    def diffattn_lowrank(q, k, v, F, G, lam, causal=True):
        q, k, v = (m._f64(t) for t in (q, k, v))
        lam = np.asarray(lam, dtype=np.float64).reshape(-1)
        B, H, Lq, _ = q.shape
        Hkv = k.shape[1]
        out = np.empty((B, H, Lq, v.shape[3]))
        for b in range(B):
            for h in range(H):
                g = h % Hkv
                out[b, h] = m.lowrank_head(q[b, h], k[b, g], v[b, g], F[h], G[h], lam[h], causal)
        return out
    m.diffattn_lowrank = diffattn_lowrank


MUTATIONS = [_mut_mask_ignored_in_normaliser, _mut_columns_normalised, _mut_no_zero_mass_guard,
             _mut_query_factor_twice, _mut_top_left_causal, _mut_plus_lambda, _mut_no_score_scale, _mut_gqa_modulo]


def _failures(m):
    failed = []
    for pin, args in PINS:
        try:
            pin(m, *args)
        except Exception:   # an assertion, or the mistake's own error
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda f: f.__name__)
def test_mutation_is_caught(mutate):
    m = _fresh()
    mutate(m)
    assert _failures(m), f"no pin catches {mutate.__name__}"


def test_unmutated_copy_passes():
    assert _failures(_fresh()) == []
