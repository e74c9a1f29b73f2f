"""Pins of the fp64 oracle of the fixed low-rank substitute for A2 (no GPU).

Each test checks the oracle against something that does not share its code:
the closed form of the uniform case (prefix means by cumulative sums), the
limit of the softmax map A2 as its scores vanish, the rank of the unmasked
map, the prefix-sum (linear-attention) evaluation a kernel would use, and a
pure-Python loop twin on a tiny case."""

import math

import numpy as np
import pytest

from oracle import diffattn as orc
from oracle import lowrank


def _rng(seed):
    return np.random.default_rng(seed)


def pin_uniform_case_is_the_prefix_mean(lr, Lq, Lk):
    rng = _rng(Lq + Lk)
    v = rng.standard_normal((Lk, 5))
    N = lr.noise_map(np.ones((Lq, 1)), np.ones((Lk, 1)), Lq, Lk, causal=True)
    csum = np.cumsum(v, axis=0)
    last = np.arange(Lq) + (Lk - Lq)                 # last key row i sees
    want = csum[last] / (last + 1)[:, None]
    assert np.allclose(N @ v, want, rtol=1e-13, atol=1e-14)
    # non-causal: every row is the plain mean
    Nn = lr.noise_map(np.ones((Lq, 1)), np.ones((Lk, 1)), Lq, Lk, causal=False)
    assert np.allclose(Nn @ v, np.broadcast_to(v.mean(axis=0), (Lq, 5)), rtol=1e-13, atol=1e-14)


def pin_softmax_map_tends_to_the_uniform_substitute(lr):
    """As Q2 K2^T -> 0, A2 -> the r = 1, F = G = 1 map, at rate O(eps)."""
    rng = _rng(3)
    L, d = 12, 8
    q1, k1, q2, k2 = (rng.standard_normal((L, d)) for _ in range(4))
    U = lr.noise_map(np.ones((L, 1)), np.ones((L, 1)), L, L, causal=True)
    errs = []
    for eps in (1e-2, 1e-3, 1e-4):
        _, A2 = orc.maps(q1, k1, eps * q2, k2, causal=True)
        errs.append(np.max(np.abs(A2 - U)))
    assert errs[0] < 1e-1 and errs[2] < 1e-3
    assert errs[1] / errs[0] == pytest.approx(0.1, rel=0.05) and errs[2] / errs[1] == pytest.approx(0.1, rel=0.05)


def pin_unmasked_map_has_rank_r_and_unit_rows(lr, r):
    rng = _rng(10 + r)
    F, G = rng.random((20, r)) + 0.1, rng.random((30, r)) + 0.1
    N = lr.noise_map(F, G, 20, 30, causal=False)
    s = np.linalg.svd(N, compute_uv=False)
    assert np.sum(s > 1e-12 * s[0]) == r
    assert np.allclose(N.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert np.all(N >= 0)


def pin_prefix_sum_evaluation_matches_the_map(lr):
    """(N V)_i = f_i^T S_i / f_i^T z_i with S_i = sum_{j<=i} g_j v_j^T, z_i = sum_{j<=i} g_j:
    the linear-time evaluation of the causal map."""
    rng = _rng(21)
    L, r, dv = 16, 4, 6
    F, G, v = rng.random((L, r)), rng.random((L, r)), rng.standard_normal((L, dv))
    S = np.cumsum(G[:, :, None] * v[:, None, :], axis=0)     # [L, r, dv]
    z = np.cumsum(G, axis=0)                                   # [L, r]
    scan = np.einsum("ir,ird->id", F, S) / np.einsum("ir,ir->i", F, z)[:, None]
    assert np.allclose(lr.noise_map(F, G, L, L, causal=True) @ v, scan, rtol=1e-12, atol=1e-13)


def pin_loop_twin_and_rows(lr):
    rng = _rng(5)
    Lq, Lk, d, dv, r, lam = 3, 5, 4, 2, 2, 0.7
    q, k, v = rng.standard_normal((Lq, d)), rng.standard_normal((Lk, d)), rng.standard_normal((Lk, dv))
    F, G = rng.random((Lq, r)), rng.random((Lk, r))
    got = lr.lowrank_head(q, k, v, F, G, lam, causal=True)
    for i in range(Lq):
        vis = [j for j in range(Lk) if j <= i + (Lk - Lq)]
        s = [sum(q[i, c] * k[j, c] for c in range(d)) / math.sqrt(d) for j in vis]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        a1 = [x / sum(e) for x in e]
        w = [sum(F[i, t] * G[j, t] for t in range(r)) for j in vis]
        n = [x / sum(w) for x in w]
        for c in range(dv):
            want = sum((a1[t] - lam * n[t]) * v[j, c] for t, j in enumerate(vis))
            assert got[i, c] == pytest.approx(want, rel=1e-12, abs=1e-14)
    # rows of A1 - lam N sum to 1 - lam: with V = ones the output is 1 - lam
    ones = lr.lowrank_head(q, k, np.ones((Lk, 1)), F, G, lam, causal=True)
    assert np.allclose(ones, 1 - lam, rtol=0, atol=1e-14)


def pin_zero_mass_rows_and_bad_factors(lr):
    F = np.array([[0.0], [1.0]])
    N = lr.noise_map(F, np.ones((2, 1)), 2, 2, causal=True)
    assert np.all(N[0] == 0) and np.allclose(N[1], [0.5, 0.5])
    with pytest.raises(ValueError):
        lr.noise_map(-F, np.ones((2, 1)), 2, 2, causal=True)


def pin_batched_layout_matches_heads(lr):
    rng = _rng(8)
    B, H, Hkv, L, d, dv, r = 2, 4, 2, 6, 4, 3, 2
    q, k, v = rng.standard_normal((B, H, L, d)), rng.standard_normal((B, Hkv, L, d)), rng.standard_normal((B, Hkv, L, dv))
    F, G = rng.random((H, L, r)), rng.random((H, L, r))
    lam = np.array([0.1, 0.5, -0.2, 0.9])
    out = lr.diffattn_lowrank(q, k, v, F, G, lam, causal=True)
    for b in range(B):
        for h in range(H):
            assert np.array_equal(out[b, h], lr.lowrank_head(q[b, h], k[b, h // 2], v[b, h // 2], F[h], G[h], lam[h], True))


# Every pin with its arguments; test_oracle_lowrank_mutations.py runs the same
# list against planted mistakes.
PINS = [
    (pin_uniform_case_is_the_prefix_mean, (7, 7)),
    (pin_uniform_case_is_the_prefix_mean, (4, 9)),
    (pin_softmax_map_tends_to_the_uniform_substitute, ()),
    (pin_unmasked_map_has_rank_r_and_unit_rows, (1,)),
    (pin_unmasked_map_has_rank_r_and_unit_rows, (3,)),
    (pin_prefix_sum_evaluation_matches_the_map, ()),
    (pin_loop_twin_and_rows, ()),
    (pin_zero_mass_rows_and_bad_factors, ()),
    (pin_batched_layout_matches_heads, ()),
]


@pytest.mark.parametrize("pin,args", PINS, ids=lambda x: getattr(x, "__name__", str(x)))
def test_pin(pin, args):
    pin(lowrank, *args)
