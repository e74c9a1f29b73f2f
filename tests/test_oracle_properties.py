"""Property-based pins of the fp64 oracles (no GPU).

Each property follows from the mathematics of the method, not from the
oracle's code, and holds for any sizes: hypothesis draws small shapes, masks,
lambdas and seeds.  A wrong mask, a scale applied to the wrong operand, a
sign error, a crossed map or a broken GQA index breaks at least one of them.

  * softmax ignores a per-row shift of the scores: adding one vector w to
    every key of a map shifts row i's scores by q_i.w / sqrt(d), so O does
    not change;
  * without a mask, permuting the keys together with their values leaves O
    unchanged;
  * O is linear in V and affine in lambda;
  * swapping the two maps and replacing lambda by 1/lambda gives -O / lambda;
  * causality: row i does not depend on keys (or values) it cannot see;
  * GQA: a KV head shared by several query heads gives the same output as
    separate copies of it;
  * with eps = 0 the RMSNorm output does not depend on the scale of V;
  * the key gradient of each map sums to zero over the keys (softmax rows
    are shift invariant), so dK sums to zero in the V2 layout;
  * the low-rank map is unchanged by positive scalings of F's rows (each
    row of N is normalised), by one positive scale of G, and by permuting
    the rank index of both factors together."""

import math

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import backward as bwd
from oracle import diffattn as orc
from oracle import lowrank as lr

SETTINGS = settings(max_examples=25, deadline=None, derandomize=True)   # reproducible runs


@st.composite
def v1_case(draw, causal=None):
    Lq = draw(st.integers(1, 7))
    Lk = draw(st.integers(1, 9))
    d = draw(st.integers(1, 6))
    dv = draw(st.integers(1, 5))
    c = draw(st.booleans()) if causal is None else causal
    lam = draw(st.floats(-1.5, 1.5))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    rng = np.random.default_rng(seed)
    q1, q2 = rng.standard_normal((1, 1, Lq, d)), rng.standard_normal((1, 1, Lq, d))
    k1, k2 = rng.standard_normal((1, 1, Lk, d)), rng.standard_normal((1, 1, Lk, d))
    v = rng.standard_normal((1, 1, Lk, dv))
    return dict(q1=q1, k1=k1, q2=q2, k2=k2, v=v, lam=np.array([lam]), causal=c, rng=rng)


def _out(c, **over):
    a = dict(c)
    a.update(over)
    return orc.diffattn_v1(a["q1"], a["k1"], a["q2"], a["k2"], a["v"], a["lam"], causal=a["causal"],
                           rms=a.get("rms", False), eps=a.get("eps", 1e-5))


def _close(a, b, tol=1e-10):
    a, b = np.nan_to_num(a), np.nan_to_num(b)
    return np.max(np.abs(a - b)) <= tol * max(1.0, np.max(np.abs(b)))


@SETTINGS
@given(v1_case())
def test_shifting_every_key_leaves_the_output(c):
    w1 = c["rng"].standard_normal(c["k1"].shape[-1])
    w2 = c["rng"].standard_normal(c["k2"].shape[-1])
    assert _close(_out(c, k1=c["k1"] + w1, k2=c["k2"] + w2), _out(c))


@SETTINGS
@given(v1_case(causal=False))
def test_unmasked_key_permutation(c):
    p = c["rng"].permutation(c["k1"].shape[2])
    assert _close(_out(c, k1=c["k1"][:, :, p], k2=c["k2"][:, :, p], v=c["v"][:, :, p]), _out(c))


@SETTINGS
@given(v1_case(), st.floats(-3, 3), st.floats(-2, 2))
def test_linear_in_v_and_affine_in_lambda(c, alpha, lam_b):
    v2 = c["rng"].standard_normal(c["v"].shape)
    assert _close(_out(c, v=c["v"] + alpha * v2), _out(c) + alpha * _out(c, v=v2), 1e-9)
    # O(lambda) - O(lambda_b) = (lambda_b - lambda) A2 V, and A2 V = O(0) - O(1)
    a2v = _out(c, lam=np.array([0.0])) - _out(c, lam=np.array([1.0]))
    lam = float(c["lam"][0])
    assert _close(_out(c) - _out(c, lam=np.array([lam_b])), (lam_b - lam) * a2v, 1e-9)


@SETTINGS
@given(v1_case())
def test_swapping_the_maps(c):
    lam = float(c["lam"][0])
    if abs(lam) < 0.05:
        lam = 0.5
    base = _out(c, lam=np.array([lam]))
    swapped = _out(c, q1=c["q2"], k1=c["k2"], q2=c["q1"], k2=c["k1"], lam=np.array([1.0 / lam]))
    assert _close(swapped, -base / lam, 1e-9)


@SETTINGS
@given(v1_case(causal=True))
def test_rows_do_not_see_later_keys(c):
    Lq, Lk = c["q1"].shape[2], c["k1"].shape[2]
    off = Lk - Lq
    out = _out(c)
    k1, k2, v = c["k1"].copy(), c["k2"].copy(), c["v"].copy()
    for i in range(Lq):
        last = i + off                      # last key row i sees
        if last + 1 < Lk:
            k1b, k2b, vb = k1.copy(), k2.copy(), v.copy()
            k1b[:, :, last + 1:] += 3.0
            k2b[:, :, last + 1:] -= 2.0
            vb[:, :, last + 1:] *= -5.0
            assert _close(_out(c, k1=k1b, k2=k2b, v=vb)[:, :, i], out[:, :, i])


@SETTINGS
@given(st.integers(1, 3), st.integers(1, 3), st.integers(1, 6), st.booleans(), st.integers(0, 2 ** 31 - 1))
def test_gqa_equals_replicated_kv_heads(Hkv, pairs_per_group, L, causal, seed):
    rng = np.random.default_rng(seed)
    grp = 2 * pairs_per_group
    Hq = Hkv * grp
    q = rng.standard_normal((1, Hq, L, 4))
    k, v = rng.standard_normal((1, Hkv, L, 4)), rng.standard_normal((1, Hkv, L, 4))
    lam = rng.uniform(-1, 1, Hq // 2)
    shared = orc.diffattn_v2(q, k, v, lam, causal=causal)
    # one KV copy per pair: pair h reads KV head h of the replicated tensors
    kr = np.repeat(k, pairs_per_group, axis=1)
    vr = np.repeat(v, pairs_per_group, axis=1)
    assert _close(orc.diffattn_v2(q, kr, vr, lam, causal=causal), shared)
    # the V1 layout: head h reads KV head h // (H / Hkv)
    q1, q2 = q[:, 0::2], q[:, 1::2]
    H = Hq // 2
    k1 = rng.standard_normal((1, Hkv, L, 4))
    v1 = orc.diffattn_v1(q1, k1, q2, k, v, lam, causal=causal)
    rep = H // Hkv
    assert _close(orc.diffattn_v1(q1, np.repeat(k1, rep, axis=1), q2, np.repeat(k, rep, axis=1),
                                  np.repeat(v, rep, axis=1), lam, causal=causal), v1)


@SETTINGS
@given(v1_case(), st.floats(0.01, 100))
def test_rmsnorm_ignores_the_scale_of_v(c, scale):
    a = _out(c, rms=True, eps=0.0)
    b = _out(c, v=c["v"] * scale, rms=True, eps=0.0)
    assert _close(a, b, 1e-9)


@SETTINGS
@given(st.integers(1, 5), st.integers(1, 6), st.booleans(), st.integers(0, 2 ** 31 - 1))
def test_key_gradients_sum_to_zero(L, d, causal, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 4, L, d))
    k, v = rng.standard_normal((1, 1, L, d)), rng.standard_normal((1, 1, L, d))
    lam = rng.uniform(-1, 1, 2)
    dout = rng.standard_normal((1, 2, L, d))
    _, dk, _, _ = bwd.diffattn_v2_backward(q, k, v, lam, dout, causal=causal)
    assert np.max(np.abs(dk.sum(axis=2))) <= 1e-10 * max(1.0, np.max(np.abs(dk)))


@SETTINGS
@given(st.integers(1, 6), st.integers(1, 8), st.integers(1, 4), st.booleans(), st.integers(0, 2 ** 31 - 1))
def test_lowrank_map_ignores_row_scalings(Lq, Lk, r, causal, seed):
    rng = np.random.default_rng(seed)
    F, G = rng.random((Lq, r)) + 0.05, rng.random((Lk, r)) + 0.05
    N = lr.noise_map(F, G, Lq, Lk, causal)
    cF = rng.uniform(0.1, 10, (Lq, 1))
    assert _close(lr.noise_map(F * cF, G, Lq, Lk, causal), N)
    cG = rng.uniform(0.1, 10)
    assert _close(lr.noise_map(F, G * cG, Lq, Lk, causal), N)
    p = rng.permutation(r)
    assert _close(lr.noise_map(F[:, p], G[:, p], Lq, Lk, causal), N)
    # rows with a visible key sum to 1
    vis = [i for i in range(Lq) if (not causal) or i + (Lk - Lq) >= 0]
    assert np.allclose(N[vis].sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert math.isfinite(float(N.sum()))
