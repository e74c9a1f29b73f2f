"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each ``pin_*`` takes the oracle module (normally ``oracle.diffattn``) and
raises AssertionError when the oracle breaks the fact.  ``test_oracle.py``
runs them on the real oracle; ``test_oracle_mutations.py`` runs them on
deliberately broken copies to show that each plausible mistake is caught.

What pins what (page title, section):
  * lambda_init: the value 0.2 at layer 1 stated for the tiny V1 workload, the
    0.8 asymptote and the exp(-0.3) geometric decay of the schedule in
    "Differential Transformer" (mcipr.com) section 3 工程实践.
  * lambda: closed forms (exp(ln 2) = 2, exp(0) = 1), antisymmetry under
    swapping the two maps, the tutorial's default lambda_init = 0.5
    ("差分注意力" Step 4), and high-precision evaluation with mpmath.
  * lambda = 0 reduces to standard softmax attention ("差分注意力" section
    Softmax 的噪声底): compared with torch's scaled_dot_product_attention in
    fp64, including its own GQA head mapping.
  * Q2 = Q1, K2 = K1, lambda = 1 gives exactly zero; V = ones gives 1 - lambda
    (softmax rows sum to one, section Softmax 的噪声底).
  * softmax never yields an exact zero (same section): every visible weight is
    positive, every masked weight is exactly zero.
  * the 1/sqrt(d) scale ("差分注意力" section 差分思路): two-key closed form.
  * causal alignment: the last n rows of a causal prefill equal a causal
    query of those n rows against all keys (suffix consistency), and a single
    query sees the whole cache.
  * RMSNorm: ||y||^2 / dv = ms / (ms + eps).
  * the pure-Python loop twin on tiny ragged GQA shapes.
  * the noise probe's SNR and noise fraction ("差分注意力" Step 1 and Step 3):
    closed forms on constructions where every noise key gets the same score.
"""

from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

from oracle import brute


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


# ----------------------------------------------------------------------------
def pin_lambda_init(orc):
    # 0.2 at layer 1: stated for the tiny V1 workload (layer = 1).
    assert abs(orc.lambda_init(1) - 0.2) < 1e-15, orc.lambda_init(1)
    vals = [orc.lambda_init(l) for l in range(1, 60)]
    # increasing towards 0.8
    assert all(b > a for a, b in zip(vals, vals[1:])), "lambda_init not increasing"
    assert 0.8 - vals[-1] < 1e-6 and all(v < 0.8 for v in vals), "asymptote is not 0.8"
    # geometric decay of the gap with ratio exp(-0.3)
    r = math.exp(-0.3)
    for a, b in zip(vals, vals[1:20]):
        assert abs((0.8 - b) / (0.8 - a) - r) < 1e-12, "decay ratio is not exp(-0.3)"
    # the 12th and 24th layer values used by the bf16 workloads (mpmath, 30 digits)
    import mpmath as mp
    mp.mp.dps = 30
    for l in (12, 24):
        ref = mp.mpf("0.8") - mp.mpf("0.6") * mp.e ** (mp.mpf("-0.3") * (l - 1))
        assert abs(orc.lambda_init(l) - float(ref)) < 1e-15


def pin_lambda(orc):
    H, d = 3, 8
    z = np.zeros((H, d))
    # all-zero parameters: lambda == lambda_init; the tutorial's default is 0.5
    lam = orc.lambda_(z, z, z, z, 0.5)
    assert lam.dtype == np.float32 and np.all(lam == np.float32(0.5))
    # exp(ln2 * 1) - exp(0) + init = 1 + init
    lq1 = z.copy(); lk1 = z.copy()
    lq1[:, 0] = math.log(2.0); lk1[:, 0] = 1.0
    lam = orc.lambda_(lq1, lk1, z, z, 0.2)
    assert np.all(lam == np.float32(1.2)), lam
    # swapping the maps: lambda(a,b) + lambda(b,a) = 2*init
    rng = _rng(5)
    a1, b1, a2, b2 = (rng.normal(0, 0.3, (H, d)) for _ in range(4))
    l_ab = orc.lambda_(a1, b1, a2, b2, 0.7).astype(np.float64)
    l_ba = orc.lambda_(a2, b2, a1, b1, 0.7).astype(np.float64)
    assert np.all(np.abs(l_ab + l_ba - 1.4) < 4e-7)
    # high-precision reference, rounded once to fp32, must agree bitwise
    import mpmath as mp
    mp.mp.dps = 40
    for h in range(H):
        t1 = mp.fsum(mp.mpf(float(x)) * mp.mpf(float(y)) for x, y in zip(a1[h], b1[h]))
        t2 = mp.fsum(mp.mpf(float(x)) * mp.mpf(float(y)) for x, y in zip(a2[h], b2[h]))
        ref = np.float32(float(mp.e ** t1 - mp.e ** t2 + mp.mpf(0.7)))
        assert ref == np.float32(l_ab[h]), (h, ref, l_ab[h])


def pin_standard_attention(orc):
    """lambda = 0 is softmax attention: torch SDPA in fp64 (incl. its GQA map)."""
    rng = _rng(11)
    B, Hq, Hkv, L, D = 2, 8, 2, 9, 16
    q = rng.normal(size=(B, Hq, L, D)); k = rng.normal(size=(B, Hkv, L, D))
    v = rng.normal(size=(B, Hkv, L, D))
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    for causal in (True, False):
        ref = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, enable_gqa=True).numpy()
        # lambda = 0: pair h is head 2h alone
        out = orc.diffattn_v2(q, k, v, np.zeros(Hq // 2), causal=causal)
        _close(out, ref[:, 0::2], 1e-12, f"V2 lambda=0 causal={causal}")
        # lambda = -1: A1 + A2, i.e. head 2h plus head 2h+1
        out = orc.diffattn_v2(q, k, v, -np.ones(Hq // 2), causal=causal)
        _close(out, ref[:, 0::2] + ref[:, 1::2], 1e-12, f"V2 lambda=-1 causal={causal}")
    # V1 layout with lambda = 0 against SDPA of map 1, and lambda = -1
    H = 4
    q1 = rng.normal(size=(B, H, L, D)); q2 = rng.normal(size=(B, H, L, D))
    k1 = rng.normal(size=(B, Hkv, L, D)); k2 = rng.normal(size=(B, Hkv, L, D))
    v = rng.normal(size=(B, Hkv, L, 24))
    t = lambda x: torch.from_numpy(x)  # noqa: E731
    r1 = F.scaled_dot_product_attention(t(q1), t(k1), t(v), is_causal=True, enable_gqa=True).numpy()
    r2 = F.scaled_dot_product_attention(t(q2), t(k2), t(v), is_causal=True, enable_gqa=True).numpy()
    _close(orc.diffattn_v1(q1, k1, q2, k2, v, np.zeros(H)), r1, 1e-12, "V1 lambda=0")
    _close(orc.diffattn_v1(q1, k1, q2, k2, v, np.full(H, 0.3)), r1 - 0.3 * r2, 1e-12, "V1 lambda=0.3")
    # single-token decode sees the whole cache: non-causal SDPA
    qd = rng.normal(size=(B, Hq, D))
    T = 13
    kc = rng.normal(size=(B, Hkv, T, D)); vc = rng.normal(size=(B, Hkv, T, D))
    ref = F.scaled_dot_product_attention(t(qd[:, :, None]), t(kc), t(vc), enable_gqa=True).numpy()[:, :, 0]
    lam = rng.normal(size=Hq // 2)
    _close(orc.decode_v2(qd, kc, vc, lam), ref[:, 0::2] - lam[None, :, None] * ref[:, 1::2],
           1e-12, "decode")


def pin_exact_zero(orc):
    rng = _rng(12)
    q = rng.normal(size=(1, 2, 7, 8)); k = rng.normal(size=(1, 1, 7, 8)); v = rng.normal(size=(1, 1, 7, 5))
    out = orc.diffattn_v1(q, k, q, k, v, np.ones(2), causal=True)
    assert np.all(out == 0.0), "Q2=Q1, K2=K1, lambda=1 must give exactly 0"


def pin_row_sums(orc):
    rng = _rng(13)
    B, H, Lq, Lk, d = 1, 3, 6, 10, 8
    lam = np.array([0.2, -0.4, 0.9])
    args = [rng.normal(size=s) for s in ((B, H, Lq, d), (B, H, Lk, d), (B, H, Lq, d), (B, H, Lk, d))]
    ones = np.ones((B, H, Lk, 4))
    for causal in (True, False):
        out = orc.diffattn_v1(args[0], args[1], args[2], args[3], ones, lam, causal=causal)
        _close(out, (1 - lam)[None, :, None, None] * np.ones_like(out), 1e-13, "V=ones")


def pin_masks_and_positivity(orc):
    """V = I makes O the map itself: masked entries exactly 0, visible > 0."""
    rng = _rng(14)
    Lq, Lk, d = 5, 9, 8
    q = rng.normal(size=(1, 1, Lq, d)); k = rng.normal(size=(1, 1, Lk, d))
    eye = np.eye(Lk)[None, None]
    A = orc.diffattn_v1(q, k, q, k, eye, np.zeros(1), causal=True)[0, 0]
    # causal with Lq < Lk: each visible set is a prefix, and consecutive rows see one more key
    nz = (A != 0.0).sum(axis=1)
    for i in range(Lq):
        assert np.all(A[i, :nz[i]] > 0.0) and np.all(A[i, nz[i]:] == 0.0), "visible set is not a prefix"
    assert np.all(np.diff(nz) == 1) and nz[-1] == Lk, "last row must see every key"
    _close(A.sum(axis=1), np.ones(Lq), 1e-14, "rows sum to 1")
    # non-causal: all weights strictly positive
    A = orc.diffattn_v1(q, k, q, k, eye, np.zeros(1), causal=False)[0, 0]
    assert np.all(A > 0.0)


def pin_suffix_consistency(orc):
    """Rows [a, L) of a causal prefill equal a causal query of those rows alone."""
    rng = _rng(15)
    L, d, a = 11, 8, 7
    q1 = rng.normal(size=(1, 1, L, d)); q2 = rng.normal(size=(1, 1, L, d))
    k1 = rng.normal(size=(1, 1, L, d)); k2 = rng.normal(size=(1, 1, L, d)); v = rng.normal(size=(1, 1, L, 6))
    lam = np.array([0.37])
    full = orc.diffattn_v1(q1, k1, q2, k2, v, lam, causal=True)
    tail = orc.diffattn_v1(q1[:, :, a:], k1, q2[:, :, a:], k2, v, lam, causal=True)
    _close(tail, full[:, :, a:], 1e-13, "suffix consistency")


def pin_uniform_keys(orc):
    """Identical keys: each map is uniform over the visible keys."""
    rng = _rng(16)
    Lq = Lk = 6
    d = 8
    q1 = rng.normal(size=(1, 1, Lq, d)); q2 = rng.normal(size=(1, 1, Lq, d))
    k = np.repeat(rng.normal(size=(1, 1, 1, d)), Lk, axis=2)
    v = rng.normal(size=(1, 1, Lk, 3))
    lam = 0.25
    out = orc.diffattn_v1(q1, k, q2, k, v, np.array([lam]), causal=True)[0, 0]
    for i in range(Lq):
        _close(out[i], (1 - lam) * v[0, 0, :i + 1].mean(axis=0), 1e-13, "uniform keys")


def pin_scale(orc):
    """Two keys: weight of key 0 is 1 / (1 + exp((s1 - s0)/sqrt(d)))."""
    import mpmath as mp
    mp.mp.dps = 30
    for d in (16, 64, 128):
        q = np.zeros((1, 1, 1, d)); q[..., 0] = 1.5
        k = np.zeros((1, 1, 2, d)); k[0, 0, 0, 0] = 2.0; k[0, 0, 1, 0] = -1.0
        eye = np.eye(2)[None, None]
        A = orc.diffattn_v1(q, k, q, k, eye, np.zeros(1), causal=False)[0, 0, 0]
        ref = 1 / (1 + mp.e ** ((mp.mpf(-1.5) - mp.mpf(3.0)) / mp.sqrt(d)))
        assert abs(A[0] - float(ref)) < 1e-15, (d, A[0], float(ref))


def pin_rmsnorm(orc):
    rng = _rng(17)
    q1 = rng.normal(size=(1, 2, 5, 8)); q2 = rng.normal(size=(1, 2, 5, 8))
    k1 = rng.normal(size=(1, 2, 5, 8)); k2 = rng.normal(size=(1, 2, 5, 8)); v = rng.normal(size=(1, 2, 5, 16))
    lam = np.array([0.5, 0.1])
    eps = 1e-2
    x = orc.diffattn_v1(q1, k1, q2, k2, v, lam, causal=True)
    y = orc.diffattn_v1(q1, k1, q2, k2, v, lam, causal=True, rms=True, eps=eps)
    ms = np.mean(x * x, axis=-1)
    _close(np.mean(y * y, axis=-1), ms / (ms + eps), 1e-13, "RMSNorm energy")
    # y is a positive multiple of x
    ratio = y / x
    assert np.all(ratio > 0)
    _close(ratio, ratio[..., :1] * np.ones_like(ratio), 1e-12, "RMSNorm direction")


def pin_brute(orc):
    rng = _rng(18)
    # V1, GQA 4 heads over 2 KV heads, ragged Lq < Lk, with and without RMSNorm
    B, H, Hkv, Lq, Lk, d, dv = 2, 4, 2, 5, 7, 6, 3
    q1 = rng.normal(size=(B, H, Lq, d)); q2 = rng.normal(size=(B, H, Lq, d))
    k1 = rng.normal(size=(B, Hkv, Lk, d)); k2 = rng.normal(size=(B, Hkv, Lk, d))
    v = rng.normal(size=(B, Hkv, Lk, dv))
    lam = rng.normal(size=H)
    for causal in (True, False):
        for rms in (False, True):
            ref = np.array(brute.v1(q1.tolist(), k1.tolist(), q2.tolist(), k2.tolist(), v.tolist(),
                                    lam.tolist(), causal, rms))
            out = orc.diffattn_v1(q1, k1, q2, k2, v, lam, causal=causal, rms=rms)
            _close(out, ref, 1e-12, f"brute V1 causal={causal} rms={rms}")
    # V2, 8 Q heads (4 pairs) over 2 KV heads
    Hq = 8
    q = rng.normal(size=(B, Hq, Lq, d)); k = rng.normal(size=(B, Hkv, Lk, d)); v = rng.normal(size=(B, Hkv, Lk, d))
    lam = rng.normal(size=Hq // 2)
    for causal in (True, False):
        ref = np.array(brute.v2(q.tolist(), k.tolist(), v.tolist(), lam.tolist(), causal))
        _close(orc.diffattn_v2(q, k, v, lam, causal=causal), ref, 1e-12, f"brute V2 causal={causal}")
    # lambda
    a = [rng.normal(0, 0.1, (3, 5)) for _ in range(4)]
    ref = np.array(brute.lam(*[x.tolist() for x in a], 0.3), dtype=np.float32)
    got = orc.lambda_(*a, 0.3)
    assert np.all(np.abs(got.astype(np.float64) - ref.astype(np.float64)) <= 1e-7)


def pin_noise_probe_closed_form(orc):
    """Step 3's SNR (weight at the signal key over the mean weight at the noise
    keys) and Step 1's noise fraction on constructions with a closed form: the
    query meets the signal key with score s0 and every noise key with one
    score sn (the noise keys differ only in directions orthogonal to the
    query), so with Z = e^s0 + (N-1) e^sn the plain row is e^s0/Z at the
    signal key and e^sn/Z at each noise key: SNR_plain = e^(s0-sn) for every
    N, the noise fraction is (N-1) e^sn/Z, and the difference's SNR is
    (A1[0] - lam A2[0]) / (A1[j] - lam A2[j]).  Evaluated with mpmath at 40
    digits.  A sum in place of the mean, the signal key counted as noise, or
    a missing 1/sqrt(d) each miss it."""
    import mpmath as mp
    mp.mp.dps = 40
    d, lam = 4, 0.5
    cases = ((5, (1.5, 2.0, 0.25), (0.5, 0.75, -1.0)), (12, (2.0, 3.0, -0.5), (1.0, -0.5, 0.125)),
             (1000, (2.5, 4.0, 0.0), (1.0, 1.0, 1.0)))
    for N, p1, p2 in cases:
        rng = _rng(N)

        def keys(a, b, c):
            q = np.array([a, 0.0, 0.0, 0.0])
            k = np.zeros((N, d))
            k[0, 0], k[1:, 0] = b, c
            k[1:, 1:] = rng.normal(size=(N - 1, d - 1))
            return q, k

        def row(a, b, c):
            s0, sn = mp.mpf(a) * b / mp.sqrt(d), mp.mpf(a) * c / mp.sqrt(d)
            Z = mp.e ** s0 + (N - 1) * mp.e ** sn
            return mp.e ** s0 / Z, mp.e ** sn / Z

        (q1, k1), (q2, k2) = keys(*p1), keys(*p2)
        r = orc.noise_probe(q1[None], k1[None], q2[None], k2[None], lam)
        a0, an = row(*p1)
        b0, bn = row(*p2)
        want = {"snr_plain": a0 / an, "snr_diff": (a0 - lam * b0) / (an - lam * bn),
                "noise_fraction_plain": (N - 1) * an}
        assert abs(want["snr_plain"] - mp.e ** ((mp.mpf(p1[0]) * p1[1] - mp.mpf(p1[0]) * p1[2]) / 2)) < 1e-30
        for key, w in want.items():
            got = float(r[key][0])
            assert abs(got - float(w)) <= 1e-12 * abs(float(w)), (N, key, got, float(w))


ALL_PINS = [pin_lambda_init, pin_lambda, pin_standard_attention, pin_exact_zero, pin_row_sums,
            pin_masks_and_positivity, pin_suffix_consistency, pin_uniform_keys, pin_scale,
            pin_rmsnorm, pin_brute, pin_noise_probe_closed_form]
