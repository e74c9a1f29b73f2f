"""Backward of the V2 forward (training forward, dQ, dK, dV, dlambda, lambda's
parameter gradients) against the fp64 oracle.  Needs a B200.

Tolerance as for the forward: max|g - g_ref| <= 2e-2 max|g_ref| per gradient
tensor (bf16 outputs of fp32 arithmetic)."""

import math

import numpy as np
import pytest
import torch

import differential_attention_transformers_b200 as da
from differential_attention_transformers_b200 import inputs
from oracle import backward as bwd
from oracle import diffattn as orc
from tests.test_parity_gpu import BF16_TOL, DEV, lam_gpu_and_ref

pytestmark = pytest.mark.gpu


def _rel(got, ref):
    got = got.double().cpu().numpy() if hasattr(got, "cpu") else np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref))) / scale if scale > 0 else float(np.max(np.abs(got)))


# dlambda sums Lq * dv products of the upstream gradient (dO, or with RMSNorm
# the f32 dX) and the forward's stored bf16 map-2 output, rounded to 2^-9
# relative.  Its error therefore scales with the terms, not with their sum.
# With RMSNorm the forward stores map 2's part orthogonal to the difference
# output X (dX is orthogonal to X), so the terms are dX * (O_2 - c X), small
# when the maps are alike even though dX * O_2 is not.  Bound: the output
# tolerance plus ten unit roundings of those terms' 2-norm (a dropped term or
# a sign error misses it by far more).
DLAM_ROUND = 10 * 2.0 ** -9


def _dlam_ok(got, ref, term_norms):
    got = got.double().cpu().numpy()
    ref = np.asarray(ref, dtype=np.float64)
    bound = BF16_TOL * np.max(np.abs(ref)) + DLAM_ROUND * np.asarray(term_norms)
    return bool(np.all(np.abs(got - ref) <= bound)), np.abs(got - ref), bound


def _case(B, Hq, Hkv, Lq, Lk, seed, lam_lo=-0.2, lam_hi=1.0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    s = 1 / math.sqrt(128)
    mk = lambda *shape, std=s: (torch.randn(*shape, generator=g) * std).to(torch.bfloat16).to(DEV)  # noqa: E731
    q, k, v = mk(B, Hq, Lq, 128), mk(B, Hkv, Lk, 128), mk(B, Hkv, Lk, 128)
    dout = mk(B, Hq // 2, Lq, 128, std=1.0)
    lam = (torch.rand(Hq // 2, generator=g) * (lam_hi - lam_lo) + lam_lo).to(DEV)
    return q, k, v, dout, lam


CASES = [
    # B, Hq, Hkv, Lq, Lk, causal
    (1, 4, 1, 200, 200, True),      # ragged tails, one KV head for both pairs
    (2, 8, 2, 300, 300, False),     # non-causal, GQA groups of 4 Q heads
    (1, 4, 2, 130, 257, True),      # Lq < Lk: bottom-right causal offset
    (1, 4, 2, 257, 130, True),      # Lq > Lk: the first rows see no key (a row block with no key tile)
    (1, 8, 1, 64, 64, True),        # a single tile
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,causal", CASES)
def test_backward_matches_oracle(B, Hq, Hkv, Lq, Lk, causal):
    q, k, v, dout, lam = _case(B, Hq, Hkv, Lq, Lk, seed=Lq + 7 * Lk + Hq)
    out, lse, om = da.fwd_v2_train(q, k, v, lam, causal=causal)
    assert torch.equal(out, da.fwd_v2(q, k, v, lam, causal=causal))   # the training forward is the forward
    dq, dk, dv, dlam = da.bwd_v2(q, k, v, lam, dout, lse, om, causal=causal)
    torch.cuda.synchronize()
    assert da.last_status() == da.OK
    rq, rk, rv, rl = bwd.diffattn_v2_backward(q, k, v, lam.cpu().numpy(), dout, causal=causal)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        assert torch.isfinite(got.float()).all(), name
        assert _rel(got, ref) <= BF16_TOL, (name, _rel(got, ref))
    assert _rel(dlam, rl) <= BF16_TOL, ("dlambda", dlam.cpu().numpy(), rl)


def test_training_forward_statistics():
    q, k, v, dout, lam = _case(1, 4, 2, 190, 190, seed=31)
    out, lse, om = da.fwd_v2_train(q, k, v, lam, causal=True)
    qd, kd, vd = (orc._f64(t) for t in (q, k, v))
    sl = math.log2(math.e) / math.sqrt(128)
    for h in range(2):
        for m in range(2):
            qh = 2 * h + m
            g = qh // 2
            S = qd[0, qh] @ kd[0, g].T * sl
            vis = np.tril(np.ones((190, 190), dtype=bool))
            S = np.where(vis, S, -np.inf)
            mx = S.max(axis=1, keepdims=True)
            ref_lse = (mx + np.log2(np.sum(np.exp2(S - mx), axis=1, keepdims=True)))[:, 0]
            assert np.max(np.abs(lse[0, h, m].cpu().numpy() - ref_lse)) <= 1e-3
            A = np.exp2(S - ref_lse[:, None])
            assert _rel(om[0, h, m], A @ vd[0, g]) <= BF16_TOL


def test_lambda_parameter_gradients():
    g = torch.Generator(device="cpu").manual_seed(5)
    p = [(torch.randn(6, 32, generator=g) * 0.1).to(DEV) for _ in range(4)]
    dlam = torch.randn(6, generator=g).to(DEV)
    got = da.lambda_backward(*p, dlam)
    ref = bwd.lambda_backward(*[t.cpu().numpy() for t in p], dlam.cpu().numpy())
    for a, b in zip(got, ref):
        assert np.allclose(a.cpu().numpy(), b, rtol=1e-5, atol=1e-7)


def test_backward_full_size_sampled():
    # the V2 prefill workload; one KV group of one batch entry against the oracle
    w = inputs.WORKLOADS["v2_prefill"]
    x = inputs.make(w, device=DEV)
    lam, lref = lam_gpu_and_ref(w)
    gen = torch.Generator(device=DEV).manual_seed(77)
    dout = torch.randn((w.B, w.pairs, w.Lq, w.dv), generator=gen, device=DEV).to(torch.bfloat16)
    out, lse, om = da.fwd_v2_train(x["q"], x["k"], x["v"], lam, causal=True)
    dq, dk, dv, dlam = da.bwd_v2(x["q"], x["k"], x["v"], lam, dout, lse, om, causal=True)
    torch.cuda.synchronize()
    assert da.last_status() == da.OK
    for t in (dq, dk, dv, dlam):
        assert torch.isfinite(t.float()).all()
    b, g = 1, 3
    grp = w.H // w.Hkv
    rk, rv = 0.0, 0.0
    for h in range(g * grp // 2, (g + 1) * grp // 2):
        h1, h2 = 2 * h, 2 * h + 1
        a = bwd.head_backward(x["q"][b, h1], x["k"][b, g], x["q"][b, h2], x["k"][b, g], x["v"][b, g], float(lref[h]),
                              dout[b, h], causal=True)
        assert _rel(dq[b, h1], a[0]) <= BF16_TOL, ("dq", h1)
        assert _rel(dq[b, h2], a[2]) <= BF16_TOL, ("dq", h2)
        rk = rk + a[1] + a[3]
        rv = rv + a[4]
    assert _rel(dk[b, g], rk) <= BF16_TOL
    assert _rel(dv[b, g], rv) <= BF16_TOL


@pytest.mark.parametrize("lam_value", [0.97, 1.0, 0.86, 1.14])
def test_backward_near_unit_lambda_with_similar_maps(lam_value):
    """The hardest case for bf16 P and dS: near-uniform, nearly identical maps and
    lambda close to 1, where A_1 - lambda A_2 cancels."""
    g = torch.Generator(device="cpu").manual_seed(int(lam_value * 1000) + 1)
    s = 1 / math.sqrt(128)
    q1 = torch.randn(1, 1, 512, 128, generator=g) * s
    q2 = q1 + 0.05 * s * torch.randn(1, 1, 512, 128, generator=g)
    q = torch.cat([q1, q2], dim=1).to(torch.bfloat16).to(DEV)
    k = (torch.randn(1, 1, 512, 128, generator=g) * s).to(torch.bfloat16).to(DEV)
    v = (torch.randn(1, 1, 512, 128, generator=g) * s).to(torch.bfloat16).to(DEV)
    dout = torch.randn(1, 1, 512, 128, generator=g).to(torch.bfloat16).to(DEV)
    lam = torch.tensor([lam_value], device=DEV)
    _, lse, om = da.fwd_v2_train(q, k, v, lam, causal=True)
    dq, dk, dv, dlam = da.bwd_v2(q, k, v, lam, dout, lse, om, causal=True)
    rq, rk, rv, rl = bwd.diffattn_v2_backward(q, k, v, np.array([lam_value]), dout, causal=True)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        assert _rel(got, ref) <= BF16_TOL, (name, lam_value, _rel(got, ref))


# ----------------------------------------------------------------- V1 layout --
def _case_v1(B, H, Hkv, Lq, Lk, seed, lam_lo=-0.2, lam_hi=1.0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    s = 1 / math.sqrt(64)
    mk = lambda *shape, std=s: (torch.randn(*shape, generator=g) * std).to(torch.bfloat16).to(DEV)  # noqa: E731
    q1, q2 = mk(B, H, Lq, 64), mk(B, H, Lq, 64)
    k1, k2 = mk(B, Hkv, Lk, 64), mk(B, Hkv, Lk, 64)
    v = mk(B, Hkv, Lk, 128)
    dout = mk(B, H, Lq, 128, std=1.0)
    lam = (torch.rand(H, generator=g) * (lam_hi - lam_lo) + lam_lo).to(DEV)
    return q1, k1, q2, k2, v, dout, lam


CASES_V1 = [
    # B, H, Hkv, Lq, Lk, causal, rmsnorm
    (1, 2, 1, 200, 200, True, False),    # ragged tails, two heads share a KV head
    (2, 4, 2, 300, 300, False, True),    # non-causal, RMSNorm
    (1, 2, 2, 130, 257, True, True),     # Lq < Lk: bottom-right causal offset
    (1, 2, 1, 257, 130, True, True),     # Lq > Lk: the first rows see no key
    (1, 4, 4, 64, 64, True, False),      # a single tile
]


@pytest.mark.parametrize("B,H,Hkv,Lq,Lk,causal,rms", CASES_V1)
def test_v1_backward_matches_oracle(B, H, Hkv, Lq, Lk, causal, rms):
    q1, k1, q2, k2, v, dout, lam = _case_v1(B, H, Hkv, Lq, Lk, seed=3 * Lq + Lk + H)
    out, lse, om, rstd, o2c = da.fwd_v1_train(q1, k1, q2, k2, v, lam, causal=causal, rmsnorm=rms)
    inf = da.fwd_v1(q1, k1, q2, k2, v, lam, causal=causal, rmsnorm=rms)
    if rms:   # the training forward keeps P's residual on every head: equal up to P's rounding
        assert _rel(out, orc.diffattn_v1(q1, k1, q2, k2, v, lam.cpu().numpy(), causal=causal, rms=True)) <= BF16_TOL
        assert _rel(out, inf.double().cpu().numpy()) <= BF16_TOL
    else:     # the training forward is the forward
        assert torch.equal(out, inf)
    grads = da.bwd_v1(q1, k1, q2, k2, v, lam, dout, out, lse, om, rstd, o2c, causal=causal, rmsnorm=rms)
    torch.cuda.synchronize()
    assert da.last_status() == da.OK
    lr = lam.cpu().numpy()
    ref = bwd.diffattn_v1_backward(q1, k1, q2, k2, v, lr, dout, causal=causal, rms=rms, eps=1e-5)
    for name, got, r in zip(("dq1", "dk1", "dq2", "dk2", "dv"), grads, ref):
        assert torch.isfinite(got.float()).all(), name
        assert _rel(got, r) <= BF16_TOL, (name, _rel(got, r))
    grp = H // Hkv
    norms = [np.sqrt(sum(np.sum(bwd.dlambda_terms(q1[b, h], k1[b, h // grp], q2[b, h], k2[b, h // grp],
                                                  v[b, h // grp], lr[h], dout[b, h], causal, rms=rms,
                                                  orthogonal=True) ** 2)
                         for b in range(B))) for h in range(H)]
    ok, err, bound = _dlam_ok(grads[5], ref[5], norms)
    assert ok, ("dlambda", err, bound)


def test_v1_training_forward_statistics():
    q1, k1, q2, k2, v, dout, lam = _case_v1(1, 2, 1, 190, 190, seed=41)
    out, lse, om, rstd, o2c = da.fwd_v1_train(q1, k1, q2, k2, v, lam, causal=True, rmsnorm=True)
    sl = math.log2(math.e) / 8.0
    vis = np.tril(np.ones((190, 190), dtype=bool))
    vd = orc._f64(v[0, 0])
    for h in range(2):
        A = []
        for m, (q, k) in enumerate(((q1, k1), (q2, k2))):
            S = np.where(vis, orc._f64(q[0, h]) @ orc._f64(k[0, 0]).T * sl, -np.inf)
            mx = S.max(axis=1, keepdims=True)
            ref_lse = (mx + np.log2(np.sum(np.exp2(S - mx), axis=1, keepdims=True)))[:, 0]
            assert np.max(np.abs(lse[0, h, m].cpu().numpy() - ref_lse)) <= 1e-3
            A.append(np.exp2(S - ref_lse[:, None]))
        x = (A[0] - float(lam[h]) * A[1]) @ vd
        r = 1.0 / np.sqrt(np.mean(x * x, axis=1) + 1e-5)
        assert np.max(np.abs(rstd[0, h].cpu().numpy() - r) / r) <= 1e-2
        assert _rel(om[0, h, 0], A[0] @ vd) <= BF16_TOL
        # map 2 is stored as its part orthogonal to x, with c eps r^2 per row.
        # That part is a small difference of the kernel's own O_2 and x, which
        # carry the bf16 rounding of P: its error is on the scale of O_2.
        o2 = A[1] @ vd
        c = np.sum(o2 * x, axis=1) / np.sum(x * x, axis=1)
        perp = o2 - c[:, None] * x
        got_perp = om[0, h, 1].double().cpu().numpy()
        assert np.max(np.abs(got_perp - perp)) <= BF16_TOL * np.max(np.abs(o2))
        assert np.max(np.abs(np.sum(got_perp * x, axis=1))) <= 2e-2 * np.max(np.abs(np.sum(o2 * x, axis=1)))
        assert _rel(o2c[0, h], c * 1e-5 * r * r) <= BF16_TOL


@pytest.mark.parametrize("lam_value", [0.3, 0.5, 0.7])
def test_v1_dlambda_rmsnorm_alike_maps(lam_value):
    """dlambda with RMSNorm when the two maps are alike (near-uniform maps from
    small scores, the V1 workload's input scale): X = O_1 - lambda O_2 is then
    nearly parallel to O_2, and the sum of dX . O_2 is a small remainder of
    terms over 5x larger in 2-norm.  With map 2's orthogonal part stored (and
    P's residual kept), the error scales with the terms dX * (O_2 - c X): it
    stays within the output tolerance plus ten roundings of their 2-norm (at
    least five times smaller than the terms dX * O_2 here), and within the
    plain 2e-2 |dlambda| wherever |dlambda| is above twice their 2-norm."""
    q1, k1, q2, k2, v, dout, _ = _case_v1(1, 2, 1, 1024, 1024, seed=int(lam_value * 100) + 9)
    lam = torch.full((2,), lam_value, device=DEV)
    out, lse, om, rstd, o2c = da.fwd_v1_train(q1, k1, q2, k2, v, lam, causal=True, rmsnorm=True)
    grads = da.bwd_v1(q1, k1, q2, k2, v, lam, dout, out, lse, om, rstd, o2c, causal=True, rmsnorm=True)
    torch.cuda.synchronize()
    assert da.last_status() == da.OK
    lr = lam.cpu().numpy().astype(np.float64)
    ref = bwd.diffattn_v1_backward(q1, k1, q2, k2, v, lr, dout, causal=True, rms=True, eps=1e-5)
    for h in range(2):
        full = bwd.dlambda_terms(q1[0, h], k1[0, 0], q2[0, h], k2[0, 0], v[0, 0], lr[h], dout[0, h], True, rms=True)
        perp = bwd.dlambda_terms(q1[0, h], k1[0, 0], q2[0, h], k2[0, 0], v[0, 0], lr[h], dout[0, h], True, rms=True,
                                 orthogonal=True)
        n_full, n_perp = np.sqrt(np.sum(full ** 2)), np.sqrt(np.sum(perp ** 2))
        assert n_perp < 0.2 * n_full   # the case is ill-conditioned for the terms dX * O_2
        err = abs(float(grads[5][h]) - ref[5][h])
        bound = BF16_TOL * abs(ref[5][h]) + DLAM_ROUND * n_perp
        assert err <= bound, (h, err, bound)
        if abs(ref[5][h]) > 2 * n_perp:
            assert err <= BF16_TOL * abs(ref[5][h]), (h, err, ref[5][h])
