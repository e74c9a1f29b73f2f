"""Pins of the fp64 backward oracle (no GPU).

The oracle writes out the chain rule of the forward.  These tests pin it to
things that do not share its derivation: central finite differences of the
forward oracle, and torch.autograd applied to a separate masked-softmax forward
written with torch ops.  A dropped term (the D correction, the -lambda factor
of map 2, the RMSNorm projection), a transposed product or a wrong mask
fails them."""

import math

import numpy as np
import pytest
import torch

from oracle import backward as bwd
from oracle import diffattn as orc


def _rand(shape, rng, scale=1.0):
    return rng.standard_normal(shape) * scale


def _fd(f, x, eps=1e-6):
    """Central differences of the scalar f with respect to every entry of x (in place)."""
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        fp = f()
        x[i] = old - eps
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


def pin_v2_finite_differences(b, causal, Lq, Lk):
    rng = np.random.default_rng(11 + Lq + Lk)
    q = _rand((1, 4, Lq, 3), rng)
    k = _rand((1, 1, Lk, 3), rng)
    v = _rand((1, 1, Lk, 3), rng)
    lam = np.array([0.7, -0.2])
    dout = _rand((1, 2, Lq, 3), rng)
    loss = lambda: float(np.sum(dout * orc.diffattn_v2(q, k, v, lam, causal=causal)))  # noqa: E731
    dq, dk, dv, dlam = b.diffattn_v2_backward(q, k, v, lam, dout, causal=causal)
    for got, x in ((dq, q), (dk, k), (dv, v), (dlam, lam)):
        want = _fd(loss, x)
        assert np.allclose(got, want, rtol=1e-6, atol=1e-8)


def pin_v1_finite_differences(b, rms):
    rng = np.random.default_rng(23 + rms)
    q1, q2 = _rand((2, 2, 4, 3), rng), _rand((2, 2, 4, 3), rng)
    k1, k2 = _rand((2, 1, 4, 3), rng), _rand((2, 1, 4, 3), rng)
    v = _rand((2, 1, 4, 5), rng)
    lam = np.array([0.45, 1.1])
    dout = _rand((2, 2, 4, 5), rng)
    loss = lambda: float(np.sum(dout * orc.diffattn_v1(q1, k1, q2, k2, v, lam, causal=True,  # noqa: E731
                                                         rms=rms, eps=1e-5)))
    grads = b.diffattn_v1_backward(q1, k1, q2, k2, v, lam, dout, causal=True, rms=rms, eps=1e-5)
    for got, x in zip(grads, (q1, k1, q2, k2, v, lam)):
        assert np.allclose(got, _fd(loss, x), rtol=1e-6, atol=1e-8)


def pin_lambda_parameters(b):
    rng = np.random.default_rng(5)
    p = [_rand((3, 4), rng, 0.3) for _ in range(4)]
    dlam = np.array([0.5, -1.5, 2.0])

    def lam64():
        a = np.exp(np.sum(p[0] * p[1], axis=1))
        b = np.exp(np.sum(p[2] * p[3], axis=1))
        return a - b + 0.2

    loss = lambda: float(np.sum(dlam * lam64()))  # noqa: E731
    for got, x in zip(b.lambda_backward(*p, dlam), p):
        assert np.allclose(got, _fd(loss, x), rtol=1e-7, atol=1e-10)


def _torch_forward_v2(q, k, v, lam, causal):
    """Independent forward with torch ops (masked softmax by -inf fill)."""
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    grp = Hq // Hkv
    outs = []
    for h in range(Hq // 2):
        g = (2 * h) // grp
        s1 = q[:, 2 * h] @ k[:, g].transpose(-1, -2) / math.sqrt(D)
        s2 = q[:, 2 * h + 1] @ k[:, g].transpose(-1, -2) / math.sqrt(D)
        if causal:
            i = torch.arange(Lq)[:, None]
            j = torch.arange(Lk)[None, :]
            mask = j > i + (Lk - Lq)
            s1 = s1.masked_fill(mask, float("-inf"))
            s2 = s2.masked_fill(mask, float("-inf"))
        outs.append((torch.softmax(s1, -1) - lam[h] * torch.softmax(s2, -1)) @ v[:, g])
    return torch.stack(outs, dim=1)


def pin_autograd_with_gqa(b):
    g = torch.Generator().manual_seed(3)
    q = torch.randn(2, 8, 33, 16, generator=g, dtype=torch.float64, requires_grad=True)
    k = torch.randn(2, 2, 33, 16, generator=g, dtype=torch.float64, requires_grad=True)
    v = torch.randn(2, 2, 33, 16, generator=g, dtype=torch.float64, requires_grad=True)
    lam = torch.tensor([0.3, 0.9, -0.1, 0.6], dtype=torch.float64, requires_grad=True)
    dout = torch.randn(2, 4, 33, 16, generator=g, dtype=torch.float64)
    _torch_forward_v2(q, k, v, lam, True).backward(dout)
    dq, dk, dv, dlam = b.diffattn_v2_backward(q.detach(), k.detach(), v.detach(), lam.detach(), dout)
    for got, ref in ((dq, q.grad), (dk, k.grad), (dv, v.grad), (dlam, lam.grad)):
        assert np.allclose(got, ref.numpy(), rtol=1e-10, atol=1e-12)


# The pins above with their arguments; test_oracle_backward_mutations.py runs
# the same list against planted mistakes.
PINS = [
    (pin_v2_finite_differences, (True, 5, 5)),
    (pin_v2_finite_differences, (False, 4, 6)),
    (pin_v2_finite_differences, (True, 3, 6)),
    (pin_v1_finite_differences, (False,)),
    (pin_v1_finite_differences, (True,)),
    (pin_lambda_parameters, ()),
    (pin_autograd_with_gqa, ()),
]


@pytest.mark.parametrize("pin,args", PINS, ids=lambda x: getattr(x, "__name__", str(x)))
def test_pin(pin, args):
    pin(bwd, *args)


def test_zero_upstream_gives_zero_gradients_and_linearity():
    rng = np.random.default_rng(9)
    q, k, v = _rand((1, 2, 6, 4), rng), _rand((1, 1, 6, 4), rng), _rand((1, 1, 6, 4), rng)
    lam = np.array([0.8])
    zero = bwd.diffattn_v2_backward(q, k, v, lam, np.zeros((1, 1, 6, 4)))
    assert all(np.count_nonzero(t) == 0 for t in zero)
    d1, d2 = _rand((1, 1, 6, 4), rng), _rand((1, 1, 6, 4), rng)
    a = bwd.diffattn_v2_backward(q, k, v, lam, d1)
    b = bwd.diffattn_v2_backward(q, k, v, lam, d2)
    c = bwd.diffattn_v2_backward(q, k, v, lam, 2 * d1 - d2)
    for x, y, z in zip(a, b, c):
        assert np.allclose(z, 2 * x - y, rtol=1e-12, atol=1e-12)


def test_v1_gradients_are_v2_gradients_of_the_packed_layout():
    """The V1 and V2 oracle backwards agree through the packing identity: a V1
    head is the V2 pair [Q1|0], [0|Q2] over [K1|K2].  With d = 64 and the V2
    scale 1/sqrt(128), Q' is multiplied by sqrt(2) so that the scores are
    Q_m K_m^T / 8; the V1 gradients are then fixed halves of the packed ones.
    (Each backward is pinned on its own elsewhere; this ties the two.)"""
    rng = np.random.default_rng(29)
    B, H, Hkv, Lq, Lk, d = 1, 4, 2, 7, 9, 64
    q1, q2 = _rand((B, H, Lq, d), rng, 0.3), _rand((B, H, Lq, d), rng, 0.3)
    k1, k2 = _rand((B, Hkv, Lk, d), rng, 0.3), _rand((B, Hkv, Lk, d), rng, 0.3)
    v = _rand((B, Hkv, Lk, 2 * d), rng)
    lam = np.array([0.3, 0.9, -0.1, 1.2])
    dout = _rand((B, H, Lq, 2 * d), rng)
    want = bwd.diffattn_v1_backward(q1, k1, q2, k2, v, lam, dout, causal=True)

    c = math.sqrt(2.0)
    qp = np.zeros((B, 2 * H, Lq, 2 * d))
    qp[:, 0::2, :, :d] = c * q1
    qp[:, 1::2, :, d:] = c * q2
    kp = np.concatenate([k1, k2], axis=-1)
    dqp, dkp, dv, dlam = bwd.diffattn_v2_backward(qp, kp, v, lam, dout, causal=True)
    got = (c * dqp[:, 0::2, :, :d], dkp[:, :, :, :d], c * dqp[:, 1::2, :, d:], dkp[:, :, :, d:], dv, dlam)
    for a, b in zip(got, want):
        assert np.allclose(a, b, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("rms", [False, True])
def test_dlambda_terms_sum_to_dlambda(rms):
    """dlambda_terms (the error scale of dlambda in the GPU tests) sums to the
    finite-difference-pinned dlambda; without RMSNorm its terms are dO * O_2."""
    rng = np.random.default_rng(31 + rms)
    q1, q2, k1, k2 = (_rand((6, 3), rng) for _ in range(4))
    v, dout = _rand((6, 5), rng), _rand((6, 5), rng)
    t = bwd.dlambda_terms(q1, k1, q2, k2, v, 0.6, dout, True, rms=rms)
    assert np.isclose(-t.sum(), bwd.head_backward(q1, k1, q2, k2, v, 0.6, dout, True, rms=rms)[5], rtol=1e-12)
    if not rms:
        _, A2 = orc.maps(q1, k1, q2, k2, True)
        assert np.allclose(t, dout * (A2 @ v), rtol=1e-13, atol=0)


def test_dlambda_orthogonal_terms_sum_to_dlambda_up_to_eps():
    """With RMSNorm, the terms dX * (O_2 - c X) sum to -dlambda up to
    c dX . X = c <y, dY> eps r^2, which vanishes with eps; and they are
    smaller than dX * O_2 when the maps are alike."""
    rng = np.random.default_rng(37)
    q1, k1 = _rand((40, 8), rng, 0.05), _rand((40, 8), rng, 0.05)     # small scores: near-uniform maps
    q2, k2 = _rand((40, 8), rng, 0.05), _rand((40, 8), rng, 0.05)
    v, dout = _rand((40, 6), rng), _rand((40, 6), rng)
    for eps in (1e-5, 0.0):
        full = bwd.dlambda_terms(q1, k1, q2, k2, v, 0.5, dout, True, rms=True, eps=eps)
        perp = bwd.dlambda_terms(q1, k1, q2, k2, v, 0.5, dout, True, rms=True, eps=eps, orthogonal=True)
        dlam = bwd.head_backward(q1, k1, q2, k2, v, 0.5, dout, True, rms=True, eps=eps)[5]
        assert np.isclose(-full.sum(), dlam, rtol=1e-12)
        tol = 1e-12 if eps == 0.0 else 1e-3
        assert abs(-perp.sum() - dlam) <= tol * np.abs(full).sum()
        assert np.linalg.norm(perp) < 0.5 * np.linalg.norm(full)
