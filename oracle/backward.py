"""Definition-level fp64 gradients of the differential attention forward.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): nothing on the product
path imports this module.

The forward is the one in ``oracle/diffattn.py`` ("差分注意力" tutorial,
section 差分思路 and Step 2; V1/V2 layouts from its section V1 到 V2 的 diff):

    S_m = Q_m K_m^T / sqrt(d),  A_m = softmax(S_m) (masked),  O_m = A_m V
    X   = O_1 - lambda O_2,     O = X  or  RMSNorm(X)

λ is learnable (tutorial, Step 4 λ 参数化: λ = exp(lq1.lk1) - exp(lq2.lk2) +
λ_init), so training needs its gradient too.  The pages print no backward;
what follows is the chain rule of that forward, written out per head with a
given upstream gradient dO:

    RMSNorm (when used), r = (mean(X^2) + eps)^-1/2 over the value width n:
        dX = r dO - (r^3 / n) X <X, dO>            (per row)
    dV    = (A_1 - lambda A_2)^T dX
    dW    = dX V^T                                  (gradient of A_1 - lambda A_2)
    D_m   = rowsum(dX * O_m)                        (= rowsum(dW * A_m))
    dS_1  =  A_1 * (dW - D_1)
    dS_2  = -lambda A_2 * (dW - D_2)
    dQ_m  = dS_m K_m / sqrt(d),  dK_m = dS_m^T Q_m / sqrt(d)
    dlambda = -sum(dX * O_2)
    and for λ's parameters, with e_1 = exp(lq1.lk1), e_2 = exp(lq2.lk2):
        dlq1 = dlambda e_1 lk1, dlk1 = dlambda e_1 lq1,
        dlq2 = -dlambda e_2 lk2, dlk2 = -dlambda e_2 lq2.

Masked entries have A = 0, so their dS is 0; a row that sees no key
contributes nothing.  In the V2 layout the two maps of a pair and every pair of
a KV group share K and V, so their dK and dV add up; λ is per head (V1) or per
pair (V2) and its gradient sums over batch and rows.

Pinned in tests/test_oracle_backward.py against central finite differences of
the forward oracle and against an independent autograd derivation.
"""

from __future__ import annotations

import numpy as np

from .diffattn import ROW_CHUNK, _f64, _pair_heads, maps


def head_backward(q1, k1, q2, k2, v, lam: float, dout, causal: bool, rms: bool = False, eps: float = 1e-5):
    """Gradients for one head.  q* [Lq, d], k* [Lk, d], v [Lk, dv], dout [Lq, dv].

    Returns (dq1, dk1, dq2, dk2, dv, dlam) in fp64.  Rows are processed in
    chunks; dK, dV and dlam accumulate over them.
    """
    q1, k1, q2, k2, v, dout = (_f64(t) for t in (q1, k1, q2, k2, v, dout))
    lam = float(lam)
    Lq, d = q1.shape
    s = 1.0 / np.sqrt(d)
    dq1, dq2 = np.zeros_like(q1), np.zeros_like(q2)
    dk1, dk2, dv = np.zeros_like(k1), np.zeros_like(k2), np.zeros_like(v)
    dlam = 0.0
    for r0 in range(0, Lq, ROW_CHUNK):
        r1 = min(Lq, r0 + ROW_CHUNK)
        A1, A2 = maps(q1[r0:r1], k1, q2[r0:r1], k2, causal, r0, Lq)
        O1, O2 = A1 @ v, A2 @ v
        dx = dout[r0:r1]
        if rms:
            x = O1 - lam * O2
            n = x.shape[1]
            r = 1.0 / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + eps)
            dx = r * dx - (r ** 3 / n) * x * np.sum(x * dx, axis=1, keepdims=True)
        dv += (A1 - lam * A2).T @ dx
        dW = dx @ v.T
        D1 = np.sum(dx * O1, axis=1, keepdims=True)
        D2 = np.sum(dx * O2, axis=1, keepdims=True)
        dS1 = A1 * (dW - D1)
        dS2 = -lam * A2 * (dW - D2)
        dq1[r0:r1] = s * (dS1 @ k1)
        dq2[r0:r1] = s * (dS2 @ k2)
        dk1 += s * (dS1.T @ q1[r0:r1])
        dk2 += s * (dS2.T @ q2[r0:r1])
        dlam -= float(np.sum(dx * O2))
    return dq1, dk1, dq2, dk2, dv, dlam


def dlambda_terms(q1, k1, q2, k2, v, lam: float, dout, causal: bool, rms: bool = False, eps: float = 1e-5,
                  orthogonal: bool = False):
    """The products dX * O_2 whose sum, negated, is one head's dlambda ([Lq, dv] fp64).

    Used to state the error a bf16 implementation can reach: dlambda sums
    Lq * dv products of two stored bf16 operands, so its rounding scales with
    the terms' size, not with the sum's.  With RMSNorm, dX is orthogonal to X
    (up to eps), and when the two maps are alike O_2 is nearly parallel to X,
    so the sum is a small remainder of large terms.

    orthogonal=True (with rms): the products dX * (O_2 - c X), c = <O_2, X> /
    <X, X> per row, i.e. with map 2's output reduced to its part orthogonal
    to X.  Their sum differs from that of dX * O_2 only by c dX . X, which
    is of order eps; an implementation that stores that part instead of O_2
    has rounding of these terms' size."""
    q1, k1, q2, k2, v, dout = (_f64(t) for t in (q1, k1, q2, k2, v, dout))
    A1, A2 = maps(q1, k1, q2, k2, causal, 0, q1.shape[0])
    O1, O2 = A1 @ v, A2 @ v
    dx = dout
    if rms:
        x = O1 - float(lam) * O2
        r = 1.0 / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + eps)
        dx = r * dx - (r ** 3 / x.shape[1]) * x * np.sum(x * dx, axis=1, keepdims=True)
        if orthogonal:
            xx = np.sum(x * x, axis=1, keepdims=True)
            c = np.divide(np.sum(O2 * x, axis=1, keepdims=True), xx, out=np.zeros_like(xx), where=xx > 0)
            return dx * (O2 - c * x)
    return dx * O2


def diffattn_v2_backward(q, k, v, lam, dout, causal=True):
    """V2 layout.  q [B,Hq,Lq,D]; k,v [B,Hkv,Lk,D]; lam [Hq/2]; dout [B,Hq/2,Lq,D].

    Returns dq [B,Hq,Lq,D], dk, dv [B,Hkv,Lk,D], dlam [Hq/2] (fp64).
    """
    q, k, v, dout = (_f64(t) for t in (q, k, v, dout))
    lam = np.asarray(_f64(lam), dtype=np.float64).reshape(-1)
    B, Hq, Lq, D = q.shape
    Hkv = k.shape[1]
    grp = Hq // Hkv
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dlam = np.zeros(Hq // 2)
    for b in range(B):
        for h in range(Hq // 2):
            h1, h2 = _pair_heads(h)
            g = h1 // grp
            g1, gk1, g2, gk2, gv, gl = head_backward(q[b, h1], k[b, g], q[b, h2], k[b, g], v[b, g], lam[h],
                                                     dout[b, h], causal)
            dq[b, h1], dq[b, h2] = g1, g2
            dk[b, g] += gk1 + gk2
            dv[b, g] += gv
            dlam[h] += gl
    return dq, dk, dv, dlam


def diffattn_v1_backward(q1, k1, q2, k2, v, lam, dout, causal=True, rms=False, eps=1e-5):
    """V1 layout.  q1,q2 [B,H,Lq,d]; k1,k2 [B,Hkv,Lk,d]; v [B,Hkv,Lk,dv]; lam [H];
    dout [B,H,Lq,dv].  Returns dq1, dk1, dq2, dk2, dv, dlam [H] (fp64)."""
    q1, k1, q2, k2, v, dout = (_f64(t) for t in (q1, k1, q2, k2, v, dout))
    lam = np.asarray(_f64(lam), dtype=np.float64).reshape(-1)
    B, H = q1.shape[:2]
    Hkv = k1.shape[1]
    grp = H // Hkv
    dq1, dq2 = np.zeros_like(q1), np.zeros_like(q2)
    dk1, dk2, dv = np.zeros_like(k1), np.zeros_like(k2), np.zeros_like(v)
    dlam = np.zeros(H)
    for b in range(B):
        for h in range(H):
            g = h // grp
            a, bk1, c, bk2, bv, bl = head_backward(q1[b, h], k1[b, g], q2[b, h], k2[b, g], v[b, g], lam[h],
                                                   dout[b, h], causal, rms, eps)
            dq1[b, h], dq2[b, h] = a, c
            dk1[b, g] += bk1
            dk2[b, g] += bk2
            dv[b, g] += bv
            dlam[h] += bl
    return dq1, dk1, dq2, dk2, dv, dlam


def lambda_backward(lq1, lk1, lq2, lk2, dlam):
    """Gradients of λ = exp(lq1.lk1) - exp(lq2.lk2) + λ_init with respect to its
    four parameter vectors, given dlam [H].  Returns (dlq1, dlk1, dlq2, dlk2)."""
    lq1, lk1, lq2, lk2 = (np.asarray(_f64(t), dtype=np.float64) for t in (lq1, lk1, lq2, lk2))
    g = np.asarray(_f64(dlam), dtype=np.float64).reshape(-1, 1)
    e1 = np.exp(np.sum(lq1 * lk1, axis=1, keepdims=True))
    e2 = np.exp(np.sum(lq2 * lk2, axis=1, keepdims=True))
    return g * e1 * lk1, g * e1 * lq1, -g * e2 * lk2, -g * e2 * lq2
