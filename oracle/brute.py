"""Pure-Python per-element twin of the oracle, for tiny shapes only.

TEST INFRASTRUCTURE ONLY: nothing on the product path imports this module.

It restates the same definition as ``oracle.diffattn`` with scalar loops and
``math.exp`` and no NumPy at all, so that a slip in the vectorised oracle (a
transposed operand, a wrong head mapping, a broadcasting error, a mask off by
one) shows up as a disagreement between the two.  Sources as in
``oracle/__init__.py``: "差分注意力" tutorial, section 差分思路 and Step 2;
the V1/V2 layouts from its section V1 到 V2 的 diff.

Inputs are nested Python lists of floats.
"""

from __future__ import annotations

import math


def _row_weights(q, keys, limit):
    """Softmax weights of one query over keys[0..limit] (inclusive); zeros after."""
    d = len(q)
    n = len(keys)
    w = [0.0] * n
    if limit < 0:
        return w
    scores = []
    for j in range(limit + 1):
        s = 0.0
        for t in range(d):
            s += q[t] * keys[j][t]
        scores.append(s / math.sqrt(d))
    m = max(scores)
    z = 0.0
    for j in range(limit + 1):
        w[j] = math.exp(scores[j] - m)
        z += w[j]
    for j in range(limit + 1):
        w[j] /= z
    return w


def head(q1, k1, q2, k2, v, lam, causal, rms=False, eps=1e-5):
    """One head: q* [Lq][d], k* [Lk][d], v [Lk][dv] -> [Lq][dv]."""
    Lq, Lk = len(q1), len(k1)
    dv = len(v[0]) if Lk else 0
    out = []
    for i in range(Lq):
        limit = min(Lk - 1, i + (Lk - Lq)) if causal else Lk - 1
        w1 = _row_weights(q1[i], k1, limit)
        w2 = _row_weights(q2[i], k2, limit)
        row = []
        for c in range(dv):
            acc = 0.0
            for j in range(Lk):
                acc += (w1[j] - lam * w2[j]) * v[j][c]
            row.append(acc)
        if rms:
            ms = sum(x * x for x in row) / dv
            r = 1.0 / math.sqrt(ms + eps)
            row = [x * r for x in row]
        out.append(row)
    return out


def v1(q1, k1, q2, k2, v, lam, causal, rms=False, eps=1e-5):
    """q1,q2 [B][H][Lq][d]; k1,k2 [B][Hkv][Lk][d]; v [B][Hkv][Lk][dv]; lam [H]."""
    B, H, Hkv = len(q1), len(q1[0]), len(k1[0])
    grp = H // Hkv
    return [[head(q1[b][h], k1[b][h // grp], q2[b][h], k2[b][h // grp], v[b][h // grp],
                  lam[h], causal, rms, eps) for h in range(H)] for b in range(B)]


def v2(q, k, v, lam, causal):
    """q [B][Hq][Lq][D]; k,v [B][Hkv][Lk][D]; lam [Hq/2]; pair h = Q heads 2h, 2h+1."""
    B, Hq, Hkv = len(q), len(q[0]), len(k[0])
    grp = Hq // Hkv
    out = []
    for b in range(B):
        pairs = []
        for h in range(Hq // 2):
            g = (2 * h) // grp
            pairs.append(head(q[b][2 * h], k[b][g], q[b][2 * h + 1], k[b][g], v[b][g],
                              lam[h], causal))
        out.append(pairs)
    return out


def lam(lq1, lk1, lq2, lk2, lam_init):
    """exp(lq1.lk1) - exp(lq2.lk2) + lam_init per head, in Python floats."""
    res = []
    for h in range(len(lq1)):
        a = sum(x * y for x, y in zip(lq1[h], lk1[h]))
        b = sum(x * y for x, y in zip(lq2[h], lk2[h]))
        res.append(math.exp(a) - math.exp(b) + lam_init)
    return res
