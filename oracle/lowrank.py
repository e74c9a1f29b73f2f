"""fp64 oracle of the fixed low-rank substitute for the second attention map.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): nothing on the product
path imports this module.

Source: the paper note "Understanding Differential Transformer Unchains
Pretrained Self-Attentions", sections 基于分析的改进建议 and 亮点与洞察.  The
note finds the noise component that A2 removes to be low-rank, and proposes a
cheaper differential variant that does without a second full QK attention:
a fixed low-rank matrix in place of A2.  It gives no form for that matrix.

Reading (the plainest one that keeps the rest of the method intact):

  * N replaces A2 and is a map like A2: non-negative, zero on masked keys,
    each row summing to 1 over the keys it sees, so that rows of A1 - lambda N
    still sum to 1 - lambda.
  * N is fixed (it does not depend on the input) and of rank <= r.  It is
    given by non-negative positional factors F [Lq, r] (query positions) and
    G [Lk, r] (key positions):

        N[i, j] = (f_i . g_j) / sum_{j' visible from i} (f_i . g_j')   for visible j,
        N[i, j] = 0 otherwise, and N[i, :] = 0 when that sum is 0.

    Without a mask, N = diag(1 / (F G^T 1)) F G^T has rank <= r.  With the
    causal mask it is the masked low-rank matrix that causal linear attention
    with fixed features produces.
  * O = (A1 - lambda N) V, with A1 = softmax(Q1 K1^T / sqrt(d)) as in the
    forward (oracle.diffattn).

  r = 1 with F = G = 1 makes N the uniform map over the visible keys: the
  limit of A2 as its scores vanish, i.e. softmax's noise floor (tutorial,
  Step 1).
"""

from __future__ import annotations

import numpy as np

from .diffattn import _f64, _scale, _softmax_masked, _visible


def noise_map(F, G, Lq: int, Lk: int, causal: bool) -> np.ndarray:
    """The explicit fixed map N [Lq, Lk] from factors F [Lq, r], G [Lk, r] (>= 0)."""
    F = np.asarray(F, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    if np.any(F < 0) or np.any(G < 0):
        raise ValueError("the factors must be non-negative")
    W = np.where(_visible(np.arange(Lq), Lq, Lk, causal), F @ G.T, 0.0)
    z = W.sum(axis=1, keepdims=True)
    return np.divide(W, z, out=np.zeros_like(W), where=z > 0)


def lowrank_head(q1, k1, v, F, G, lam: float, causal: bool) -> np.ndarray:
    """O = (A1 - lam N) V for one head: q1 [Lq, d], k1 [Lk, d], v [Lk, dv]."""
    q1, k1, v = (_f64(t) for t in (q1, k1, v))
    Lq, d = q1.shape
    Lk = k1.shape[0]
    A1 = _softmax_masked((q1 @ k1.T) * _scale(d), _visible(np.arange(Lq), Lq, Lk, causal))
    return (A1 - float(lam) * noise_map(F, G, Lq, Lk, causal)) @ v


def diffattn_lowrank(q, k, v, F, G, lam, causal: bool = True) -> np.ndarray:
    """Batched layout: q [B, H, Lq, d]; k [B, Hkv, Lk, d]; v [B, Hkv, Lk, dv];
    F [H, Lq, r], G [H, Lk, r] per head; lam [H].  Head h reads KV head
    h // (H // Hkv).  Returns [B, H, Lq, dv] fp64."""
    q, k, v = (_f64(t) for t in (q, k, v))
    lam = np.asarray(_f64(lam), dtype=np.float64).reshape(-1)
    B, H, Lq, _ = q.shape
    Hkv = k.shape[1]
    if H % Hkv:
        raise ValueError("H must be a multiple of Hkv")
    grp = H // Hkv
    out = np.empty((B, H, Lq, v.shape[3]))
    for b in range(B):
        for h in range(H):
            g = h // grp
            out[b, h] = lowrank_head(q[b, h], k[b, g], v[b, g], F[h], G[h], lam[h], causal)
    return out
