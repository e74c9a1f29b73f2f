"""Definition-level fp64 oracle of the differential attention forward.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): nothing on the product
path imports this module.

What it computes, with the passage each step follows:

  lambda_init(l) = 0.8 - 0.6 * exp(-0.3 * (l - 1))
      "Differential Transformer：用“差分降噪”重塑LLM注意力机制", section 3
      (工程实践), the progressive lambda initialisation.  ``layer`` is 1-based,
      so layer 1 gives 0.2.

  lambda = exp(lq1 . lk1) - exp(lq2 . lk2) + lambda_init
      "差分注意力" tutorial, section 差分思路 (last sentence) and Step 4
      (λ 参数化).  Computed in fp64 and rounded once to fp32.

  A1 = softmax(Q1 K1^T / sqrt(d)),  A2 = softmax(Q2 K2^T / sqrt(d))
  O  = (A1 - lambda * A2) V
      "差分注意力" tutorial, section 差分思路 (the two maps and their
      difference) and Step 2 (差分注意力); the paper note "Understanding
      Differential Transformer Unchains Pretrained Self-Attentions", section
      关键设计, writes the same difference A_diff = A1 - lambda*A2.
      d is the contraction width of Q1 K1^T (the half-head width in the V1
      layout, the head width in the V2 layout).

  V1 layout: separate half-width Q1,K1,Q2,K2 per head, one V, optional per-head
  RMSNorm of the difference output; V2 layout: Q heads (2h, 2h+1) are the two
  maps of pair h, both maps share the pair's K and V head, no norm.
      "差分注意力" tutorial, section V1 到 V2 的 diff.

Readings where the pages are silent:
  * causal mask, bottom-right aligned: query row i sees key j iff
    j <= i + (Lk - Lq).  Lq == Lk gives j <= i; Lq == 1 sees every key.
  * a row that sees no key at all (only possible when Lq > Lk under the causal
    mask, or Lk == 0) has A1 = A2 = 0, hence O = 0.
  * RMSNorm: y = x / sqrt(mean(x^2) + eps) over the value width, unit weight.
  * GQA head mapping: V1 head h reads KV head h // (H // Hkv); V2 pair h reads
    KV head (2h) // (Hq // Hkv).

Arithmetic: everything in fp64 (inputs are upcast), softmax with max
subtraction, one library matmul per product.  Rows are processed in chunks of
``ROW_CHUNK`` to bound memory; the chunking does not change what is computed.
"""

from __future__ import annotations

import math

import numpy as np

ROW_CHUNK = 512


# ----------------------------------------------------------------------------
# lambda
# ----------------------------------------------------------------------------
def lambda_init(layer: int) -> float:
    """0.8 - 0.6 * exp(-0.3 * (layer - 1)), layer counted from 1.

    Differential Transformer (mcipr.com) section 3 工程实践.
    """
    if layer < 1:
        raise ValueError("layer is 1-based")
    return 0.8 - 0.6 * math.exp(-0.3 * (layer - 1))


def lambda_(lq1, lk1, lq2, lk2, lam_init: float) -> np.ndarray:
    """Per-head lambda, fp64 arithmetic, rounded once to fp32.

    lq1, lk1, lq2, lk2: arrays [H, dl].  Each dot product is a sequential fp64
    sum in index order; exp is the libm exponential.  "差分注意力" tutorial,
    Step 4 (λ 参数化) and section 差分思路.
    """
    lq1 = np.asarray(lq1, dtype=np.float64)
    lk1 = np.asarray(lk1, dtype=np.float64)
    lq2 = np.asarray(lq2, dtype=np.float64)
    lk2 = np.asarray(lk2, dtype=np.float64)
    H = lq1.shape[0]
    out = np.empty(H, dtype=np.float32)
    for h in range(H):
        d1 = 0.0
        for a, b in zip(lq1[h].tolist(), lk1[h].tolist()):
            d1 += a * b
        d2 = 0.0
        for a, b in zip(lq2[h].tolist(), lk2[h].tolist()):
            d2 += a * b
        out[h] = np.float32(math.exp(d1) - math.exp(d2) + lam_init)
    return out


# ----------------------------------------------------------------------------
# attention maps
# ----------------------------------------------------------------------------
def _scale(d: int) -> float:
    """Score scale 1/sqrt(d) ("差分注意力" tutorial, section 差分思路)."""
    return 1.0 / math.sqrt(d)


def _visible(rows: np.ndarray, Lq: int, Lk: int, causal: bool) -> np.ndarray:
    """Boolean [len(rows), Lk]: may query row i see key j.

    Bottom-right aligned causal mask: j <= i + (Lk - Lq).
    """
    cols = np.arange(Lk)[None, :]
    if not causal:
        return np.ones((rows.shape[0], Lk), dtype=bool)
    return cols <= (rows[:, None] + (Lk - Lq))


def _softmax_masked(S: np.ndarray, visible: np.ndarray) -> np.ndarray:
    """Row softmax over the visible entries, exact zeros elsewhere.

    A row with no visible entry is all zeros.
    """
    if S.shape[-1] == 0:
        return np.zeros_like(S)
    S = np.where(visible, S, -np.inf)
    m = S.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    E = np.where(visible, np.exp(S - m), 0.0)
    z = E.sum(axis=-1, keepdims=True)
    return np.divide(E, z, out=np.zeros_like(E), where=z > 0)


def maps(q1, k1, q2, k2, causal: bool, row0: int = 0, Lq: int | None = None):
    """A1 and A2 for one head: q* [n, d] (rows row0.. of a Lq-row query), k* [Lk, d]."""
    q1 = np.asarray(q1, dtype=np.float64)
    q2 = np.asarray(q2, dtype=np.float64)
    k1 = np.asarray(k1, dtype=np.float64)
    k2 = np.asarray(k2, dtype=np.float64)
    n, d = q1.shape
    Lk = k1.shape[0]
    if Lq is None:
        Lq = n
    rows = np.arange(row0, row0 + n)
    vis = _visible(rows, Lq, Lk, causal)
    s = _scale(d)
    A1 = _softmax_masked((q1 @ k1.T) * s, vis)
    A2 = _softmax_masked((q2 @ k2.T) * s, vis)
    return A1, A2


def rmsnorm(x: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) over the last axis, unit weight."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps)


def diff_head(q1, k1, q2, k2, v, lam: float, causal: bool,
              rms: bool = False, eps: float = 1e-5) -> np.ndarray:
    """O = (A1 - lam*A2) V for one head, optional RMSNorm. Returns [Lq, dv] fp64."""
    q1 = np.asarray(q1, dtype=np.float64)
    Lq = q1.shape[0]
    v = np.asarray(v, dtype=np.float64)
    out = np.empty((Lq, v.shape[1]), dtype=np.float64)
    lam = float(lam)
    for r0 in range(0, Lq, ROW_CHUNK):
        r1 = min(Lq, r0 + ROW_CHUNK)
        A1, A2 = maps(q1[r0:r1], k1, np.asarray(q2)[r0:r1], k2, causal, r0, Lq)
        o = (A1 - lam * A2) @ v
        out[r0:r1] = rmsnorm(o, eps) if rms else o
    return out


# ----------------------------------------------------------------------------
# layouts
# ----------------------------------------------------------------------------
def _f64(x):
    if hasattr(x, "detach"):  # torch tensor (possibly bf16)
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def diffattn_v1(q1, k1, q2, k2, v, lam, causal=True, rms=False, eps=1e-5,
                heads=None, batches=None) -> np.ndarray:
    """V1 layout.  q1,q2 [B,H,Lq,d]; k1,k2 [B,Hkv,Lk,d]; v [B,Hkv,Lk,dv]; lam [H].

    Head h reads KV head h // (H // Hkv).  Returns [B,H,Lq,dv] fp64, or only
    the (b, h) slices requested by ``batches`` x ``heads`` (others left NaN).
    """
    q1, k1, q2, k2, v = (_f64(t) for t in (q1, k1, q2, k2, v))
    lam = np.asarray(_f64(lam), dtype=np.float64).reshape(-1)
    B, H, Lq, d = q1.shape
    Hkv = k1.shape[1]
    if H % Hkv:
        raise ValueError("H must be a multiple of Hkv")
    grp = H // Hkv
    out = np.full((B, H, Lq, v.shape[3]), np.nan)
    for b in (range(B) if batches is None else batches):
        for h in (range(H) if heads is None else heads):
            g = h // grp
            out[b, h] = diff_head(q1[b, h], k1[b, g], q2[b, h], k2[b, g], v[b, g],
                                  lam[h], causal, rms, eps)
    return out


def diffattn_v2(q, k, v, lam, causal=True, pairs=None, batches=None) -> np.ndarray:
    """V2 layout.  q [B,Hq,Lq,D]; k,v [B,Hkv,Lk,D]; lam [Hq/2].

    Pair h uses Q heads 2h (map 1) and 2h+1 (map 2), both against KV head
    (2h) // (Hq // Hkv).  Returns [B,Hq/2,Lq,D] fp64 (unrequested slices NaN).
    """
    q, k, v = (_f64(t) for t in (q, k, v))
    lam = np.asarray(_f64(lam), dtype=np.float64).reshape(-1)
    B, Hq, Lq, D = q.shape
    Hkv = k.shape[1]
    if Hq % 2 or Hq % Hkv or (Hq // Hkv) % 2:
        raise ValueError("Hq must be even and each KV group must hold whole pairs")
    grp = Hq // Hkv
    Hp = Hq // 2
    out = np.full((B, Hp, Lq, v.shape[3]), np.nan)
    for b in (range(B) if batches is None else batches):
        for h in (range(Hp) if pairs is None else pairs):
            h1, h2 = _pair_heads(h)
            g = h1 // grp
            out[b, h] = diff_head(q[b, h1], k[b, g], q[b, h2], k[b, g], v[b, g],
                                  lam[h], causal)
    return out


def _pair_heads(h: int):
    """Q heads of diff pair h in the V2 layout: (2h, 2h+1) = (map 1, map 2)."""
    return 2 * h, 2 * h + 1


def decode_v2(q, kc, vc, lam, batches=None, pairs=None) -> np.ndarray:
    """Single-token V2 decode: q [B,Hq,D] against the whole cache kc,vc [B,Hkv,T,D].

    A one-row query under the bottom-right causal mask sees every cached key,
    so this is ``diffattn_v2`` with Lq = 1.  Returns [B,Hq/2,D] fp64.
    """
    q = _f64(q)
    out = diffattn_v2(q[:, :, None, :], kc, vc, lam, causal=True, pairs=pairs, batches=batches)
    return out[:, :, 0, :]


def gather_pages(pages, table_row, n: int) -> np.ndarray:
    """The first ``n`` cached tokens of one sequence, read from a page pool.

    pages [num_pages, page_size, Hkv, D] (token-major pages: each page holds
    page_size consecutive tokens, every KV head of a token side by side);
    table_row lists the sequence's page ids in token order.  Returns
    [Hkv, n, D] fp64.
    """
    pages = _f64(pages)
    ps = pages.shape[1]
    npg = -(-n // ps)
    if npg == 0:
        return np.zeros((pages.shape[2], 0, pages.shape[3]))
    toks = np.concatenate([pages[int(p)] for p in np.asarray(table_row)[:npg]], axis=0)[:n]
    return np.transpose(toks, (1, 0, 2))


def decode_v2_paged(q, k_pages, v_pages, block_table, seq_lens, lam) -> np.ndarray:
    """Single-token V2 decode of B sequences whose K/V caches live in a shared
    pool of fixed-size pages, each sequence with its own length.

    Serving layout (the tutorial's V1 到 V2 的 diff section names the
    vLLM/SGLang integration; the pages give no layout, so this follows the
    common token-major page pool): k_pages, v_pages [num_pages, page_size,
    Hkv, D]; block_table [B, max_pages] page ids; seq_lens [B].  Sequence b is
    its first seq_lens[b] tokens in page order, and its output is
    ``decode_v2`` against exactly that cache (a length of 0 gives zeros).
    Returns [B, Hq/2, D] fp64.
    """
    q = _f64(q)
    bt = np.asarray(block_table.cpu() if hasattr(block_table, "cpu") else block_table)
    sl = np.asarray(seq_lens.cpu() if hasattr(seq_lens, "cpu") else seq_lens)
    B, Hq, D = q.shape
    out = np.zeros((B, Hq // 2, D))
    for b in range(B):
        n = max(0, int(sl[b]))
        if n == 0:
            continue
        kc = gather_pages(k_pages, bt[b], n)[None]
        vc = gather_pages(v_pages, bt[b], n)[None]
        out[b] = decode_v2(q[b:b + 1], kc, vc, lam)[0]
    return out


def decode_v1(q1, k1, q2, k2, v, lam, batches=None, heads=None) -> np.ndarray:
    """Single-token V1-layout decode: q1,q2 [B,H,d]; k1,k2 [B,Hkv,T,d]; v [B,Hkv,T,dv]."""
    q1, q2 = _f64(q1), _f64(q2)
    out = diffattn_v1(q1[:, :, None, :], k1, q2[:, :, None, :], k2, v, lam, causal=True,
                      heads=heads, batches=batches)
    return out[:, :, 0, :]


# ----------------------------------------------------------------------------
# noise-floor probe ("差分注意力" tutorial, Step 1 and Step 3)
# ----------------------------------------------------------------------------
def noise_probe(q1, k1, q2, k2, lam: float):
    """Per-instance signal/noise report of the tutorial's toy construction.

    q1 [n, d] queries, k1 [n, N, d] keys with key 0 the strong match, q2/k2 the
    independent second map.  For each instance: the plain-softmax row A1, the
    difference row A1 - lam*A2, and SNR = weight at position 0 / mean weight
    over positions 1..N-1 (Step 3).  Returns a dict of arrays.

    Parity unpinned: the tutorial's claimed noise fractions (about 8 % at 1k
    keys rising past 30 % at 100k) and its claim that the difference SNR is
    much higher than the plain one are not reproduced by the literal
    construction at d = 64; these values are reported only.
    The row-sum identity and positivity below are pinned.
    """
    q1, k1, q2, k2 = (_f64(t) for t in (q1, k1, q2, k2))
    n = q1.shape[0]
    plain, diff = [], []
    for i in range(n):
        A1, A2 = maps(q1[i:i + 1], k1[i], q2[i:i + 1], k2[i], causal=False)
        plain.append(A1[0])
        diff.append(A1[0] - lam * A2[0])
    plain = np.stack(plain)
    diff = np.stack(diff)
    snr_plain = plain[:, 0] / plain[:, 1:].mean(axis=1)
    snr_diff = diff[:, 0] / diff[:, 1:].mean(axis=1)
    return {
        "plain": plain,
        "diff": diff,
        "noise_fraction_plain": plain[:, 1:].sum(axis=1),
        "snr_plain": snr_plain,
        "snr_diff": snr_diff,
    }
