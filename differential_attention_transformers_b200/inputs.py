"""Seeded synthetic inputs for the differential attention workloads.

This module only draws random numbers and arranges them in the layouts the
library takes; it holds none of the method's arithmetic.  Both the CUDA path
(tests, bench) and the fp64 oracle consume what it returns.

Workloads (shapes, value distributions):

  v1_tiny      V1 layout, fp32: B1 H1 Lq=Lk=128 d32 dv64, causal, all N(0,1),
               lambda from lq/lk in R^32 ~ N(0, 0.1) at layer 1.
  noise_probe  fp32, 64 independent instances of the tutorial's toy
               construction ("差分注意力", Step 1 / Step 3): q ~ N(0,1) in d=64,
               1000 keys ~ N(0,1) with key 0 = 5q, an independent second map
               (Q2, K2 ~ N(0,1)), V = the 1000x1000 identity, lambda = 0.5.
               Laid out as V1 with B=64, H=1, Lq=1, Lk=1000, non-causal.
  v1_prefill   V1, bf16: B8 H16 (Hkv16) N4096 d64 dv128, causal,
               N(0,1)/sqrt(64), layer 12, RMSNorm eps 1e-5.
  v2_prefill   V2, bf16: B2 Hq64 Hkv8 N8192 D128, causal, N(0,1)/sqrt(128),
               layer 24.
  v2_decode    V2 single-token decode, bf16: B16 Hq64 Hkv8 T65536 D128,
               N(0,1)/sqrt(128), layer 24.
  v1_decode    the same decode shape in the V1 layout: 32 heads over 8 KV
               heads, Q1/Q2/K1/K2 width 64, V width 128.
  lowrank      (lowrank_inputs) the fixed low-rank substitute for A2 on the
               V2 prefill's attention shape with one Q head per output head:
               B2 H32 Hkv8 N8192 D128 causal, N(0,1)/sqrt(128); positional
               factors F [H, N, r], G [H, N, r] ~ U(0, 1), r = 16.
  serving      (serving_cache) a serving-shaped paged V2 decode: 256
               sequences with lengths drawn uniformly from 16..4096 tokens,
               one query token each (Hq64 Hkv8 D128), their K/V in a shared,
               shuffled pool of 16-token pages; N(0,1)/sqrt(128), layer 24.
  noise sweep  (noise_sweep / sweep_prefix) the noise_probe construction at
               context lengths 1k..256k keys (tutorial exercise 1), in bf16 for
               the V1 decode layout: 64 instances, each a query q ~ N(0,1) in
               d=64 with key 0 = 5q among N(0,1) keys and an independent second
               map; shorter contexts are prefixes of the longest one.  V has
               width 128: column 0 is 1 at key 0, column 1 is 1 at keys 1..N-1,
               the rest 0, so the output holds the row's weight on the signal
               key and its total weight on the noise keys.

bf16 tensors are drawn in fp32 and rounded to bf16 (round-to-nearest-even);
the oracle receives those rounded values.  lq/lk are fp32 N(0,1)*0.1 with the
QK width as their length.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    layout: str            # "v1" | "v2" | "v1_decode" | "v2_decode"
    dtype: torch.dtype
    B: int
    H: int                 # V1: heads; V2: Q heads (pairs = H // 2)
    Hkv: int
    Lq: int
    Lk: int
    d: int                 # QK contraction width
    dv: int                # value width
    causal: bool
    layer: int             # lambda_init layer (1-based); 0 = explicit lambda
    rmsnorm: bool
    std: float
    seed: int
    explicit_lambda: float | None = None

    @property
    def pairs(self) -> int:
        return self.H // 2 if self.layout.startswith("v2") else self.H


WORKLOADS = {
    "v1_tiny": Workload("v1_tiny", "v1", torch.float32, 1, 1, 1, 128, 128, 32, 64,
                        True, 1, False, 1.0, 1001),
    "noise_probe": Workload("noise_probe", "v1", torch.float32, 64, 1, 1, 1, 1000, 64, 1000,
                            False, 0, False, 1.0, 1002, explicit_lambda=0.5),
    "v1_prefill": Workload("v1_prefill", "v1", torch.bfloat16, 8, 16, 16, 4096, 4096, 64, 128,
                           True, 12, True, 1.0 / math.sqrt(64), 1003),
    "v2_prefill": Workload("v2_prefill", "v2", torch.bfloat16, 2, 64, 8, 8192, 8192, 128, 128,
                           True, 24, False, 1.0 / math.sqrt(128), 1004),
    "v2_decode": Workload("v2_decode", "v2_decode", torch.bfloat16, 16, 64, 8, 1, 65536, 128, 128,
                          True, 24, False, 1.0 / math.sqrt(128), 1005),
    "v1_decode": Workload("v1_decode", "v1_decode", torch.bfloat16, 16, 32, 8, 1, 65536, 64, 128,
                          True, 24, False, 1.0 / math.sqrt(64), 1006),
}


def with_shape(w: Workload, **kw) -> Workload:
    """A copy of ``w`` with some fields replaced (smaller parity cases)."""
    d = dict(w.__dict__)
    d.update(kw)
    return Workload(**d)


def _randn(gen, shape, std, dtype, device):
    x = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def lambda_params(w: Workload, device="cpu", seed_offset: int = 0):
    """lq1, lk1, lq2, lk2 [pairs, d] fp32 ~ N(0, 0.1)."""
    gen = torch.Generator(device=device).manual_seed(w.seed * 7 + 13 + seed_offset)
    return tuple(_randn(gen, (w.pairs, w.d), 0.1, torch.float32, device) for _ in range(4))


def make(w: Workload, device="cpu"):
    """Draw the attention inputs of workload ``w`` on ``device``.

    Returns a dict.  V1: q1, k1, q2, k2, v.  V2: q, k, v.  Decode layouts drop
    the query length axis (q [B, H, d]).
    """
    gen = torch.Generator(device=device).manual_seed(w.seed)
    dt, std = w.dtype, w.std
    if w.name == "noise_probe":
        n, N, d = w.B, w.Lk, w.d
        q1 = _randn(gen, (n, 1, 1, d), 1.0, torch.float32, device)
        k1 = _randn(gen, (n, 1, N, d), 1.0, torch.float32, device)
        k1[:, 0, 0, :] = 5.0 * q1[:, 0, 0, :]
        q2 = _randn(gen, (n, 1, 1, d), 1.0, torch.float32, device)
        k2 = _randn(gen, (n, 1, N, d), 1.0, torch.float32, device)
        v = torch.eye(N, dtype=torch.float32, device=device).expand(n, 1, N, N).contiguous()
        return {"q1": q1, "k1": k1, "q2": q2, "k2": k2, "v": v}
    if w.layout == "v1":
        return {
            "q1": _randn(gen, (w.B, w.H, w.Lq, w.d), std, dt, device),
            "k1": _randn(gen, (w.B, w.Hkv, w.Lk, w.d), std, dt, device),
            "q2": _randn(gen, (w.B, w.H, w.Lq, w.d), std, dt, device),
            "k2": _randn(gen, (w.B, w.Hkv, w.Lk, w.d), std, dt, device),
            "v": _randn(gen, (w.B, w.Hkv, w.Lk, w.dv), std, dt, device),
        }
    if w.layout == "v2":
        return {
            "q": _randn(gen, (w.B, w.H, w.Lq, w.d), std, dt, device),
            "k": _randn(gen, (w.B, w.Hkv, w.Lk, w.d), std, dt, device),
            "v": _randn(gen, (w.B, w.Hkv, w.Lk, w.dv), std, dt, device),
        }
    if w.layout == "v2_decode":
        return {
            "q": _randn(gen, (w.B, w.H, w.d), std, dt, device),
            "k": _randn(gen, (w.B, w.Hkv, w.Lk, w.d), std, dt, device),
            "v": _randn(gen, (w.B, w.Hkv, w.Lk, w.dv), std, dt, device),
        }
    if w.layout == "v1_decode":
        return {
            "q1": _randn(gen, (w.B, w.H, w.d), std, dt, device),
            "k1": _randn(gen, (w.B, w.Hkv, w.Lk, w.d), std, dt, device),
            "q2": _randn(gen, (w.B, w.H, w.d), std, dt, device),
            "k2": _randn(gen, (w.B, w.Hkv, w.Lk, w.d), std, dt, device),
            "v": _randn(gen, (w.B, w.Hkv, w.Lk, w.dv), std, dt, device),
        }
    raise ValueError(w.layout)


def paged_cache(kc, vc, page_size: int, seed: int, spare_pages: int = 3, lens=None):
    """Scatter contiguous caches kc, vc [B, Hkv, T, D] into a shuffled pool of
    token-major pages [num_pages, page_size, Hkv, D] (the serving layout).

    Sequence b keeps its first lens[b] tokens (default: all T) in
    ceil(lens[b] / page_size) pages drawn at random from the pool; spare pages
    and the unused rows of each sequence's last page hold NaN, so a reader that
    touches anything outside a sequence shows it.  Returns (k_pages, v_pages,
    block_table [B, max_pages] int32, seq_lens [B] int32) on kc's device.
    Pure data movement: no arithmetic of the method.
    """
    B, Hkv, T, D = kc.shape
    lens = [T] * B if lens is None else [int(x) for x in lens]
    need = [-(-n // page_size) for n in lens]
    max_pages = max(1, -(-T // page_size))
    num_pages = sum(need) + spare_pages
    gen = torch.Generator(device="cpu").manual_seed(seed)
    perm = torch.randperm(num_pages, generator=gen).tolist()
    kp = torch.full((num_pages, page_size, Hkv, D), float("nan"), dtype=kc.dtype, device=kc.device)
    vp = torch.full_like(kp, float("nan"))
    if all(n == T for n in lens) and T % page_size == 0:
        # every sequence full and page-aligned: one scatter of all pages at once
        npg = T // page_size
        ids = torch.tensor(perm[: B * npg], dtype=torch.long, device=kc.device)
        for src, dst in ((kc, kp), (vc, vp)):
            dst[ids] = src.reshape(B, Hkv, npg, page_size, D).permute(0, 2, 3, 1, 4).reshape(B * npg, page_size, Hkv, D)
        table = torch.tensor(perm[: B * npg], dtype=torch.int32).reshape(B, npg)
        return kp, vp, table.to(kc.device), torch.tensor(lens, dtype=torch.int32, device=kc.device)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    nxt = 0
    for b in range(B):
        for i in range(need[b]):
            pid = perm[nxt]
            nxt += 1
            table[b, i] = pid
            t0, t1 = i * page_size, min((i + 1) * page_size, lens[b])
            kp[pid, : t1 - t0] = kc[b, :, t0:t1].transpose(0, 1)
            vp[pid, : t1 - t0] = vc[b, :, t0:t1].transpose(0, 1)
    return kp, vp, table.to(kc.device), torch.tensor(lens, dtype=torch.int32, device=kc.device)



SWEEP_LENGTHS = tuple(1024 << i for i in range(9))    # 1k, 2k, ..., 256k keys
SWEEP_INSTANCES = 64


def noise_sweep(n: int = SWEEP_INSTANCES, N: int = SWEEP_LENGTHS[-1], seed: int = 1010, device="cpu"):
    """The noise-floor construction over N keys for n instances, bf16, V1
    decode layout: q1, q2 [n, 1, 64]; k1, k2 [n, 1, N, 64]; v [n, 1, N, 128]
    (indicator columns, see the module notes).  Key 0 of k1 is 5 q1, formed in
    fp32 before the rounding to bf16."""
    gen = torch.Generator(device=device).manual_seed(seed)
    d = 64
    q1 = _randn(gen, (n, 1, d), 1.0, torch.float32, device)
    k1 = _randn(gen, (n, 1, N, d), 1.0, torch.float32, device)
    k1[:, 0, 0, :] = 5.0 * q1[:, 0, :]
    q2 = _randn(gen, (n, 1, d), 1.0, torch.float32, device)
    k2 = _randn(gen, (n, 1, N, d), 1.0, torch.float32, device)
    v = torch.zeros((n, 1, N, 128), dtype=torch.bfloat16, device=device)
    v[:, 0, 0, 0] = 1.0
    v[:, 0, 1:, 1] = 1.0
    bf = torch.bfloat16
    return {"q1": q1.to(bf), "k1": k1.to(bf), "q2": q2.to(bf), "k2": k2.to(bf), "v": v}


def sweep_prefix(x, N: int):
    """The same instances over their first N keys (contiguous copies)."""
    out = {"q1": x["q1"], "q2": x["q2"]}
    for name in ("k1", "k2", "v"):
        out[name] = x[name][:, :, :N].contiguous()
    return out


LOWRANK_SHAPE = dict(B=2, H=32, Hkv=8, L=8192, r=16)


def lowrank_inputs(B=2, H=32, Hkv=8, L=8192, r=16, seed=1011, device="cpu"):
    """q [B, H, L, 128], k, v [B, Hkv, L, 128] bf16 ~ N(0,1)/sqrt(128); F, G
    [H, L, r] fp32 ~ U(0, 1)."""
    gen = torch.Generator(device=device).manual_seed(seed)
    s = 1.0 / math.sqrt(128)
    q = _randn(gen, (B, H, L, 128), s, torch.bfloat16, device)
    k = _randn(gen, (B, Hkv, L, 128), s, torch.bfloat16, device)
    v = _randn(gen, (B, Hkv, L, 128), s, torch.bfloat16, device)
    F = torch.rand((H, L, r), generator=gen, device=device, dtype=torch.float32)
    G = torch.rand((H, L, r), generator=gen, device=device, dtype=torch.float32)
    return {"q": q, "k": k, "v": v, "F": F, "G": G}


SERVING_SHAPE = dict(B=256, Hq=64, Hkv=8, min_len=16, max_len=4096, page_size=16)


def serving_cache(B=256, Hq=64, Hkv=8, min_len=16, max_len=4096, page_size=16, seed=1013, device="cpu"):
    """A serving-shaped paged decode batch: B sequences with lengths drawn
    uniformly from [min_len, max_len], each holding ceil(len / page_size)
    pages drawn at random from one pool [num_pages, page_size, Hkv, 128]
    (three spare pages).  Values ~ N(0,1)/sqrt(128) bf16; the rows of a
    sequence's last page past its length and the spare pages hold NaN, so a
    reader that touches them shows it.  Returns q [B, Hq, 128], k_pages,
    v_pages, block_table [B, ceil(max_len / page_size)] int32 (-1 past a
    sequence's pages) and seq_lens [B] int32, on ``device``."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    lens = torch.randint(min_len, max_len + 1, (B,), generator=gen)
    need = (lens + page_size - 1) // page_size
    num_pages = int(need.sum()) + 3
    perm = torch.randperm(num_pages, generator=gen)
    max_pages = -(-max_len // page_size)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        n = int(need[b])
        table[b, :n] = perm[off:off + n].to(torch.int32)
        off += n
    dgen = torch.Generator(device=device).manual_seed(seed + 1)
    s = 1.0 / math.sqrt(128)
    q = _randn(dgen, (B, Hq, 128), s, torch.bfloat16, device)
    kp = _randn(dgen, (num_pages, page_size, Hkv, 128), s, torch.bfloat16, device)
    vp = _randn(dgen, (num_pages, page_size, Hkv, 128), s, torch.bfloat16, device)
    for b in range(B):
        n = int(need[b])
        used = int(lens[b]) - (n - 1) * page_size
        if used < page_size:
            last = int(table[b, n - 1])
            kp[last, used:] = float("nan")
            vp[last, used:] = float("nan")
    spare = perm[off:].to(device)
    kp[spare] = float("nan")
    vp[spare] = float("nan")
    return {"q": q, "k_pages": kp, "v_pages": vp, "block_table": table.to(device),
            "seq_lens": lens.to(torch.int32).to(device)}
