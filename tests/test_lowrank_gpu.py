"""The low-rank substitute for A2 (out = A1 V - lambda N V, N fixed from
positional factors) on the GPU against the fp64 oracle.  Needs a B200.

A1 V runs on the prefill's training variant (heads in pairs over a KV head)
and N V on the scan kernels, whose host runs are checked in
tests/test_lowrank_host.py.  Tolerance: max|O - O_ref| <= 2e-2 max|O_ref| per
(batch, head) slice, the bf16 output bound of the forward."""

import math

import numpy as np
import pytest
import torch

import differential_attention_transformers_b200 as da
from oracle import lowrank as lr
from tests.test_parity_gpu import BF16_TOL, DEV

pytestmark = pytest.mark.gpu


def _case(B, H, Hkv, Lq, Lk, r, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    s = 1 / math.sqrt(128)
    mk = lambda *shape: (torch.randn(*shape, generator=g) * s).to(torch.bfloat16).to(DEV)  # noqa: E731
    q, k, v = mk(B, H, Lq, 128), mk(B, Hkv, Lk, 128), mk(B, Hkv, Lk, 128)
    F = torch.rand(H, Lq, r, generator=g).to(DEV)
    G = torch.rand(H, Lk, r, generator=g).to(DEV)
    lam = (torch.rand(H, generator=g) * 1.2 - 0.2).to(DEV)
    return q, k, v, F, G, lam


def _rel(got, ref):
    got = got.double().cpu().numpy()
    scale = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref))) / scale if scale > 0 else float(np.max(np.abs(got)))


CASES = [
    # B, H, Hkv, Lq, Lk, r, causal
    (1, 4, 2, 600, 600, 5, True),     # ragged chunks, two heads per KV head
    (2, 4, 1, 300, 700, 3, True),     # Lq < Lk: bottom-right causal offset
    (1, 2, 1, 700, 300, 1, True),     # Lq > Lk: the first rows see no key
    (1, 4, 2, 300, 600, 16, False),   # unmasked, largest rank
    (1, 2, 1, 64, 0, 2, True),        # no keys: zero output
]


@pytest.mark.parametrize("B,H,Hkv,Lq,Lk,r,causal", CASES)
def test_lowrank_matches_oracle(B, H, Hkv, Lq, Lk, r, causal):
    q, k, v, F, G, lam = _case(B, H, Hkv, Lq, Lk, r, seed=Lq + 3 * Lk + r)
    out = da.fwd_lowrank(q, k, v, F, G, lam, causal=causal)
    torch.cuda.synchronize()
    assert da.last_status() == da.OK
    ref = lr.diffattn_lowrank(q, k, v, F.cpu().numpy(), G.cpu().numpy(), lam.cpu().numpy(), causal=causal)
    assert torch.isfinite(out.float()).all()
    if Lk == 0:
        assert torch.all(out == 0)
        return
    for b in range(B):
        for h in range(H):
            assert _rel(out[b, h], ref[b, h]) <= BF16_TOL, (b, h, _rel(out[b, h], ref[b, h]))
    again = da.fwd_lowrank(q, k, v, F, G, lam, causal=causal)
    assert torch.equal(out, again)                 # no atomics: bitwise repeatable


def test_lowrank_uniform_factors_reduce_to_the_prefix_mean():
    """r = 1, F = G = 1: N is the uniform causal map, so out = A1 V - lambda *
    (prefix mean of V); with lambda = 0 the output is plain attention."""
    q, k, v, F, G, lam = _case(1, 2, 1, 333, 333, 1, seed=5)
    ones_f, ones_g = torch.ones_like(F), torch.ones_like(G)
    lam = torch.tensor([0.0, 1.0], device=DEV)
    out = da.fwd_lowrank(q, k, v, ones_f, ones_g, lam, causal=True).double().cpu().numpy()
    vd = v[0, 0].double().cpu().numpy()
    prefix_mean = np.cumsum(vd, axis=0) / np.arange(1, 334)[:, None]
    a1v = lr.diffattn_lowrank(q, k, v, ones_f.cpu().numpy(), ones_g.cpu().numpy(), np.zeros(2), causal=True)[0]
    assert np.max(np.abs(out[0, 0] - a1v[0])) <= BF16_TOL * np.max(np.abs(a1v[0]))
    want = a1v[1] - prefix_mean
    assert np.max(np.abs(out[0, 1] - want)) <= BF16_TOL * np.max(np.abs(want))


def test_lowrank_full_size_sampled():
    """B2 H32 Hkv8 N8192 r16, causal: one (batch, head) slice against the oracle."""
    B, H, Hkv, L, r = 2, 32, 8, 8192, 16
    q, k, v, F, G, lam = _case(B, H, Hkv, L, L, r, seed=8192)
    out = da.fwd_lowrank(q, k, v, F, G, lam, causal=True)
    torch.cuda.synchronize()
    assert da.last_status() == da.OK
    assert torch.isfinite(out.float()).all()
    b, h = 1, 13
    g = h // (H // Hkv)
    ref = lr.lowrank_head(q[b, h], k[b, g], v[b, g], F[h].cpu().numpy(), G[h].cpu().numpy(), float(lam[h]), True)
    assert _rel(out[b, h], ref) <= BF16_TOL
