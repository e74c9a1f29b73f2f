"""The low-rank substitute for A2 (out = A1 V - lambda N V, N fixed from
positional factors) on the GPU against the fp64 oracle.  Needs a B200.

A1 V runs on the prefill's training variant (heads in pairs over a KV head),
which rounds P to bf16 and stores A1 V in bf16; N V runs on the scan kernels
(their host runs are checked in tests/test_lowrank_host.py) in f32.

Error bound.  The output is A1 V - lambda N V, and A1 V carries two bf16
roundings (P and the stored value), each up to 2^-9 of A1 V's own scale.
When N is close to A1 and lambda close to 1, the difference is small against
A1 V and those roundings dominate it.  The bound is therefore the bf16 output
bound, 2e-2 max|O_ref|, plus four roundings of A1 V, 2^-7 max|A1 V|; an error
in the pairing, lambda, the head mapping or the workspace misses it by far.
N V itself is checked tightly: two calls that differ only in lambda (0 and 1)
share the same bf16 A1 V, so their difference is N V up to the rounding of the
lambda = 1 output."""

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


def _ratio(got, ref, a1v):
    """Error over the bound 2e-2 max|O_ref| + 2^-7 max|A1 V| (<= 1 passes)."""
    got = got.double().cpu().numpy()
    bound = BF16_TOL * float(np.max(np.abs(ref))) + 2.0 ** -7 * float(np.max(np.abs(a1v)))
    return float(np.max(np.abs(got - ref))) / bound if bound > 0 else float(np.max(np.abs(got)))


def _oracle(q, k, v, F, G, lam, causal):
    args = (q, k, v, F.cpu().numpy(), G.cpu().numpy())
    ref = lr.diffattn_lowrank(*args, lam.cpu().numpy(), causal=causal)
    a1v = lr.diffattn_lowrank(*args, np.zeros(lam.shape[0]), causal=causal)
    return ref, a1v


CASES = [
    # B, H, Hkv, Lq, Lk, r, causal
    (1, 4, 2, 600, 600, 5, True),     # ragged chunks, two heads per KV head
    (2, 4, 1, 300, 700, 3, True),     # Lq < Lk: bottom-right causal offset
    (1, 2, 1, 700, 300, 1, True),     # Lq > Lk: the first rows see no key
    (1, 4, 2, 300, 600, 16, False),   # unmasked, largest rank
    (1, 2, 1, 40, 1000, 4, True),     # decode-like: 960 leading keys every row sees
    (1, 2, 1, 64, 0, 2, True),        # no keys: zero output
]


@pytest.mark.parametrize("B,H,Hkv,Lq,Lk,r,causal", CASES)
def test_lowrank_matches_oracle(B, H, Hkv, Lq, Lk, r, causal):
    q, k, v, F, G, lam = _case(B, H, Hkv, Lq, Lk, r, seed=Lq + 3 * Lk + r)
    out = da.fwd_lowrank(q, k, v, F, G, lam, causal=causal)
    torch.cuda.synchronize()
    assert da.last_status() == da.OK
    ref, a1v = _oracle(q, k, v, F, G, lam, causal)
    assert torch.isfinite(out.float()).all()
    if Lk == 0:
        assert torch.all(out == 0)
        return
    for b in range(B):
        for h in range(H):
            assert _ratio(out[b, h], ref[b, h], a1v[b, h]) <= 1.0, (b, h, _ratio(out[b, h], ref[b, h], a1v[b, h]))
    again = da.fwd_lowrank(q, k, v, F, G, lam, causal=causal)
    assert torch.equal(out, again)                 # no atomics: bitwise repeatable


@pytest.mark.parametrize("B,H,Hkv,Lq,Lk,r,causal", [c for c in CASES if c[4] > 0])
def test_lowrank_nv_part_is_exact_to_the_output_rounding(B, H, Hkv, Lq, Lk, r, causal):
    """out(lambda=0) - out(lambda=1) = N V: the bf16 A1 V is the same in both
    calls, so the only rounding left is that of the lambda = 1 output (2^-9 of
    its value), plus the fp32 sums over keys (2^-14 of N |V|).  One key too
    many or too few in N V misses this bound."""
    q, k, v, F, G, _ = _case(B, H, Hkv, Lq, Lk, r, seed=Lq + 3 * Lk + r + 1)
    out0 = da.fwd_lowrank(q, k, v, F, G, torch.zeros(H, device=DEV), causal=causal).double().cpu().numpy()
    out1 = da.fwd_lowrank(q, k, v, F, G, torch.ones(H, device=DEV), causal=causal).double().cpu().numpy()
    grp = H // Hkv
    vd = v.double().cpu().numpy()
    for b in range(B):
        for h in range(H):
            N = lr.noise_map(F[h].double().cpu().numpy(), G[h].double().cpu().numpy(), Lq, Lk, causal)
            nv, na = N @ vd[b, h // grp], N @ np.abs(vd[b, h // grp])
            err = np.abs((out0[b, h] - out1[b, h]) - nv)
            assert np.all(err <= 2.0 ** -8 * np.abs(out1[b, h]) + 2.0 ** -14 * na), (b, h, float(np.max(err)))


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
    # lambda = 1 cancels the mean part: the bound is relative to A1 V (see the module notes)
    want = a1v[1] - prefix_mean
    assert np.max(np.abs(out[0, 1] - want)) <= BF16_TOL * np.max(np.abs(want)) + 2.0 ** -7 * np.max(np.abs(a1v[1]))


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
    args = (q[b, h], k[b, g], v[b, g], F[h].cpu().numpy(), G[h].cpu().numpy())
    ref = lr.lowrank_head(*args, float(lam[h]), True)
    a1v = lr.lowrank_head(*args, 0.0, True)
    assert _ratio(out[b, h], ref, a1v) <= 1.0
