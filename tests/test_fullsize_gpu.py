"""Full-size workloads, in the launch configuration the bench times, against the
fp64 oracle on sampled (batch, head) slices over every query row (prefill) or
on every head (decode).  Needs a B200."""

import math

import numpy as np
import pytest
import torch

import differential_attention_transformers_b200 as da
from differential_attention_transformers_b200 import inputs
from oracle import diffattn as orc
from tests.test_parity_gpu import BF16_TOL, DEV, PREFILL_RESID_TAU, lam_gpu_and_ref, rel_err

pytestmark = pytest.mark.gpu


def _sample(n, k, seed, must):
    rng = np.random.default_rng(seed)
    picks = set(int(i) for i in rng.choice(n, size=k, replace=False))
    picks.update(must)
    return sorted(picks)


@pytest.fixture(scope="module")
def v2_prefill():
    w = inputs.WORKLOADS["v2_prefill"]
    x = inputs.make(w, device=DEV)
    lam, lref = lam_gpu_and_ref(w)
    out = da.fwd_v2(x["q"], x["k"], x["v"], lam, causal=True)
    torch.cuda.synchronize()
    return w, x, lref, out


def test_v2_prefill_full_sampled(v2_prefill):
    w, x, lref, out = v2_prefill
    grp = w.H // w.Hkv
    for b, h in [(0, 0), (w.B - 1, w.pairs - 1), (1, 13)]:
        g = (2 * h) // grp
        ref = orc.diffattn_v2(x["q"][b:b + 1, 2 * h:2 * h + 2].cpu(), x["k"][b:b + 1, g:g + 1].cpu(),
                              x["v"][b:b + 1, g:g + 1].cpu(), lref[h:h + 1], causal=True)
        assert rel_err(out[b:b + 1, h:h + 1], ref) <= BF16_TOL, (b, h)


def test_v2_prefill_full_properties(v2_prefill):
    w, x, lref, out = v2_prefill
    assert torch.isfinite(out.float()).all()
    # first row sees only key 0: O = (1 - lambda) v[0] exactly up to bf16 rounding
    grp = w.H // w.Hkv
    for h in (0, 7, 31):
        g = (2 * h) // grp
        row0 = out[:, h, 0].float().cpu()
        ref = (1 - lref[h]) * x["v"][:, g, 0].float().cpu()
        assert torch.max(torch.abs(row0 - ref)) <= 1e-2 * torch.max(torch.abs(ref)) + 1e-6


@pytest.fixture(scope="module")
def v1_prefill():
    w = inputs.WORKLOADS["v1_prefill"]
    x = inputs.make(w, device=DEV)
    lam, lref = lam_gpu_and_ref(w)
    out = da.fwd_v1(x["q1"], x["k1"], x["q2"], x["k2"], x["v"], lam, causal=True, rmsnorm=True, eps=1e-5)
    torch.cuda.synchronize()
    return w, x, lref, out


def test_v1_prefill_full_sampled(v1_prefill):
    w, x, lref, out = v1_prefill
    for b, h in [(0, 0), (w.B - 1, w.H - 1), (3, 9)]:
        sl = lambda t: t[b:b + 1, h:h + 1].cpu()  # noqa: E731  (MHA: Hkv == H)
        ref = orc.diffattn_v1(sl(x["q1"]), sl(x["k1"]), sl(x["q2"]), sl(x["k2"]), sl(x["v"]), lref[h:h + 1],
                              causal=True, rms=True, eps=1e-5)
        assert rel_err(out[b:b + 1, h:h + 1], ref) <= BF16_TOL, (b, h)
    # RMSNorm: every row's mean square is ms/(ms+eps) <= 1 (bf16 output rounding aside)
    msq = (out.float() ** 2).mean(dim=-1)
    assert torch.all(msq <= 1.0 + 2e-2)


def test_v2_decode_full_all_heads():
    w = inputs.WORKLOADS["v2_decode"]
    x = inputs.make(w, device=DEV)
    lam, lref = lam_gpu_and_ref(w)
    out = da.decode_v2(x["q"], x["k"], x["v"], lam).float().cpu().numpy()
    grp = w.H // w.Hkv
    for b in range(w.B):
        for g in range(w.Hkv):
            pairs = list(range(g * grp // 2, (g + 1) * grp // 2))
            ref = orc.decode_v2(x["q"][b:b + 1, g * grp:(g + 1) * grp].cpu(), x["k"][b:b + 1, g:g + 1].cpu(),
                                x["v"][b:b + 1, g:g + 1].cpu(), lref[pairs])
            for i, h in enumerate(pairs):   # tolerance per output head
                err = float(np.max(np.abs(out[b, h] - ref[0, i])))
                assert err <= BF16_TOL * float(np.max(np.abs(ref[0, i]))), (b, h, err)


def test_v1_decode_full_sampled():
    w = inputs.WORKLOADS["v1_decode"]
    x = inputs.make(w, device=DEV)
    lam, lref = lam_gpu_and_ref(w)
    grp = w.H // w.Hkv
    for fused in (True, False):
        out = da.decode_v1(x["q1"], x["k1"], x["q2"], x["k2"], x["v"], lam, fused=fused).float().cpu().numpy()
        for b in (0, w.B - 1):
            for g in (0, w.Hkv - 1):
                hs = list(range(g * grp, (g + 1) * grp))
                sl = lambda t: t[b:b + 1, g:g + 1].cpu()  # noqa: E731
                ref = orc.decode_v1(x["q1"][b:b + 1, hs].cpu(), sl(x["k1"]), x["q2"][b:b + 1, hs].cpu(),
                                    sl(x["k2"]), sl(x["v"]), lref[hs])
                assert np.max(np.abs(out[b:b + 1, hs] - ref)) <= BF16_TOL * np.max(np.abs(ref)), (fused, b, g)


def _hardest_heads(lref, tau=PREFILL_RESID_TAU):
    """The head nearest lambda = 1 (residual path, largest amplification) and the
    non-residual head nearest the threshold (bf16-only path, largest amplification)."""
    d = np.abs(1.0 - lref.astype(np.float64))
    with_resid = int(np.argmin(d))
    outside = np.where(d >= tau)[0]
    without = int(outside[np.argmin(d[outside])]) if outside.size else None
    return with_resid, without


def test_v2_prefill_precision_policy_extremes(v2_prefill):
    w, x, lref, out = v2_prefill
    grp = w.H // w.Hkv
    for h in _hardest_heads(lref):
        if h is None:
            continue
        g = (2 * h) // grp
        for b in range(w.B):
            ref = orc.diffattn_v2(x["q"][b:b + 1, 2 * h:2 * h + 2].cpu(), x["k"][b:b + 1, g:g + 1].cpu(),
                                  x["v"][b:b + 1, g:g + 1].cpu(), lref[h:h + 1], causal=True)
            assert rel_err(out[b:b + 1, h:h + 1], ref) <= BF16_TOL, (b, h, float(lref[h]))


def test_v1_prefill_precision_policy_extremes(v1_prefill):
    w, x, lref, out = v1_prefill
    for h in _hardest_heads(lref):
        if h is None:
            continue
        for b in (0, w.B - 1):
            sl = lambda t: t[b:b + 1, h:h + 1].cpu()  # noqa: E731
            ref = orc.diffattn_v1(sl(x["q1"]), sl(x["k1"]), sl(x["q2"]), sl(x["k2"]), sl(x["v"]), lref[h:h + 1],
                                  causal=True, rms=True, eps=1e-5)
            assert rel_err(out[b:b + 1, h:h + 1], ref) <= BF16_TOL, (b, h, float(lref[h]))
