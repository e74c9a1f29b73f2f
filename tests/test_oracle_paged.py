"""Pins of the paged, variable-length decode oracle (no GPU).

The oracle reads each sequence's first seq_lens[b] tokens out of a shuffled
pool of token-major pages and applies the V2 decode definition.  These tests
pin the paging reading to the contiguous reading and to invariants that a
gather mistake (a wrong page order, a transposed token/head axis, an off-by-one
length, rows read past the sequence) would break."""

import math

import numpy as np
import pytest
import torch

from differential_attention_transformers_b200 import inputs
from oracle import brute
from oracle import diffattn


def _case(B=3, Hq=8, Hkv=2, T=150, D=16, seed=0):
    g = torch.Generator().manual_seed(seed)
    s = 1 / math.sqrt(D)
    q = torch.randn(B, Hq, D, generator=g, dtype=torch.float64) * s
    kc = torch.randn(B, Hkv, T, D, generator=g, dtype=torch.float64) * s
    vc = torch.randn(B, Hkv, T, D, generator=g, dtype=torch.float64)
    lam = np.linspace(0.3, 0.9, Hq // 2)
    return q, kc, vc, lam


def pin_identity_reading_full_lengths_equals_contiguous_decode(orc):
    q, kc, vc, lam = _case()
    for ps in (16, 64):
        kp, vp, bt, sl = inputs.paged_cache(kc, vc, ps, seed=ps)
        got = orc.decode_v2_paged(q, kp, vp, bt, sl, lam)
        ref = orc.decode_v2(q, kc, vc, lam)
        assert np.allclose(got, ref, rtol=0, atol=1e-13)


def pin_variable_lengths_equal_truncated_contiguous_decode(orc):
    q, kc, vc, lam = _case(T=200)
    lens = [200, 1, 77]
    kp, vp, bt, sl = inputs.paged_cache(kc, vc, 32, seed=5, lens=lens)
    got = orc.decode_v2_paged(q, kp, vp, bt, sl, lam)
    for b, n in enumerate(lens):
        ref = orc.decode_v2(q[b:b + 1], kc[b:b + 1, :, :n], vc[b:b + 1, :, :n], lam)[0]
        assert np.allclose(got[b], ref, rtol=0, atol=1e-13)
        assert np.all(np.isfinite(got[b]))     # NaN rows past the length never read


def pin_page_permutation_invariance(orc):
    q, kc, vc, lam = _case(T=96)
    a = orc.decode_v2_paged(q, *inputs.paged_cache(kc, vc, 16, seed=1), lam)
    b = orc.decode_v2_paged(q, *inputs.paged_cache(kc, vc, 16, seed=2), lam)
    assert np.array_equal(a, b)


def pin_zero_length_sequence_gives_zeros(orc):
    q, kc, vc, lam = _case(T=40)
    kp, vp, bt, sl = inputs.paged_cache(kc, vc, 16, seed=3, lens=[40, 0, 17])
    got = orc.decode_v2_paged(q, kp, vp, bt, sl, lam)
    assert np.array_equal(got[1], np.zeros_like(got[1]))
    assert np.all(np.isfinite(got))


def pin_single_token_sequence_is_one_minus_lambda_times_value(orc):
    # one visible key: both maps put weight 1 on it, O = (1 - lambda) v
    q, kc, vc, lam = _case(B=1, T=5)
    kp, vp, bt, sl = inputs.paged_cache(kc, vc, 16, seed=4, lens=[1])
    got = orc.decode_v2_paged(q, kp, vp, bt, sl, lam)
    grp = q.shape[1] // kc.shape[1]
    for h in range(q.shape[1] // 2):
        g = (2 * h) // grp
        assert np.allclose(got[0, h], (1 - lam[h]) * vc[0, g, 0].numpy(), rtol=0, atol=1e-14)


def pin_brute_force_twin_on_a_tiny_paged_case(orc):
    q, kc, vc, lam = _case(B=2, Hq=4, Hkv=1, T=21, D=4)
    lens = [21, 9]
    kp, vp, bt, sl = inputs.paged_cache(kc, vc, 16, seed=6, lens=lens)
    got = orc.decode_v2_paged(q, kp, vp, bt, sl, lam)
    for b, n in enumerate(lens):
        qq = [[[q[b, h].tolist()] for h in range(4)]]
        kk = [[kc[b, 0, :n].tolist()]]
        vv = [[vc[b, 0, :n].tolist()]]
        ref = np.array(brute.v2(qq, kk, vv, list(lam), causal=True))[0, :, 0]
        assert np.allclose(got[b], ref, rtol=0, atol=1e-12)


# The pins above; test_oracle_paged_mutations.py runs them against planted
# gather mistakes.
PINS = [pin_identity_reading_full_lengths_equals_contiguous_decode, pin_variable_lengths_equal_truncated_contiguous_decode, pin_page_permutation_invariance, pin_zero_length_sequence_gives_zeros, pin_single_token_sequence_is_one_minus_lambda_times_value, pin_brute_force_twin_on_a_tiny_paged_case]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(diffattn)
