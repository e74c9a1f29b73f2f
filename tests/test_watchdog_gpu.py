"""Bounded device waits: a wait limit of 0 makes the kernels' first unsatisfied
mbarrier wait expire.  The kernel must then record DIFFATTN_ERR_TIMEOUT in the
device status word, let its in-flight copies and MMAs finish, free its tensor
memory and return -- no trap, no hang -- and the context must stay usable."""

import math

import numpy as np
import pytest
import torch

import differential_attention_transformers_b200 as da
from oracle import diffattn as orc
from tests.test_parity_gpu import BF16_TOL, DEV, bf16, rel_err

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT = 2_000_000_000


def _inputs(seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    s = 1 / math.sqrt(128)
    return bf16(1, 4, 2048, 128, g=g, std=s), bf16(1, 2, 2048, 128, g=g, std=s), bf16(1, 2, 2048, 128, g=g, std=s)


def test_prefill_wait_timeout_is_reported_and_recoverable():
    q, k, v = _inputs(41)
    lam = torch.tensor([0.4, 0.7], device=DEV)
    assert da.last_status() == da.OK
    da.set_wait_limit_ns(0)
    try:
        da.fwd_v2(q, k, v, lam, causal=True)
        st = da.last_status()
    finally:
        da.set_wait_limit_ns(DEFAULT_LIMIT)
    assert st == da.ERR_TIMEOUT
    out = da.fwd_v2(q, k, v, lam, causal=True)
    assert da.last_status() == da.OK
    ref = orc.diffattn_v2(q, k, v, lam.cpu().numpy(), causal=True)
    assert rel_err(out, ref) <= BF16_TOL


def test_decode_wait_timeout_is_reported_and_recoverable():
    g = torch.Generator(device="cpu").manual_seed(42)
    s = 1 / math.sqrt(128)
    q, kc, vc = bf16(2, 8, 128, g=g, std=s), bf16(2, 2, 20000, 128, g=g, std=s), bf16(2, 2, 20000, 128, g=g, std=s)
    lam = torch.tensor([0.1, 0.2, 0.3, 0.4], device=DEV)
    da.set_wait_limit_ns(0)
    try:
        da.decode_v2(q, kc, vc, lam)
        st = da.last_status()
    finally:
        da.set_wait_limit_ns(DEFAULT_LIMIT)
    assert st == da.ERR_TIMEOUT
    out = da.decode_v2(q, kc, vc, lam)
    assert da.last_status() == da.OK
    ref = orc.decode_v2(q, kc, vc, lam.cpu().numpy())
    assert rel_err(out, ref) <= BF16_TOL
