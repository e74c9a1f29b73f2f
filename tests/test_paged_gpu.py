"""Paged, variable-length V2 decode (diffattn_decode_v2_paged) against the fp64
oracle and against the contiguous decode.  Needs a B200.

The page pools come from inputs.paged_cache: pages in shuffled order, NaN in
every spare page and in the unused rows of each sequence's last page, so a
kernel that reads anything outside a sequence produces NaN."""

import math

import numpy as np
import pytest
import torch

import differential_attention_transformers_b200 as da
from differential_attention_transformers_b200 import inputs
from oracle import diffattn as orc
from tests.test_parity_gpu import BF16_TOL, DEV, lam_gpu_and_ref

pytestmark = pytest.mark.gpu


def _qkv(B, Hq, Hkv, T, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    s = 1 / math.sqrt(128)
    mk = lambda *shape: (torch.randn(*shape, generator=g) * s).to(torch.bfloat16).to(DEV)  # noqa: E731
    lam = (torch.rand(Hq // 2, generator=g) * 1.2 - 0.2).to(DEV)
    return mk(B, Hq, 128), mk(B, Hkv, T, 128), mk(B, Hkv, T, 128), lam


def _check_against_oracle(out, q, kp, vp, bt, sl, lam, what):
    ref = orc.decode_v2_paged(q, kp, vp, bt, sl, lam.cpu().numpy())
    got = out.float().cpu().numpy()
    assert np.all(np.isfinite(got)), what
    for b in range(ref.shape[0]):
        scale = float(np.max(np.abs(ref[b])))
        err = float(np.max(np.abs(got[b] - ref[b])))
        if scale == 0.0:
            assert err == 0.0, (what, b)          # empty sequence: exact zeros
        else:
            assert err <= BF16_TOL * scale, (what, b, err / scale)


@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
def test_paged_variable_lengths_match_oracle(page_size):
    lens = [700, 0, 1, 63, 64, 65, 333]
    q, kc, vc, lam = _qkv(len(lens), 16, 2, 700, seed=page_size)
    kp, vp, bt, sl = inputs.paged_cache(kc, vc, page_size, seed=page_size + 1, lens=lens)
    out = da.decode_v2_paged(q, kp, vp, bt, sl, lam)
    torch.cuda.synchronize()
    assert da.last_status() == da.OK
    _check_against_oracle(out, q, kp, vp, bt, sl, lam, f"page_size {page_size}")


def test_paged_many_short_sequences_match_oracle():
    # many segments per CTA range: the record slot of every (CTA, segment) pair is distinct
    g = torch.Generator(device="cpu").manual_seed(77)
    lens = torch.randint(0, 200, (300,), generator=g).tolist()
    q, kc, vc, lam = _qkv(300, 4, 2, 200, seed=78)
    kp, vp, bt, sl = inputs.paged_cache(kc, vc, 32, seed=79, lens=lens)
    out = da.decode_v2_paged(q, kp, vp, bt, sl, lam)
    _check_against_oracle(out, q, kp, vp, bt, sl, lam, "300 short sequences")


def test_paged_one_long_many_short():
    lens = [12000] + [5] * 40
    q, kc, vc, lam = _qkv(len(lens), 8, 1, 12000, seed=81)
    kp, vp, bt, sl = inputs.paged_cache(kc, vc, 16, seed=82, lens=lens)
    out = da.decode_v2_paged(q, kp, vp, bt, sl, lam)
    _check_against_oracle(out, q, kp, vp, bt, sl, lam, "one long, many short")


def test_paged_all_empty_gives_zeros():
    q, kc, vc, lam = _qkv(3, 8, 2, 64, seed=90)
    kp, vp, bt, sl = inputs.paged_cache(kc, vc, 64, seed=91, lens=[0, 0, 0])
    out = da.decode_v2_paged(q, kp, vp, bt, sl, lam)
    assert torch.count_nonzero(out).item() == 0


@pytest.mark.parametrize("page_size", [16, 64, 256])
def test_paged_full_lengths_bitwise_equal_contiguous_decode(page_size):
    # same tiles, same split of the block space, same merge order: identical bits
    q, kc, vc, lam = _qkv(4, 16, 2, 4096, seed=100 + page_size)
    kp, vp, bt, sl = inputs.paged_cache(kc, vc, page_size, seed=7)
    paged = da.decode_v2_paged(q, kp, vp, bt, sl, lam)
    contiguous = da.decode_v2(q, kc, vc, lam)
    assert torch.equal(paged, contiguous)


def test_paged_full_size_workload():
    # the V2 decode workload (B16 Hq64 Hkv8 T65536) in 16-token pages
    w = inputs.WORKLOADS["v2_decode"]
    x = inputs.make(w, device=DEV)
    lam, lref = lam_gpu_and_ref(w)
    kp, vp, bt, sl = inputs.paged_cache(x["k"], x["v"], 16, seed=5)
    out = da.decode_v2_paged(x["q"], kp, vp, bt, sl, lam)
    assert torch.equal(out, da.decode_v2(x["q"], x["k"], x["v"], lam))
    grp = w.H // w.Hkv
    got = out.float().cpu().numpy()
    for b, gk in ((0, 0), (w.B - 1, w.Hkv - 1), (7, 3)):
        pairs = list(range(gk * grp // 2, (gk + 1) * grp // 2))
        ref = orc.decode_v2(x["q"][b:b + 1, gk * grp:(gk + 1) * grp].cpu(), x["k"][b:b + 1, gk:gk + 1].cpu(),
                            x["v"][b:b + 1, gk:gk + 1].cpu(), lref[pairs])
        for i, h in enumerate(pairs):
            err = float(np.max(np.abs(got[b, h] - ref[0, i])))
            assert err <= BF16_TOL * float(np.max(np.abs(ref[0, i]))), (b, h, err)


def test_paged_serving_shaped_batch():
    """The bench's serving-shaped batch in its launch configuration: 256
    sequences of lengths 16..4096 in one pool of 16-token pages.  A seeded
    sample of 24 sequences (the shortest and longest among them) against the
    oracle, and the whole batch bitwise repeatable."""
    x = inputs.serving_cache(**inputs.SERVING_SHAPE, device=DEV)
    Hq = inputs.SERVING_SHAPE["Hq"]
    lam = (torch.rand(Hq // 2, generator=torch.Generator().manual_seed(77)) * 1.2 - 0.2).to(DEV)
    args = (x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"], lam)
    out = da.decode_v2_paged(*args)
    torch.cuda.synchronize()
    assert da.last_status() == da.OK
    assert torch.equal(out, da.decode_v2_paged(*args))
    lens = x["seq_lens"].cpu()
    pick = torch.randperm(lens.numel(), generator=torch.Generator().manual_seed(5))[:22].tolist()
    pick += [int(lens.argmin()), int(lens.argmax())]
    idx = torch.tensor(sorted(set(pick)), device=DEV)
    _check_against_oracle(out[idx], x["q"][idx], x["k_pages"], x["v_pages"], x["block_table"][idx],
                          x["seq_lens"][idx], lam, "serving batch")
