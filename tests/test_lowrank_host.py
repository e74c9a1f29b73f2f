"""The low-rank scan kernels' bodies, run on the host over every index
(tests/host/lowrank_host.cu includes the library's lowrank.cuh), against the
fp64 oracle of the fixed low-rank substitute for A2.  No GPU.

The harness takes A1 V as an f32 input (the prefill writes it in f32) and
returns out = A1 V - lambda N V in bf16, its only rounding to bf16.  The checks are per element: with A1 V = 0 and lambda = 1, N V is
within two bf16 roundings of its own value plus the fp32 summation bound
(one key too many or too few shows), and so is the combination.
That covers the chunk boundaries, the causal offset on both sides (Lq < Lk,
Lq > Lk), the unmasked total, ranks 1 to 16, rows whose factor row is zero,
and empty key sets."""

import os
import subprocess

import numpy as np
import pytest
import torch

from differential_attention_transformers_b200 import build
from oracle import lowrank as lr

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "host", "lowrank_host.cu")


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    try:
        nvcc = build.nvcc()
    except RuntimeError:
        pytest.skip("nvcc not available")
    exe = str(tmp_path_factory.mktemp("lowrank") / "lowrank_host")
    res = subprocess.run([nvcc, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a", SRC, "-o", exe],
                         capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    return exe


def _bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy()


def _bf16_values(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _run(exe, tmp_path, B, H, Hkv, Lq, Lk, r, causal, v, F, G, lam, a1v):
    fin, fout = tmp_path / "in.bin", tmp_path / "out.bin"
    with open(fin, "wb") as f:
        f.write(np.array([B, H, Hkv, Lq, Lk, r, int(causal)], dtype=np.int32).tobytes())
        f.write(_bf16_bits(v).tobytes())
        f.write(np.ascontiguousarray(F, dtype=np.float32).tobytes())
        f.write(np.ascontiguousarray(G, dtype=np.float32).tobytes())
        f.write(np.ascontiguousarray(lam, dtype=np.float32).tobytes())
        f.write(np.ascontiguousarray(a1v, dtype=np.float32).tobytes())
    res = subprocess.run([exe, str(fin), str(fout)], capture_output=True, text=True)
    assert res.returncode == 0, (res.returncode, res.stderr)
    bits = np.fromfile(fout, dtype=np.int16).reshape(B, H, Lq, 128)
    return torch.from_numpy(bits).view(torch.bfloat16).double().numpy()


CASES = [
    # B, H, Hkv, Lq, Lk, r, causal
    (2, 4, 2, 600, 600, 5, True),     # ragged last chunk, two heads per KV head
    (1, 2, 1, 300, 700, 3, True),     # Lq < Lk: offset 400, beyond one chunk
    (1, 2, 2, 700, 300, 1, True),     # Lq > Lk: the first 400 rows see no key
    (1, 2, 1, 300, 600, 16, False),   # unmasked, largest rank
    (1, 2, 1, 40, 1000, 4, True),     # decode-like: 960 leading keys, four slots, the last partial
    (1, 2, 1, 70, 0, 2, True),        # no keys
    (1, 2, 1, 70, 0, 2, False),
]


@pytest.mark.parametrize("B,H,Hkv,Lq,Lk,r,causal", CASES)
def test_scan_matches_oracle(harness, tmp_path, B, H, Hkv, Lq, Lk, r, causal):
    rng = np.random.default_rng(Lq * 7 + Lk + r)
    v = _bf16_values(rng.standard_normal((B, Hkv, Lk, 128)) * 0.3)
    F = rng.random((H, Lq, r)).astype(np.float32)
    G = rng.random((H, Lk, r)).astype(np.float32)
    F[0, min(5, Lq - 1)] = 0.0                      # a row with zero mass: N's row is 0
    grp = H // Hkv
    maps = [lr.noise_map(F[h].astype(np.float64), G[h].astype(np.float64), Lq, Lk, causal) for h in range(H)]
    NV = np.stack([np.stack([maps[h] @ v[b, h // grp] for h in range(H)]) for b in range(B)])
    NA = np.stack([np.stack([maps[h] @ np.abs(v[b, h // grp]) for h in range(H)]) for b in range(B)])
    # Error model: the bf16 rounding of the output (2^-9 of each value, twice
    # for margin) plus the fp32 sums over up to Lk keys, bounded by 2^-14 of
    # the sum of the absolute terms, N |V|.  One key too many or too few moves
    # an element by about |v| / Lk, far above the second term.
    # N V alone (A1 V = 0, lambda = 1):
    got = _run(harness, tmp_path, B, H, Hkv, Lq, Lk, r, causal, v, F, G, np.ones(H, np.float32),
               np.zeros((B, H, Lq, 128)))
    err = np.abs(-got - NV)
    assert np.all(err <= 2.0 ** -8 * np.abs(NV) + 2.0 ** -14 * NA), float(np.max(err - 2.0 ** -8 * np.abs(NV)))
    # the combination with A1 V and lambda
    lam = np.linspace(-0.3, 1.2, H).astype(np.float32)
    a1v = (rng.standard_normal((B, H, Lq, 128)) * 0.2).astype(np.float32).astype(np.float64)   # stands in for A1 V
    got = _run(harness, tmp_path, B, H, Hkv, Lq, Lk, r, causal, v, F, G, lam, a1v)
    lam64 = lam[None, :, None, None].astype(np.float64)
    want = a1v - lam64 * NV
    assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 2.0 ** -14 * (np.abs(a1v) + np.abs(lam64) * NA))
    if Lk == 0 or (causal and Lq > Lk):
        # rows without a visible key keep A1 V unchanged
        first = Lq if Lk == 0 else Lq - Lk
        assert np.array_equal(got[:, :, :first], _bf16_values(a1v[:, :, :first]))
    assert np.array_equal(got[:, 0, min(5, Lq - 1)], _bf16_values(a1v[:, 0, min(5, Lq - 1)]))


def test_whole_substitute_against_oracle(harness, tmp_path):
    """With A1 V from the oracle's attention, the harness output is the oracle's
    (A1 - lambda N) V within the bf16 output tolerance."""
    rng = np.random.default_rng(99)
    B, H, Hkv, L, r = 1, 2, 1, 520, 4
    q = _bf16_values(rng.standard_normal((B, H, L, 128)) / np.sqrt(128))
    k = _bf16_values(rng.standard_normal((B, Hkv, L, 128)) / np.sqrt(128))
    v = _bf16_values(rng.standard_normal((B, Hkv, L, 128)) / np.sqrt(128))
    F, G = rng.random((H, L, r)).astype(np.float32), rng.random((H, L, r)).astype(np.float32)
    lam = np.array([0.5, 0.8], dtype=np.float32)
    a1v = lr.diffattn_lowrank(q, k, v, F, G, np.zeros(H), causal=True)
    got = _run(harness, tmp_path, B, H, Hkv, L, L, r, True, v, F, G, lam, a1v)
    ref = lr.diffattn_lowrank(q, k, v, F, G, lam, causal=True)
    assert np.max(np.abs(got - ref)) <= 2e-2 * np.max(np.abs(ref))


def test_near_cancellation_keeps_f32_precision(harness, tmp_path):
    """A1 V close to N V and lambda = 1: the output is a small difference of two
    near-equal terms.  With A1 V in f32 its error is the fp32 sums' (about
    Lk 2^-24 of N |V|) plus the one bf16 rounding of the output, far inside
    2e-2 of the output's own scale; a bf16 A1 V (2^-9 of its value) would not
    be."""
    rng = np.random.default_rng(7)
    B, H, Hkv, L, r = 1, 2, 1, 600, 1
    v = _bf16_values(rng.standard_normal((B, Hkv, L, 128)) / np.sqrt(128))
    F, G = np.ones((H, L, r), np.float32), np.ones((H, L, r), np.float32)   # N = the causal mean
    N = lr.noise_map(F[0].astype(np.float64), G[0].astype(np.float64), L, L, True)
    nv = N @ v[0, 0]
    small = rng.standard_normal((B, H, L, 128)) * 1e-3 * np.abs(nv).max()
    a1v = (nv[None, None] + small).astype(np.float32).astype(np.float64)
    got = _run(harness, tmp_path, B, H, Hkv, L, L, r, True, v, F, G, np.ones(H, np.float32), a1v)
    want = a1v - nv[None, None]
    assert np.max(np.abs(got - want)) <= 2e-2 * np.max(np.abs(want))
    # the same output through a bf16 A1 V misses that bound
    coarse = _bf16_values(a1v) - nv[None, None]
    assert np.max(np.abs(coarse - want)) > 2e-2 * np.max(np.abs(want))
