"""diffattn_decode_v2_noalloc: the decode entry point that allocates nothing.

Some callers cannot call cudaMalloc at the point where they decode: code that
runs inside a custom memory pool or an allocator callback (re-entering the
allocator there deadlocks or corrupts the pool), or a serving runtime that owns
every byte of device memory and only lends this library its tensors.  For them
the library keeps a fixed 4 MiB scratch array in device memory and the entry
point takes no workspace argument.

This file is collected last on purpose (the name sorts after every other test
file): the entry point keeps state in the library's shared scratch, so it is
checked both after everything else has run and, when run alone, in a fresh
process.  It calls the new entry point through the C ABI (ctypes) and compares
it with the existing workspace-taking entry point, on two calls in a row with
different inputs, within the bf16 tolerance used by the other parity tests.
"""

import ctypes
import math

import pytest
import torch

import differential_attention_transformers_b200 as da

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
DEV = "cuda"


def _inputs(seed, B, Hq, Hkv, T):
    g = torch.Generator(device="cpu").manual_seed(seed)
    s = 1 / math.sqrt(128)
    mk = lambda *shape: (torch.randn(*shape, generator=g) * s).to(torch.bfloat16).to(DEV)  # noqa: E731
    lam = (torch.rand(Hq // 2, generator=g) * 1.2 - 0.2).to(DEV)
    return mk(B, Hq, 128), mk(B, Hkv, T, 128), mk(B, Hkv, T, 128), lam


def _noalloc(q, kc, vc, lam):
    L = da.load()
    B, Hq, D = q.shape
    Hkv, T = kc.shape[1], kc.shape[2]
    out = torch.empty((B, Hq // 2, D), dtype=torch.bfloat16, device=DEV)
    st = L.diffattn_decode_v2_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()),
                                      ctypes.c_void_p(vc.data_ptr()), ctypes.c_void_p(lam.data_ptr()),
                                      ctypes.c_void_p(out.data_ptr()), da.BF16, B, Hq, Hkv, T, D,
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == da.OK, da.last_error()
    return out


def _rel(a, b):
    a, b = a.float(), b.float()
    return (torch.max(torch.abs(a - b)) / torch.max(torch.abs(b))).item()


def test_noalloc_decode_matches_workspace_decode_twice():
    cases = [(_inputs(101, 16, 64, 8, 4099), "ragged 4099-token cache"),
             (_inputs(202, 3, 16, 2, 20000), "20000-token cache, 8 heads per group")]
    outs = []
    for (q, kc, vc, lam), _ in cases:                 # two calls in a row on the shared scratch
        outs.append(_noalloc(q, kc, vc, lam))
    torch.cuda.synchronize()
    assert da.last_status() == da.OK
    for ((q, kc, vc, lam), what), got in zip(cases, outs):
        ref = da.decode_v2(q, kc, vc, lam)
        assert torch.isfinite(got.float()).all(), what
        assert _rel(got, ref) <= BF16_TOL, what


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = da.load()
    P = ctypes.c_void_p(256)  # never dereferenced: the size check comes first
    # 4000 sequences x 8 KV heads x 64 tokens: far more partial records than 4 MiB holds
    st = L.diffattn_decode_v2_noalloc(P, P, P, P, P, da.BF16, 4000, 64, 8, 64, 128, ctypes.c_void_p(0))
    assert st == da.ERR_UNSUPPORTED
    assert "scratch" in da.last_error()
