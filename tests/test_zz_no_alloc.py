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
different inputs.  Both run the same kernels with the same split of the keys,
so the outputs must agree bit for bit; one case is also checked against the
fp64 oracle within the bf16 tolerance of the other parity tests.  A call made
after the first must leave the device's free memory (cudaMemGetInfo) and
torch's allocated bytes unchanged.
"""

import ctypes
import math

import pytest
import torch

import differential_attention_transformers_b200 as da
from oracle import diffattn as orc

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
DEV = "cuda"


def _inputs(seed, B, Hq, Hkv, T):
    g = torch.Generator(device="cpu").manual_seed(seed)
    s = 1 / math.sqrt(128)
    mk = lambda *shape: (torch.randn(*shape, generator=g) * s).to(torch.bfloat16).to(DEV)  # noqa: E731
    lam = (torch.rand(Hq // 2, generator=g) * 1.2 - 0.2).to(DEV)
    return mk(B, Hq, 128), mk(B, Hkv, T, 128), mk(B, Hkv, T, 128), lam


def _noalloc(q, kc, vc, lam, out=None):
    L = da.load()
    B, Hq, D = q.shape
    Hkv, T = kc.shape[1], kc.shape[2]
    if out is None:
        out = torch.empty((B, Hq // 2, D), dtype=torch.bfloat16, device=DEV)
    st = L.diffattn_decode_v2_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()),
                                      ctypes.c_void_p(vc.data_ptr()), ctypes.c_void_p(lam.data_ptr()),
                                      ctypes.c_void_p(out.data_ptr()), da.BF16, B, Hq, Hkv, T, D,
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == da.OK, da.last_error()
    return out


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
        assert torch.equal(got, ref), what            # same kernels, same split: bit for bit
    # the second case against the fp64 oracle, every head
    (q, kc, vc, lam), _ = cases[1]
    want = orc.decode_v2(q, kc, vc, lam.double().cpu().numpy())
    got = outs[1].double().cpu().numpy()
    for b in range(want.shape[0]):
        for h in range(want.shape[1]):
            err = abs(got[b, h] - want[b, h]).max()
            assert err <= BF16_TOL * abs(want[b, h]).max(), (b, h, err)


def test_noalloc_call_allocates_nothing():
    """After a first call (the one-time set-up), a call changes neither the
    device's free memory nor torch's allocated bytes."""
    q, kc, vc, lam = _inputs(303, 4, 64, 8, 9000)
    out = torch.empty((4, 32, 128), dtype=torch.bfloat16, device=DEV)
    _noalloc(q, kc, vc, lam, out)
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    _noalloc(q, kc, vc, lam, out)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0
    assert da.last_status() == da.OK
    assert torch.equal(out, da.decode_v2(q, kc, vc, lam))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = da.load()
    P = ctypes.c_void_p(256)  # never dereferenced: the size check comes first
    # 4000 sequences x 8 KV heads x 64 tokens: far more partial records than 4 MiB holds
    st = L.diffattn_decode_v2_noalloc(P, P, P, P, P, da.BF16, 4000, 64, 8, 64, 128, ctypes.c_void_p(0))
    assert st == da.ERR_UNSUPPORTED
    assert "scratch" in da.last_error()
