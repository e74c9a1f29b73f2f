"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200).

Tolerances (stated by the workload definition, written here):
  bf16 inputs: max|O - O_ref| <= 2e-2 * max|O_ref|
  f32 inputs : max|O - O_ref| <= 1e-5 * max|O_ref|
  lambda     : bitwise equal to the oracle's fp64-then-round value
  masks      : exact zeros exactly where the oracle's map is masked.
"""

import math

import numpy as np
import pytest
import torch

import differential_attention_transformers_b200 as da
from differential_attention_transformers_b200 import inputs
from oracle import diffattn as orc

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
F32_TOL = 1e-5
DEV = "cuda"


def rel_err(out, ref):
    out = out.detach().double().cpu().numpy() if hasattr(out, "detach") else np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    assert out.shape == ref.shape, (out.shape, ref.shape)
    assert np.all(np.isfinite(out)), "non-finite output"
    scale = np.max(np.abs(ref))
    err = np.max(np.abs(out - ref)) if out.size else 0.0
    return err / scale if scale > 0 else err


def lam_gpu_and_ref(w, device=DEV):
    if w.explicit_lambda is not None:
        lam = torch.full((w.pairs,), w.explicit_lambda, dtype=torch.float32, device=device)
        return lam, lam.cpu().numpy()
    p = inputs.lambda_params(w, device=device)
    init = orc.lambda_init(w.layer)
    lam = da.compute_lambda(*p, init)
    ref = orc.lambda_(*[t.double().cpu().numpy() for t in p], init)
    return lam, ref


def rand_lam(n, seed, device=DEV):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.rand(n, generator=g) * 1.2 - 0.2).to(device)


# ----------------------------------------------------------------------------- lambda
@pytest.mark.parametrize("name", ["v1_tiny", "v1_prefill", "v2_prefill", "v2_decode", "v1_decode"])
def test_lambda_bitwise(name):
    w = inputs.WORKLOADS[name]
    lam, ref = lam_gpu_and_ref(w)
    got = lam.cpu().numpy()
    assert got.dtype == np.float32 and np.array_equal(got.view(np.uint32), ref.view(np.uint32)), (got, ref)


def test_lambda_bitwise_wide():
    g = torch.Generator(device="cpu").manual_seed(77)
    p = [(torch.randn(256, 128, generator=g) * 0.3).to(DEV) for _ in range(4)]
    for init in (0.2, 0.5, orc.lambda_init(24)):
        got = da.compute_lambda(*p, init).cpu().numpy()
        ref = orc.lambda_(*[t.double().cpu().numpy() for t in p], init)
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


# ----------------------------------------------------------------------------- f32 (SIMT)
def test_f32_v1_tiny():
    w = inputs.WORKLOADS["v1_tiny"]
    x = {k: t.to(DEV) for k, t in inputs.make(w).items()}
    lam, lref = lam_gpu_and_ref(w)
    out = da.fwd_v1(x["q1"], x["k1"], x["q2"], x["k2"], x["v"], lam, causal=True)
    ref = orc.diffattn_v1(x["q1"], x["k1"], x["q2"], x["k2"], x["v"], lref, causal=True)
    assert rel_err(out, ref) <= F32_TOL


def test_f32_noise_probe():
    w = inputs.WORKLOADS["noise_probe"]
    x = {k: t.to(DEV) for k, t in inputs.make(w).items()}
    lam = torch.full((1,), 0.5, dtype=torch.float32, device=DEV)
    out = da.fwd_v1(x["q1"], x["k1"], x["q2"], x["k2"], x["v"], lam, causal=False)
    ref = orc.diffattn_v1(x["q1"], x["k1"], x["q2"], x["k2"], x["v"], np.array([0.5]), causal=False)
    assert rel_err(out, ref) <= F32_TOL
    rows = out[:, 0, 0].double().cpu().numpy()
    assert np.max(np.abs(rows.sum(axis=1) - 0.5)) <= F32_TOL          # rows of A1 - lambda A2 sum to 1 - lambda
    plain = da.fwd_v1(x["q1"], x["k1"], x["q2"], x["k2"], x["v"], torch.zeros_like(lam), causal=False)
    plain = plain[:, 0, 0].double().cpu().numpy()
    assert np.all(plain > 0.0)                                          # softmax never yields an exact zero


@pytest.mark.parametrize("causal", [True, False])
def test_f32_v2_and_rms(causal):
    g = torch.Generator(device="cpu").manual_seed(5)
    q = torch.randn(2, 8, 37, 48, generator=g).to(DEV)
    k = torch.randn(2, 2, 53, 48, generator=g).to(DEV)
    v = torch.randn(2, 2, 53, 48, generator=g).to(DEV)
    lam = rand_lam(4, 6)
    out = da.fwd_v2(q, k, v, lam, causal=causal)
    ref = orc.diffattn_v2(q, k, v, lam.cpu().numpy(), causal=causal)
    assert rel_err(out, ref) <= F32_TOL
    q1, q2 = q[:, :4].contiguous(), q[:, 4:].contiguous()
    k2 = torch.randn(2, 2, 53, 48, generator=g).to(DEV)
    out = da.fwd_v1(q1, k, q2, k2, v, lam, causal=causal, rmsnorm=True, eps=1e-5)
    ref = orc.diffattn_v1(q1, k, q2, k2, v, lam.cpu().numpy(), causal=causal, rms=True, eps=1e-5)
    assert rel_err(out, ref) <= F32_TOL


# ----------------------------------------------------------------------------- bf16 prefill
def bf16(*shape, g, std=1.0):
    return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16).to(DEV)


V2_CASES = [
    # B, Hq, Hkv, Lq, Lk, causal
    (1, 4, 2, 300, 300, True),     # 3 tiles with a ragged tail
    (2, 8, 2, 257, 257, False),
    (1, 4, 1, 100, 333, True),     # Lq < Lk: bottom-right alignment
    (1, 4, 2, 200, 130, True),     # Lq > Lk: the first 70 rows see nothing
    (1, 2, 1, 1, 1000, True),      # one query row
    (1, 16, 4, 128, 128, True),    # exactly one tile
    (2, 4, 2, 640, 640, True),     # several row blocks, longest first
]


@pytest.mark.parametrize("case", V2_CASES, ids=lambda c: "B%d_Hq%d_Hkv%d_Lq%d_Lk%d_c%d" % c)
def test_bf16_v2_small(case):
    B, Hq, Hkv, Lq, Lk, causal = case
    g = torch.Generator(device="cpu").manual_seed(hash(case) % 2**31)
    s = 1 / math.sqrt(128)
    q, k, v = bf16(B, Hq, Lq, 128, g=g, std=s), bf16(B, Hkv, Lk, 128, g=g, std=s), bf16(B, Hkv, Lk, 128, g=g, std=s)
    lam = rand_lam(Hq // 2, 9)
    out = da.fwd_v2(q, k, v, lam, causal=causal)
    ref = orc.diffattn_v2(q, k, v, lam.cpu().numpy(), causal=causal)
    assert rel_err(out, ref) <= BF16_TOL
    if causal and Lq > Lk:
        assert torch.all(out[:, :, : Lq - Lk] == 0)


V1_CASES = [
    # B, H, Hkv, Lq, Lk, d, causal, rms
    (1, 4, 2, 401, 401, 64, True, True),
    (2, 2, 2, 129, 129, 64, False, False),
    (1, 2, 1, 300, 300, 128, True, False),
    (1, 2, 2, 50, 700, 64, True, True),
]


@pytest.mark.parametrize("case", V1_CASES, ids=lambda c: "B%d_H%d_Hkv%d_Lq%d_Lk%d_d%d_c%d_r%d" % c)
def test_bf16_v1_small(case):
    B, H, Hkv, Lq, Lk, d, causal, rms = case
    g = torch.Generator(device="cpu").manual_seed(hash(case) % 2**31)
    s = 1 / math.sqrt(d)
    q1, q2 = bf16(B, H, Lq, d, g=g, std=s), bf16(B, H, Lq, d, g=g, std=s)
    k1, k2 = bf16(B, Hkv, Lk, d, g=g, std=s), bf16(B, Hkv, Lk, d, g=g, std=s)
    v = bf16(B, Hkv, Lk, 128, g=g, std=s)
    lam = rand_lam(H, 10)
    out = da.fwd_v1(q1, k1, q2, k2, v, lam, causal=causal, rmsnorm=rms, eps=1e-5)
    ref = orc.diffattn_v1(q1, k1, q2, k2, v, lam.cpu().numpy(), causal=causal, rms=rms, eps=1e-5)
    assert rel_err(out, ref) <= BF16_TOL


@pytest.mark.parametrize("Lq", [128, 40])
def test_bf16_masks_exact(Lq):
    """V = I makes the output the map itself: zeros exactly where masked."""
    g = torch.Generator(device="cpu").manual_seed(21)
    Lk = 128
    q = bf16(1, 2, Lq, 128, g=g, std=0.1)
    k = bf16(1, 1, Lk, 128, g=g, std=0.1)
    eye = torch.eye(Lk, dtype=torch.bfloat16, device=DEV)[None, None].contiguous()
    out = da.fwd_v2(q, k, eye, torch.zeros(1, device=DEV), causal=True)[0, 0].float().cpu().numpy()
    ref = orc.diffattn_v2(q, k, eye, np.zeros(1), causal=True)[0, 0]
    assert np.array_equal(out == 0.0, ref == 0.0)
    assert np.all(out[ref != 0.0] > 0.0)
    # V1 layout, same check with RMSNorm off
    q1, q2 = bf16(1, 1, Lq, 64, g=g, std=0.1), bf16(1, 1, Lq, 64, g=g, std=0.1)
    k1, k2 = bf16(1, 1, Lk, 64, g=g, std=0.1), bf16(1, 1, Lk, 64, g=g, std=0.1)
    out = da.fwd_v1(q1, k1, q2, k2, eye, torch.zeros(1, device=DEV), causal=True)[0, 0].float().cpu().numpy()
    ref = orc.diffattn_v1(q1, k1, q2, k2, eye, np.zeros(1), causal=True)[0, 0]
    assert np.array_equal(out == 0.0, ref == 0.0)


def test_bf16_exact_zero_when_maps_equal():
    g = torch.Generator(device="cpu").manual_seed(22)
    q = bf16(1, 2, 300, 128, g=g, std=0.09)
    q = torch.cat([q, q], dim=1)[:, [0, 2, 1, 3]].contiguous()   # heads (0,1) equal, (2,3) equal
    k, v = bf16(1, 1, 300, 128, g=g, std=0.09), bf16(1, 1, 300, 128, g=g, std=0.09)
    out = da.fwd_v2(q, k, v, torch.ones(2, device=DEV), causal=True)
    assert torch.all(out == 0)
    q1 = bf16(1, 2, 200, 64, g=g, std=0.12)
    k1, v = bf16(1, 2, 200, 64, g=g, std=0.12), bf16(1, 2, 200, 128, g=g, std=0.12)
    out = da.fwd_v1(q1, k1, q1, k1, v, torch.ones(2, device=DEV), causal=True)
    assert torch.all(out == 0)


def test_bf16_v_ones_gives_one_minus_lambda():
    g = torch.Generator(device="cpu").manual_seed(23)
    q, k = bf16(1, 4, 260, 128, g=g, std=0.09), bf16(1, 2, 260, 128, g=g, std=0.09)
    v = torch.ones(1, 2, 260, 128, dtype=torch.bfloat16, device=DEV)
    lam = torch.tensor([0.2, -0.3], device=DEV)
    out = da.fwd_v2(q, k, v, lam, causal=True).float().cpu()
    target = (1 - lam.cpu())[None, :, None, None].expand_as(out)
    assert torch.max(torch.abs(out - target)) <= BF16_TOL * 1.3


def test_bf16_degenerate_sizes():
    g = torch.Generator(device="cpu").manual_seed(24)
    q = bf16(1, 4, 64, 128, g=g)
    k = torch.empty(1, 2, 0, 128, dtype=torch.bfloat16, device=DEV)
    out = da.fwd_v2(q, k, k, torch.ones(2, device=DEV), causal=True)
    assert out.shape == (1, 2, 64, 128) and torch.all(out == 0)
    q0 = torch.empty(1, 4, 0, 128, dtype=torch.bfloat16, device=DEV)
    k1 = bf16(1, 2, 10, 128, g=g)
    assert da.fwd_v2(q0, k1, k1, torch.ones(2, device=DEV)).shape == (1, 2, 0, 128)
    qb = torch.empty(0, 4, 16, 128, dtype=torch.bfloat16, device=DEV)
    assert da.fwd_v2(qb, k1[:0], k1[:0], torch.ones(2, device=DEV)).shape == (0, 2, 16, 128)


def test_bf16_deterministic_and_streams():
    g = torch.Generator(device="cpu").manual_seed(25)
    q, k, v = bf16(2, 8, 500, 128, g=g, std=0.09), bf16(2, 2, 500, 128, g=g, std=0.09), bf16(2, 2, 500, 128, g=g, std=0.09)
    lam = rand_lam(4, 26)
    a = da.fwd_v2(q, k, v, lam)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = da.fwd_v2(q, k, v, lam)
    s.synchronize()
    assert torch.equal(a, b)


def test_host_buffers_match_device_path():
    g = torch.Generator(device="cpu").manual_seed(27)
    q = (torch.randn(1, 4, 200, 128, generator=g) * 0.09).to(torch.bfloat16)
    k = (torch.randn(1, 2, 200, 128, generator=g) * 0.09).to(torch.bfloat16)
    v = (torch.randn(1, 2, 200, 128, generator=g) * 0.09).to(torch.bfloat16)
    lam = torch.tensor([0.3, 0.6])
    host = da.fwd_v2(q, k, v, lam)
    assert host.device.type == "cpu"
    dev = da.fwd_v2(q.to(DEV), k.to(DEV), v.to(DEV), lam.to(DEV)).cpu()
    assert torch.equal(host, dev)


def test_abi_errors_on_device():
    g = torch.Generator(device="cpu").manual_seed(28)
    buf = bf16(1, 4, 64, 128 + 8, g=g)
    # a view starting 2 bytes into the allocation: not 16-byte aligned
    flat = bf16(4 * 64 * 128 + 8, g=g)
    q_bad = flat[1:1 + 4 * 64 * 128].view(1, 4, 64, 128)
    k = bf16(1, 2, 64, 128, g=g)
    with pytest.raises(da.DiffAttnError) as e:
        da.fwd_v2(q_bad, k, k, torch.ones(2, device=DEV))
    assert e.value.code == da.ERR_MISALIGNED
    del buf
    # decode workspace too small
    q = bf16(2, 8, 128, g=g)
    kc = bf16(2, 2, 1000, 128, g=g)
    with pytest.raises(da.DiffAttnError) as e:
        da.decode_v2(q, kc, kc, torch.ones(4, device=DEV), workspace=torch.empty(16, dtype=torch.uint8, device=DEV))
    assert e.value.code == da.ERR_WORKSPACE


# ----------------------------------------------------------------------------- decode
DEC_CASES = [
    # B, Hq, Hkv, T
    (3, 8, 2, 1000),    # ragged tail of 40 keys
    (2, 16, 2, 5000),   # 8 Q heads per KV group
    (1, 4, 2, 64),      # one block
    (2, 4, 1, 1),       # one key
    (2, 8, 4, 0),       # empty cache -> zeros
    (4, 12, 2, 777),    # 6 heads per group
]


@pytest.mark.parametrize("case", DEC_CASES, ids=lambda c: "B%d_Hq%d_Hkv%d_T%d" % c)
def test_decode_v2_small(case):
    B, Hq, Hkv, T = case
    g = torch.Generator(device="cpu").manual_seed(hash(case) % 2**31)
    s = 1 / math.sqrt(128)
    q, kc, vc = bf16(B, Hq, 128, g=g, std=s), bf16(B, Hkv, T, 128, g=g, std=s), bf16(B, Hkv, T, 128, g=g, std=s)
    lam = rand_lam(Hq // 2, 31)
    out = da.decode_v2(q, kc, vc, lam)
    if T == 0:
        assert torch.all(out == 0)
        return
    ref = orc.decode_v2(q, kc, vc, lam.cpu().numpy())
    assert rel_err(out, ref) <= BF16_TOL


@pytest.mark.parametrize("B,Hq,T", [(16, 64, 65536), (3, 16, 4097), (1, 4, 1), (2, 12, 0)])
def test_decode_v2_workspace_size_covers_every_kv_head_count(B, Hq, T):
    """diffattn_decode_v2_workspace_size(B, Hq, T, D) is at least the exact
    size for every valid Hkv, and a decode given exactly that many bytes runs
    (the Hkv the caller ends up with is one of them)."""
    L = da.load()
    n = L.diffattn_decode_v2_workspace_size(B, Hq, T, 128)
    valid = [h for h in range(1, Hq // 2 + 1) if Hq % h == 0 and (Hq // h) % 2 == 0 and Hq // h <= 8]
    assert valid and n == max(L.diffattn_decode_workspace_size(B, h, T, 128) for h in valid)
    Hkv = valid[0]
    g = torch.Generator(device="cpu").manual_seed(B * 1000 + Hq + T)
    s = 1 / math.sqrt(128)
    q, kc, vc = bf16(B, Hq, 128, g=g, std=s), bf16(B, Hkv, T, 128, g=g, std=s), bf16(B, Hkv, T, 128, g=g, std=s)
    lam = rand_lam(Hq // 2, 7)
    ws = torch.empty(max(int(n), 16), dtype=torch.uint8, device=DEV)
    out = da.decode_v2(q, kc, vc, lam, workspace=ws)
    assert torch.equal(out, da.decode_v2(q, kc, vc, lam))


@pytest.mark.parametrize("fused", [1, 0])
@pytest.mark.parametrize("case", [(2, 8, 2, 1000), (1, 4, 4, 130), (3, 16, 4, 4097)],
                         ids=lambda c: "B%d_H%d_Hkv%d_T%d" % c)
def test_decode_v1_small(case, fused):
    B, H, Hkv, T = case
    g = torch.Generator(device="cpu").manual_seed(hash(case) % 2**31 + fused)
    s = 1 / 8
    q1, q2 = bf16(B, H, 64, g=g, std=s), bf16(B, H, 64, g=g, std=s)
    k1, k2 = bf16(B, Hkv, T, 64, g=g, std=s), bf16(B, Hkv, T, 64, g=g, std=s)
    v = bf16(B, Hkv, T, 128, g=g, std=s)
    lam = rand_lam(H, 32)
    out = da.decode_v1(q1, k1, q2, k2, v, lam, fused=bool(fused))
    ref = orc.decode_v1(q1, k1, q2, k2, v, lam.cpu().numpy())
    assert rel_err(out, ref) <= BF16_TOL


# |1 - lambda| below which the prefill keeps the bf16 residual of P
PREFILL_RESID_TAU = 0.15


@pytest.mark.parametrize("lam_value", [0.97, 1.0, 1.03, 0.86, 1.14, 0.84, 1.16, 0.74, 1.26])
def test_bf16_near_unit_lambda_with_similar_maps(lam_value):
    """The hardest case for bf16 P: near-uniform, nearly identical maps and lambda
    close to 1, where O1/l1 - lambda*O2/l2 cancels.  0.97/1.0/1.03 and 0.86/1.14 take
    the residual path; 0.84/1.16 sit just outside its threshold (|1 - lambda| = 0.16)
    and use bf16 P alone, as do 0.74/1.26."""
    g = torch.Generator(device="cpu").manual_seed(int(lam_value * 1000))
    s = 1 / math.sqrt(128)
    q1 = torch.randn(1, 1, 1024, 128, generator=g) * s
    q2 = q1 + 0.05 * s * torch.randn(1, 1, 1024, 128, generator=g)       # map 2 close to map 1
    q = torch.cat([q1, q2], dim=1).to(torch.bfloat16).to(DEV)
    k = bf16(1, 1, 1024, 128, g=g, std=s)
    v = bf16(1, 1, 1024, 128, g=g, std=s)
    lam = torch.tensor([lam_value], device=DEV)
    out = da.fwd_v2(q, k, v, lam, causal=True)
    ref = orc.diffattn_v2(q, k, v, np.array([lam_value]), causal=True)
    assert rel_err(out, ref) <= BF16_TOL


def test_host_pipelined_prefill_matches_device_path(monkeypatch):
    """CPU inputs take the chunked path (copies overlapping kernels); forced on
    here for small shapes with many chunks, it must give the device path's bits."""
    monkeypatch.setattr(da, "_PIPELINE_MIN_BYTES", 0)
    monkeypatch.setattr(da, "_PIPELINE_CHUNK_UNITS", 3)
    g = torch.Generator(device="cpu").manual_seed(404)
    s = 1 / math.sqrt(128)
    mk = lambda *shape, std=s: (torch.randn(*shape, generator=g) * std).to(torch.bfloat16)  # noqa: E731
    q, k, v = mk(2, 8, 300, 128), mk(2, 4, 300, 128), mk(2, 4, 300, 128)
    lam = torch.rand(4, generator=g) * 0.8
    host = da.fwd_v2(q, k, v, lam, causal=True)
    dev = da.fwd_v2(q.to(DEV), k.to(DEV), v.to(DEV), lam.to(DEV), causal=True)
    assert host.device.type == "cpu" and torch.equal(host, dev.cpu())
    q1, q2 = mk(2, 6, 200, 64, std=0.125), mk(2, 6, 200, 64, std=0.125)
    k1, k2, vv = mk(2, 3, 200, 64, std=0.125), mk(2, 3, 200, 64, std=0.125), mk(2, 3, 200, 128, std=0.125)
    lam1 = torch.rand(6, generator=g) * 0.8
    host = da.fwd_v1(q1, k1, q2, k2, vv, lam1, causal=True, rmsnorm=True)
    dev = da.fwd_v1(q1.to(DEV), k1.to(DEV), q2.to(DEV), k2.to(DEV), vv.to(DEV), lam1.to(DEV), causal=True,
                    rmsnorm=True)
    assert torch.equal(host, dev.cpu())
