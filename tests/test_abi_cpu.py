"""The C ABI library without a GPU: it loads, exports every declared symbol,
and rejects bad arguments before touching the device."""

import ctypes
import os
import re

import pytest

import differential_attention_transformers_b200 as da
from differential_attention_transformers_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "diffattn.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return da.load()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(diffattn_\w+)\s*\(", text)))


@pytest.mark.parametrize("lang,std", [("c", "c99"), ("c++", "c++11")])
def test_header_is_plain_c(lang, std):
    """The boundary header needs no CUDA, torch or C++ types: it compiles alone
    as C99 and as C++11, warnings as errors."""
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    res = subprocess.run([cc, "-fsyntax-only", "-x", lang, f"-std={std}", "-Wall", "-Wextra", "-pedantic", "-Werror",
                          HEADER], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


def test_header_declares_the_binding_exports():
    assert declared_symbols() == sorted(da.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
    # and nothing else of ours leaks out (hidden visibility for internals)
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", da.LIB_PATH], capture_output=True, text=True).stdout
    ours = sorted({l.split()[-1] for l in out.splitlines() if l.split()[-1].startswith("diffattn_")})
    assert ours == declared_symbols()


def test_version_and_lambda_init(L):
    assert "sm_100a" in da.version()
    assert da.lambda_init(1) == pytest.approx(0.2, abs=1e-15)
    import math
    for l in (1, 2, 12, 24):
        assert da.lambda_init(l) == 0.8 - 0.6 * math.exp(-0.3 * (l - 1))
    assert math.isnan(da.lambda_init(0))


def test_argument_errors_before_any_device_call(L):
    P = ctypes.c_void_p(64)  # never dereferenced: validation fails first
    s = ctypes.c_void_p(0)
    # Hq odd
    assert L.diffattn_fwd_v2(P, P, P, P, P, da.BF16, 1, 3, 1, 8, 8, 128, 1, s) == da.ERR_INVALID_ARG
    # a pair straddling two KV groups (Hq/Hkv odd)
    assert L.diffattn_fwd_v2(P, P, P, P, P, da.BF16, 1, 6, 2, 8, 8, 128, 1, s) == da.ERR_INVALID_ARG
    assert "Hq" in da.last_error()
    # null pointer
    assert L.diffattn_fwd_v2(None, P, P, P, P, da.BF16, 1, 4, 2, 8, 8, 128, 1, s) == da.ERR_INVALID_ARG
    # negative sizes
    assert L.diffattn_fwd_v1(P, P, P, P, P, P, P, da.BF16, 1, 2, 1, -1, 8, 64, 128, 1, 0, 1e-5, s) == da.ERR_INVALID_ARG
    # H not a multiple of Hkv
    assert L.diffattn_fwd_v1(P, P, P, P, P, P, P, da.BF16, 1, 3, 2, 8, 8, 64, 128, 1, 0, 1e-5, s) == da.ERR_INVALID_ARG
    # unknown dtype
    assert L.diffattn_fwd_v2(P, P, P, P, P, 7, 1, 4, 2, 8, 8, 128, 1, s) == da.ERR_INVALID_ARG
    # unsupported bf16 widths
    assert L.diffattn_fwd_v2(P, P, P, P, P, da.BF16, 1, 4, 2, 8, 8, 96, 1, s) == da.ERR_UNSUPPORTED
    assert L.diffattn_fwd_v1(P, P, P, P, P, P, P, da.BF16, 1, 2, 1, 8, 8, 32, 128, 1, 0, 1e-5, s) == da.ERR_UNSUPPORTED
    # misaligned bf16 pointer (16-byte rule of tensor-map copies)
    Pm = ctypes.c_void_p(66)
    assert L.diffattn_fwd_v2(Pm, P, P, P, P, da.BF16, 1, 4, 2, 8, 8, 128, 1, s) == da.ERR_MISALIGNED
    # lambda: bad sizes / null
    assert L.diffattn_lambda(P, P, P, P, 0, 8, 0.2, P, s) == da.ERR_INVALID_ARG
    assert L.diffattn_lambda(None, P, P, P, 2, 8, 0.2, P, s) == da.ERR_INVALID_ARG
    # decode
    assert L.diffattn_decode_v2(P, P, P, P, P, da.BF16, 1, 5, 1, 64, 128, P, 1 << 20, s) == da.ERR_INVALID_ARG
    assert L.diffattn_decode_v2(P, P, P, P, P, da.BF16, 1, 32, 2, 64, 128, P, 1 << 20, s) == da.ERR_UNSUPPORTED
    assert L.diffattn_decode_v1(P, P, P, P, P, P, P, da.BF16, 1, 16, 2, 64, 64, 128, 1, P, 1 << 20, s) == da.ERR_UNSUPPORTED
    # paged decode: (q, k_pages, v_pages, table, lens, lambda, out, dtype, B, Hq, Hkv, num_pages, page_size,
    # max_pages, ws, ws_bytes, stream)
    pg = lambda *args: L.diffattn_decode_v2_paged(*args)  # noqa: E731
    assert pg(P, P, P, P, P, P, P, da.BF16, 0, 16, 2, 8, 16, 4, P, 1 << 20, s) == da.ERR_INVALID_ARG     # B = 0
    assert pg(P, P, P, P, P, P, P, da.BF16, 4096, 16, 2, 8, 16, 4, P, 1 << 20, s) == da.ERR_INVALID_ARG  # B > 2048
    assert pg(P, P, P, P, P, P, P, da.BF16, 2, 6, 2, 8, 16, 4, P, 1 << 20, s) == da.ERR_INVALID_ARG      # Hq/Hkv odd
    assert pg(P, P, P, P, P, P, P, da.BF16, 2, 16, 2, 0, 16, 4, P, 1 << 20, s) == da.ERR_INVALID_ARG     # no pages
    assert pg(P, P, P, P, P, P, P, da.BF16, 2, 16, 2, 8, 48, 4, P, 1 << 20, s) == da.ERR_UNSUPPORTED     # page size
    assert "page_size" in da.last_error()
    assert pg(P, P, P, P, P, P, P, da.F32, 2, 16, 2, 8, 16, 4, P, 1 << 20, s) == da.ERR_UNSUPPORTED      # f32
    assert pg(P, P, P, P, P, P, P, da.BF16, 2, 32, 2, 8, 16, 4, P, 1 << 20, s) == da.ERR_UNSUPPORTED     # 16 per group
    assert pg(P, P, P, None, P, P, P, da.BF16, 2, 16, 2, 8, 16, 4, P, 1 << 20, s) == da.ERR_INVALID_ARG  # null table
    assert pg(Pm, P, P, P, P, P, P, da.BF16, 2, 16, 2, 8, 16, 4, P, 1 << 20, s) == da.ERR_MISALIGNED     # q
    Pi = ctypes.c_void_p(66)
    assert pg(P, P, P, Pi, P, P, P, da.BF16, 2, 16, 2, 8, 16, 4, P, 1 << 20, s) == da.ERR_MISALIGNED     # table
    assert pg(P, P, P, P, P, P, P, da.BF16, 2048, 16, 8, 8, 256, 1 << 20, P, 1 << 20, s) == da.ERR_UNSUPPORTED
    assert "2^31" in da.last_error()
    # training forward and backward: (q, k, v, lambda, out, lse, o_maps, dtype, B, Hq, Hkv, Lq, Lk, D, causal, s)
    assert L.diffattn_fwd_v2_train(P, P, P, P, P, P, P, da.F32, 1, 4, 2, 8, 8, 128, 1, s) == da.ERR_UNSUPPORTED
    assert L.diffattn_fwd_v2_train(P, P, P, P, P, None, P, da.BF16, 1, 4, 2, 8, 8, 128, 1, s) == da.ERR_INVALID_ARG
    assert L.diffattn_fwd_v2_train(P, P, P, P, P, P, P, da.BF16, 1, 6, 2, 8, 8, 128, 1, s) == da.ERR_INVALID_ARG
    assert L.diffattn_fwd_v2_train(P, P, P, P, P, P, P, da.BF16, 1, 4, 2, 8, 8, 64, 1, s) == da.ERR_UNSUPPORTED
    bw = lambda *args: L.diffattn_bwd_v2(*args)  # noqa: E731
    # (q, k, v, lambda, dout, lse, o_maps, dq, dk, dv, dlambda, dtype, B, Hq, Hkv, Lq, Lk, D, causal, ws, bytes, s)
    assert bw(P, P, P, P, P, P, P, P, P, P, P, da.F32, 1, 4, 2, 8, 8, 128, 1, P, 1 << 20, s) == da.ERR_UNSUPPORTED
    assert bw(P, P, P, P, P, P, P, P, P, P, P, da.BF16, 1, 4, 3, 8, 8, 128, 1, P, 1 << 20, s) == da.ERR_INVALID_ARG
    # Hq/Hkv odd: a diff pair's two maps must share a KV head (the key-stationary kernel takes them in
    # consecutive steps and shares dP between them)
    assert bw(P, P, P, P, P, P, P, P, P, P, P, da.BF16, 1, 6, 2, 8, 8, 128, 1, P, 1 << 20, s) == da.ERR_INVALID_ARG
    assert bw(P, P, P, P, P, None, P, P, P, P, P, da.BF16, 1, 4, 2, 8, 8, 128, 1, P, 1 << 20, s) == da.ERR_INVALID_ARG
    assert bw(P, P, P, P, P, P, P, Pm, P, P, P, da.BF16, 1, 4, 2, 8, 8, 128, 1, P, 1 << 20, s) == da.ERR_MISALIGNED
    assert L.diffattn_bwd_v2_workspace_size(2, 64, 8192) > 0
    assert L.diffattn_bwd_v2_workspace_size(2, 63, 8192) == 0
    # V1 training forward: (q1, k1, q2, k2, v, lambda, out, lse, o_maps, rstd, o2_coef, dtype, B, H, Hkv, Lq, Lk,
    # d, dv, causal, rmsnorm, eps, s)
    f1 = lambda *args: L.diffattn_fwd_v1_train(*args)  # noqa: E731
    assert f1(P, P, P, P, P, P, P, P, P, P, P, da.F32, 1, 2, 1, 8, 8, 64, 128, 1, 0, 1e-5, s) == da.ERR_UNSUPPORTED
    assert f1(P, P, P, P, P, P, P, P, P, P, P, da.BF16, 1, 2, 1, 8, 8, 128, 128, 1, 0, 1e-5, s) == da.ERR_UNSUPPORTED
    assert f1(P, P, P, P, P, P, P, P, P, None, P, da.BF16, 1, 2, 1, 8, 8, 64, 128, 1, 1, 1e-5, s) == da.ERR_INVALID_ARG
    assert f1(P, P, P, P, P, P, P, P, P, P, None, da.BF16, 1, 2, 1, 8, 8, 64, 128, 1, 1, 1e-5, s) == da.ERR_INVALID_ARG
    assert f1(P, P, P, P, P, P, P, P, P, P, P, da.BF16, 1, 3, 2, 8, 8, 64, 128, 1, 0, 1e-5, s) == da.ERR_INVALID_ARG
    assert f1(P, P, P, P, P, P, P, P, Pm, P, P, da.BF16, 1, 2, 1, 8, 8, 64, 128, 1, 0, 1e-5, s) == da.ERR_MISALIGNED
    # V1 backward: (q1, k1, q2, k2, v, lambda, dout, out, lse, o_maps, rstd, o2_coef, dq1, dk1, dq2, dk2, dv,
    # dlambda, dtype, B, H, Hkv, Lq, Lk, d, dv, causal, rmsnorm, ws, bytes, s)
    b1 = lambda *args: L.diffattn_bwd_v1(*args)  # noqa: E731
    ptrs = [P] * 18
    assert b1(*ptrs, da.F32, 1, 2, 1, 8, 8, 64, 128, 1, 0, P, 1 << 20, s) == da.ERR_UNSUPPORTED
    assert b1(*ptrs, da.BF16, 1, 2, 1, 8, 8, 128, 128, 1, 0, P, 1 << 20, s) == da.ERR_UNSUPPORTED
    assert b1(*ptrs, da.BF16, 1, 4, 3, 8, 8, 64, 128, 1, 0, P, 1 << 20, s) == da.ERR_INVALID_ARG
    no_out = ptrs[:7] + [None] + ptrs[8:]        # RMSNorm needs the forward output
    assert b1(*no_out, da.BF16, 1, 2, 1, 8, 8, 64, 128, 1, 1, P, 1 << 20, s) == da.ERR_INVALID_ARG
    no_coef = ptrs[:11] + [None] + ptrs[12:]     # ... and the stored coefficient
    assert b1(*no_coef, da.BF16, 1, 2, 1, 8, 8, 64, 128, 1, 1, P, 1 << 20, s) == da.ERR_INVALID_ARG
    bad_dq = ptrs[:12] + [Pm] + ptrs[13:]
    assert b1(*bad_dq, da.BF16, 1, 2, 1, 8, 8, 64, 128, 1, 0, P, 1 << 20, s) == da.ERR_MISALIGNED
    w_rms = L.diffattn_bwd_v1_workspace_size(8, 16, 16, 4096, 4096, 1)
    w_plain = L.diffattn_bwd_v1_workspace_size(8, 16, 16, 4096, 4096, 0)
    assert w_rms == w_plain + 8 * 16 * 4096 * (256 + 8) and w_plain == L.diffattn_bwd_v2_workspace_size(8, 32, 4096)
    assert L.diffattn_bwd_v1_workspace_size(1, 3, 2, 8, 8, 0) == 0
    assert L.diffattn_lambda_backward(P, P, P, P, P, 0, 8, P, P, P, P, s) == da.ERR_INVALID_ARG
    assert L.diffattn_lambda_backward(P, P, P, None, P, 2, 8, P, P, P, P, s) == da.ERR_INVALID_ARG
    # low-rank forward: (q, k, v, F, G, lambda, out, dtype, B, H, Hkv, Lq, Lk, D, r, causal, ws, bytes, s)
    lrf = lambda *args: L.diffattn_fwd_lowrank(*args)  # noqa: E731
    p7 = [P] * 7
    assert lrf(*p7, da.BF16, 1, 6, 2, 8, 8, 128, 4, 1, P, 1 << 20, s) == da.ERR_INVALID_ARG    # H/Hkv odd
    assert lrf(*p7, da.F32, 1, 4, 2, 8, 8, 128, 4, 1, P, 1 << 20, s) == da.ERR_UNSUPPORTED
    assert lrf(*p7, da.BF16, 1, 4, 2, 8, 8, 64, 4, 1, P, 1 << 20, s) == da.ERR_UNSUPPORTED
    assert lrf(*p7, da.BF16, 1, 4, 2, 8, 8, 128, 17, 1, P, 1 << 20, s) == da.ERR_UNSUPPORTED   # r > 16
    assert lrf(*p7, da.BF16, 1, 4, 2, 8, 8, 128, 0, 1, P, 1 << 20, s) == da.ERR_INVALID_ARG
    no_f = [P, P, P, None, P, P, P]
    assert lrf(*no_f, da.BF16, 1, 4, 2, 8, 8, 128, 4, 1, P, 1 << 20, s) == da.ERR_INVALID_ARG
    bad_out = [P] * 6 + [Pm]
    assert lrf(*bad_out, da.BF16, 1, 4, 2, 8, 8, 128, 4, 1, P, 1 << 20, s) == da.ERR_MISALIGNED
    assert lrf(*p7, da.BF16, 1, 4, 2, 8, 8, 128, 4, 1, P, 16, s) == da.ERR_WORKSPACE
    w1 = L.diffattn_fwd_lowrank_workspace_size(2, 32, 8192, 8192, 16, 1)
    assert w1 > 2 * 32 * 8192 * 256 and L.diffattn_fwd_lowrank_workspace_size(2, 32, 8192, 8192, 17, 1) == 0


def test_binding_has_no_cpu_fallback(monkeypatch):
    """With the library missing, the product path raises instead of computing elsewhere."""
    monkeypatch.setattr(da, "_lib", None)
    monkeypatch.setattr(da, "LIB_PATH", "/nonexistent/libdiffattn.so")
    with pytest.raises(RuntimeError, match="missing"):
        da.load()


def test_plain_c_client_links_and_runs(L, tmp_path):
    """A C program built against the header and linked to the library (no
    Python) gets the version, lambda_init, argument errors and workspace sizes."""
    import shutil
    import subprocess
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no host compiler")
    exe = str(tmp_path / "abi_c_client")
    libdir = os.path.dirname(da.LIB_PATH)
    res = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", os.path.join(ROOT, "tests", "host", "abi_c_client.c"),
                          "-I", os.path.join(ROOT, "include"), "-L", libdir, "-ldiffattn", "-lm", "-o", exe],
                         capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    env = dict(os.environ, LD_LIBRARY_PATH=libdir + os.pathsep + os.environ.get("LD_LIBRARY_PATH", ""))
    run = subprocess.run([exe], capture_output=True, text=True, env=env)
    assert run.returncode == 0 and run.stdout.strip() == "ok", (run.returncode, run.stderr)
