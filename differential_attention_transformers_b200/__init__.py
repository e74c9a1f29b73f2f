"""B200-native differential attention forward: thin Python binding of libdiffattn.so.

The operation is O = (softmax(Q1 K1^T/sqrt(d)) - lambda softmax(Q2 K2^T/sqrt(d))) V
with lambda = exp(lq1.lk1) - exp(lq2.lk2) + lambda_init ("差分注意力" tutorial,
sections 差分思路, Step 2 and Step 4).  Every step runs in the CUDA kernels
of ``libdiffattn.so`` (C ABI in ``include/diffattn.h``); this module only
marshals torch tensors (device memory, the current stream) into that ABI.
There is no CPU fallback: if the library is missing, every call raises.

Inputs may be CUDA tensors (results stay on the device) or CPU tensors (they
are copied to the current CUDA device, the kernels run there, and the result
is copied back: the end-to-end path).  For large CPU inputs the prefill
entry points overlap the copies with the kernels: the work is cut into chunks
of (batch, KV-head group), each uploaded, computed and downloaded on its own
stream, so chunk c computes while chunk c+1 uploads and chunk c-1 downloads.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdiffattn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_MISALIGNED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = 0, -1, -2, -3, -4, -5, -6
F32, BF16 = 0, 1

EXPORTS = ["diffattn_version", "diffattn_lambda_init", "diffattn_lambda", "diffattn_fwd_v1", "diffattn_fwd_v2",
           "diffattn_decode_workspace_size", "diffattn_decode_v2_workspace_size", "diffattn_decode_v2",
           "diffattn_decode_v1", "diffattn_last_error",
           "diffattn_last_status", "diffattn_set_wait_limit_ns", "diffattn_decode_v2_noalloc",
           "diffattn_decode_paged_workspace_size", "diffattn_decode_v2_paged", "diffattn_fwd_v2_train",
           "diffattn_bwd_v2_workspace_size", "diffattn_bwd_v2", "diffattn_lambda_backward",
           "diffattn_fwd_v1_train", "diffattn_bwd_v1_workspace_size", "diffattn_bwd_v1",
           "diffattn_fwd_lowrank_workspace_size", "diffattn_fwd_lowrank"]

_lib = None


class DiffAttnError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"diffattn error {code}: {msg}")
        self.code = code


def load():
    """Load libdiffattn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m differential_attention_transformers_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, D, Z, U = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_double, ctypes.c_size_t, ctypes.c_ulonglong
    sig = {
        "diffattn_version": (ctypes.c_char_p, []),
        "diffattn_lambda_init": (D, [I]),
        "diffattn_lambda": (I, [P, P, P, P, I, I, D, P, P]),
        "diffattn_fwd_v1": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, F, P]),
        "diffattn_fwd_v2": (I, [P, P, P, P, P, I, I, I, I, I, I, I, I, P]),
        "diffattn_decode_workspace_size": (Z, [I, I, I, I]),
        "diffattn_decode_v2_workspace_size": (Z, [I, I, I, I]),
        "diffattn_decode_v2": (I, [P, P, P, P, P, I, I, I, I, I, I, P, Z, P]),
        "diffattn_decode_v1": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, Z, P]),
        "diffattn_last_error": (ctypes.c_char_p, []),
        "diffattn_last_status": (I, [P]),
        "diffattn_set_wait_limit_ns": (None, [U]),
        "diffattn_decode_v2_noalloc": (I, [P, P, P, P, P, I, I, I, I, I, I, P]),
        "diffattn_decode_paged_workspace_size": (Z, [I, I]),
        "diffattn_decode_v2_paged": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, Z, P]),
        "diffattn_fwd_v2_train": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P]),
        "diffattn_bwd_v2_workspace_size": (Z, [I, I, I]),
        "diffattn_bwd_v2": (I, [P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, Z, P]),
        "diffattn_lambda_backward": (I, [P, P, P, P, P, I, I, P, P, P, P, P]),
        "diffattn_fwd_v1_train": (I, [P] * 11 + [I] * 10 + [F, P]),
        "diffattn_bwd_v1_workspace_size": (Z, [I] * 6),
        "diffattn_bwd_v1": (I, [P] * 18 + [I] * 10 + [P, Z, P]),
        "diffattn_fwd_lowrank_workspace_size": (Z, [I] * 6),
        "diffattn_fwd_lowrank": (I, [P] * 7 + [I] * 9 + [P, Z, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    env = os.environ.get("DIFFATTN_WAIT_LIMIT_NS")
    if env:
        L.diffattn_set_wait_limit_ns(int(env))
    _lib = L
    return L


def _check(code):
    if code != OK:
        raise DiffAttnError(code, load().diffattn_last_error().decode())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}: use bfloat16 or float32")


def _expect(*specs):
    """Shape and dtype checks, made before anything reaches the library: the C
    ABI takes plain pointers and sizes, so a tensor smaller than the sizes say
    would be read or written out of bounds.  specs: (name, tensor, shape, dtype
    or None)."""
    for name, t, shape, dt in specs:
        if t is None:
            raise ValueError(f"{name} is required")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if dt is not None and t.dtype != dt:
            raise ValueError(f"{name} must be {dt}, got {t.dtype}")


def _dims(name, t, n):
    if t is None or t.dim() != n:
        raise ValueError(f"{name} must be a {n}-d tensor")
    return tuple(t.shape)


def _device_only(named):
    """Entry points that take device tensors: contiguous, on the current CUDA device."""
    for name, t in named:
        if t is None:
            continue
        if t.device.type != "cuda":
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    dev = torch.cuda.current_device()
    for name, t in named:
        if t is not None and t.device.index != dev:
            raise ValueError(f"{name} is on cuda:{t.device.index}, the current device is cuda:{dev}")


def _prep(tensors):
    """Move CPU inputs to the current CUDA device; report whether we did."""
    host = any(t.device.type == "cpu" for t in tensors)
    dev = torch.device("cuda", torch.cuda.current_device())
    out = []
    for t in tensors:
        if t.device.type == "cuda" and t.device.index != dev.index:
            raise ValueError(f"a tensor is on cuda:{t.device.index}, the current device is cuda:{dev.index}")
        if t.device.type == "cpu":
            t = t.pin_memory().to(dev, non_blocking=True) if not t.is_pinned() else t.to(dev, non_blocking=True)
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        out.append(t)
    return host, out


def _finish(host, out):
    if not host:
        return out
    res = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    res.copy_(out, non_blocking=True)
    torch.cuda.current_stream().synchronize()
    return res


# ----------------------------------------------------------------------------
def version() -> str:
    return load().diffattn_version().decode()


def lambda_init(layer: int) -> float:
    """0.8 - 0.6 exp(-0.3 (layer - 1)), layer counted from 1."""
    return float(load().diffattn_lambda_init(int(layer)))


def compute_lambda(lq1, lk1, lq2, lk2, lam_init: float, out=None):
    """Per-head lambda (f32 [H]) from f32 [H, dim] parameters, on the GPU."""
    host, (lq1, lk1, lq2, lk2) = _prep([lq1, lk1, lq2, lk2])
    H, dim = lq1.shape
    for t in (lq1, lk1, lq2, lk2):
        if t.dtype != torch.float32 or tuple(t.shape) != (H, dim):
            raise ValueError("lq1, lk1, lq2, lk2 must be float32 [H, dim]")
    if out is None:
        out = torch.empty(H, dtype=torch.float32, device=lq1.device)
    _check(load().diffattn_lambda(_ptr(lq1), _ptr(lk1), _ptr(lq2), _ptr(lk2), H, dim, float(lam_init),
                                  _ptr(out), _stream()))
    return _finish(host, out)


# ----------------------------------------------------------------------------
# end-to-end prefill on host tensors: chunked, with copies overlapping kernels
_PIPELINE_MIN_BYTES = 64 << 20     # smaller inputs take the plain copy-compute-copy path
_PIPELINE_CHUNK_UNITS = 256        # 128-row blocks per chunk kernel
_pipe_streams = {}


def _pipelined(tensors, out):
    return (out is None and all(t.device.type == "cpu" for t in tensors)
            and sum(t.numel() * t.element_size() for t in tensors) >= _PIPELINE_MIN_BYTES)


def _prefill_host_pipelined(v1, qs, ks, v, lam, causal, rmsnorm, eps):
    """CPU q/k/v in, pinned CPU output back.  qs: [q] (V2) or [q1, q2] (V1);
    ks: [k] or [k1, k2].  Chunk = one batch entry and a run of whole KV heads
    (with their query heads and outputs), all contiguous slices."""
    dev = torch.device("cuda", torch.cuda.current_device())
    pin = lambda t: t.contiguous() if t.is_pinned() else t.contiguous().pin_memory()  # noqa: E731
    qs, ks, v = [pin(t) for t in qs], [pin(t) for t in ks], pin(v)
    B, Hq, Lq, d = qs[0].shape
    Hkv, Lk, dv = ks[0].shape[1], ks[0].shape[2], v.shape[3]
    if Hkv < 1 or Hq % Hkv:
        raise ValueError("query heads must be a multiple of the KV heads")
    grp = Hq // Hkv
    opg = grp if v1 else grp // 2                       # output heads per KV head
    Hout = Hq if v1 else Hq // 2
    n_rb = -(-Lq // 128)
    gpc = max(1, min(Hkv, -(-_PIPELINE_CHUNK_UNITS // max(1, n_rb * opg))))
    chunks = [(b, g0, min(Hkv, g0 + gpc)) for b in range(B) for g0 in range(0, Hkv, gpc)]

    lam_d = lam.to(dev, non_blocking=False).contiguous()
    qd = [torch.empty(t.shape, dtype=t.dtype, device=dev) for t in qs]
    kd = [torch.empty(t.shape, dtype=t.dtype, device=dev) for t in ks]
    vd = torch.empty(v.shape, dtype=v.dtype, device=dev)
    out_d = torch.empty((B, Hout, Lq, dv), dtype=qs[0].dtype, device=dev)
    out_h = torch.empty(out_d.shape, dtype=out_d.dtype, pin_memory=True)
    if dev.index not in _pipe_streams:
        _pipe_streams[dev.index] = tuple(torch.cuda.Stream(device=dev) for _ in range(3))
    s_in, s_run, s_out = _pipe_streams[dev.index]
    for st in (s_in, s_run, s_out):
        st.wait_stream(torch.cuda.current_stream())
    L, dt = load(), _dtype_code(qs[0])
    for b, g0, g1 in chunks:
        hq, hk, ho = slice(g0 * grp, g1 * grp), slice(g0, g1), slice(g0 * opg, g1 * opg)
        with torch.cuda.stream(s_in):
            for dst, src in zip(qd, qs):
                dst[b, hq].copy_(src[b, hq], non_blocking=True)
            for dst, src in zip(kd, ks):
                dst[b, hk].copy_(src[b, hk], non_blocking=True)
            vd[b, hk].copy_(v[b, hk], non_blocking=True)
        s_run.wait_stream(s_in)
        with torch.cuda.stream(s_run):
            nq, nk = (g1 - g0) * grp, g1 - g0
            if v1:
                _check(L.diffattn_fwd_v1(_ptr(qd[0][b, hq]), _ptr(kd[0][b, hk]), _ptr(qd[1][b, hq]),
                                         _ptr(kd[1][b, hk]), _ptr(vd[b, hk]), _ptr(lam_d[ho]), _ptr(out_d[b, ho]),
                                         dt, 1, nq, nk, Lq, Lk, d, dv, int(causal), int(rmsnorm), float(eps),
                                         _stream()))
            else:
                _check(L.diffattn_fwd_v2(_ptr(qd[0][b, hq]), _ptr(kd[0][b, hk]), _ptr(vd[b, hk]), _ptr(lam_d[ho]),
                                         _ptr(out_d[b, ho]), dt, 1, nq, nk, Lq, Lk, d, int(causal), _stream()))
        s_out.wait_stream(s_run)
        with torch.cuda.stream(s_out):
            out_h[b, ho].copy_(out_d[b, ho], non_blocking=True)
    s_out.synchronize()
    return out_h


def fwd_v1(q1, k1, q2, k2, v, lam, causal=True, rmsnorm=False, eps=1e-5, out=None):
    """V1 layout: q1,q2 [B,H,Lq,d]; k1,k2 [B,Hkv,Lk,d]; v [B,Hkv,Lk,dv]; lam f32 [H]."""
    B, H, Lq, d = _dims("q1", q1, 4)
    _, Hkv, Lk, _ = _dims("k1", k1, 4)
    dv = _dims("v", v, 4)[3]
    _expect(("q2", q2, (B, H, Lq, d), q1.dtype), ("k1", k1, (B, Hkv, Lk, d), q1.dtype),
            ("k2", k2, (B, Hkv, Lk, d), q1.dtype), ("v", v, (B, Hkv, Lk, dv), q1.dtype),
            ("lam", lam, (H,), torch.float32))
    if out is not None:
        _expect(("out", out, (B, H, Lq, dv), q1.dtype))
    if _pipelined([q1, k1, q2, k2, v], out):
        return _prefill_host_pipelined(True, [q1, q2], [k1, k2], v, lam, causal, rmsnorm, eps)
    host, (q1, k1, q2, k2, v, lam) = _prep([q1, k1, q2, k2, v, lam])
    B, H, Lq, d = q1.shape
    Hkv, Lk, dv = k1.shape[1], k1.shape[2], v.shape[3]
    dt = _dtype_code(q1)
    if out is None:
        out = torch.empty((B, H, Lq, dv), dtype=q1.dtype, device=q1.device)
    _check(load().diffattn_fwd_v1(_ptr(q1), _ptr(k1), _ptr(q2), _ptr(k2), _ptr(v), _ptr(lam), _ptr(out), dt,
                                  B, H, Hkv, Lq, Lk, d, dv, int(causal), int(rmsnorm), float(eps), _stream()))
    return _finish(host, out)


def fwd_v2(q, k, v, lam, causal=True, out=None):
    """V2 layout: q [B,Hq,Lq,D]; k,v [B,Hkv,Lk,D]; lam f32 [Hq/2] -> [B,Hq/2,Lq,D]."""
    B, Hq, Lq, D = _dims("q", q, 4)
    _, Hkv, Lk, _ = _dims("k", k, 4)
    _expect(("k", k, (B, Hkv, Lk, D), q.dtype), ("v", v, (B, Hkv, Lk, D), q.dtype),
            ("lam", lam, (Hq // 2,), torch.float32))
    if out is not None:
        _expect(("out", out, (B, Hq // 2, Lq, D), q.dtype))
    if _pipelined([q, k, v], out):
        return _prefill_host_pipelined(False, [q], [k], v, lam, causal, False, 1e-5)
    host, (q, k, v, lam) = _prep([q, k, v, lam])
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((B, Hq // 2, Lq, D), dtype=q.dtype, device=q.device)
    _check(load().diffattn_fwd_v2(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out), dt, B, Hq, Hkv, Lq, Lk, D,
                                  int(causal), _stream()))
    return _finish(host, out)


def fwd_v2_train(q, k, v, lam, causal=True):
    """V2 forward that also returns what the backward needs: (out [B,Hq/2,Lq,D],
    lse f32 [B,Hq/2,2,Lq] (log2 units), o_maps [B,Hq/2,2,Lq,D] = O_m / l_m).  bf16, device tensors."""
    B, Hq, Lq, D = _dims("q", q, 4)
    _, Hkv, Lk, _ = _dims("k", k, 4)
    _expect(("q", q, (B, Hq, Lq, D), torch.bfloat16), ("k", k, (B, Hkv, Lk, D), torch.bfloat16),
            ("v", v, (B, Hkv, Lk, D), torch.bfloat16), ("lam", lam, (Hq // 2,), torch.float32))
    _device_only([("q", q), ("k", k), ("v", v), ("lam", lam)])
    out = torch.empty((B, Hq // 2, Lq, D), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, Hq // 2, 2, Lq), dtype=torch.float32, device=q.device)
    o_maps = torch.empty((B, Hq // 2, 2, Lq, D), dtype=q.dtype, device=q.device)
    _check(load().diffattn_fwd_v2_train(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out), _ptr(lse), _ptr(o_maps),
                                        _dtype_code(q), B, Hq, Hkv, Lq, Lk, D, int(causal), _stream()))
    return out, lse, o_maps


def bwd_v2(q, k, v, lam, dout, lse, o_maps, causal=True, workspace=None):
    """Gradients of the V2 forward: (dq, dk, dv, dlam) given dout [B,Hq/2,Lq,D] and the
    training forward's lse and o_maps.  bf16 gradients, f32 dlam.  Device tensors."""
    B, Hq, Lq, D = _dims("q", q, 4)
    _, Hkv, Lk, _ = _dims("k", k, 4)
    bf, f32, Hp = torch.bfloat16, torch.float32, Hq // 2
    _expect(("q", q, (B, Hq, Lq, D), bf), ("k", k, (B, Hkv, Lk, D), bf), ("v", v, (B, Hkv, Lk, D), bf),
            ("lam", lam, (Hp,), f32), ("dout", dout, (B, Hp, Lq, D), bf), ("lse", lse, (B, Hp, 2, Lq), f32),
            ("o_maps", o_maps, (B, Hp, 2, Lq, D), bf))
    _device_only([("q", q), ("k", k), ("v", v), ("lam", lam), ("dout", dout), ("lse", lse), ("o_maps", o_maps),
                  ("workspace", workspace)])
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dlam = torch.empty(Hq // 2, dtype=torch.float32, device=q.device)
    need = int(load().diffattn_bwd_v2_workspace_size(B, Hq, Lq))
    ws = workspace if workspace is not None else _workspace(need, q.device)
    _check(load().diffattn_bwd_v2(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(dout), _ptr(lse), _ptr(o_maps),
                                  _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlam), _dtype_code(q), B, Hq, Hkv, Lq, Lk, D,
                                  int(causal), _ptr(ws), ws.numel() * ws.element_size(), _stream()))
    return dq, dk, dv, dlam


def fwd_v1_train(q1, k1, q2, k2, v, lam, causal=True, rmsnorm=False, eps=1e-5):
    """V1 forward (bf16, d = 64, dv = 128) that also returns what bwd_v1 needs:
    (out [B,H,Lq,128], lse f32 [B,H,2,Lq], o_maps [B,H,2,Lq,128], rstd f32 [B,H,Lq],
    o2c f32 [B,H,Lq]); rstd and o2c are None without RMSNorm, and with it
    o_maps[:, :, 1] holds map 2's part orthogonal to the difference output
    (see diffattn_fwd_v1_train).  Device tensors."""
    B, H, Lq, d = _dims("q1", q1, 4)
    _, Hkv, Lk, _ = _dims("k1", k1, 4)
    dv = _dims("v", v, 4)[3]
    bf = torch.bfloat16
    _expect(("q1", q1, (B, H, Lq, d), bf), ("q2", q2, (B, H, Lq, d), bf), ("k1", k1, (B, Hkv, Lk, d), bf),
            ("k2", k2, (B, Hkv, Lk, d), bf), ("v", v, (B, Hkv, Lk, dv), bf), ("lam", lam, (H,), torch.float32))
    _device_only([("q1", q1), ("k1", k1), ("q2", q2), ("k2", k2), ("v", v), ("lam", lam)])
    out = torch.empty((B, H, Lq, dv), dtype=q1.dtype, device=q1.device)
    lse = torch.empty((B, H, 2, Lq), dtype=torch.float32, device=q1.device)
    o_maps = torch.empty((B, H, 2, Lq, dv), dtype=q1.dtype, device=q1.device)
    rstd = torch.empty((B, H, Lq), dtype=torch.float32, device=q1.device) if rmsnorm else None
    o2c = torch.empty((B, H, Lq), dtype=torch.float32, device=q1.device) if rmsnorm else None
    _check(load().diffattn_fwd_v1_train(_ptr(q1), _ptr(k1), _ptr(q2), _ptr(k2), _ptr(v), _ptr(lam), _ptr(out),
                                        _ptr(lse), _ptr(o_maps), _ptr(rstd), _ptr(o2c), _dtype_code(q1), B, H, Hkv,
                                        Lq, Lk, d, dv, int(causal), int(rmsnorm), float(eps), _stream()))
    return out, lse, o_maps, rstd, o2c


def bwd_v1(q1, k1, q2, k2, v, lam, dout, out, lse, o_maps, rstd=None, o2c=None, causal=True, rmsnorm=False,
           workspace=None):
    """Gradients of the V1 forward: (dq1, dk1, dq2, dk2, dv, dlam) given dout [B,H,Lq,128]
    and fwd_v1_train's outputs.  bf16 gradients, f32 dlam.  Device tensors."""
    B, H, Lq, d = _dims("q1", q1, 4)
    _, Hkv, Lk, _ = _dims("k1", k1, 4)
    dvw = _dims("v", v, 4)[3]
    bf, f32 = torch.bfloat16, torch.float32
    _expect(("q1", q1, (B, H, Lq, d), bf), ("q2", q2, (B, H, Lq, d), bf), ("k1", k1, (B, Hkv, Lk, d), bf),
            ("k2", k2, (B, Hkv, Lk, d), bf), ("v", v, (B, Hkv, Lk, dvw), bf), ("lam", lam, (H,), f32),
            ("dout", dout, (B, H, Lq, dvw), bf), ("lse", lse, (B, H, 2, Lq), f32),
            ("o_maps", o_maps, (B, H, 2, Lq, dvw), bf))
    if rmsnorm:
        _expect(("out", out, (B, H, Lq, dvw), bf), ("rstd", rstd, (B, H, Lq), f32), ("o2c", o2c, (B, H, Lq), f32))
    _device_only([("q1", q1), ("k1", k1), ("q2", q2), ("k2", k2), ("v", v), ("lam", lam), ("dout", dout),
                  ("out", out), ("lse", lse), ("o_maps", o_maps), ("rstd", rstd), ("o2c", o2c),
                  ("workspace", workspace)])
    dq1, dq2 = torch.empty_like(q1), torch.empty_like(q2)
    dk1, dk2, dv = torch.empty_like(k1), torch.empty_like(k2), torch.empty_like(v)
    dlam = torch.empty(H, dtype=torch.float32, device=q1.device)
    need = int(load().diffattn_bwd_v1_workspace_size(B, H, Hkv, Lq, Lk, int(rmsnorm)))
    ws = workspace if workspace is not None else _workspace(need, q1.device)
    _check(load().diffattn_bwd_v1(_ptr(q1), _ptr(k1), _ptr(q2), _ptr(k2), _ptr(v), _ptr(lam), _ptr(dout),
                                  _ptr(out), _ptr(lse), _ptr(o_maps), _ptr(rstd), _ptr(o2c), _ptr(dq1), _ptr(dk1),
                                  _ptr(dq2),
                                  _ptr(dk2), _ptr(dv), _ptr(dlam), _dtype_code(q1), B, H, Hkv, Lq, Lk, d, dvw,
                                  int(causal), int(rmsnorm), _ptr(ws), ws.numel() * ws.element_size(), _stream()))
    return dq1, dk1, dq2, dk2, dv, dlam


def fwd_lowrank(q, k, v, F, G, lam, causal=True, out=None, workspace=None):
    """Differential attention with a fixed low-rank map in place of A2:
    out = softmax(Q K^T / sqrt(128)) V - lam N V, N[i, j] = f_i.g_j / sum over
    visible j' of f_i.g_j'.  q [B,H,Lq,128], k, v [B,Hkv,Lk,128] bf16; F [H,Lq,r],
    G [H,Lk,r] f32 >= 0; lam f32 [H] -> [B,H,Lq,128].  Device tensors."""
    B, H, Lq, D = _dims("q", q, 4)
    _, Hkv, Lk, _ = _dims("k", k, 4)
    r = _dims("F", F, 3)[2]
    bf, f32 = torch.bfloat16, torch.float32
    _expect(("q", q, (B, H, Lq, D), bf), ("k", k, (B, Hkv, Lk, D), bf), ("v", v, (B, Hkv, Lk, D), bf),
            ("F", F, (H, Lq, r), f32), ("G", G, (H, Lk, r), f32), ("lam", lam, (H,), f32))
    if out is not None:
        _expect(("out", out, (B, H, Lq, D), bf))
    _device_only([("q", q), ("k", k), ("v", v), ("F", F), ("G", G), ("lam", lam), ("out", out),
                  ("workspace", workspace)])
    if out is None:
        out = torch.empty((B, H, Lq, D), dtype=bf, device=q.device)
    need = int(load().diffattn_fwd_lowrank_workspace_size(B, H, Lq, Lk, r, int(causal)))
    ws = workspace if workspace is not None else _workspace(need, q.device)
    _check(load().diffattn_fwd_lowrank(_ptr(q), _ptr(k), _ptr(v), _ptr(F), _ptr(G), _ptr(lam), _ptr(out), BF16,
                                       B, H, Hkv, Lq, Lk, D, r, int(causal), _ptr(ws), ws.numel() * ws.element_size(),
                                       _stream()))
    return out


def lambda_backward(lq1, lk1, lq2, lk2, dlam):
    """Gradients of the four lambda parameter vectors ([H, dim] f32) given dlam [H]."""
    H, dim = _dims("lq1", lq1, 2)
    f32 = torch.float32
    _expect(("lq1", lq1, (H, dim), f32), ("lk1", lk1, (H, dim), f32), ("lq2", lq2, (H, dim), f32),
            ("lk2", lk2, (H, dim), f32), ("dlam", dlam, (H,), f32))
    _device_only([("lq1", lq1), ("lk1", lk1), ("lq2", lq2), ("lk2", lk2), ("dlam", dlam)])
    outs = [torch.empty_like(lq1) for _ in range(4)]
    _check(load().diffattn_lambda_backward(_ptr(lq1), _ptr(lk1), _ptr(lq2), _ptr(lk2), _ptr(dlam), H, dim,
                                           *[_ptr(t) for t in outs], _stream()))
    return tuple(outs)


def decode_workspace_size(B: int, Hkv: int, T: int, dv: int = 128) -> int:
    return int(load().diffattn_decode_workspace_size(B, Hkv, T, dv))


_ws_cache = {}


def _workspace(nbytes, device):
    """Scratch of at least nbytes for a call on the current stream of ``device``:
    one buffer per (device, stream).  Calls on one stream run in order and can
    share it; calls on two streams may overlap, so each stream has its own."""
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def decode_v2(q, kc, vc, lam, out=None, workspace=None):
    """Single-token V2 decode: q [B,Hq,D]; kc,vc [B,Hkv,T,D]; lam [Hq/2] -> [B,Hq/2,D]."""
    B, Hq, D = _dims("q", q, 3)
    _, Hkv, T, _ = _dims("kc", kc, 4)
    _expect(("kc", kc, (B, Hkv, T, D), q.dtype), ("vc", vc, (B, Hkv, T, D), q.dtype),
            ("lam", lam, (Hq // 2,), torch.float32))
    if out is not None:
        _expect(("out", out, (B, Hq // 2, D), q.dtype))
    host, (q, kc, vc, lam) = _prep([q, kc, vc, lam])
    B, Hq, D = q.shape
    Hkv, T = kc.shape[1], kc.shape[2]
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((B, Hq // 2, D), dtype=q.dtype, device=q.device)
    need = decode_workspace_size(B, Hkv, T, D)
    ws = workspace if workspace is not None else _workspace(need, q.device)
    _check(load().diffattn_decode_v2(_ptr(q), _ptr(kc), _ptr(vc), _ptr(lam), _ptr(out), dt, B, Hq, Hkv, T, D,
                                     _ptr(ws), ws.numel() * ws.element_size(), _stream()))
    return _finish(host, out)


def decode_paged_workspace_size(B: int, Hkv: int) -> int:
    return int(load().diffattn_decode_paged_workspace_size(B, Hkv))


def decode_v2_paged(q, k_pages, v_pages, block_table, seq_lens, lam, out=None, workspace=None):
    """Paged, variable-length V2 decode: q [B,Hq,128]; k_pages, v_pages [num_pages, page_size, Hkv, 128];
    block_table int32 [B, max_pages]; seq_lens int32 [B]; lam [Hq/2] -> [B, Hq/2, 128]."""
    B, Hq, D = _dims("q", q, 3)
    P, ps, Hkv, _ = _dims("k_pages", k_pages, 4)
    M = _dims("block_table", block_table, 2)[1]
    _expect(("k_pages", k_pages, (P, ps, Hkv, D), q.dtype), ("v_pages", v_pages, (P, ps, Hkv, D), q.dtype),
            ("block_table", block_table, (B, M), torch.int32), ("seq_lens", seq_lens, (B,), torch.int32),
            ("lam", lam, (Hq // 2,), torch.float32))
    if out is not None:
        _expect(("out", out, (B, Hq // 2, D), q.dtype))
    host, (q, k_pages, v_pages, block_table, seq_lens, lam) = _prep([q, k_pages, v_pages, block_table, seq_lens,
                                                                      lam])
    B, Hq, D = q.shape
    num_pages, page_size, Hkv = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_table and seq_lens must be int32")
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((B, Hq // 2, D), dtype=q.dtype, device=q.device)
    need = decode_paged_workspace_size(B, Hkv)
    ws = workspace if workspace is not None else _workspace(need, q.device)
    _check(load().diffattn_decode_v2_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                                           _ptr(seq_lens), _ptr(lam), _ptr(out), dt, B, Hq, Hkv, num_pages,
                                           page_size, block_table.shape[1], _ptr(ws),
                                           ws.numel() * ws.element_size(), _stream()))
    return _finish(host, out)


def decode_v1(q1, k1, q2, k2, v, lam, fused=True, out=None, workspace=None):
    """Single-token V1-layout decode: q1,q2 [B,H,d]; k1,k2 [B,Hkv,T,d]; v [B,Hkv,T,dv] -> [B,H,dv]."""
    B, H, d = _dims("q1", q1, 3)
    _, Hkv, T, _ = _dims("k1", k1, 4)
    dv = _dims("v", v, 4)[3]
    _expect(("q2", q2, (B, H, d), q1.dtype), ("k1", k1, (B, Hkv, T, d), q1.dtype),
            ("k2", k2, (B, Hkv, T, d), q1.dtype), ("v", v, (B, Hkv, T, dv), q1.dtype),
            ("lam", lam, (H,), torch.float32))
    if out is not None:
        _expect(("out", out, (B, H, dv), q1.dtype))
    host, (q1, k1, q2, k2, v, lam) = _prep([q1, k1, q2, k2, v, lam])
    B, H, d = q1.shape
    Hkv, T, dv = k1.shape[1], k1.shape[2], v.shape[3]
    dt = _dtype_code(q1)
    if out is None:
        out = torch.empty((B, H, dv), dtype=q1.dtype, device=q1.device)
    need = decode_workspace_size(B, Hkv, T, dv)
    ws = workspace if workspace is not None else _workspace(need, q1.device)
    _check(load().diffattn_decode_v1(_ptr(q1), _ptr(k1), _ptr(q2), _ptr(k2), _ptr(v), _ptr(lam), _ptr(out), dt,
                                     B, H, Hkv, T, d, dv, int(fused), _ptr(ws), ws.numel() * ws.element_size(),
                                     _stream()))
    return _finish(host, out)


def last_status() -> int:
    """Synchronise the current stream and read/clear the device status word."""
    return int(load().diffattn_last_status(_stream()))


def last_error() -> str:
    return load().diffattn_last_error().decode()


def set_wait_limit_ns(ns: int) -> None:
    load().diffattn_set_wait_limit_ns(int(ns))
