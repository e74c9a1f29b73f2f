"""Runs bench.main() on the host with the GPU and the library faked, to check
the bench's control flow and the keys of its JSON line (not any number).

    python tests/host/bench_flow.py [bench arguments]

Every library call returns OK without computing and CUDA events report 1 ms;
the binding's own argument checks stay, so every call the bench makes is
checked for shape and dtype.  Workloads are shrunk: only the flow is tested.
Prints the JSON line.  Test scaffolding only: nothing else imports it."""

import contextlib
import ctypes
import io
import json
import math
import os
import sys
import types

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import differential_attention_transformers_b200 as da  # noqa: E402
from differential_attention_transformers_b200 import inputs  # noqa: E402


class _Lib:
    """Stands in for libdiffattn.so: every entry point returns OK."""

    def __getattr__(self, name):
        if name == "diffattn_last_error":
            return lambda: b"stub"
        if name == "diffattn_lambda_init":
            return lambda layer: 0.8 - 0.6 * math.exp(-0.3 * (layer - 1))
        if name.endswith("workspace_size"):
            return lambda *a: 1024
        return lambda *a: 0


class _Event:
    def __init__(self, *a, **k):
        pass

    def record(self, *a, **k):
        pass

    def elapsed_time(self, other):
        return 1.0


class _TorchOnHost(types.ModuleType):
    """torch, with CUDA devices mapped to the host and CUDA events faked."""

    def __getattr__(self, name):
        return getattr(torch, name)


def main(argv):
    da._lib = _Lib()
    da.load = lambda: da._lib
    da._prep = lambda ts: (False, list(ts))
    da._device_only = lambda named: None
    da._stream = lambda: ctypes.c_void_p(0)
    da._workspace = lambda n, device: torch.empty(max(n, 16), dtype=torch.uint8)
    da._pipelined = lambda tensors, out: False
    torch.Tensor.pin_memory = lambda self, *a, **k: self
    host_torch = _TorchOnHost("torch")
    host_torch.device = lambda *a, **k: torch.device("cpu")
    host_torch.cuda = types.SimpleNamespace(Event=_Event, synchronize=lambda *a, **k: None,
                                            set_device=lambda *a: None, current_device=lambda: 0,
                                            empty_cache=lambda: None)
    for name, kw in (("v2_prefill", dict(Lq=256, Lk=256)), ("v1_prefill", dict(Lq=256, Lk=256, B=2)),
                     ("v2_decode", dict(Lk=2048, B=2)), ("v1_decode", dict(Lk=2048, B=2))):
        inputs.WORKLOADS[name] = inputs.with_shape(inputs.WORKLOADS[name], **kw)
    inputs.LOWRANK_SHAPE.update(B=1, H=4, Hkv=2, L=256, r=3)
    inputs.SERVING_SHAPE.update(B=4, min_len=16, max_len=200)
    import bench
    bench.torch = host_torch
    bench.SETTLE_S = 0.0
    bench.SnrSweep.__init__.__defaults__ = (4, (1024, 2048))
    sys.argv = ["bench.py"] + argv
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main()
    lines = [l for l in buf.getvalue().splitlines() if l.startswith("{")]
    print(lines[-1] if lines else "{}")
    return rc


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
