"""Signal-to-noise of one attention row against context length, on the decode kernel.

("差分注意力" tutorial, Step 1, Step 3 and exercise 1.)  One query sees key 0
as its strong match among N - 1 unrelated keys.  Step 1 measures the weight
that plain softmax leaves on the unrelated keys (the noise floor); Step 3
defines SNR = weight on the signal key / mean weight on the noise keys, for
plain softmax and for the difference A1 - lambda A2; exercise 1 asks for that
curve from 1k to 256k keys.

The construction (``inputs.noise_sweep``) gives V two indicator columns, so
one bf16 V1 decode of each instance returns, in output column 0, the row's
weight on the signal key and, in column 1, its total weight on the noise keys:

    O[0] = A[0],   O[1] = sum_{j >= 1} A[j],   SNR = O[0] (N - 1) / O[1]

with A = A1 for plain softmax (lambda = 0) and A = A1 - lambda A2 for the
difference.  All attention arithmetic runs in the library's decode kernel;
this module only forms the ratios and summarises them.
"""

from __future__ import annotations

import torch

from . import decode_v1, inputs


def probe(x, lam):
    """Signal weight and total noise weight per instance ([n] f32 each) of the
    construction ``x`` (inputs.noise_sweep / sweep_prefix) under per-head
    lambda ``lam`` (f32 [1] on the device): one decode_v1 call."""
    out = decode_v1(x["q1"], x["k1"], x["q2"], x["k2"], x["v"], lam)
    return out[:, 0, 0].float(), out[:, 0, 1].float()


def snr(signal, noise, N: int):
    """SNR = signal weight / mean noise weight over the N - 1 noise keys."""
    return signal * (N - 1) / noise


def _quartiles(t):
    q = torch.quantile(t.double().cpu(), torch.tensor([0.25, 0.5, 0.75], dtype=torch.float64))
    return [float(v) for v in q]


def summarize(N: int, sig_plain, noise_plain, sig_diff, noise_diff):
    """Quartiles (25 %, median, 75 %) over the instances of one context length."""
    return {
        "N": N,
        "snr_plain": _quartiles(snr(sig_plain, noise_plain, N)),
        "snr_diff": _quartiles(snr(sig_diff, noise_diff, N)),
        "noise_fraction_plain": _quartiles(noise_plain / (sig_plain + noise_plain)),
        "signal_plain": _quartiles(sig_plain),
        "signal_diff": _quartiles(sig_diff),
        "noise_mass_diff": _quartiles(noise_diff),
    }


def sweep(lengths=inputs.SWEEP_LENGTHS, n: int = inputs.SWEEP_INSTANCES, lam_value: float = 0.5, seed: int = 1010,
          device=None):
    """The SNR curve: for each context length, the plain and difference rows of
    the same n instances (shorter contexts are prefixes of the longest).
    Returns one summary dict per length."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    x = inputs.noise_sweep(n, max(lengths), seed, device)
    lam = torch.full((1,), float(lam_value), dtype=torch.float32, device=device)
    zero = torch.zeros_like(lam)
    rows = []
    for N in lengths:
        xp = inputs.sweep_prefix(x, N)
        sp, zp = probe(xp, zero)
        sd, zd = probe(xp, lam)
        rows.append(summarize(N, sp, zp, sd, zd))
        del xp
    return rows
