"""Seeded synthetic inputs for the selective-SSM mixer core.

This module only draws random tensors; it contains none of the mixer's own
arithmetic (no convolution, no softplus of activations, no scan). Both the CUDA
path and the fp64 CPU oracle are fed from it, so that they see bit-identical
inputs.

Value recipe (Mamba-style layer, as the workloads describe it):

* x, z ~ N(0, 1); B, C ~ N(0, 1) per token (one group shared by all channels).
* conv weight ~ N(0, 0.25) read as variance 0.25 (std 0.5); conv bias 0 unless
  a random bias is asked for (then also N(0, 0.25)).
* A[c, n] = -(n + 1) (the S4D-real initialisation); D = 1.
* raw dt = 0.1 * clip(N(0, 1), -3, 3); per channel a target dt0 is drawn
  log-uniform in [1e-3 * e^0.3, 1e-1 * e^-0.3] and dt_bias is the inverse
  softplus of dt0. Because log(softplus) is 1-Lipschitz, softplus(dt + dt_bias)
  then lies in [1e-3, 1e-1].
* bf16 workloads round every activation tensor (x, z, dt, B, C and the conv
  state) to bf16 with round-to-nearest-even; A, D, dt_bias, conv weight and
  bias and the SSM state stay fp32.

Host draws use NumPy's PCG64; the very large workloads are drawn on the device
with a seeded torch generator instead (same distributions, different stream).
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

# Largest bf16 value not above 0.3: raw dt is clipped to it after rounding so
# that the [1e-3, 1e-1] bound on softplus(dt + dt_bias) survives bf16 rounding.
DT_RAW_LIMIT = 0.298828125
DT_LO, DT_HI, DT_MARGIN = 1e-3, 1e-1, 0.3


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); return float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    rounded = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16
    return (rounded.astype(np.uint32) << 16).view(np.float32).reshape(a.shape)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, stream]))


@dataclasses.dataclass
class MixerParams:
    """Per-channel parameters of one mixer layer (all float32)."""

    conv_w: np.ndarray  # (D, K)
    conv_b: np.ndarray  # (D,)
    A: np.ndarray  # (D, N)
    Dskip: np.ndarray  # (D,)
    dt_bias: np.ndarray  # (D,)


def inverse_softplus_bias(dt0: np.ndarray) -> np.ndarray:
    """dt_bias such that softplus(dt_bias) == dt0 (input recipe, not the method)."""
    dt0 = dt0.astype(np.float64)
    return (dt0 + np.log(-np.expm1(-dt0))).astype(np.float32)


def make_params(seed: int, D: int, N: int = 16, K: int = 4, random_bias: bool = False,
                random_A: bool = False, random_D: bool = False) -> MixerParams:
    rng = _rng(seed, 1)
    conv_w = (0.5 * rng.standard_normal((D, K))).astype(np.float32)
    conv_b = ((0.5 * rng.standard_normal(D)) if random_bias else np.zeros(D)).astype(np.float32)
    if random_A:
        # general negative reals (used by unit tests so that nothing relies on
        # the structure of the S4D-real initialisation)
        A = (-np.exp(rng.uniform(np.log(0.05), np.log(20.0), (D, N)))).astype(np.float32)
    else:
        A = np.tile(-(np.arange(N, dtype=np.float32) + 1.0), (D, 1))
    Dskip = (rng.standard_normal(D) if random_D else np.ones(D)).astype(np.float32)
    lo = math.log(DT_LO) + DT_MARGIN
    hi = math.log(DT_HI) - DT_MARGIN
    dt0 = np.exp(rng.uniform(lo, hi, D))
    dt_bias = inverse_softplus_bias(dt0)
    return MixerParams(conv_w, conv_b, A, Dskip, dt_bias)


def sample_lengths(seed: int, total: int, lo: int = 128, hi: int = 8192) -> np.ndarray:
    """Packed sequence lengths: log-uniform in [lo, hi] until the sum reaches
    `total`; the last length is cut so the lengths add up to exactly `total`."""
    rng = _rng(seed, 3)
    lens = []
    acc = 0
    while acc < total:
        L = int(round(math.exp(rng.uniform(math.log(lo), math.log(hi)))))
        L = min(L, total - acc)
        lens.append(L)
        acc += L
    return np.asarray(lens, dtype=np.int64)


def cu_from_lengths(lens) -> np.ndarray:
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lens, dtype=np.int64))
    return cu


def _raw_dt(rng: np.random.Generator, shape, bf16: bool) -> np.ndarray:
    dt = (0.1 * np.clip(rng.standard_normal(shape), -3.0, 3.0)).astype(np.float32)
    if bf16:
        dt = np.clip(round_bf16(dt), -DT_RAW_LIMIT, DT_RAW_LIMIT)
    return dt


def make_activations(seed: int, tok: int, D: int, N: int = 16, bf16: bool = True,
                     stream: int = 2) -> dict:
    """x, z, raw dt: (tok, D); B, C: (tok, N). float32 arrays (bf16-exact when bf16)."""
    rng = _rng(seed, stream)
    rnd = round_bf16 if bf16 else (lambda a: a.astype(np.float32))
    out = {}
    out["x"] = rnd(rng.standard_normal((tok, D), dtype=np.float32))
    out["z"] = rnd(rng.standard_normal((tok, D), dtype=np.float32))
    out["dt"] = _raw_dt(rng, (tok, D), bf16)
    out["B"] = rnd(rng.standard_normal((tok, N), dtype=np.float32))
    out["C"] = rnd(rng.standard_normal((tok, N), dtype=np.float32))
    return out


def make_states(seed: int, S: int, D: int, N: int = 16, K: int = 4, bf16: bool = True,
                scale: float = 1.0) -> dict:
    """Random initial states: h0 (S, D, N) fp32 and conv_state (S, D, K-1)."""
    rng = _rng(seed, 4)
    h0 = (scale * rng.standard_normal((S, D, N))).astype(np.float32)
    cs = rng.standard_normal((S, D, K - 1)).astype(np.float32)
    if bf16:
        cs = round_bf16(cs)
    return {"h0": h0, "conv_state": cs}


# --------------------------------------------------------------------------
# Device-side draws for the very large workloads (torch generator on the GPU).
# --------------------------------------------------------------------------

def device_activations(seed: int, tok: int, D: int, N: int = 16, device="cuda",
                       dtype=None, out=None):
    """Same distributions as make_activations, drawn on `device` in bf16.

    Draws in slabs of at most 16 Mi elements so that no fp32 copy of a whole
    large tensor is ever materialised."""
    import torch

    dtype = dtype or torch.bfloat16
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000003 + 17)
    res = out or {
        "x": torch.empty((tok, D), dtype=dtype, device=device),
        "z": torch.empty((tok, D), dtype=dtype, device=device),
        "dt": torch.empty((tok, D), dtype=dtype, device=device),
        "B": torch.empty((tok, N), dtype=dtype, device=device),
        "C": torch.empty((tok, N), dtype=dtype, device=device),
    }
    rows = max(1, (16 << 20) // max(D, 1))
    for name in ("x", "z", "dt"):
        t = res[name]
        for r0 in range(0, tok, rows):
            r1 = min(tok, r0 + rows)
            v = torch.randn((r1 - r0, D), generator=g, device=device, dtype=torch.float32)
            if name == "dt":
                v = (0.1 * v.clamp_(-3.0, 3.0)).to(dtype).clamp_(-DT_RAW_LIMIT, DT_RAW_LIMIT)
            t[r0:r1].copy_(v)
    for name in ("B", "C"):
        res[name].copy_(torch.randn((tok, N), generator=g, device=device, dtype=torch.float32))
    return res


# --------------------------------------------------------------------------
# The five workloads (shapes and structure only).
# --------------------------------------------------------------------------

WORKLOADS = {
    "mamba_tiny_fp32": dict(kind="prefill", batch=1, seqlen=64, D=32, N=16, K=4, bf16=False),
    "mamba130m_layer_b8_l2048": dict(kind="prefill", batch=8, seqlen=2048, D=1536, N=16, K=4,
                                     bf16=True),
    "packmamba_2p8b_varlen_65536": dict(kind="varlen", total=65536, D=5120, N=16, K=4,
                                        bf16=True, len_lo=128, len_hi=8192),
    "falcon_mamba7b_longctx_131072": dict(kind="chunked", batch=1, seqlen=131072, chunk=8192,
                                          D=8192, N=16, K=4, bf16=True),
    "decode_b256_d8192": dict(kind="decode", batch=256, D=8192, N=16, K=4, bf16=True,
                              prefill_len=512, steps=1000),
}
