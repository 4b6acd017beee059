"""Helpers for the GPU parity tests: move seeded inputs to the device, call the
library through its C ABI binding, and compare with the fp64 oracle.

Tolerances (max-abs error, per output element):

* fp32 activations: |gpu - oracle| <= 1e-4 * rms(oracle).
* bf16 activations with fp32 state: |gpu - oracle| <= 2e-2 * rms(oracle)
  + 2^-8 * |oracle| for outputs stored in bf16. The second term is the
  largest error of rounding the exact result to bf16: half a bf16 ulp, which
  is at most 2^-8 |y| (bf16 keeps 8 significant bits). y is heavy-tailed (max
  |y| is ~60 rms(y) on Mamba-shaped inputs), so that rounding alone can exceed
  the first term and no bf16-output implementation could meet it alone. fp32
  outputs (the SSM state) get the first term only.
"""

from __future__ import annotations

import numpy as np
import torch

import selective_state_space_causal_b200 as ssm

TOL_F32 = 1e-4
TOL_BF16 = 2e-2
BF16_ULP = 2.0 ** -8


def dev(a, dtype=torch.float32):
    if a is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda").to(dtype)


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def rms(a):
    a = np.asarray(a, np.float64)
    return float(np.sqrt(np.mean(a * a))) if a.size else 0.0


def err_ratio(gpu, ref, bf16_out: bool, tol: float):
    """max over elements of (|gpu - ref| - slack) / (tol * rms(ref)); <= 1 passes."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    scale = tol * rms(ref)
    if scale == 0.0:
        scale = tol
    excess = np.abs(gpu - ref)
    if bf16_out:
        excess = excess - BF16_ULP * np.abs(ref)
    return float(np.max(excess) / scale)


def assert_close(gpu, ref, bf16_out: bool, tol: float, what: str = ""):
    r = err_ratio(gpu, ref, bf16_out, tol)
    assert r <= 1.0, f"{what}: error is {r:.3g} x the bound"
    return r


def act_dtype(bf16: bool):
    return torch.bfloat16 if bf16 else torch.float32


def cu_tensor(lens):
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    return torch.from_numpy(cu).cuda(), cu


def run_conv(x, w, bias=None, cu=None, S=None, state_in=None, want_state=False,
             state_inplace=False, apply_silu=True):
    """x: device tensor. Returns (xc, state_out) device tensors."""
    tok, D = x.shape
    K = w.shape[1]
    xc = torch.empty_like(x)
    st_out = None
    if want_state:
        if S is None:
            S = cu.numel() - 1 if cu is not None else 1
        if state_inplace:
            st_out = state_in
        else:
            sdt = state_in.dtype if state_in is not None else x.dtype
            st_out = torch.full((S, D, K - 1), 777.0, dtype=sdt, device="cuda")
    ssm.ssm_causal_conv1d(x, xc, w, bias=bias, cu_seqlens=cu, S=S, conv_state_in=state_in,
                          conv_state_out=st_out, apply_silu=apply_silu)
    return xc, st_out


def run_scan(u, dt, A, B, C, Dskip=None, z=None, dt_bias=None, delta_softplus=True, h0=None,
             cu=None, S=None, want_state=True, inplace_state=False, workspace=False,
             y_fill=None):
    tok, D = u.shape
    N = A.shape[1]
    if S is None:
        S = cu.numel() - 1 if cu is not None else 1
    y = torch.empty_like(u) if y_fill is None else torch.full_like(u, y_fill)
    hf = None
    if want_state:
        hf = h0 if inplace_state else torch.full((S, D, N), 555.0, device="cuda")
    ws = None
    if workspace:
        nb = ssm.ssm_scan_workspace_size(tok, D, N, S)
        ws = torch.empty(max(nb, 1), dtype=torch.uint8, device="cuda")
    ssm.ssm_selective_scan_fwd(u, dt, A, B, C, y, Dskip=Dskip, z=z, dt_bias=dt_bias,
                               delta_softplus=delta_softplus, h0=h0, h_final=hf, cu_seqlens=cu,
                               S=S, workspace=ws)
    return y, hf
