"""Fused conv1d + SiLU -> selective scan on the GPU against the fp64 oracle's
conv followed by its scan (conv output kept in fp64, as the fused kernel keeps
it in fp32), and against the two-call GPU path."""

import numpy as np
import pytest
import torch

import selective_state_space_causal_b200 as ssm
from selective_state_space_causal_b200 import synth
from gpu_helpers import (TOL_BF16, TOL_F32, act_dtype, assert_close, cu_tensor, dev, host,
                         run_conv, run_scan)

pytestmark = pytest.mark.gpu


def _fused(x, w, b, dt, A, B, C, Dskip, z, dtb, h0, cs_in, cu, S, want_xc=False,
           inplace_state=False, K=4):
    tok, D = x.shape
    y = torch.full_like(x, 3.0)
    hf = torch.full((S, D, 16), 555.0, device="cuda")
    if inplace_state:
        cs_out = cs_in
    else:
        sdt = cs_in.dtype if cs_in is not None else x.dtype
        cs_out = torch.full((S, D, K - 1), 777.0, dtype=sdt, device="cuda")
    xc = torch.empty_like(x) if want_xc else None
    ssm.ssm_conv_scan_fwd(x, w, dt, A, B, C, y, conv_b=b, conv_state_in=cs_in,
                          conv_state_out=cs_out, xc=xc, Dskip=Dskip, z=z, dt_bias=dtb, h0=h0,
                          h_final=hf, cu_seqlens=cu, S=S)
    torch.cuda.synchronize()
    return y, hf, cs_out, xc


def _case(orc, bf16, K, lens, D, seed, inplace=False, want_xc=True, dense=None):
    dt_ = act_dtype(bf16)
    if dense:
        S, L = dense
        tok, cu_d, cu_h = S * L, None, None
    else:
        cu_d, cu_h = cu_tensor(lens)
        tok, S = int(cu_h[-1]), len(lens)
    prm = synth.make_params(seed, D, K=K, random_bias=True, random_A=True, random_D=True)
    act = synth.make_activations(seed, tok, D, bf16=bf16)
    st = synth.make_states(seed + 1, S, D, K=K, bf16=bf16, scale=0.3)
    cs_in = dev(st["conv_state"], dt_)
    y, hf, cs, xc = _fused(dev(act["x"], dt_), dev(prm.conv_w), dev(prm.conv_b),
                           dev(act["dt"], dt_), dev(prm.A), dev(act["B"], dt_),
                           dev(act["C"], dt_), dev(prm.Dskip), dev(act["z"], dt_),
                           dev(prm.dt_bias), dev(st["h0"]), cs_in, cu_d, S, want_xc=want_xc,
                           inplace_state=inplace, K=K)
    rxc, rcs = orc.causal_conv1d(act["x"], prm.conv_w, prm.conv_b, cu_seqlens=cu_h,
                                 S=S if dense else None, state_in=st["conv_state"],
                                 want_state=True)
    ry, rh = orc.selective_scan(rxc, act["dt"], prm.A, act["B"], act["C"], Dskip=prm.Dskip,
                                z=act["z"], dt_bias=prm.dt_bias, h0=st["h0"], cu_seqlens=cu_h,
                                S=S if dense else None, want_state=True)
    tol = TOL_BF16 if bf16 else TOL_F32
    assert_close(host(y), ry, bf16, tol, "y")
    assert_close(host(hf), rh, False, tol, "h_final")
    assert np.array_equal(host(cs), rcs), "conv state output"
    if want_xc:
        assert_close(host(xc), rxc, bf16, tol, "xc")
    assert ssm.ssm_device_status() == 0
    return y


@pytest.fixture(params=[(0, 0), (16, 12)], ids=["pick", "one_lane_per_channel"])
def fused_variant(request):
    """The kernel the library picks for the shape, and the one-lane-per-channel
    fused kernel (taken where the scan would run schedule 12), forced."""
    ssm.ssm_set_scan_variant(*request.param)
    yield request.param
    ssm.ssm_set_scan_variant(0, 0)


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("K", [2, 3, 4])
def test_fused_packed(orc, bf16, K, fused_variant):
    # empty and shorter-than-K-1 sequences, chunk edges at 64 tokens, a
    # partial channel block
    _case(orc, bf16, K, [70, 0, 1, 2, 64, 129, 5], 96, 3 + K)


def test_fused_in_place_conv_state_and_dense(orc, fused_variant):
    _case(orc, True, 4, [33, 65, 1], 64, 21, inplace=True, want_xc=False)
    _case(orc, True, 4, None, 128, 22, dense=(3, 100))


def test_fused_many_sequences(orc, fused_variant):
    """More sequences than a CTA ranks by itself (index order then), with a
    ragged channel tail over two channel blocks."""
    lens = list(np.random.default_rng(41).integers(0, 40, size=150))
    _case(orc, True, 4, lens, 200, 41)


@pytest.mark.parametrize("bf16", [False, True])
def test_fused_unaligned_rows(orc, bf16):
    """D = 36: bf16 rows are not 16-byte aligned, so the scalar layout runs."""
    _case(orc, bf16, 4, [40, 7, 90], 36, 31)


def test_fused_mamba130m_layer(orc, fused_variant):
    """The Mamba-130M layer shape: y and h_final of sampled channels against the
    oracle's conv then scan, and the conv state output and the optional xc copy
    bit for bit equal to the two-call path's (the fused kernel computes the
    conv with the conv kernel's operations). The two paths' y are not compared
    with each other: the two-call path rounds xc to bf16 between its calls,
    which alone moves y by about the bf16 bound."""
    w = synth.WORKLOADS["mamba130m_layer_b8_l2048"]
    Bn, L, D = w["batch"], w["seqlen"], w["D"]
    tok = Bn * L
    prm = synth.make_params(0, D)
    p = {k: dev(getattr(prm, k)) for k in ("conv_w", "conv_b", "A", "Dskip", "dt_bias")}
    a = synth.device_activations(0, tok, D)
    xc, cs2 = run_conv(a["x"], p["conv_w"], p["conv_b"], S=Bn, want_state=True)
    y1, h1, cs1, xc1 = _fused(a["x"], p["conv_w"], p["conv_b"], a["dt"], p["A"], a["B"], a["C"],
                              p["Dskip"], a["z"], p["dt_bias"], None, None, None, Bn,
                              want_xc=True)
    assert torch.equal(cs1, cs2)
    assert torch.equal(xc1, xc), "the fused kernel's xc rounds to the conv kernel's bits"
    rng = np.random.default_rng(0)
    ch = np.sort(rng.choice(D, size=16, replace=False))
    chd = torch.from_numpy(ch).cuda()
    sel = lambda t: host(t.index_select(1, chd))  # noqa: E731
    rxc = orc.causal_conv1d(sel(a["x"]), prm.conv_w[ch], prm.conv_b[ch], S=Bn)
    ry, rh = orc.selective_scan(rxc, sel(a["dt"]), prm.A[ch], host(a["B"]), host(a["C"]),
                                Dskip=prm.Dskip[ch], z=sel(a["z"]), dt_bias=prm.dt_bias[ch], S=Bn,
                                want_state=True)
    assert_close(sel(y1), ry, True, TOL_BF16, "y")
    assert_close(host(h1)[:, ch], rh, False, TOL_BF16, "h_final")
    assert ssm.ssm_device_status() == 0


def test_fused_packed_workload(orc):
    """The packed 65536 x 5120 workload (43 sequences) in the kernel the library
    picks for it (one lane per channel): the conv state output and the xc copy
    bit for bit equal to the conv kernel's, y and h_final of sampled channels
    (the first and last among them) against the oracle's conv then scan."""
    w = synth.WORKLOADS["packmamba_2p8b_varlen_65536"]
    D = w["D"]
    lens = synth.sample_lengths(0, w["total"], w["len_lo"], w["len_hi"])
    cu_d, cu_h = cu_tensor(lens)
    tok, S = int(cu_h[-1]), len(lens)
    prm = synth.make_params(0, D)
    p = {k: dev(getattr(prm, k)) for k in ("conv_w", "conv_b", "A", "Dskip", "dt_bias")}
    a = synth.device_activations(0, tok, D)
    xc, cs2 = run_conv(a["x"], p["conv_w"], p["conv_b"], cu=cu_d, S=S, want_state=True)
    y1, h1, cs1, xc1 = _fused(a["x"], p["conv_w"], p["conv_b"], a["dt"], p["A"], a["B"], a["C"],
                              p["Dskip"], a["z"], p["dt_bias"], None, None, cu_d, S,
                              want_xc=True)
    assert torch.equal(cs1, cs2)
    assert torch.equal(xc1, xc), "the fused kernel's xc rounds to the conv kernel's bits"
    rng = np.random.default_rng(1)
    ch = np.unique(np.concatenate([[0, D - 1], rng.choice(D, size=10, replace=False)]))
    chd = torch.from_numpy(ch).cuda()
    sel = lambda t: host(t.index_select(1, chd))  # noqa: E731
    rxc = orc.causal_conv1d(sel(a["x"]), prm.conv_w[ch], prm.conv_b[ch], cu_seqlens=cu_h)
    ry, rh = orc.selective_scan(rxc, sel(a["dt"]), prm.A[ch], host(a["B"]), host(a["C"]),
                                Dskip=prm.Dskip[ch], z=sel(a["z"]), dt_bias=prm.dt_bias[ch],
                                cu_seqlens=cu_h, want_state=True)
    assert_close(sel(y1), ry, True, TOL_BF16, "y")
    assert_close(host(h1)[:, ch], rh, False, TOL_BF16, "h_final")
    assert ssm.ssm_device_status() == 0
