"""The five Mamba-shaped workloads at full size, on the launch configuration the
benchmark uses, against the fp64 oracle.

The tiny fp32 layer and the Mamba-130M layer are checked on every output
element. The three large workloads are checked on a seeded sample of channels
(channels are independent, so the oracle can run those channels alone over
every sequence, token and decode step).
"""

import numpy as np
import pytest
import torch

import selective_state_space_causal_b200 as ssm
from selective_state_space_causal_b200 import synth
from gpu_helpers import TOL_BF16, TOL_F32, assert_close, dev, host, run_conv, run_scan

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def _dparams(prm):
    return {k: dev(getattr(prm, k)) for k in ("conv_w", "conv_b", "A", "Dskip", "dt_bias")}


def _sample_channels(D, n, seed=0):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(D, size=n, replace=False))


def _sub(prm, ch):
    return synth.MixerParams(prm.conv_w[ch], prm.conv_b[ch], prm.A[ch], prm.Dskip[ch],
                             prm.dt_bias[ch])


def test_tiny_fp32_layer(orc):
    w = synth.WORKLOADS["mamba_tiny_fp32"]
    D, L = w["D"], w["seqlen"]
    prm = synth.make_params(0, D)
    act = synth.make_activations(0, L, D, bf16=False)
    p = _dparams(prm)
    xc, _ = run_conv(dev(act["x"]), p["conv_w"], p["conv_b"])
    y, hf = run_scan(xc, dev(act["dt"]), p["A"], dev(act["B"]), dev(act["C"]), Dskip=p["Dskip"],
                     z=dev(act["z"]), dt_bias=p["dt_bias"])
    rxc = orc.causal_conv1d(act["x"], prm.conv_w, prm.conv_b)
    ry, rh = orc.selective_scan(rxc, act["dt"], prm.A, act["B"], act["C"], Dskip=prm.Dskip,
                                z=act["z"], dt_bias=prm.dt_bias, want_state=True)
    assert_close(host(xc), rxc, False, TOL_F32, "xc")
    assert_close(host(y), ry, False, TOL_F32, "y (conv and scan end to end)")
    assert_close(host(hf), rh, False, TOL_F32, "h_final")


def test_mamba130m_layer_full(orc):
    w = synth.WORKLOADS["mamba130m_layer_b8_l2048"]
    Bn, L, D = w["batch"], w["seqlen"], w["D"]
    tok = Bn * L
    prm = synth.make_params(0, D)
    act = synth.make_activations(0, tok, D, bf16=True)
    p = _dparams(prm)
    xc, cs = run_conv(dev(act["x"], BF), p["conv_w"], p["conv_b"], S=Bn, want_state=True)
    y, hf = run_scan(xc, dev(act["dt"], BF), p["A"], dev(act["B"], BF), dev(act["C"], BF),
                     Dskip=p["Dskip"], z=dev(act["z"], BF), dt_bias=p["dt_bias"], S=Bn)
    rxc, rcs = orc.causal_conv1d(act["x"], prm.conv_w, prm.conv_b, S=Bn, want_state=True)
    assert_close(host(xc), rxc, True, TOL_BF16, "xc")
    assert np.array_equal(host(cs), rcs)
    ry, rh = orc.selective_scan(host(xc), act["dt"], prm.A, act["B"], act["C"], Dskip=prm.Dskip,
                                z=act["z"], dt_bias=prm.dt_bias, S=Bn, want_state=True)
    assert_close(host(y), ry, True, TOL_BF16, "y")
    assert_close(host(hf), rh, False, TOL_BF16, "h_final")


def test_packmamba_varlen_sampled(orc):
    w = synth.WORKLOADS["packmamba_2p8b_varlen_65536"]
    D, total = w["D"], w["total"]
    lens = synth.sample_lengths(0, total, w["len_lo"], w["len_hi"])
    cu_h = synth.cu_from_lengths(lens)
    cu_d = torch.from_numpy(cu_h).cuda()
    S = len(lens)
    prm = synth.make_params(0, D)
    p = _dparams(prm)
    a = synth.device_activations(0, total, D)
    xc, cs = run_conv(a["x"], p["conv_w"], p["conv_b"], cu=cu_d, want_state=True)
    y, hf = run_scan(xc, a["dt"], p["A"], a["B"], a["C"], Dskip=p["Dskip"], z=a["z"],
                     dt_bias=p["dt_bias"], cu=cu_d, workspace=True)
    ch = _sample_channels(D, 64)
    chd = torch.from_numpy(ch).cuda()
    g = {k: host(v.index_select(1, chd)) for k, v in (("x", a["x"]), ("dt", a["dt"]),
                                                      ("z", a["z"]), ("xc", xc), ("y", y))}
    Bh, Ch = host(a["B"]), host(a["C"])
    sp = _sub(prm, ch)
    rxc, rcs = orc.causal_conv1d(g["x"], sp.conv_w, sp.conv_b, cu_seqlens=cu_h, want_state=True)
    assert_close(g["xc"], rxc, True, TOL_BF16, "xc")
    assert np.array_equal(host(cs)[:, ch], rcs)
    ry, rh = orc.selective_scan(g["xc"], g["dt"], sp.A, Bh, Ch, Dskip=sp.Dskip, z=g["z"],
                                dt_bias=sp.dt_bias, cu_seqlens=cu_h, want_state=True)
    assert_close(g["y"], ry, True, TOL_BF16, "y")
    assert_close(host(hf)[:, ch], rh, False, TOL_BF16, "h_final")
    assert S == hf.shape[0]


def test_longctx_chunked_sampled(orc):
    w = synth.WORKLOADS["falcon_mamba7b_longctx_131072"]
    D, L, chunk = w["D"], w["seqlen"], w["chunk"]
    prm = synth.make_params(0, D)
    p = _dparams(prm)
    a = synth.device_activations(0, L, D)
    cs = torch.zeros((1, D, 3), dtype=BF, device="cuda")
    h = torch.zeros((1, D, 16), device="cuda")
    ys, xcs = [], []
    for c0 in range(0, L, chunk):
        sl = slice(c0, c0 + chunk)
        xc, _ = run_conv(a["x"][sl], p["conv_w"], p["conv_b"], state_in=cs, want_state=True,
                         state_inplace=True)
        y, _ = run_scan(xc, a["dt"][sl], p["A"], a["B"][sl], a["C"][sl], Dskip=p["Dskip"],
                        z=a["z"][sl], dt_bias=p["dt_bias"], h0=h, inplace_state=True)
        ys.append(y)
        xcs.append(xc)
    y = torch.cat(ys)
    xc = torch.cat(xcs)
    ch = _sample_channels(D, 16)
    chd = torch.from_numpy(ch).cuda()
    g = {k: host(v.index_select(1, chd)) for k, v in (("x", a["x"]), ("dt", a["dt"]),
                                                      ("z", a["z"]), ("xc", xc), ("y", y))}
    sp = _sub(prm, ch)
    rxc, rcs = orc.causal_conv1d(g["x"], sp.conv_w, sp.conv_b, want_state=True)
    assert_close(g["xc"], rxc, True, TOL_BF16, "xc across 16 calls")
    assert np.array_equal(host(cs)[:, ch], rcs)
    ry, rh = orc.selective_scan(g["xc"], g["dt"], sp.A, host(a["B"]), host(a["C"]),
                                Dskip=sp.Dskip, z=g["z"], dt_bias=sp.dt_bias, want_state=True)
    assert_close(g["y"], ry, True, TOL_BF16, "y across 16 calls")
    assert_close(host(h)[:, ch], rh, False, TOL_BF16, "carried h")


def test_decode_b256_1000_steps_sampled(orc):
    w = synth.WORKLOADS["decode_b256_d8192"]
    Bt, D, L0, steps = w["batch"], w["D"], w["prefill_len"], w["steps"]
    prm = synth.make_params(0, D)
    p = _dparams(prm)
    a = synth.device_activations(0, Bt * L0, D)
    xc, cs = run_conv(a["x"], p["conv_w"], p["conv_b"], S=Bt, want_state=True)
    _, h = run_scan(xc, a["dt"], p["A"], a["B"], a["C"], Dskip=p["Dskip"], z=a["z"],
                    dt_bias=p["dt_bias"], S=Bt)
    ch = _sample_channels(D, 8)
    chd = torch.from_numpy(ch).cuda()
    sp = _sub(prm, ch)
    pre = {k: host(v.index_select(1, chd)) for k, v in (("x", a["x"]), ("dt", a["dt"]),
                                                        ("z", a["z"]))}
    rxc, rcs = orc.causal_conv1d(pre["x"], sp.conv_w, sp.conv_b, S=Bt, want_state=True)
    _, rh = orc.selective_scan(rxc, pre["dt"], sp.A, host(a["B"]), host(a["C"]), Dskip=sp.Dskip,
                               z=pre["z"], dt_bias=sp.dt_bias, S=Bt, want_state=True)
    del a, xc
    y = torch.empty((Bt, D), device="cuda", dtype=BF)
    worst = 0.0
    for step in range(steps):
        s = synth.device_activations(10_000 + step, Bt, D)
        ssm.ssm_selective_state_update(cs, h, s["x"], s["dt"], s["B"], s["C"], y, p["conv_w"],
                                       p["A"], z=s["z"], conv_b=p["conv_b"], Dskip=p["Dskip"],
                                       dt_bias=p["dt_bias"])
        g = {k: host(v.index_select(1, chd)) for k, v in (("x", s["x"]), ("dt", s["dt"]),
                                                          ("z", s["z"]), ("y", y))}
        ry, rcs, rh = orc.state_update(rcs, rh, g["x"], g["dt"], host(s["B"]), host(s["C"]),
                                       g["z"], sp.conv_w, sp.conv_b, sp.A, sp.Dskip, sp.dt_bias)
        worst = max(worst, assert_close(g["y"], ry, True, TOL_BF16, f"y at step {step}"))
    assert np.array_equal(host(cs)[:, ch], rcs)
    assert_close(host(h)[:, ch], rh, False, TOL_BF16, "ssm state after 1000 steps")
