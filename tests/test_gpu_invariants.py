"""Invariants of the method checked on the GPU path itself.

* A packed batch equals its sequences run one by one (bit for bit: each
  element sees the same operations in the same order).
* A prefill cut in two, with h and the conv state carried, equals the one-shot
  prefill (bit for bit).
* Prefill followed by k decode steps equals prefill over the extended
  sequence: with fp32 activations to the fp32 bound (the decode kernel sums
  the readout in another order); with bf16 activations the prefill stores its
  conv output in bf16 while decode keeps it in fp32, so there each step is
  checked against the oracle chained from the GPU prefill's states.
"""

import numpy as np
import pytest
import torch

import selective_state_space_causal_b200 as ssm
from selective_state_space_causal_b200 import synth
from gpu_helpers import TOL_BF16, TOL_F32, assert_close, cu_tensor, dev, host, run_conv, run_scan

pytestmark = pytest.mark.gpu

BF = torch.bfloat16


@pytest.fixture(autouse=True)
def _fixed_variant():
    # the packed and per-sequence runs must use the same kernel variant
    ssm.ssm_set_scan_variant(4, 2)
    yield
    ssm.ssm_set_scan_variant(0, 0)


def _params(seed, D):
    prm = synth.make_params(seed, D, random_bias=True, random_A=True, random_D=True)
    return {k: dev(getattr(prm, k)) for k in ("conv_w", "conv_b", "A", "Dskip", "dt_bias")}


def _prefill(p, x, dt, z, B, C, cu=None, S=None, conv_state=None, h0=None):
    xc, cs = run_conv(x, p["conv_w"], p["conv_b"], cu=cu, S=S, state_in=conv_state,
                      want_state=True)
    y, hf = run_scan(xc, dt, p["A"], B, C, Dskip=p["Dskip"], z=z, dt_bias=p["dt_bias"], h0=h0,
                     cu=cu, S=S)
    return y, hf, cs


def _acts(seed, tok, D):
    a = synth.make_activations(seed, tok, D, bf16=True)
    return {k: dev(v, BF) for k, v in a.items()}


@pytest.mark.parametrize("variant", [(4, 1), (4, 2), (4, 3), (2, 3), (8, 2), (16, 2), (4, 6), (8, 6), (4, 7), (8, 7), (2, 8), (4, 8),
                                     (2, 9), (4, 9), (8, 9), (4, 10), (8, 10), (4, 11), (16, 12)],
                         ids=lambda v: f"{v[0]}x{v[1]}")
def test_pack_equals_separate(variant):
    ssm.ssm_set_scan_variant(*variant)
    lens = [100, 0, 3, 1, 257, 64]
    D = 96
    p = _params(1, D)
    a = _acts(2, sum(lens), D)
    st = synth.make_states(3, len(lens), D, bf16=True, scale=0.3)
    cs0, h00 = dev(st["conv_state"], BF), dev(st["h0"])
    cu_d, cu_h = cu_tensor(lens)
    y, hf, cs = _prefill(p, a["x"], a["dt"], a["z"], a["B"], a["C"], cu=cu_d,
                         conv_state=cs0.clone(), h0=h00.clone())
    for s in range(len(lens)):
        s0, s1 = int(cu_h[s]), int(cu_h[s + 1])
        sl = slice(s0, s1)
        ys, hs, css = _prefill(p, a["x"][sl], a["dt"][sl], a["z"][sl], a["B"][sl], a["C"][sl],
                               S=1, conv_state=cs0[s:s + 1].clone(), h0=h00[s:s + 1].clone())
        assert torch.equal(y[sl], ys), s
        assert torch.equal(hf[s], hs[0]), s
        assert torch.equal(cs[s], css[0]), s


def test_chunked_equals_oneshot():
    L, D = 700, 64
    p = _params(4, D)
    a = _acts(5, L, D)
    y, hf, cs = _prefill(p, a["x"], a["dt"], a["z"], a["B"], a["C"], S=1)
    for L1 in (1, 2, 3, 64, 65, 333, 699):
        s1 = slice(0, L1)
        s2 = slice(L1, L)
        y1, h1, c1 = _prefill(p, a["x"][s1], a["dt"][s1], a["z"][s1], a["B"][s1], a["C"][s1], S=1)
        y2, h2, c2 = _prefill(p, a["x"][s2], a["dt"][s2], a["z"][s2], a["B"][s2], a["C"][s2], S=1,
                              conv_state=c1, h0=h1)
        assert torch.equal(torch.cat([y1, y2]), y), L1
        assert torch.equal(h2, hf), L1
        assert torch.equal(c2, cs), L1


@pytest.mark.parametrize("k", [1, 7, 100])
def test_prefill_then_decode_equals_longer_prefill_fp32(k):
    """fp32 activations: no intermediate is rounded, so decode after prefill must
    equal the longer prefill to the fp32 bound (only summation order differs)."""
    Bt, L0, D = 4, 300, 128
    L = L0 + k
    p = _params(6, D)
    a = synth.make_activations(7, Bt * L, D, bf16=True)  # bf16-exact values held in fp32
    view = {n: dev(v).view(Bt, L, -1) for n, v in a.items()}
    full = {n: t.reshape(Bt * L, -1) for n, t in view.items()}
    y_long, h_long, c_long = _prefill(p, full["x"], full["dt"], full["z"], full["B"], full["C"],
                                      S=Bt)
    head = {n: t[:, :L0].reshape(Bt * L0, -1).contiguous() for n, t in view.items()}
    _, h, c = _prefill(p, head["x"], head["dt"], head["z"], head["B"], head["C"], S=Bt)
    ys = []
    for t in range(L0, L):
        step = {n: v[:, t].contiguous() for n, v in view.items()}
        y = torch.empty((Bt, D), device="cuda")
        ssm.ssm_selective_state_update(c, h, step["x"], step["dt"], step["B"], step["C"], y,
                                       p["conv_w"], p["A"], z=step["z"], conv_b=p["conv_b"],
                                       Dskip=p["Dskip"], dt_bias=p["dt_bias"])
        ys.append(y)
    y_dec = torch.stack(ys, dim=1)  # (Bt, k, D)
    y_ref = y_long.view(Bt, L, D)[:, L0:]
    assert_close(host(y_dec), host(y_ref), False, TOL_F32, "decode y vs prefill y")
    assert_close(host(h), host(h_long), False, TOL_F32, "decode state vs prefill state")
    assert torch.equal(c, c_long), "conv state must match exactly"


@pytest.mark.parametrize("k", [1, 50])
def test_prefill_then_decode_bf16_against_oracle_chain(orc, k):
    """bf16 activations: each decode step checked against the oracle chained from
    the GPU prefill's own states."""
    Bt, L0, D = 4, 300, 128
    L = L0 + k
    prm = synth.make_params(6, D, random_bias=True, random_A=True, random_D=True)
    p = _params(6, D)
    a = synth.make_activations(8, Bt * L, D, bf16=True)
    view = {n: v.reshape(Bt, L, -1) for n, v in a.items()}
    head = {n: dev(v[:, :L0].reshape(Bt * L0, -1), BF) for n, v in view.items()}
    _, h, c = _prefill(p, head["x"], head["dt"], head["z"], head["B"], head["C"], S=Bt)
    rc, rh = host(c), host(h)
    for t in range(L0, L):
        step = {n: v[:, t] for n, v in view.items()}
        y = torch.empty((Bt, D), device="cuda", dtype=BF)
        ssm.ssm_selective_state_update(c, h, dev(step["x"], BF), dev(step["dt"], BF),
                                       dev(step["B"], BF), dev(step["C"], BF), y, p["conv_w"],
                                       p["A"], z=dev(step["z"], BF), conv_b=p["conv_b"],
                                       Dskip=p["Dskip"], dt_bias=p["dt_bias"])
        ry, rc, rh = orc.state_update(rc, rh, step["x"], step["dt"], step["B"], step["C"],
                                      step["z"], prm.conv_w, prm.conv_b, prm.A, prm.Dskip,
                                      prm.dt_bias)
        assert_close(host(y), ry, True, TOL_BF16, f"decode y at step {t - L0}")
    assert np.array_equal(host(c), rc)
    assert_close(host(h), rh, False, TOL_BF16, "state after the decode steps")


@pytest.mark.parametrize("variant", [(4, 3), (2, 3)])
def test_chunked_prefill_time_split_variant(variant):
    """The time-split kernel combines segments through their decay products, so
    a call boundary moves the segment boundaries: equal to the fp32 bound."""
    ssm.ssm_set_scan_variant(*variant)
    L, D = 700, 64
    p = _params(9, D)
    a = {k: dev(v) for k, v in synth.make_activations(10, L, D, bf16=True).items()}
    y, hf, cs = _prefill(p, a["x"], a["dt"], a["z"], a["B"], a["C"], S=1)
    for L1 in (1, 31, 33, 64, 333):
        s1, s2 = slice(0, L1), slice(L1, L)
        y1, h1, c1 = _prefill(p, a["x"][s1], a["dt"][s1], a["z"][s1], a["B"][s1], a["C"][s1], S=1)
        y2, h2, c2 = _prefill(p, a["x"][s2], a["dt"][s2], a["z"][s2], a["B"][s2], a["C"][s2], S=1,
                              conv_state=c1, h0=h1)
        assert_close(host(torch.cat([y1, y2])), host(y), False, TOL_F32, f"y split at {L1}")
        assert_close(host(h2), host(hf), False, TOL_F32, f"h split at {L1}")
        assert torch.equal(c2, cs), L1
