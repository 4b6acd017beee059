"""Replay decode on the GPU ("ReplaySSM: Cache SSM Inputs, Not State",
abstract): the checkpoint-plus-buffer kernels against the fp64 oracle's replay
step, and against the library's own eager decode bit for bit.

Tolerances: outputs and states follow the activation dtype's bound (see
gpu_helpers). Outputs computed from the bf16 checkpoint copy take the bf16
bound whatever the activation dtype, because that copy's precision is part of
the method: the oracle rounds its fp64 checkpoint to bf16 while the kernel
rounds its fp32 one, so an element near a rounding boundary may land one bf16
step apart. Buffer lengths must match exactly.
"""

import numpy as np
import pytest
import torch

import selective_state_space_causal_b200 as ssm
from selective_state_space_causal_b200 import synth
from gpu_helpers import TOL_BF16, TOL_F32, act_dtype, assert_close, dev, host

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def _same_up_to_sum_order(y_r, y_e):
    """Replay sums the 16 state terms of the readout in natural order and eager
    decode in its lane-rotated order, so the fp32 sums may differ in their last
    bits (relative to the size of the terms, which near a cancelling y is far
    above y itself: hence 1e-5 rms(y) of absolute slack) and their bf16
    roundings by one bf16 step (at most 2^-7 relative)."""
    a, b = y_r.float(), y_e.float()
    slack = 1e-5 * float(torch.sqrt(torch.mean(b * b)))
    return bool((torch.abs(a - b) <= 2.0 ** -7 * torch.abs(b) + slack).all())


def _params(seed, D, K):
    return synth.make_params(seed, D, K=K, random_bias=True, random_A=True, random_D=True)


def _dev_params(prm):
    return {k: dev(getattr(prm, k)) for k in ("conv_w", "conv_b", "A", "Dskip", "dt_bias")}


def _step(cs, rep, s, y, p, dt_, idx=None):
    ssm.ssm_replay_state_update(cs, rep, dev(s["x"], dt_), dev(s["dt"], dt_), dev(s["B"], dt_),
                                dev(s["C"], dt_), y, p["conv_w"], p["A"], z=dev(s["z"], dt_),
                                conv_b=p["conv_b"], Dskip=p["Dskip"], dt_bias=p["dt_bias"],
                                state_indices=idx)


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("K", [2, 4])
@pytest.mark.parametrize("W,keep_lo", [(1, True), (2, False), (3, False), (4, True), (8, True)])
def test_replay_matches_oracle(orc, bf16, K, W, keep_lo):
    n_slots, Bt, D, steps = 9, 6, 200, 10
    prm = _params(30 + K, D, K)
    p = _dev_params(prm)
    st = synth.make_states(31, n_slots, D, K=K, bf16=bf16, scale=0.3)
    dt_ = act_dtype(bf16)
    idx = np.array([7, -1, 0, 3, 8, 4], dtype=np.int32)
    idx_d = torch.from_numpy(idx).cuda()
    cs = dev(st["conv_state"], dt_)
    rep = ssm.replay_buffers(n_slots, D, W, "cuda", keep_lo=keep_lo)
    rep["ckpt"].copy_(dev(st["h0"]))
    ssm.ssm_replay_reset(rep)
    rcs = np.asarray(st["conv_state"], np.float64)
    rrep = orc.replay_init(st["h0"], W, keep_lo=keep_lo)
    live = idx >= 0
    used = sorted(int(i) for i in idx if i >= 0)
    unused = [s for s in range(n_slots) if s not in used]
    y = torch.full((Bt, D), 9.0, device="cuda", dtype=dt_)
    tol = TOL_BF16 if bf16 else TOL_F32
    ytol = TOL_BF16 if keep_lo else tol
    for t in range(steps):
        s = synth.make_activations(100 + t, Bt, D, bf16=bf16)
        _step(cs, rep, s, y, p, dt_, idx_d)
        ry, rcs, rrep = orc.replay_step(rcs, rrep, s["x"], s["dt"], s["B"], s["C"], s["z"],
                                        prm.conv_w, prm.conv_b, prm.A, prm.Dskip, prm.dt_bias,
                                        state_indices=idx.astype(np.int64),
                                        y_init=np.full((Bt, D), 9.0))
        gy = host(y)
        assert_close(gy[live], ry[live], bf16, ytol, f"y at step {t}")
        assert np.all(gy[~live] == 9.0), "skipped rows keep their y"
        assert np.array_equal(host(rep["buf_len"]), rrep["len"]), f"buffer lengths at step {t}"
        assert np.array_equal(host(cs), rcs), f"conv state at step {t}"
        assert np.all(host(rep["tickets"]) == 0), "tickets return to zero"
    assert_close(host(rep["ckpt"])[used], rrep["ck"][used], False, tol, "checkpoint")
    assert np.array_equal(host(rep["ckpt"])[unused], np.asarray(st["h0"], np.float64)[unused])
    if keep_lo:
        lo = host(rep["ckpt_lo"])
        # the copy is the checkpoint rounded to bf16 (within half a bf16 step of
        # the exact checkpoint; the oracle's own copy may sit one step away)
        assert_close(lo[used], rrep["ck"][used], True, tol, "bf16 checkpoint copy")
    # the state each slot stands for: materialised by a flush, against the oracle
    ssm.ssm_replay_flush(rep, p["A"])
    assert np.all(host(rep["buf_len"]) == 0)
    assert_close(host(rep["ckpt"])[used], orc.replay_state(rrep, prm.A)[used], False, tol,
                 "flushed state")
    assert ssm.ssm_device_status() == 0


@pytest.mark.parametrize("keep_lo", [False, True])
def test_replay_checkpoint_is_eager_state_bitwise(keep_lo):
    """Eager decode and replay decode on the same tokens: every checkpoint
    step writes exactly the eager state, the conv state matches at every step,
    and without the bf16 copy every output matches up to the order of the
    readout sum."""
    Bt, D, K, W, steps = 12, 512, 4, 4, 13
    prm = synth.make_params(40, D, K=K, random_bias=True)
    p = _dev_params(prm)
    st = synth.make_states(41, Bt, D, K=K, bf16=True, scale=0.5)
    cs_e, h_e = dev(st["conv_state"], BF), dev(st["h0"])
    cs_r = cs_e.clone()
    rep = ssm.replay_buffers(Bt, D, W, "cuda", keep_lo=keep_lo)
    rep["ckpt"].copy_(h_e)
    ssm.ssm_replay_reset(rep)
    y_e = torch.empty((Bt, D), device="cuda", dtype=BF)
    y_r = torch.empty_like(y_e)
    for t in range(steps):
        s = synth.make_activations(200 + t, Bt, D, bf16=True)
        ssm.ssm_selective_state_update(cs_e, h_e, dev(s["x"], BF), dev(s["dt"], BF),
                                       dev(s["B"], BF), dev(s["C"], BF), y_e, p["conv_w"],
                                       p["A"], z=dev(s["z"], BF), conv_b=p["conv_b"],
                                       Dskip=p["Dskip"], dt_bias=p["dt_bias"])
        _step(cs_r, rep, s, y_r, p, BF)
        flush = (t + 1) % W == 0
        assert torch.equal(cs_r, cs_e), t
        if flush or not keep_lo:
            assert _same_up_to_sum_order(y_r, y_e), t
        if flush:
            assert torch.equal(rep["ckpt"], h_e), t
            if keep_lo:
                assert torch.equal(rep["ckpt_lo"], h_e.to(BF)), t
    # mid-window: a flush materialises the eager state exactly
    assert int(host(rep["buf_len"])[0]) == steps % W
    ssm.ssm_replay_flush(rep, p["A"])
    assert torch.equal(rep["ckpt"], h_e)


def test_replay_slots_at_different_window_positions(orc):
    """Rows join at different steps (state_indices subsets), so slots sit at
    different buffer lengths; flushing a subset touches exactly those slots,
    and stepping on afterwards still matches eager decode."""
    n_slots, D, K, W = 8, 256, 4, 4
    prm = _params(50, D, K)
    p = _dev_params(prm)
    st = synth.make_states(51, n_slots, D, K=K, bf16=True, scale=0.3)
    cs_e, h_e = dev(st["conv_state"], BF), dev(st["h0"])
    cs_r = cs_e.clone()
    rep = ssm.replay_buffers(n_slots, D, W, "cuda", keep_lo=False)
    rep["ckpt"].copy_(h_e)
    ssm.ssm_replay_reset(rep)
    plan = [[0, 1, 2, 3, 4, 5, 6, 7], [1, 3, 5], [0, 1, 2], [7, 1], [1, 2, 3, 4], [6, 5, 4]]
    y_e = torch.empty((n_slots, D), device="cuda", dtype=BF)
    y_r = torch.empty_like(y_e)
    lens = np.zeros(n_slots, np.int64)
    for t, rows in enumerate(plan):
        idx = torch.tensor(rows, dtype=torch.int32, device="cuda")
        s = synth.make_activations(300 + t, len(rows), D, bf16=True)
        ye, yr = y_e[:len(rows)], y_r[:len(rows)]
        ssm.ssm_selective_state_update(cs_e, h_e, dev(s["x"], BF), dev(s["dt"], BF),
                                       dev(s["B"], BF), dev(s["C"], BF), ye, p["conv_w"], p["A"],
                                       z=dev(s["z"], BF), conv_b=p["conv_b"], Dskip=p["Dskip"],
                                       dt_bias=p["dt_bias"], state_indices=idx)
        _step(cs_r, rep, s, yr, p, BF, idx)
        for r in rows:
            lens[r] = (lens[r] + 1) % W
        assert _same_up_to_sum_order(yr, ye), t
        assert np.array_equal(host(rep["buf_len"]), lens), t
    sub = torch.tensor([1, 6], dtype=torch.int32, device="cuda")
    before = rep["ckpt"].clone()
    ssm.ssm_replay_flush(rep, p["A"], slots=sub)
    for sl in range(n_slots):
        if sl in (1, 6):
            assert torch.equal(rep["ckpt"][sl], h_e[sl]), sl
            assert int(host(rep["buf_len"])[sl]) == 0
        else:
            assert torch.equal(rep["ckpt"][sl], before[sl]), sl
            assert int(host(rep["buf_len"])[sl]) == lens[sl]
    lens[[1, 6]] = 0
    s = synth.make_activations(399, n_slots, D, bf16=True)
    ssm.ssm_selective_state_update(cs_e, h_e, dev(s["x"], BF), dev(s["dt"], BF), dev(s["B"], BF),
                                   dev(s["C"], BF), y_e, p["conv_w"], p["A"], z=dev(s["z"], BF),
                                   conv_b=p["conv_b"], Dskip=p["Dskip"], dt_bias=p["dt_bias"])
    _step(cs_r, rep, s, y_r, p, BF)
    assert _same_up_to_sum_order(y_r, y_e)
    ssm.ssm_replay_flush(rep, p["A"])
    assert torch.equal(rep["ckpt"], h_e)
    assert ssm.ssm_device_status() == 0


def test_replay_decode_b256_sampled(orc):
    """The batch-256 decode workload through replay decode (W = 4, bf16
    checkpoint copy): states from a 512-token prefill, 1000 steps with fresh
    inputs, checked against the oracle's replay step on sampled channels."""
    w = synth.WORKLOADS["decode_b256_d8192"]
    Bt, D, L0, steps = w["batch"], w["D"], w["prefill_len"], w["steps"]
    W = 4
    prm = synth.make_params(0, D)
    p = _dev_params(prm)
    a = synth.device_activations(0, Bt * L0, D)
    xc = torch.empty_like(a["x"])
    cs = torch.empty((Bt, D, 3), dtype=BF, device="cuda")
    ssm.ssm_causal_conv1d(a["x"], xc, p["conv_w"], bias=p["conv_b"], S=Bt, conv_state_out=cs)
    rep = ssm.replay_buffers(Bt, D, W, "cuda", keep_lo=True)
    yp = torch.empty_like(xc)
    ssm.ssm_selective_scan_fwd(xc, a["dt"], p["A"], a["B"], a["C"], yp, Dskip=p["Dskip"],
                               z=a["z"], dt_bias=p["dt_bias"], h_final=rep["ckpt"], S=Bt)
    ssm.ssm_replay_reset(rep)
    rng = np.random.default_rng(0)
    ch = np.sort(rng.choice(D, size=8, replace=False))
    chd = torch.from_numpy(ch).cuda()
    sp = synth.MixerParams(prm.conv_w[ch], prm.conv_b[ch], prm.A[ch], prm.Dskip[ch],
                           prm.dt_bias[ch])
    pre = {k: host(v.index_select(1, chd)) for k, v in (("x", a["x"]), ("dt", a["dt"]),
                                                        ("z", a["z"]))}
    rxc, rcs = orc.causal_conv1d(pre["x"], sp.conv_w, sp.conv_b, S=Bt, want_state=True)
    _, rh = orc.selective_scan(rxc, pre["dt"], sp.A, host(a["B"]), host(a["C"]), Dskip=sp.Dskip,
                               z=pre["z"], dt_bias=sp.dt_bias, S=Bt, want_state=True)
    rrep = orc.replay_init(rh, W, keep_lo=True)
    del a, xc, yp
    y = torch.empty((Bt, D), device="cuda", dtype=BF)
    for step in range(steps):
        s = synth.device_activations(10_000 + step, Bt, D)
        ssm.ssm_replay_state_update(cs, rep, s["x"], s["dt"], s["B"], s["C"], y, p["conv_w"],
                                    p["A"], z=s["z"], conv_b=p["conv_b"], Dskip=p["Dskip"],
                                    dt_bias=p["dt_bias"])
        g = {k: host(v.index_select(1, chd)) for k, v in (("x", s["x"]), ("dt", s["dt"]),
                                                          ("z", s["z"]), ("y", y))}
        ry, rcs, rrep = orc.replay_step(rcs, rrep, g["x"], g["dt"], host(s["B"]), host(s["C"]),
                                        g["z"], sp.conv_w, sp.conv_b, sp.A, sp.Dskip,
                                        sp.dt_bias)
        if step % 50 == 0 or step == steps - 1:
            assert_close(g["y"], ry, True, TOL_BF16, f"y at step {step}")
    assert np.all(host(rep["buf_len"]) == steps % W)
    ssm.ssm_replay_flush(rep, p["A"])
    assert_close(host(rep["ckpt"].index_select(1, chd)), orc.replay_state(rrep, sp.A), False,
                 TOL_BF16, "state after 1000 steps")
    assert np.array_equal(host(cs.index_select(1, chd)), rcs)
    assert ssm.ssm_device_status() == 0


def test_replay_many_rows_per_cta_bitwise():
    """2048 rows of 8192 channels: each CTA walks about 186 rows, more than
    the 128 rows whose slots and lengths it holds at once, so the row batches
    hand over mid-call. Checkpoints still equal eager decode bit for bit,
    outputs up to the readout's sum order (no bf16 copy), and every length
    advances once per step."""
    Bt, D, W, steps = 2048, 8192, 3, 4
    prm = synth.make_params(60, D)
    p = _dev_params(prm)
    g = torch.Generator(device="cuda")
    g.manual_seed(61)
    h_e = 0.3 * torch.randn((Bt, D, 16), device="cuda", generator=g)
    cs_e = torch.randn((Bt, D, 3), device="cuda", generator=g).to(BF)
    cs_r = cs_e.clone()
    rep = ssm.replay_buffers(Bt, D, W, "cuda", keep_lo=False)
    rep["ckpt"].copy_(h_e)
    ssm.ssm_replay_reset(rep)
    y_e = torch.empty((Bt, D), device="cuda", dtype=BF)
    y_r = torch.empty_like(y_e)
    for t in range(steps):
        s = synth.device_activations(700 + t, Bt, D)
        ssm.ssm_selective_state_update(cs_e, h_e, s["x"], s["dt"], s["B"], s["C"], y_e,
                                       p["conv_w"], p["A"], z=s["z"], conv_b=p["conv_b"],
                                       Dskip=p["Dskip"], dt_bias=p["dt_bias"])
        ssm.ssm_replay_state_update(cs_r, rep, s["x"], s["dt"], s["B"], s["C"], y_r, p["conv_w"],
                                    p["A"], z=s["z"], conv_b=p["conv_b"], Dskip=p["Dskip"],
                                    dt_bias=p["dt_bias"])
        assert _same_up_to_sum_order(y_r, y_e), t
        assert bool((rep["buf_len"] == (t + 1) % W).all()), t
        if (t + 1) % W == 0:
            assert torch.equal(rep["ckpt"], h_e), t
    assert torch.equal(cs_r, cs_e)
    assert bool((rep["tickets"] == 0).all())
    assert ssm.ssm_device_status() == 0


@pytest.mark.parametrize("K", [3, 4])
def test_replay_mixed_dtypes_and_bare_options(orc, K):
    """bf16 activations with an fp32 conv state; no gate, no Dskip, no conv
    bias, no dt_bias and the softplus off (the raw input is the step size)."""
    n_slots, Bt, D, W, steps = 5, 5, 64, 3, 7
    prm = _params(70 + K, D, K)
    p = _dev_params(prm)
    st = synth.make_states(71, n_slots, D, K=K, bf16=False, scale=0.3)
    cs = dev(st["conv_state"])  # fp32 conv state
    rep = ssm.replay_buffers(n_slots, D, W, "cuda", keep_lo=False)
    rep["ckpt"].copy_(dev(st["h0"]))
    ssm.ssm_replay_reset(rep)
    rcs = np.asarray(st["conv_state"], np.float64)
    rrep = orc.replay_init(st["h0"], W, keep_lo=False)
    y = torch.empty((Bt, D), device="cuda", dtype=BF)
    for t in range(steps):
        s = synth.make_activations(400 + t, Bt, D, bf16=True)
        delta = synth.round_bf16(np.logaddexp(0.0, s["dt"].astype(np.float64)
                                              + prm.dt_bias[None, :]).astype(np.float32))
        ssm.ssm_replay_state_update(cs, rep, dev(s["x"], BF), dev(delta, BF), dev(s["B"], BF),
                                    dev(s["C"], BF), y, p["conv_w"], p["A"],
                                    delta_softplus=False)
        ry, rcs, rrep = orc.replay_step(rcs, rrep, s["x"], delta, s["B"], s["C"], None,
                                        prm.conv_w, None, prm.A, None, None,
                                        delta_softplus=False)
        assert_close(host(y), ry, True, TOL_BF16, f"y at step {t}")
        assert_close(host(cs), rcs, False, TOL_F32, f"fp32 conv state at step {t}")
        assert np.array_equal(host(rep["buf_len"]), rrep["len"])
    ssm.ssm_replay_flush(rep, p["A"])
    assert_close(host(rep["ckpt"]), orc.replay_state(rrep, prm.A), False, TOL_BF16, "state")


def test_replay_skips_out_of_range_slots_and_clamps_lengths(orc):
    """A slot index >= n_slots skips its row like -1; a buffer length outside
    0..W-1 (corrupt) is clamped into range, so the call stays in bounds."""
    n_slots, Bt, D, W = 4, 3, 128, 3
    prm = _params(80, D, 4)
    p = _dev_params(prm)
    st = synth.make_states(81, n_slots, D, bf16=True, scale=0.3)
    cs = dev(st["conv_state"], BF)
    rep = ssm.replay_buffers(n_slots, D, W, "cuda", keep_lo=True)
    rep["ckpt"].copy_(dev(st["h0"]))
    ssm.ssm_replay_reset(rep)
    rep["buf_len"][2] = 100  # corrupt: clamped to W-1, a checkpoint step
    idx = torch.tensor([2, 9, 0], dtype=torch.int32, device="cuda")
    s = synth.make_activations(500, Bt, D, bf16=True)
    y = torch.full((Bt, D), 5.0, device="cuda", dtype=BF)
    before = {k: rep[k].clone() for k in ("ckpt", "ckpt_lo", "buf")}
    _step(cs, rep, s, y, p, BF, idx)
    torch.cuda.synchronize()
    assert bool((y[1] == 5.0).all()), "the out-of-range row keeps its y"
    lens = host(rep["buf_len"])
    assert lens[2] == 0 and lens[0] == 1 and lens[1] == 0 and lens[3] == 0
    assert torch.equal(rep["ckpt"][1], before["ckpt"][1])
    assert torch.equal(rep["ckpt"][3], before["ckpt"][3])
    assert not torch.equal(rep["ckpt"][2], before["ckpt"][2]), "slot 2 took a checkpoint step"
    assert ssm.ssm_device_status() == 0
