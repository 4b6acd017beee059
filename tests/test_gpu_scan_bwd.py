"""Backward of the selective scan on the GPU against the fp64 oracle's
backward (itself pinned to finite differences of the forward), for training on
packed sequences (PackMamba abstract).

Tolerances follow gpu_helpers: outputs stored in the activation dtype (du,
ddelta, dz) take the bf16 bound with one bf16 step of slack for bf16
activations and 1e-4 rms for fp32; the fp32 outputs (dB, dC, dA, dDskip,
ddt_bias, dh0) take the bare bound of the activation dtype.
"""

import numpy as np
import pytest
import torch

import selective_state_space_causal_b200 as ssm
from selective_state_space_causal_b200 import synth
from gpu_helpers import TOL_BF16, TOL_F32, act_dtype, assert_close, cu_tensor, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[1, 2], ids=["lanes4", "thread"])
def variant(request):
    """Every test runs on both kernels: 4 lanes per channel, and one thread per
    channel with all 16 states."""
    ssm.ssm_set_scan_bwd_variant(request.param)
    yield request.param
    ssm.ssm_set_scan_bwd_variant(0)


def _run_bwd(u, dt, A, B, C, dy, Dskip, z, dt_bias, h0, dh_final, cu, S, softplus=True,
             from_fwd=False):
    """from_fwd: the workspace is filled by ssm_selective_scan_fwd_ckpt first,
    whose y and h_final must be those of ssm_selective_scan_fwd bit for bit,
    and the backward reads its checkpoints (ssm_selective_scan_bwd_ckpt)."""
    tok, D = u.shape
    N = A.shape[1]
    f32 = dict(device="cuda", dtype=torch.float32)
    g = {"du": torch.full_like(u, 7.0), "ddelta": torch.full_like(u, 7.0),
         "dz": torch.full_like(u, 7.0) if z is not None else None,
         "dB": torch.full((tok, N), 7.0, **f32), "dC": torch.full((tok, N), 7.0, **f32),
         "dA": torch.full((D, N), 7.0, **f32), "dDskip": torch.full((D,), 7.0, **f32),
         "ddt_bias": torch.full((D,), 7.0, **f32), "dh0": torch.full((S, D, N), 7.0, **f32)}
    ws = torch.empty(max(1, ssm.ssm_scan_bwd_workspace_size(tok, D, N, S)), dtype=torch.uint8,
                     device="cuda")
    if from_fwd:
        fws = torch.empty(max(1, ssm.ssm_scan_workspace_size(tok, D, N, S)), dtype=torch.uint8,
                          device="cuda")
        ys = [torch.full_like(u, 3.0) for _ in range(2)]
        hs = [torch.full((S, D, N), 3.0, device="cuda") for _ in range(2)]
        kw = dict(Dskip=Dskip, z=z, dt_bias=dt_bias, delta_softplus=softplus, h0=h0,
                  cu_seqlens=cu, S=S, workspace=fws)
        ws.fill_(0xFF)  # NaN everywhere a checkpoint is not written
        ssm.ssm_selective_scan_fwd_ckpt(u, dt, A, B, C, ys[0], ws, h_final=hs[0], **kw)
        ssm.ssm_selective_scan_fwd(u, dt, A, B, C, ys[1], h_final=hs[1], **kw)
        torch.cuda.synchronize()
        assert torch.equal(ys[0], ys[1]), "y of the checkpointing forward"
        assert torch.equal(hs[0], hs[1]), "h_final of the checkpointing forward"
    ssm.ssm_selective_scan_bwd(u, dt, A, B, C, dy, g, Dskip=Dskip, z=z, dt_bias=dt_bias,
                               delta_softplus=softplus, h0=h0, dh_final=dh_final, cu_seqlens=cu,
                               S=S, workspace=ws, from_fwd_ckpt=from_fwd)
    torch.cuda.synchronize()
    return g


def _check(orc, bf16, lens, D, gate=True, softplus=True, dense_rows=None, seed=0,
           from_fwd=False):
    dt_ = act_dtype(bf16)
    if dense_rows:
        tok = dense_rows[0] * dense_rows[1]
        cu_d, cu_h, S = None, None, dense_rows[0]
    else:
        cu_d, cu_h = cu_tensor(lens)
        tok, S = int(cu_h[-1]), len(lens)
    prm = synth.make_params(seed, D, random_bias=True, random_A=True, random_D=True)
    act = synth.make_activations(seed, tok, D, bf16=bf16)
    rng = np.random.default_rng(seed + 7)
    dy = rng.standard_normal((tok, D)).astype(np.float32)
    if bf16:
        dy = synth.round_bf16(dy)
    st = synth.make_states(seed + 1, S, D, bf16=bf16, scale=0.3)
    dhf = (0.3 * rng.standard_normal((S, D, 16))).astype(np.float32)
    z = act["z"] if gate else None
    delta, dtb = act["dt"], prm.dt_bias
    if not softplus:
        # without the softplus the input is the step size itself: positive values
        delta = np.logaddexp(0.0, act["dt"].astype(np.float64) + prm.dt_bias[None, :])
        delta = synth.round_bf16(delta.astype(np.float32)) if bf16 else delta.astype(np.float32)
        dtb = None
    g = _run_bwd(dev(act["x"], dt_), dev(delta, dt_), dev(prm.A), dev(act["B"], dt_),
                 dev(act["C"], dt_), dev(dy, dt_), dev(prm.Dskip), dev(z, dt_) if gate else None,
                 dev(dtb), dev(st["h0"]), dev(dhf), cu_d, S, softplus, from_fwd)
    r = orc.selective_scan_bwd(act["x"], delta, prm.A, act["B"], act["C"], dy,
                               Dskip=prm.Dskip, z=z, dt_bias=dtb, delta_softplus=softplus,
                               h0=st["h0"], cu_seqlens=None if dense_rows else cu_h,
                               S=S if dense_rows else None, dh_final=dhf)
    tol = TOL_BF16 if bf16 else TOL_F32
    assert_close(host(g["du"]), r["du"], bf16, tol, "du")
    assert_close(host(g["ddelta"]), r["ddt"], bf16, tol, "ddelta")
    if gate:
        assert_close(host(g["dz"]), r["dz"], bf16, tol, "dz")
    for k, rk in (("dB", "dB"), ("dC", "dC"), ("dA", "dA"), ("dDskip", "dDskip"),
                  ("ddt_bias", "ddt_bias"), ("dh0", "dh0")):
        if k == "ddt_bias" and dtb is None:
            continue
        assert_close(host(g[k]), r[rk], False, tol, k)
    assert ssm.ssm_device_status() == 0
    return g


@pytest.mark.parametrize("bf16", [False, True])
def test_bwd_packed_matches_oracle(orc, bf16, variant):
    # chunk edges at 8 and 16 tokens: lengths below, at, across and far beyond
    # them; an empty and a one-token sequence; a partial channel block
    _check(orc, bf16, [37, 0, 1, 130, 16, 17, 5], 40)


@pytest.mark.parametrize("bf16", [False, True])
def test_bwd_no_gate_no_softplus(orc, bf16, variant):
    _check(orc, bf16, [20, 3, 48], 64, gate=False, softplus=False, seed=3)


def test_bwd_dense_rows(orc, variant):
    _check(orc, True, None, 96, dense_rows=(3, 80), seed=5)


def test_bwd_deterministic_outputs(variant):
    """Two runs agree bit for bit on the per-token gradients and dh0; the
    atomically summed ones agree to fp32 rounding."""
    lens = [300, 77, 1000]
    cu_d, cu_h = cu_tensor(lens)
    tok, S, D = int(cu_h[-1]), len(lens), 256
    prm = synth.make_params(9, D, random_bias=True)
    a = synth.device_activations(9, tok, D)
    dy = synth.device_activations(10, tok, D)["x"]
    p = {k: dev(getattr(prm, k)) for k in ("A", "Dskip", "dt_bias")}
    runs = [_run_bwd(a["x"], a["dt"], p["A"], a["B"], a["C"], dy, p["Dskip"], a["z"],
                     p["dt_bias"], None, None, cu_d, S) for _ in range(2)]
    for k in ("du", "ddelta", "dz", "dh0"):
        assert torch.equal(runs[0][k], runs[1][k]), k
    for k in ("dB", "dC", "dA", "dDskip", "ddt_bias"):
        x, y = runs[0][k], runs[1][k]
        assert torch.allclose(x, y, rtol=1e-5, atol=1e-5 * float(y.abs().max())), k


@pytest.mark.parametrize("from_fwd", [False, True], ids=["own_ckpt", "fwd_ckpt"])
def test_bwd_packmamba_workload_sampled(orc, variant, from_fwd):
    """The packed 65536-token, 5120-channel training shape: per-token gradients,
    dA, dDskip, ddt_bias and dh0 of sampled channels against the oracle run on
    those channels alone (channels are independent for these); also with the
    checkpoints written by the forward (2.7 GB of them at this shape)."""
    w = synth.WORKLOADS["packmamba_2p8b_varlen_65536"]
    D, tot = w["D"], w["total"]
    lens = synth.sample_lengths(0, tot, w["len_lo"], w["len_hi"])
    cu_d, cu_h = cu_tensor(lens)
    S = len(lens)
    prm = synth.make_params(0, D)
    p = {k: dev(getattr(prm, k)) for k in ("A", "Dskip", "dt_bias")}
    a = synth.device_activations(0, tot, D)
    dy = synth.device_activations(1, tot, D)["x"]
    g = _run_bwd(a["x"], a["dt"], p["A"], a["B"], a["C"], dy, p["Dskip"], a["z"], p["dt_bias"],
                 None, None, cu_d, S, from_fwd=from_fwd)
    rng = np.random.default_rng(0)
    ch = np.sort(rng.choice(D, size=6, replace=False))
    chd = torch.from_numpy(ch).cuda()
    sel = lambda t: host(t.index_select(1, chd))  # noqa: E731
    r = orc.selective_scan_bwd(sel(a["x"]), sel(a["dt"]), prm.A[ch], host(a["B"]), host(a["C"]),
                               sel(dy), Dskip=prm.Dskip[ch], z=sel(a["z"]),
                               dt_bias=prm.dt_bias[ch], cu_seqlens=cu_h)
    for k, rk in (("du", "du"), ("ddelta", "ddt"), ("dz", "dz")):
        assert_close(sel(g[k]), r[rk], True, TOL_BF16, k)
    assert_close(host(g["dA"])[ch], r["dA"], False, TOL_BF16, "dA")
    assert_close(host(g["dDskip"])[ch], r["dDskip"], False, TOL_BF16, "dDskip")
    assert_close(host(g["ddt_bias"])[ch], r["ddt_bias"], False, TOL_BF16, "ddt_bias")
    assert_close(host(g["dh0"])[:, ch], r["dh0"], False, TOL_BF16, "dh0")
    assert ssm.ssm_device_status() == 0


@pytest.mark.parametrize("bf16", [False, True])
def test_bwd_unaligned_rows_scalar_staging(orc, bf16, variant):
    """D = 36: bf16 rows are not a multiple of 16 bytes, so the chunk inputs are
    staged with scalar loads (fp32 rows of 144 bytes still take the copies)."""
    _check(orc, bf16, [19, 40, 2], 36, seed=11)


def test_bwd_optional_inputs_absent(orc, variant):
    """No Dskip, dt_bias, h0, dh_final and no dz output: the remaining gradients
    still match the oracle, which takes the same absences as zeros."""
    lens = [33, 9]
    cu_d, cu_h = cu_tensor(lens)
    tok, S, D = int(cu_h[-1]), len(lens), 48
    prm = synth.make_params(12, D, random_A=True)
    act = synth.make_activations(12, tok, D, bf16=True)
    dy = synth.round_bf16(np.random.default_rng(13).standard_normal((tok, D)).astype(np.float32))
    BF = torch.bfloat16
    f32 = dict(device="cuda", dtype=torch.float32)
    u = dev(act["x"], BF)
    g = {"du": torch.empty_like(u), "ddelta": torch.empty_like(u), "dz": None,
         "dB": torch.empty((tok, 16), **f32), "dC": torch.empty((tok, 16), **f32),
         "dA": torch.empty((D, 16), **f32)}
    ws = torch.empty(ssm.ssm_scan_bwd_workspace_size(tok, D, 16, S), dtype=torch.uint8,
                     device="cuda")
    ssm.ssm_selective_scan_bwd(u, dev(act["dt"], BF), dev(prm.A), dev(act["B"], BF),
                               dev(act["C"], BF), dev(dy, BF), g, z=dev(act["z"], BF),
                               cu_seqlens=cu_d, workspace=ws)
    torch.cuda.synchronize()
    r = orc.selective_scan_bwd(act["x"], act["dt"], prm.A, act["B"], act["C"], dy,
                               z=act["z"], cu_seqlens=cu_h)
    assert_close(host(g["du"]), r["du"], True, TOL_BF16, "du")
    assert_close(host(g["ddelta"]), r["ddt"], True, TOL_BF16, "ddelta")
    for k in ("dB", "dC", "dA"):
        assert_close(host(g[k]), r[k], False, TOL_BF16, k)
    assert ssm.ssm_device_status() == 0


def test_bwd_many_channel_blocks_and_odd_sums(orc, variant):
    """Several 128-channel blocks with a partial last one (D = 300), sequence
    lengths around the 8- and 16-token chunks and an fp32 dB / dC pair that is
    only 4-byte aligned (scalar atomics)."""
    lens = [8, 7, 9, 64, 65, 3, 200]
    cu_d, cu_h = cu_tensor(lens)
    tok, S, D = int(cu_h[-1]), len(lens), 300
    prm = synth.make_params(21, D, random_bias=True, random_A=True, random_D=True)
    act = synth.make_activations(21, tok, D, bf16=True)
    dy = synth.round_bf16(np.random.default_rng(22).standard_normal((tok, D)).astype(np.float32))
    BF = torch.bfloat16
    f32 = dict(device="cuda", dtype=torch.float32)
    u = dev(act["x"], BF)
    flat = torch.zeros(2 * tok * 16 + 2, **f32)
    g = {"du": torch.empty_like(u), "ddelta": torch.empty_like(u), "dz": torch.empty_like(u),
         "dB": flat[1:1 + tok * 16].view(tok, 16),
         "dC": flat[2 + tok * 16:2 + 2 * tok * 16].view(tok, 16),
         "dA": torch.empty((D, 16), **f32), "dDskip": torch.empty((D,), **f32),
         "ddt_bias": torch.empty((D,), **f32), "dh0": torch.empty((S, D, 16), **f32)}
    assert g["dB"].data_ptr() % 16 != 0 and g["dC"].data_ptr() % 16 != 0
    ws = torch.empty(ssm.ssm_scan_bwd_workspace_size(tok, D, 16, S), dtype=torch.uint8,
                     device="cuda")
    ssm.ssm_selective_scan_bwd(u, dev(act["dt"], BF), dev(prm.A), dev(act["B"], BF),
                               dev(act["C"], BF), dev(dy, BF), g, Dskip=dev(prm.Dskip),
                               z=dev(act["z"], BF), dt_bias=dev(prm.dt_bias), cu_seqlens=cu_d,
                               workspace=ws)
    torch.cuda.synchronize()
    r = orc.selective_scan_bwd(act["x"], act["dt"], prm.A, act["B"], act["C"], dy,
                               Dskip=prm.Dskip, z=act["z"], dt_bias=prm.dt_bias, cu_seqlens=cu_h)
    for k, rk in (("du", "du"), ("ddelta", "ddt"), ("dz", "dz")):
        assert_close(host(g[k]), r[rk], True, TOL_BF16, k)
    for k in ("dB", "dC", "dA", "dDskip", "ddt_bias", "dh0"):
        assert_close(host(g[k]), r[k], False, TOL_BF16, k)
    assert ssm.ssm_device_status() == 0


def test_bwd_many_short_sequences_past_the_sort_limit(orc, variant):
    """5000 packed sequences of 0 to 6 tokens: more than the longest-first sort
    handles (the order stays as given), with h0 and dh_final for each."""
    lens = list(np.random.default_rng(23).integers(0, 7, size=5000))
    _check(orc, True, lens, 128, seed=23)


@pytest.fixture(params=[(0, 0), (2, 9), (4, 10), (8, 9), (4, 11), (4, 1), (16, 12)],
                ids=["fwd_pick", "pipe2", "pipe4", "pipe8", "pipe4_255reg", "fwd_sched1", "wide16"])
def fwd_sched(request):
    """The forward that writes the checkpoints: the library's pick, the
    pipelined kernel at 2, 4 and 8 states per lane (it writes them as it goes),
    schedule 1 (no checkpoint output: the library adds its checkpointing
    pass) and schedule 12 (one lane per channel, also writing them as it
    goes)."""
    ssm.ssm_set_scan_variant(*request.param)
    yield request.param
    ssm.ssm_set_scan_variant(0, 0)


@pytest.mark.parametrize("bf16", [False, True])
def test_bwd_from_forward_checkpoints(orc, bf16, variant, fwd_sched):
    """ssm_selective_scan_fwd_ckpt then ssm_selective_scan_bwd_ckpt: the same
    y and h_final as the plain forward, gradients against the oracle; chunk
    and checkpoint edges (8, 16, 32 tokens) below, at and across, an empty and
    a one-token sequence, a partial channel block. The workspace starts as
    NaN, so a checkpoint the forward fails to write shows up."""
    _check(orc, bf16, [37, 0, 1, 130, 16, 17, 5, 64, 33], 40, from_fwd=True)


def test_bwd_from_forward_checkpoints_dense_wide(orc, variant, fwd_sched):
    """Dense rows over several channel blocks with a ragged channel tail."""
    _check(orc, True, None, 200, dense_rows=(2, 96), seed=4, from_fwd=True)


@pytest.mark.parametrize("bf16", [False, True])
def test_bwd_from_forward_checkpoints_unaligned(orc, bf16, variant):
    """D = 36: no pipelined forward for bf16 rows of 72 bytes; the
    checkpointing pass writes them."""
    _check(orc, bf16, [19, 40, 2], 36, seed=11, from_fwd=True)
