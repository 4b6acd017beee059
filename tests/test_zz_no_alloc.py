"""ssm_selective_scan_fwd_noalloc: the scan for callers that cannot allocate.

Some callers cannot allocate device memory at the moment they run the scan:
an inference engine that reserves all of its device memory at start-up and
forbids allocation afterwards, or a plugin whose host framework owns the
device allocator. For them the library keeps the scan's schedule scratch in a
fixed device array instead of a caller-provided workspace. Only packed calls of
two or more sequences use that array (at most 4096 sequences); dense calls and
single sequences need no schedule and take any number of rows.

This file is collected last on purpose, so that a run that stops at the first
failure has already run every other test. It must pass both alone, in a fresh
process (the first call on the device then looks the array up), and after the
other tests.
"""

import numpy as np
import pytest
import torch

import selective_state_space_causal_b200 as ssm
from selective_state_space_causal_b200 import synth

A16 = 0x10000  # fake, 16-byte aligned addresses: rejected calls launch nothing


@pytest.mark.parametrize("S", [4097, 5000])
def test_noalloc_rejects_too_many_packed_sequences(S):
    """More packed sequences than the fixed scratch holds: rejected before any
    launch (fake addresses; nothing reaches a device)."""
    code = ssm.lib.ssm_selective_scan_fwd_noalloc(
        A16, A16 + 0x200000, A16, A16, A16, None, None, None, 1, None, A16, S,
        A16 + 0x400000, None, S, 32, 16, 1, None)
    assert code == -1
    assert "4096" in ssm.ssm_last_error()


def _inputs(seed, tok, D, S):
    prm = synth.make_params(seed, D, random_bias=True, random_A=True, random_D=True)
    act = synth.make_activations(seed, tok, D, bf16=True)
    st = synth.make_states(seed + 1, S, D, bf16=True, scale=0.3)
    bf = torch.bfloat16
    t = {k: torch.from_numpy(act[k]).cuda().to(bf) for k in ("x", "dt", "z", "B", "C")}
    t["A"], t["Dskip"], t["dt_bias"] = (torch.from_numpy(v).cuda()
                                        for v in (prm.A, prm.Dskip, prm.dt_bias))
    t["h0"] = torch.from_numpy(st["h0"]).cuda()
    return t


def _with_workspace(t, cu, S):
    """The existing entry point, with a caller-allocated workspace."""
    tok, D = t["x"].shape
    ws = torch.empty(max(1, ssm.ssm_scan_workspace_size(tok, D, 16, S)), dtype=torch.uint8,
                     device="cuda")
    y = torch.empty_like(t["x"])
    h = torch.empty((S, D, 16), device="cuda")
    ssm.ssm_selective_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], y, Dskip=t["Dskip"],
                               z=t["z"], dt_bias=t["dt_bias"], h0=t["h0"], h_final=h,
                               cu_seqlens=cu, S=S, workspace=ws)
    return y, h


def _check_twice(t, cu, S):
    """Two no-allocation calls in a row, each against the workspace entry point."""
    from gpu_helpers import TOL_BF16, assert_close, host

    y_ref, h_ref = _with_workspace(t, cu, S)
    D = t["x"].shape[1]
    for _ in range(2):
        y = torch.full_like(t["x"], -5.0)
        h = torch.full((S, D, 16), 77.0, device="cuda")
        ssm.ssm_selective_scan_fwd_noalloc(t["x"], t["dt"], t["A"], t["B"], t["C"], y,
                                           Dskip=t["Dskip"], z=t["z"], dt_bias=t["dt_bias"],
                                           h0=t["h0"], h_final=h, cu_seqlens=cu, S=S)
        torch.cuda.synchronize()
        assert_close(host(y), host(y_ref), True, TOL_BF16, "y")
        assert_close(host(h), host(h_ref), False, TOL_BF16, "h_final")
    assert ssm.ssm_device_status(clear=True) == 0


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    ssm.ssm_set_scan_variant(0, 0)
    lens = [300, 0, 17, 129, 1, 64, 250, 9]
    t = _inputs(3, sum(lens), 192, len(lens))
    cu = torch.from_numpy(synth.cu_from_lengths(lens)).cuda()
    _check_twice(t, cu, len(lens))


@pytest.mark.gpu
def test_noalloc_full_scratch_4096_packed_sequences():
    """The largest packed call the fixed array holds: 4096 sequences (the
    longest-first sort still runs at this size), mostly of length 0 or 1."""
    ssm.ssm_set_scan_variant(0, 0)
    rng = np.random.default_rng(11)
    lens = rng.choice([0, 1, 1, 2, 5], size=4096).tolist()
    lens[7], lens[2000], lens[4095] = 130, 64, 33
    t = _inputs(5, sum(lens), 64, len(lens))
    cu = torch.from_numpy(synth.cu_from_lengths(lens)).cuda()
    _check_twice(t, cu, len(lens))


@pytest.mark.gpu
def test_noalloc_dense_rows_beyond_the_packed_limit():
    """Dense rows need no schedule: 5000 rows of 3 tokens run, and match both
    the workspace entry point and the oracle on sampled channels."""
    from gpu_helpers import TOL_BF16, assert_close, host

    import oracle

    ssm.ssm_set_scan_variant(0, 0)
    S, L, D = 5000, 3, 32
    t = _inputs(7, S * L, D, S)
    _check_twice(t, None, S)

    y = torch.empty_like(t["x"])
    h = torch.empty((S, D, 16), device="cuda")
    ssm.ssm_selective_scan_fwd_noalloc(t["x"], t["dt"], t["A"], t["B"], t["C"], y,
                                       Dskip=t["Dskip"], z=t["z"], dt_bias=t["dt_bias"],
                                       h0=t["h0"], h_final=h, S=S)
    torch.cuda.synchronize()
    ch = np.array([0, 13, 31])
    hv = lambda k: host(t[k])  # noqa: E731
    y_ref, h_ref = oracle.load().selective_scan(
        hv("x")[:, ch], hv("dt")[:, ch], hv("A")[ch], hv("B"), hv("C"), Dskip=hv("Dskip")[ch],
        z=hv("z")[:, ch], dt_bias=hv("dt_bias")[ch], h0=hv("h0")[:, ch], S=S, want_state=True)
    assert_close(host(y)[:, ch], y_ref, True, TOL_BF16, "y against the oracle")
    assert_close(host(h)[:, ch], h_ref, False, TOL_BF16, "h_final against the oracle")
    assert ssm.ssm_device_status(clear=True) == 0


@pytest.mark.gpu
def test_noalloc_rejects_4097_packed_sequences_on_the_device():
    """One sequence more than the array holds, with real device buffers: the
    call is refused and nothing is written."""
    lens = [1] * 4097
    t = _inputs(9, sum(lens), 16, len(lens))
    cu = torch.from_numpy(synth.cu_from_lengths(lens)).cuda()
    y = torch.full_like(t["x"], 3.0)
    with pytest.raises(RuntimeError, match="4096"):
        ssm.ssm_selective_scan_fwd_noalloc(t["x"], t["dt"], t["A"], t["B"], t["C"], y,
                                           cu_seqlens=cu, S=len(lens))
    torch.cuda.synchronize()
    assert bool((y == 3.0).all())
