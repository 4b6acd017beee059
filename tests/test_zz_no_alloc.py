"""ssm_selective_scan_fwd_noalloc: the scan for callers that cannot allocate.

Some callers cannot allocate device memory at the moment they run the scan:
an inference engine that reserves all of its device memory at start-up and
forbids allocation afterwards, or a plugin whose host framework owns the
device allocator. For them the library keeps the scan's schedule scratch in a
fixed device array instead of a caller-provided workspace.

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


def test_noalloc_rejects_too_many_sequences():
    """More packed sequences than the fixed scratch holds: rejected before any
    launch (fake addresses; nothing reaches a device)."""
    A16 = 0x10000
    code = ssm.lib.ssm_selective_scan_fwd_noalloc(
        A16, A16 + 0x200000, A16, A16, A16, None, None, None, 1, None, A16, 5000,
        A16 + 0x400000, None, 5000, 32, 16, 1, None)
    assert code == -1
    assert "4096" in ssm.ssm_last_error()


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    from gpu_helpers import TOL_BF16, assert_close, host

    ssm.ssm_set_scan_variant(0, 0)
    lens = [300, 0, 17, 129, 1, 64, 250, 9]
    D = 192
    tok = sum(lens)
    cu = torch.from_numpy(synth.cu_from_lengths(lens)).cuda()
    S = len(lens)
    prm = synth.make_params(3, D, random_bias=True, random_A=True, random_D=True)
    act = synth.make_activations(3, tok, D, bf16=True)
    st = synth.make_states(4, S, D, bf16=True, scale=0.3)
    bf = torch.bfloat16
    u, dt, z = (torch.from_numpy(act[k]).cuda().to(bf) for k in ("x", "dt", "z"))
    Bm, Cm = (torch.from_numpy(act[k]).cuda().to(bf) for k in ("B", "C"))
    A, Dk, dtb = (torch.from_numpy(v).cuda() for v in (prm.A, prm.Dskip, prm.dt_bias))
    h0 = torch.from_numpy(st["h0"]).cuda()

    # the existing entry point, with a caller-allocated workspace
    ws = torch.empty(ssm.ssm_scan_workspace_size(tok, D, 16, S), dtype=torch.uint8, device="cuda")
    y_ref = torch.empty_like(u)
    h_ref = torch.empty((S, D, 16), device="cuda")
    ssm.ssm_selective_scan_fwd(u, dt, A, Bm, Cm, y_ref, Dskip=Dk, z=z, dt_bias=dtb, h0=h0,
                               h_final=h_ref, cu_seqlens=cu, S=S, workspace=ws)

    # the no-allocation entry point, twice in a row
    for _ in range(2):
        y = torch.full_like(u, -5.0)
        h = torch.full((S, D, 16), 77.0, device="cuda")
        ssm.ssm_selective_scan_fwd_noalloc(u, dt, A, Bm, Cm, y, Dskip=Dk, z=z, dt_bias=dtb,
                                           h0=h0, h_final=h, cu_seqlens=cu, S=S)
        torch.cuda.synchronize()
        assert_close(host(y), host(y_ref), True, TOL_BF16, "y")
        assert_close(host(h), host(h_ref), False, TOL_BF16, "h_final")
    assert ssm.ssm_device_status(clear=True) == 0
