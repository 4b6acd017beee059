"""Failure detection on the device: a bounded wait that runs out reports it.

Every TMA-staged kernel waits for its tiles on an mbarrier with a bounded
number of suspending tries; when they run out it sets a status bit and returns
instead of hanging. Here a self-test kernel waits on a barrier that expects
bytes no copy delivers, with the limit lowered, so the wait must run out: the
kernel returns, the status bit is set, and after clearing it the library's
kernels run and the status stays clean. Nothing faults, traps or hangs.
"""

import pytest
import torch

import selective_state_space_causal_b200 as ssm

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports(orc):
    from gpu_helpers import TOL_BF16, assert_close, cu_tensor, dev, host, run_scan

    from selective_state_space_causal_b200 import synth

    assert ssm.ssm_device_status(clear=True) == 0
    ssm.ssm_selftest_wait_timeout(64)
    torch.cuda.synchronize()
    assert ssm.ssm_device_status() == 16          # only the self-test's bit
    assert ssm.ssm_device_status(clear=True) == 16
    assert ssm.ssm_device_status() == 0

    # the context is still usable: a TMA-staged scan runs and matches the oracle
    lens = [100, 3, 57]
    D = 64
    prm = synth.make_params(21, D, random_A=True)
    act = synth.make_activations(21, sum(lens), D, bf16=True)
    cu_d, cu_h = cu_tensor(lens)
    bf = torch.bfloat16
    y, hf = run_scan(dev(act["x"], bf), dev(act["dt"], bf), dev(prm.A), dev(act["B"], bf),
                     dev(act["C"], bf), Dskip=dev(prm.Dskip), z=dev(act["z"], bf),
                     dt_bias=dev(prm.dt_bias), cu=cu_d)
    ry, rh = orc.selective_scan(act["x"], act["dt"], prm.A, act["B"], act["C"], Dskip=prm.Dskip,
                                z=act["z"], dt_bias=prm.dt_bias, cu_seqlens=cu_h, want_state=True)
    assert_close(host(y), ry, True, TOL_BF16, "y")
    assert_close(host(hf), rh, False, TOL_BF16, "h_final")
    assert ssm.ssm_device_status() == 0


def test_wait_selftest_rejects_bad_limits():
    for tries in (0, -1, (1 << 17) + 1):
        with pytest.raises(ssm.SsmError):
            ssm.ssm_selftest_wait_timeout(tries)
