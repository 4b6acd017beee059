"""One conv call and one scan call whose (tokens, channels) tensors hold more
than 2^31 elements (270336 tokens x 8192 channels, 4.4 GB each in bf16), so
that any 32-bit element offset in the index arithmetic of either kernel would
wrap: the conv output, the scan output and the final state of sampled
channels (the first and the last channel among them) against the fp64 oracle
over every token. About 23 GB of device memory."""

import numpy as np
import pytest
import torch

import selective_state_space_causal_b200 as ssm
from selective_state_space_causal_b200 import synth
from gpu_helpers import TOL_BF16, assert_close, dev, host, run_conv, run_scan

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[(0, 0), (16, 12)], ids=["pick", "one_lane_per_channel"])
def scan_variant(request):
    """The library's pick for one 8192-channel sequence (4 states per lane),
    and schedule 12 forced (one lane per channel), whose offsets are computed
    apart from the other schedules'."""
    ssm.ssm_set_scan_variant(*request.param)
    yield request.param
    ssm.ssm_set_scan_variant(0, 0)


def test_conv_and_scan_past_2_31_elements(orc, scan_variant):
    D, L = 8192, 270336
    assert L * D > 2 ** 31
    prm = synth.make_params(7, D)
    p = {k: dev(getattr(prm, k)) for k in ("conv_w", "conv_b", "A", "Dskip", "dt_bias")}
    a = synth.device_activations(7, L, D)
    xc, _ = run_conv(a["x"], p["conv_w"], p["conv_b"])
    y, hf = run_scan(xc, a["dt"], p["A"], a["B"], a["C"], Dskip=p["Dskip"], z=a["z"],
                     dt_bias=p["dt_bias"])
    torch.cuda.synchronize()
    rng = np.random.default_rng(7)
    ch = np.unique(np.concatenate([[0, D - 1], rng.choice(D, size=4, replace=False)]))
    chd = torch.from_numpy(ch).cuda()
    g = {k: host(v.index_select(1, chd)) for k, v in (("x", a["x"]), ("dt", a["dt"]),
                                                      ("z", a["z"]), ("xc", xc), ("y", y))}
    sp = synth.MixerParams(prm.conv_w[ch], prm.conv_b[ch], prm.A[ch], prm.Dskip[ch],
                           prm.dt_bias[ch])
    rxc = orc.causal_conv1d(g["x"], sp.conv_w, sp.conv_b)
    assert_close(g["xc"], rxc, True, TOL_BF16, "xc past 2^31 elements")
    ry, rh = orc.selective_scan(g["xc"], g["dt"], sp.A, host(a["B"]), host(a["C"]),
                                Dskip=sp.Dskip, z=g["z"], dt_bias=sp.dt_bias, want_state=True)
    assert_close(g["y"], ry, True, TOL_BF16, "y past 2^31 elements")
    assert_close(host(hf)[:, ch], rh, False, TOL_BF16, "h_final past 2^31 elements")
    # the last tokens (the highest offsets) in particular
    assert_close(g["y"][-64:], ry[-64:], True, TOL_BF16, "y of the last 64 tokens")
