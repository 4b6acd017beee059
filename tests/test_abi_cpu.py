"""The C-ABI library on the host: it loads without a GPU, exports every symbol
the header declares, and rejects bad arguments before touching any device."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import selective_state_space_causal_b200 as ssm
from selective_state_space_causal_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm_causal.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(ssm_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_three_operations():
    names = declared_functions()
    for op in ("ssm_causal_conv1d", "ssm_selective_scan_fwd", "ssm_selective_state_update"):
        assert op in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIBRARY], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(_lib.lib, name)


def test_binding_covers_every_declared_symbol():
    bound = {name for name, _, _ in _lib.SIGNATURES}
    assert bound == set(declared_functions())


# --- argument validation (fake device addresses; nothing reaches a device) ---
L = _lib.lib
A16 = 0x10000  # 16-byte aligned fake address


def _err():
    return ssm.ssm_last_error()


def conv(**kw):
    args = dict(x=A16, xc=A16 + 0x100000, w=A16, b=None, tok=64, D=32, K=4, cu=None, S=1,
                si=None, so=None, silu=1, xdt=1, sdt=1)
    args.update(kw)
    return L.ssm_causal_conv1d(args["x"], args["xc"], args["w"], args["b"], args["tok"],
                               args["D"], args["K"], args["cu"], args["S"], args["si"],
                               args["so"], args["silu"], args["xdt"], args["sdt"], None)


def scan(**kw):
    a = dict(u=A16, dt=A16 + 0x200000, A=A16, B=A16, C=A16, Dsk=None, z=None, dtb=None, sp=1,
             h0=None, cu=None, S=1, y=A16 + 0x400000, hf=None, tok=64, D=32, N=16, adt=1,
             ws=None, wsb=0)
    a.update(kw)
    return L.ssm_selective_scan_fwd(a["u"], a["dt"], a["A"], a["B"], a["C"], a["Dsk"], a["z"],
                                    a["dtb"], a["sp"], a["h0"], a["cu"], a["S"], a["y"], a["hf"],
                                    a["tok"], a["D"], a["N"], a["adt"], a["ws"], a["wsb"], None)


def decode(**kw):
    a = dict(cs=A16, ss=A16, x=A16, dt=A16, B=A16, C=A16, z=None, w=A16, b=None, A=A16, Dsk=None,
             dtb=None, sp=1, idx=None, slots=8, y=A16, Bt=8, D=32, N=16, K=4, adt=1, cdt=1)
    a.update(kw)
    return L.ssm_selective_state_update(a["cs"], a["ss"], a["x"], a["dt"], a["B"], a["C"],
                                        a["z"], a["w"], a["b"], a["A"], a["Dsk"], a["dtb"],
                                        a["sp"], a["idx"], a["slots"], a["y"], a["Bt"], a["D"],
                                        a["N"], a["K"], a["adt"], a["cdt"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(K=5), -1), (dict(K=1), -1), (dict(S=0), -1), (dict(tok=63, S=2), -1),
    (dict(D=0), -1), (dict(x=None), -1), (dict(w=None), -1), (dict(xc=A16 + 1), -3),
    (dict(xdt=7), -2), (dict(xc=A16 + 64), -1), (dict(S=70000, tok=70000), -1),
    (dict(cu=A16 + 2), -3),
])
def test_conv_rejects(kw, code):
    assert conv(**kw) == code
    assert _err()


@pytest.mark.parametrize("kw,code", [
    (dict(N=8), -1), (dict(N=32), -1), (dict(u=None), -1), (dict(A=None), -1),
    (dict(B=A16 + 8), -3), (dict(u=A16 + 1), -3), (dict(adt=3), -2),
    (dict(y=A16 + 0x200000), -1), (dict(S=3, tok=64), -1),
    (dict(cu=A16, S=4, ws=A16, wsb=8), -5), (dict(cu=A16, S=4, ws=A16 + 16, wsb=4096), -3),
])
def test_scan_rejects(kw, code):
    assert scan(**kw) == code
    assert _err()


@pytest.mark.parametrize("kw,code", [
    (dict(N=4), -1), (dict(K=6), -1), (dict(slots=4), -1), (dict(ss=A16 + 4), -3),
    (dict(A=A16 + 4), -3), (dict(B=A16 + 8), -3), (dict(w=A16 + 4), -3),
    (dict(x=None), -1), (dict(cdt=5), -2), (dict(Bt=70000, slots=70000), -1),
])
def test_decode_rejects(kw, code):
    assert decode(**kw) == code
    assert _err()


def test_workspace_size():
    assert ssm.ssm_scan_workspace_size(100, 64, 16, 1) == 0
    n = ssm.ssm_scan_workspace_size(65536, 5120, 16, 34)
    assert n >= 34 * 4 and n % 256 == 0


def test_check_cu_seqlens_host():
    import torch

    good = torch.tensor([0, 3, 3, 10], dtype=torch.int32)
    ssm.ssm_check_cu_seqlens(good, 10)
    for bad, tok in (([1, 3, 10], 10), ([0, 5, 3, 10], 10), ([0, 3, 9], 10)):
        with pytest.raises(ssm.SsmError) as ei:
            ssm.ssm_check_cu_seqlens(torch.tensor(bad, dtype=torch.int32), tok)
        assert ei.value.code == -4


def test_tuning_knob():
    for n, c in ((0, 0), (2, 1), (4, 1), (4, 2), (4, 3), (8, 2), (16, 1), (16, 2), (16, 12)):
        ssm.ssm_set_scan_variant(n, c)
    for n, c in ((3, 1), (16, 13), (4, -1)):
        with pytest.raises(ssm.SsmError):
            ssm.ssm_set_scan_variant(n, c)
    ssm.ssm_set_scan_variant(0, 0)


def test_bwd_variant_knob_and_choice():
    """The backward takes one thread per channel once S * ceil(D / 128) CTAs
    fill every SM twice (148 SMs when no device is visible), else four lanes
    per channel; a forced kernel is reported as forced."""
    ssm.ssm_set_scan_bwd_variant(0)
    assert ssm.ssm_scan_bwd_variant_for(43, 5120) == 2    # packed 65536 x 5120
    assert ssm.ssm_scan_bwd_variant_for(32, 5120) == 2    # 32 x 2048 x 5120
    assert ssm.ssm_scan_bwd_variant_for(8, 1536) == 1     # 8 x 2048 x 1536 layer
    assert ssm.ssm_scan_bwd_variant_for(1, 8192) == 1
    for v in (1, 2):
        ssm.ssm_set_scan_bwd_variant(v)
        assert ssm.ssm_scan_bwd_variant_for(1, 16) == v
    ssm.ssm_set_scan_bwd_variant(0)
    for v in (-1, 3):
        with pytest.raises(ssm.SsmError) as ei:
            ssm.ssm_set_scan_bwd_variant(v)
        assert ei.value.code == -1
    for S, D in ((0, 16), (4, 0)):
        with pytest.raises(ssm.SsmError):
            ssm.ssm_scan_bwd_variant_for(S, D)


def test_variant_choice():
    """The automatic choice follows (sequence, channel, state) recurrences per
    SM (148 SMs when no device is visible): one lane per channel (schedule 12)
    with at least two waves of its three 128-lane CTAs per SM, else 8 states
    per lane in the pipelined kernel with 16-token chunks when the GPU holds
    about 20 warps per SM of them, else 4 states per lane with 32-token chunks while that still gives
    every SM a block (with the two-CTAs-per-SM register budget when the grid
    has at most two CTAs per SM), else 2 states per lane. A forced variant is
    reported as forced."""
    ssm.ssm_set_scan_variant(0, 0)
    assert ssm.ssm_scan_variant_for(8, 1536) == (4, 10)     # 8 x 2048 x 1536 layer
    assert ssm.ssm_scan_variant_for(43, 5120) == (16, 12)   # packed 65536 x 5120
    assert ssm.ssm_scan_variant_for(32, 5120) == (16, 12)   # 32 x 2048 x 5120
    assert ssm.ssm_scan_variant_for(16, 5120) == (8, 9)     # below two waves of schedule 12
    assert ssm.ssm_scan_variant_for(1, 8192) == (4, 11)     # one 8192-channel sequence
    assert ssm.ssm_scan_variant_for(4, 8192) == (4, 10)
    assert ssm.ssm_scan_variant_for(1, 2048) == (2, 9)
    assert ssm.ssm_scan_variant_for(1, 32) == (2, 9)
    ssm.ssm_set_scan_variant(16, 7)
    assert ssm.ssm_scan_variant_for(1, 32) == (16, 7)
    ssm.ssm_set_scan_variant(0, 0)
    for S, D in ((0, 16), (4, 0)):
        with pytest.raises(ssm.SsmError) as ei:
            ssm.ssm_scan_variant_for(S, D)
        assert ei.value.code == -1


def replay(**kw):
    a = dict(cs=A16, ck=A16, lo=A16, buf=A16, bB=A16, ln=A16, tk=A16, W=4, x=A16, dt=A16, B=A16,
             C=A16, z=None, w=A16, b=None, A=A16, Dsk=None, dtb=None, sp=1, idx=None, slots=8,
             y=A16, Bt=8, D=32, N=16, K=4, adt=1, cdt=1)
    a.update(kw)
    return L.ssm_replay_state_update(a["cs"], a["ck"], a["lo"], a["buf"], a["bB"], a["ln"], a["tk"],
                                     a["W"], a["x"], a["dt"], a["B"], a["C"], a["z"], a["w"],
                                     a["b"], a["A"], a["Dsk"], a["dtb"], a["sp"], a["idx"],
                                     a["slots"], a["y"], a["Bt"], a["D"], a["N"], a["K"], a["adt"],
                                     a["cdt"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(W=0), -1), (dict(W=9), -1), (dict(N=8), -1), (dict(K=5), -1), (dict(slots=4), -1),
    (dict(ck=None), -1), (dict(tk=None), -1), (dict(ln=None), -1), (dict(buf=None), -1),
    (dict(bB=None), -1), (dict(ck=A16 + 4), -3), (dict(lo=A16 + 8), -3), (dict(buf=A16 + 8), -3),
    (dict(D=36), -3), (dict(D=4, adt=0, cdt=1, K=4), -3), (dict(x=A16 + 2), -3), (dict(adt=4), -2),
    (dict(Bt=70000, slots=70000), -1),
])
def test_replay_rejects(kw, code):
    assert replay(**kw) == code
    assert _err()


def test_replay_window_one_needs_no_buffer():
    # W == 1 takes no buffer; with Bt == 0 nothing is launched, so this runs without a GPU
    assert replay(W=1, buf=None, bB=None, Bt=0) == 0


@pytest.mark.parametrize("fn,kw,code", [
    ("reset", dict(N=8), -1), ("reset", dict(n=9, slots_ptr=None), -1),
    ("reset", dict(ln=None), -1), ("reset", dict(lo=A16 + 8), -3),
    ("reset", dict(slots_ptr=A16 + 2), -3),
    ("flush", dict(W=0), -1), ("flush", dict(A=None), -1), ("flush", dict(buf=None), -1),
    ("flush", dict(ck=A16 + 4), -3), ("flush", dict(n=-1), -1),
])
def test_replay_reset_flush_reject(fn, kw, code):
    a = dict(ck=A16, lo=A16, buf=A16, bB=A16, ln=A16, tk=A16, A=A16, W=4, slots_ptr=None, n=8,
             n_slots=8, D=32, N=16)
    a.update(kw)
    if fn == "reset":
        rc = L.ssm_replay_reset(a["ck"], a["lo"], a["ln"], a["tk"], a["slots_ptr"], a["n"],
                                a["n_slots"], a["D"], a["N"], None)
    else:
        rc = L.ssm_replay_flush(a["ck"], a["lo"], a["buf"], a["bB"], a["ln"], a["tk"], a["A"],
                                a["W"], a["slots_ptr"], a["n"], a["n_slots"], a["D"], a["N"], None)
    assert rc == code
    assert _err()


def bwd(**kw):
    a = dict(u=A16, dt=A16 + 0x200000, A=A16, B=A16, C=A16, Dsk=None, z=None, dtb=None, sp=1,
             h0=None, cu=None, S=1, dy=A16 + 0x400000, dhf=None, du=A16 + 0x600000,
             ddt=A16 + 0x800000, dz=None, dB=A16, dC=A16, dA=A16, dDsk=None, ddtb=None,
             dh0=None, tok=64, D=32, N=16, adt=1, ws=A16, wsb=1 << 30)
    a.update(kw)
    return L.ssm_selective_scan_bwd(a["u"], a["dt"], a["A"], a["B"], a["C"], a["Dsk"], a["z"],
                                    a["dtb"], a["sp"], a["h0"], a["cu"], a["S"], a["dy"],
                                    a["dhf"], a["du"], a["ddt"], a["dz"], a["dB"], a["dC"],
                                    a["dA"], a["dDsk"], a["ddtb"], a["dh0"], a["tok"], a["D"],
                                    a["N"], a["adt"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(N=8), -1), (dict(dA=None), -1), (dict(dB=None), -1), (dict(dy=None), -1),
    (dict(du=None), -1), (dict(ws=None), -5), (dict(wsb=64), -5), (dict(ws=A16 + 16), -3),
    (dict(u=A16 + 1), -3), (dict(dA=A16 + 2), -3), (dict(adt=5), -2), (dict(S=0), -1),
    (dict(du=A16 + 0x200000), -1), (dict(tok=63, S=2), -1),
])
def test_scan_bwd_rejects(kw, code):
    assert bwd(**kw) == code
    assert _err()


def test_scan_bwd_overlap_uses_bc_extent():
    """B and C are (tok, N): a gradient right after B's tok x N elements does not
    overlap it, one that starts inside does."""
    B = A16 + 0x1000000
    assert bwd(B=B, C=B, du=B + 64 * 16 * 2 - 2) == -1  # inside B (bf16)
    assert "overlaps" in _err()
    bwd(B=B, C=B, du=B + 64 * 16 * 2)  # just past B: no overlap (fails later without a GPU)
    assert "overlaps" not in _err()


def bwd_ckpt(**kw):
    a = dict(u=A16, dt=A16 + 0x200000, A=A16, B=A16, C=A16, Dsk=None, z=None, dtb=None, sp=1,
             h0=None, cu=None, S=1, dy=A16 + 0x400000, dhf=None, du=A16 + 0x600000,
             ddt=A16 + 0x800000, dz=None, dB=A16, dC=A16, dA=A16, dDsk=None, ddtb=None,
             dh0=None, tok=64, D=32, N=16, adt=1, ws=A16, wsb=1 << 30)
    a.update(kw)
    return L.ssm_selective_scan_bwd_ckpt(a["u"], a["dt"], a["A"], a["B"], a["C"], a["Dsk"],
                                         a["z"], a["dtb"], a["sp"], a["h0"], a["cu"], a["S"],
                                         a["dy"], a["dhf"], a["du"], a["ddt"], a["dz"], a["dB"],
                                         a["dC"], a["dA"], a["dDsk"], a["ddtb"], a["dh0"],
                                         a["tok"], a["D"], a["N"], a["adt"], a["ws"], a["wsb"],
                                         None)


@pytest.mark.parametrize("kw,code", [
    (dict(N=8), -1), (dict(dA=None), -1), (dict(ws=None), -5), (dict(wsb=64), -5),
    (dict(ws=A16 + 16), -3), (dict(u=A16 + 1), -3), (dict(adt=5), -2),
    (dict(du=A16 + 0x200000), -1),
])
def test_scan_bwd_ckpt_rejects(kw, code):
    """The backward that reads the forward's checkpoints checks its arguments
    as ssm_selective_scan_bwd does."""
    assert bwd_ckpt(**kw) == code
    assert "ssm_selective_scan_bwd_ckpt" in _err()


def fwd_ckpt(**kw):
    need = ssm.ssm_scan_bwd_workspace_size(64, 32, 16, 1)
    a = dict(u=A16, dt=A16 + 0x200000, A=A16, B=A16, C=A16, Dsk=None, z=None, dtb=None, sp=1,
             h0=None, cu=None, S=1, y=A16 + 0x400000, hf=None, tok=64, D=32, N=16, adt=1,
             ws=None, wsb=0, bws=A16 + 0x600000, bwsb=need)
    a.update(kw)
    return L.ssm_selective_scan_fwd_ckpt(a["u"], a["dt"], a["A"], a["B"], a["C"], a["Dsk"],
                                         a["z"], a["dtb"], a["sp"], a["h0"], a["cu"], a["S"],
                                         a["y"], a["hf"], a["tok"], a["D"], a["N"], a["adt"],
                                         a["ws"], a["wsb"], a["bws"], a["bwsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(bws=None), -5), (dict(bwsb=64), -5), (dict(bws=A16 + 0x600000 + 16), -3),
    (dict(ws=A16 + 0x600000, wsb=256), -1), (dict(N=8), -1), (dict(A=None), -1),
    (dict(u=A16 + 1), -3), (dict(adt=5), -2), (dict(y=A16 + 0x200000), -1),
])
def test_scan_fwd_ckpt_rejects(kw, code):
    """The forward that writes checkpoints for the backward needs a 256-byte
    aligned backward workspace of ssm_scan_bwd_workspace_size() bytes apart
    from its own workspace, and checks the rest as ssm_selective_scan_fwd."""
    assert fwd_ckpt(**kw) == code
    assert _err()


def test_scan_bwd_workspace_size():
    n = ssm.ssm_scan_bwd_workspace_size(16384, 1536, 16, 8)
    # a 64-byte state per 8 tokens, sequence and channel, plus the sequence order
    assert n % 256 == 0 and n >= (16384 // 8 + 8) * 1536 * 64 + 8 * 4
    assert ssm.ssm_scan_bwd_workspace_size(100, 64, 8, 1) == 0


def conv_scan(**kw):
    a = dict(x=A16, w=A16, b=None, si=None, so=None, xc=None, K=4, sdt=1, dt=A16 + 0x200000,
             A=A16, B=A16, C=A16, Dsk=None, z=None, dtb=None, sp=1, h0=None, cu=None, S=1,
             y=A16 + 0x400000, hf=None, tok=64, D=32, N=16, adt=1)
    a.update(kw)
    return L.ssm_conv_scan_fwd(a["x"], a["w"], a["b"], a["si"], a["so"], a["xc"], a["K"], a["sdt"],
                               a["dt"], a["A"], a["B"], a["C"], a["Dsk"], a["z"], a["dtb"],
                               a["sp"], a["h0"], a["cu"], a["S"], a["y"], a["hf"], a["tok"],
                               a["D"], a["N"], a["adt"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(K=5), -1), (dict(N=8), -1), (dict(w=None), -1), (dict(x=None), -1), (dict(y=None), -1),
    (dict(B=A16 + 8), -3), (dict(x=A16 + 1), -3), (dict(adt=7), -2), (dict(sdt=7), -2),
    (dict(y=A16), -1), (dict(xc=A16 + 0x400000), -1), (dict(S=3, tok=64), -1),
])
def test_conv_scan_rejects(kw, code):
    assert conv_scan(**kw) == code
    assert _err()


@pytest.mark.parametrize("chunk", [8, 16])
def test_bwd_checkpoint_slots_are_distinct_and_fit_the_workspace(chunk):
    """The backward kernels keep sequence s's checkpoint k (k < ceil(len/chunk))
    at slot floor(start/chunk) + s + k, 64 bytes per channel, in a workspace of
    ssm_scan_bwd_workspace_size bytes (the thread-per-channel kernels use
    8-token chunks, the lane-split one 16): no two checkpoints share a slot, and
    every slot and the sequence order after them fit."""
    rng = np.random.default_rng(5)
    for trial in range(200):
        S = int(rng.integers(1, 60))
        lens = rng.integers(0, 300, size=S) * (rng.random(S) > 0.2)  # some empty
        starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
        tok = int(lens.sum())
        slots = [start // chunk + s + k
                 for s, (start, n) in enumerate(zip(starts, lens)) for k in range(-(-n // chunk))]
        assert len(slots) == len(set(slots))
        D = 8
        ws = ssm.ssm_scan_bwd_workspace_size(max(tok, 0), D, 16, S)
        top = (max(slots) + 1) if slots else 0
        assert top * D * 64 + S * 4 <= ws
