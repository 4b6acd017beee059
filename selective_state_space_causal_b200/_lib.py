"""ctypes binding of libssm_causal.so (argument marshalling only).

Each function here has the name of the C entry point it calls and does
nothing but turn tensors into pointers, dtypes into enums and the current
torch stream into a stream handle; every step of the computation runs in the
library's CUDA kernels. There is no fallback: if the library is missing the
import fails, and a failing call raises SsmError with the library's message.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(HERE, "libssm_causal.so")

SSM_F32, SSM_BF16 = 0, 1
STATUS = {0: "SSM_OK", -1: "SSM_ERR_INVALID_ARGUMENT", -2: "SSM_ERR_UNSUPPORTED_DTYPE",
          -3: "SSM_ERR_MISALIGNED", -4: "SSM_ERR_BAD_SEQLENS", -5: "SSM_ERR_WORKSPACE",
          -6: "SSM_ERR_CUDA"}

# (name, restype, argtypes) of every symbol include/ssm_causal.h declares
_vp, _i64, _int, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
SIGNATURES = [
    ("ssm_last_error", ctypes.c_char_p, []),
    ("ssm_version", _int, []),
    ("ssm_launch_count", ctypes.c_ulonglong, []),
    ("ssm_set_scan_variant", _int, [_int, _int]),
    ("ssm_scan_variant_for", _int, [_i64, _i64, ctypes.POINTER(_int), ctypes.POINTER(_int)]),
    ("ssm_device_status", _int, [_int]),
    ("ssm_check_cu_seqlens", _int, [_vp, _i64, _i64]),
    ("ssm_causal_conv1d", _int, [_vp, _vp, _vp, _vp, _i64, _i64, _int, _vp, _i64, _vp, _vp, _int,
                                 _int, _int, _vp]),
    ("ssm_scan_workspace_size", _sz, [_i64, _i64, _int, _i64]),
    ("ssm_selective_scan_fwd", _int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp, _vp, _i64,
                                      _vp, _vp, _i64, _i64, _int, _int, _vp, _sz, _vp]),
    ("ssm_selective_scan_fwd_ckpt", _int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp, _vp,
                                           _i64, _vp, _vp, _i64, _i64, _int, _int, _vp, _sz, _vp,
                                           _sz, _vp]),
    ("ssm_selective_scan_fwd_noalloc", _int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp,
                                              _vp, _i64, _vp, _vp, _i64, _i64, _int, _int, _vp]),
    ("ssm_selective_state_update", _int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                          _vp, _int, _vp, _i64, _vp, _i64, _i64, _int, _int, _int,
                                          _int, _vp]),
    ("ssm_conv_scan_fwd", _int, [_vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _vp, _vp, _vp, _vp,
                                 _vp, _vp, _vp, _int, _vp, _vp, _i64, _vp, _vp, _i64, _i64, _int,
                                 _int, _vp]),
    ("ssm_scan_bwd_workspace_size", _sz, [_i64, _i64, _int, _i64]),
    ("ssm_set_scan_bwd_variant", _int, [_int]),
    ("ssm_scan_bwd_variant_for", _int, [_i64, _i64, ctypes.POINTER(_int)]),
    ("ssm_selective_scan_bwd", _int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp, _vp, _i64,
                                      _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64,
                                      _i64, _int, _int, _vp, _sz, _vp]),
    ("ssm_selective_scan_bwd_ckpt", _int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp, _vp,
                                           _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                           _vp, _i64, _i64, _int, _int, _vp, _sz, _vp]),
    ("ssm_replay_state_update", _int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp, _vp, _vp, _vp,
                                       _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp, _i64, _vp, _i64,
                                       _i64, _int, _int, _int, _int, _vp]),
    ("ssm_replay_reset", _int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp]),
    ("ssm_replay_flush", _int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp, _i64, _i64, _i64,
                                _int, _vp]),
    ("ssm_selftest_wait_timeout", _int, [_int, _vp]),
    ("ssm_probe_sink_floats", _i64, []),
    ("ssm_probe_rate", _int, [_int, _int, _int, _vp, _i64, ctypes.POINTER(ctypes.c_double), _vp]),
]


class SsmError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"{STATUS.get(code, code)}: {message}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIBRARY):
        raise ImportError(
            f"{LIBRARY} is missing: build it with `python selective_state_space_causal_b200/build.py`"
        )
    lib = ctypes.CDLL(LIBRARY)
    for name, res, args in SIGNATURES:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _check(code: int) -> None:
    if code != 0:
        raise SsmError(code, lib.ssm_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dtype(t) -> int:
    import torch

    if t.dtype == torch.bfloat16:
        return SSM_BF16
    if t.dtype == torch.float32:
        return SSM_F32
    raise SsmError(-2, f"unsupported tensor dtype {t.dtype}")


def _stream(stream):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch

    return torch.cuda.current_stream().cuda_stream


def ssm_last_error() -> str:
    return lib.ssm_last_error().decode()


def ssm_version() -> int:
    return lib.ssm_version()


def ssm_launch_count() -> int:
    return int(lib.ssm_launch_count())


def ssm_set_scan_variant(states_per_lane: int, schedule: int = 0) -> None:
    _check(lib.ssm_set_scan_variant(int(states_per_lane), int(schedule)))


def ssm_scan_variant_for(S: int, D: int) -> tuple[int, int]:
    """(states per lane, schedule) the scan picks for S sequences of D channels."""
    npt, sched = _int(0), _int(0)
    _check(lib.ssm_scan_variant_for(int(S), int(D), ctypes.byref(npt), ctypes.byref(sched)))
    return npt.value, sched.value


def ssm_probe_sink_floats() -> int:
    return int(lib.ssm_probe_sink_floats())


def ssm_probe_rate(kind: int, iters: int, sink, warps_per_sm: int = 64, stream=None) -> float:
    """Launches throughput probe `kind` (0 ex2, 1 packed fp32x2 FMA, 2 fp32
    FMA, 3 the recurrence mix) with `warps_per_sm` resident warps per SM on the
    current stream; returns its operation count. The caller times the launch."""
    ops = ctypes.c_double(0.0)
    _check(lib.ssm_probe_rate(int(kind), int(iters), int(warps_per_sm), _ptr(sink), sink.numel(),
                              ctypes.byref(ops), _stream(stream)))
    return ops.value


def ssm_selftest_wait_timeout(tries: int = 64, stream=None) -> None:
    """Launches the bounded-wait self-test (its wait must run out)."""
    _check(lib.ssm_selftest_wait_timeout(int(tries), _stream(stream)))


def ssm_device_status(clear: bool = False) -> int:
    code = lib.ssm_device_status(int(bool(clear)))
    if code < 0:
        _check(code)
    return code


def ssm_check_cu_seqlens(cu_seqlens_host, tok: int) -> None:
    """Check a host (CPU, int32, contiguous) copy of cu_seqlens."""
    S = cu_seqlens_host.numel() - 1
    _check(lib.ssm_check_cu_seqlens(_ptr(cu_seqlens_host), S, int(tok)))


def ssm_scan_workspace_size(tok: int, D: int, N: int, S: int) -> int:
    return int(lib.ssm_scan_workspace_size(tok, D, N, S))


def ssm_causal_conv1d(x, xc, weight, bias=None, cu_seqlens=None, S=None, conv_state_in=None,
                      conv_state_out=None, apply_silu=True, stream=None):
    """x, xc: (tok, D); weight (D, K) fp32; states (S, D, K-1)."""
    tok, D = x.shape
    K = weight.shape[1]
    if S is None:
        S = (cu_seqlens.numel() - 1) if cu_seqlens is not None else 1
    st = conv_state_in if conv_state_in is not None else conv_state_out
    sdt = _dtype(st) if st is not None else _dtype(x)
    _check(lib.ssm_causal_conv1d(_ptr(x), _ptr(xc), _ptr(weight), _ptr(bias), tok, D, K,
                                 _ptr(cu_seqlens), S, _ptr(conv_state_in), _ptr(conv_state_out),
                                 int(bool(apply_silu)), _dtype(x), sdt, _stream(stream)))


def ssm_selective_scan_fwd(u, delta, A, B, C, y, Dskip=None, z=None, dt_bias=None,
                           delta_softplus=True, h0=None, h_final=None, cu_seqlens=None, S=None,
                           workspace=None, stream=None):
    """u, delta, z, y: (tok, D); A (D, N); B, C (tok, N); h0 / h_final (S, D, N) fp32."""
    tok, D = u.shape
    N = A.shape[1]
    if S is None:
        S = (cu_seqlens.numel() - 1) if cu_seqlens is not None else 1
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ssm_selective_scan_fwd(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                                      _ptr(Dskip), _ptr(z), _ptr(dt_bias), int(bool(delta_softplus)),
                                      _ptr(h0), _ptr(cu_seqlens), S, _ptr(y), _ptr(h_final), tok, D,
                                      N, _dtype(u), _ptr(workspace), ws_bytes, _stream(stream)))


def ssm_selective_scan_fwd_ckpt(u, delta, A, B, C, y, bwd_workspace, Dskip=None, z=None,
                                dt_bias=None, delta_softplus=True, h0=None, h_final=None,
                                cu_seqlens=None, S=None, workspace=None, stream=None):
    """ssm_selective_scan_fwd that also writes, into `bwd_workspace` (a device
    byte tensor of ssm_scan_bwd_workspace_size() bytes), the state checkpoints
    that ssm_selective_scan_bwd_ckpt reads instead of recomputing them."""
    tok, D = u.shape
    N = A.shape[1]
    if S is None:
        S = (cu_seqlens.numel() - 1) if cu_seqlens is not None else 1
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    bws_bytes = 0 if bwd_workspace is None else bwd_workspace.numel() * bwd_workspace.element_size()
    _check(lib.ssm_selective_scan_fwd_ckpt(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip), _ptr(z), _ptr(dt_bias),
        int(bool(delta_softplus)), _ptr(h0), _ptr(cu_seqlens), S, _ptr(y), _ptr(h_final), tok, D,
        N, _dtype(u), _ptr(workspace), ws_bytes, _ptr(bwd_workspace), bws_bytes, _stream(stream)))


def ssm_selective_scan_fwd_noalloc(u, delta, A, B, C, y, Dskip=None, z=None, dt_bias=None,
                                   delta_softplus=True, h0=None, h_final=None, cu_seqlens=None,
                                   S=None, stream=None):
    """ssm_selective_scan_fwd with the library's fixed scratch instead of a workspace.

    For callers that cannot allocate device memory at call time (an engine
    that reserved all device memory at start-up, or a plugin whose framework
    owns the allocator). At most 4096 packed sequences per call; concurrent
    calls on one GPU share the scratch and race."""
    tok, D = u.shape
    N = A.shape[1]
    if S is None:
        S = (cu_seqlens.numel() - 1) if cu_seqlens is not None else 1
    _check(lib.ssm_selective_scan_fwd_noalloc(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip), _ptr(z), _ptr(dt_bias),
        int(bool(delta_softplus)), _ptr(h0), _ptr(cu_seqlens), S, _ptr(y), _ptr(h_final), tok, D,
        N, _dtype(u), _stream(stream)))


def ssm_selective_state_update(conv_state, ssm_state, x, dt, B, C, y, conv_w, A, z=None,
                               conv_b=None, Dskip=None, dt_bias=None, delta_softplus=True,
                               state_indices=None, stream=None):
    """conv_state (slots, D, K-1); ssm_state (slots, D, N) fp32; x, dt, z, y (Bt, D)."""
    Bt, D = x.shape
    N = A.shape[1]
    K = conv_w.shape[1]
    _check(lib.ssm_selective_state_update(
        _ptr(conv_state), _ptr(ssm_state), _ptr(x), _ptr(dt), _ptr(B), _ptr(C), _ptr(z),
        _ptr(conv_w), _ptr(conv_b), _ptr(A), _ptr(Dskip), _ptr(dt_bias), int(bool(delta_softplus)),
        _ptr(state_indices), ssm_state.shape[0], _ptr(y), Bt, D, N, K, _dtype(x),
        _dtype(conv_state), _stream(stream)))


def replay_buffers(n_slots: int, D: int, W: int, device, N: int = 16, keep_lo: bool = True):
    """Allocate the replay representation's tensors (torch, on `device`) in the
    layouts ssm_replay_state_update documents: ckpt (n_slots, D, N) fp32,
    ckpt_lo (n_slots, D, N) bf16 or None, buf (n_slots, W-1, D, 2) fp32,
    buf_B (n_slots, W-1, N) fp32, buf_len (n_slots) int32, tickets (n_slots)
    int32 used as uint32. Values are zero; fill ckpt, then call ssm_replay_reset."""
    import torch

    e = max(W - 1, 1)
    return {
        "ckpt": torch.zeros((n_slots, D, N), dtype=torch.float32, device=device),
        "ckpt_lo": torch.zeros((n_slots, D, N), dtype=torch.bfloat16, device=device)
        if keep_lo else None,
        "buf": torch.zeros((n_slots, e, D, 2), dtype=torch.float32, device=device),
        "buf_B": torch.zeros((n_slots, e, N), dtype=torch.float32, device=device),
        "buf_len": torch.zeros(n_slots, dtype=torch.int32, device=device),
        "tickets": torch.zeros(n_slots, dtype=torch.int32, device=device),
        "W": int(W),
    }


def ssm_replay_state_update(conv_state, rep, x, dt, B, C, y, conv_w, A, z=None, conv_b=None,
                            Dskip=None, dt_bias=None, delta_softplus=True, state_indices=None,
                            stream=None):
    """One replay decode step; `rep` holds the tensors of replay_buffers()."""
    Bt, D = x.shape
    N = A.shape[1]
    K = conv_w.shape[1]
    ck = rep["ckpt"]
    _check(lib.ssm_replay_state_update(
        _ptr(conv_state), _ptr(ck), _ptr(rep["ckpt_lo"]), _ptr(rep["buf"]), _ptr(rep["buf_B"]),
        _ptr(rep["buf_len"]), _ptr(rep["tickets"]), int(rep["W"]), _ptr(x), _ptr(dt), _ptr(B),
        _ptr(C), _ptr(z), _ptr(conv_w), _ptr(conv_b), _ptr(A), _ptr(Dskip), _ptr(dt_bias),
        int(bool(delta_softplus)), _ptr(state_indices), ck.shape[0], _ptr(y), Bt, D, N, K,
        _dtype(x), _dtype(conv_state), _stream(stream)))


def ssm_replay_reset(rep, slots=None, n=None, stream=None):
    """Start the listed slots' windows (all slots if None) at the states in rep['ckpt']."""
    ck = rep["ckpt"]
    n_slots, D, N = ck.shape
    n = (slots.numel() if slots is not None else n_slots) if n is None else n
    _check(lib.ssm_replay_reset(_ptr(ck), _ptr(rep["ckpt_lo"]), _ptr(rep["buf_len"]),
                                _ptr(rep["tickets"]), _ptr(slots), n, n_slots, D, N,
                                _stream(stream)))


def ssm_replay_flush(rep, A, slots=None, n=None, stream=None):
    """Replay the listed slots' buffers into rep['ckpt'] and empty them."""
    ck = rep["ckpt"]
    n_slots, D, N = ck.shape
    n = (slots.numel() if slots is not None else n_slots) if n is None else n
    _check(lib.ssm_replay_flush(_ptr(ck), _ptr(rep["ckpt_lo"]), _ptr(rep["buf"]),
                                _ptr(rep["buf_B"]), _ptr(rep["buf_len"]), _ptr(rep["tickets"]),
                                _ptr(A), int(rep["W"]), _ptr(slots), n, n_slots, D, N,
                                _stream(stream)))


def ssm_scan_bwd_workspace_size(tok: int, D: int, N: int, S: int) -> int:
    return int(lib.ssm_scan_bwd_workspace_size(tok, D, N, S))


def ssm_set_scan_bwd_variant(variant: int) -> None:
    """0: library's choice; 1: four lanes per channel; 2: one thread per channel."""
    _check(lib.ssm_set_scan_bwd_variant(int(variant)))


def ssm_scan_bwd_variant_for(S: int, D: int) -> int:
    v = ctypes.c_int(0)
    _check(lib.ssm_scan_bwd_variant_for(int(S), int(D), ctypes.byref(v)))
    return v.value


def ssm_selective_scan_bwd(u, delta, A, B, C, dy, grads, Dskip=None, z=None, dt_bias=None,
                           delta_softplus=True, h0=None, dh_final=None, cu_seqlens=None, S=None,
                           workspace=None, stream=None, from_fwd_ckpt=False):
    """Backward of ssm_selective_scan_fwd. `grads` holds the output tensors:
    du, ddelta (like u), dz (like u, or None), dB, dC (tok, N) fp32, dA (D, N)
    fp32, dDskip, ddt_bias (D) fp32 or None, dh0 (S, D, N) fp32 or None.
    `workspace` is a device byte tensor of ssm_scan_bwd_workspace_size() bytes.
    from_fwd_ckpt: the workspace holds the checkpoints that
    ssm_selective_scan_fwd_ckpt wrote for the same inputs
    (ssm_selective_scan_bwd_ckpt)."""
    tok, D = u.shape
    N = A.shape[1]
    if S is None:
        S = (cu_seqlens.numel() - 1) if cu_seqlens is not None else 1
    g = grads
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    fn = lib.ssm_selective_scan_bwd_ckpt if from_fwd_ckpt else lib.ssm_selective_scan_bwd
    _check(fn(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip), _ptr(z), _ptr(dt_bias),
        int(bool(delta_softplus)), _ptr(h0), _ptr(cu_seqlens), S, _ptr(dy), _ptr(dh_final),
        _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g.get("dz")), _ptr(g["dB"]), _ptr(g["dC"]),
        _ptr(g["dA"]), _ptr(g.get("dDskip")), _ptr(g.get("ddt_bias")), _ptr(g.get("dh0")), tok, D,
        N, _dtype(u), _ptr(workspace), ws_bytes, _stream(stream)))


def ssm_conv_scan_fwd(x, conv_w, delta, A, B, C, y, conv_b=None, conv_state_in=None,
                      conv_state_out=None, xc=None, Dskip=None, z=None, dt_bias=None,
                      delta_softplus=True, h0=None, h_final=None, cu_seqlens=None, S=None,
                      stream=None):
    """Fused conv1d + SiLU -> selective scan. x, delta, z, y, xc: (tok, D);
    conv_w (D, K) fp32; conv states (S, D, K-1); A (D, N); B, C (tok, N)."""
    tok, D = x.shape
    N = A.shape[1]
    K = conv_w.shape[1]
    if S is None:
        S = (cu_seqlens.numel() - 1) if cu_seqlens is not None else 1
    st = conv_state_in if conv_state_in is not None else conv_state_out
    sdt = _dtype(st) if st is not None else _dtype(x)
    _check(lib.ssm_conv_scan_fwd(
        _ptr(x), _ptr(conv_w), _ptr(conv_b), _ptr(conv_state_in), _ptr(conv_state_out), _ptr(xc),
        K, sdt, _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip), _ptr(z), _ptr(dt_bias),
        int(bool(delta_softplus)), _ptr(h0), _ptr(cu_seqlens), S, _ptr(y), _ptr(h_final), tok, D,
        N, _dtype(x), _stream(stream)))
