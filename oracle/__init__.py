"""fp64 CPU oracle of the selective-SSM mixer core (TEST INFRASTRUCTURE).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package. It wraps ``ssm_oracle.c`` (plain C, double
precision) through ctypes and shares nothing with the CUDA path. Every
function takes NumPy arrays, converts them to float64, calls the C routine
and returns new arrays; the wrappers do data marshalling only.

Parity pins: the closed-form geometric series, the brute-force unrolled sum,
``numpy.correlate`` for the convolution, the packing, chunking and decode
invariants, the equality of replay decode with eager decode, bit-level bf16
rounding, central finite differences of the forward scan (for its backward) and
a hand-worked dyadic example all pin these routines (see the
``tests/test_oracle_*.py`` files). No function here is "parity unpinned".
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "ssm_oracle.c")
LIBRARY = os.path.join(_HERE, "libssm_oracle.so")

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64
_int = ctypes.c_int


def compile_oracle(source: str = SOURCE, output: str = LIBRARY) -> str:
    """Compile the C oracle (plain -O2, no fast-math, no FMA contraction)."""
    cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-o", output, source, "-lm"]
    subprocess.run(cmd, check=True)
    return output


def _stale(lib: str, src: str) -> bool:
    return (not os.path.exists(lib)) or os.path.getmtime(lib) < os.path.getmtime(src)


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(_dp)


def _iptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(_ip)


def _cu(cu_seqlens, tok, S):
    if cu_seqlens is None:
        if S is None:
            S = 1
        assert tok % S == 0, "dense layout needs tok divisible by the row count"
        L = tok // S
        return np.arange(S + 1, dtype=np.int64) * L
    return np.ascontiguousarray(cu_seqlens, dtype=np.int64)


class Oracle:
    """Handle to one compiled copy of the oracle library."""

    def __init__(self, path: str = LIBRARY):
        self.path = path
        lib = ctypes.CDLL(path)
        lib.oracle_causal_conv1d.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _int, _ip, _i64,
                                             _dp, _dp, _int]
        lib.oracle_causal_conv1d.restype = None
        lib.oracle_selective_scan.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _int, _dp,
                                              _ip, _i64, _i64, _i64, _int, _dp, _dp]
        lib.oracle_selective_scan.restype = None
        lib.oracle_state_update.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                            _dp, _dp, _int, _ip, _i64, _dp, _i64, _i64, _int,
                                            _int]
        lib.oracle_state_update.restype = None
        lib.oracle_round_bf16.argtypes = [_dp, _dp, _i64]
        lib.oracle_round_bf16.restype = None
        lib.oracle_replay_state.argtypes = [_dp, _dp, _dp, _dp, _ip, _dp, _i64, _int, _i64, _int,
                                            _dp]
        lib.oracle_replay_state.restype = None
        lib.oracle_replay_step.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _ip, _int, _dp, _dp, _dp,
                                           _dp, _dp, _dp, _dp, _dp, _dp, _dp, _int, _ip, _i64, _dp,
                                           _i64, _i64, _int, _int]
        lib.oracle_replay_step.restype = None
        lib.oracle_selective_scan_bwd.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _int,
                                                  _dp, _ip, _i64, _i64, _i64, _int, _dp, _dp,
                                                  _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                                  _dp]
        lib.oracle_selective_scan_bwd.restype = None
        lib.oracle_num_threads.restype = _int
        lib.oracle_set_num_threads.argtypes = [_int]
        self.lib = lib

    # -- threads -----------------------------------------------------------
    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))

    # -- conv --------------------------------------------------------------
    def causal_conv1d(self, x, w, bias=None, cu_seqlens=None, S=None, state_in=None,
                      want_state=False, apply_silu=True):
        """x (tok, D); w (D, K); returns xc (tok, D) [, state_out (S, D, K-1)]."""
        x = _f64(x)
        tok, D = x.shape
        w = _f64(w)
        K = w.shape[1]
        cu = _cu(cu_seqlens, tok, S)
        S = len(cu) - 1
        bias = _f64(bias)
        state_in = _f64(state_in)
        xc = np.zeros((tok, D), dtype=np.float64)
        st = np.zeros((S, D, K - 1), dtype=np.float64) if want_state else None
        self.lib.oracle_causal_conv1d(_ptr(x), _ptr(xc), _ptr(w), _ptr(bias), tok, D, K,
                                      _iptr(cu), S, _ptr(state_in), _ptr(st), int(apply_silu))
        return (xc, st) if want_state else xc

    # -- scan --------------------------------------------------------------
    def selective_scan(self, u, delta, A, B, C, Dskip=None, z=None, dt_bias=None,
                       delta_softplus=True, h0=None, cu_seqlens=None, S=None,
                       want_state=False, y_init=None):
        """u, delta, z: (tok, D); A (D, N); B, C (tok, N). Returns y [, h_final]."""
        u = _f64(u)
        tok, D = u.shape
        A = _f64(A)
        N = A.shape[1]
        cu = _cu(cu_seqlens, tok, S)
        S = len(cu) - 1
        y = np.zeros((tok, D)) if y_init is None else _f64(y_init).copy()
        hf = np.zeros((S, D, N)) if want_state else None
        args = [_f64(a) for a in (delta, B, C, Dskip, z, dt_bias, h0)]
        self.lib.oracle_selective_scan(_ptr(u), _ptr(args[0]), _ptr(A), _ptr(args[1]),
                                       _ptr(args[2]), _ptr(args[3]), _ptr(args[4]),
                                       _ptr(args[5]), int(delta_softplus), _ptr(args[6]),
                                       _iptr(cu), S, tok, D, N, _ptr(y), _ptr(hf))
        return (y, hf) if want_state else y

    def selective_scan_bwd(self, u, delta, A, B, C, dy, Dskip=None, z=None, dt_bias=None,
                           delta_softplus=True, h0=None, cu_seqlens=None, S=None,
                           dh_final=None):
        """Gradients of sum(dy * y) + sum(dh_final * h_final) with respect to every
        input of selective_scan. Returns a dict: du, ddt, dz (or None), dB, dC, dA,
        dDskip, ddt_bias, dh0."""
        u = _f64(u)
        tok, D = u.shape
        A = _f64(A)
        N = A.shape[1]
        cu = _cu(cu_seqlens, tok, S)
        S = len(cu) - 1
        out = {"du": np.zeros((tok, D)), "ddt": np.zeros((tok, D)),
               "dz": np.zeros((tok, D)) if z is not None else None,
               "dB": np.zeros((tok, N)), "dC": np.zeros((tok, N)), "dA": np.zeros((D, N)),
               "dDskip": np.zeros(D), "ddt_bias": np.zeros(D), "dh0": np.zeros((S, D, N))}
        work = np.zeros(((tok + S + 1) * N,))
        args = [_f64(a) for a in (delta, B, C, Dskip, z, dt_bias, h0, dy, dh_final)]
        self.lib.oracle_selective_scan_bwd(
            _ptr(u), _ptr(args[0]), _ptr(A), _ptr(args[1]), _ptr(args[2]), _ptr(args[3]),
            _ptr(args[4]), _ptr(args[5]), int(delta_softplus), _ptr(args[6]), _iptr(cu), S, tok,
            D, N, _ptr(args[7]), _ptr(args[8]), _ptr(out["du"]), _ptr(out["ddt"]),
            _ptr(out["dz"]), _ptr(out["dB"]), _ptr(out["dC"]), _ptr(out["dA"]),
            _ptr(out["dDskip"]), _ptr(out["ddt_bias"]), _ptr(out["dh0"]), _ptr(work))
        return out

    # -- decode ------------------------------------------------------------
    def state_update(self, conv_state, ssm_state, x, dt, B, C, z, conv_w, conv_b, A, Dskip,
                     dt_bias, delta_softplus=True, state_indices=None, y_init=None):
        """Returns (y, conv_state', ssm_state'); the inputs are not modified."""
        cs = _f64(conv_state).copy()
        ss = _f64(ssm_state).copy()
        x = _f64(x)
        Bt, D = x.shape
        A = _f64(A)
        N = A.shape[1]
        K = cs.shape[2] + 1
        idx = None if state_indices is None else np.ascontiguousarray(state_indices, np.int64)
        y = np.zeros((Bt, D)) if y_init is None else _f64(y_init).copy()
        args = [_f64(a) for a in (dt, B, C, z, conv_w, conv_b, Dskip, dt_bias)]
        self.lib.oracle_state_update(_ptr(cs), _ptr(ss), _ptr(x), _ptr(args[0]), _ptr(args[1]),
                                     _ptr(args[2]), _ptr(args[3]), _ptr(args[4]), _ptr(args[5]),
                                     _ptr(A), _ptr(args[6]), _ptr(args[7]), int(delta_softplus),
                                     _iptr(idx), cs.shape[0], _ptr(y), Bt, D, N, K)
        return y, cs, ss

    # -- replay decode -------------------------------------------------------
    def round_bf16(self, v):
        """Nearest bf16 value of each element (ties to even), as float64."""
        v = _f64(v)
        out = np.empty_like(v)
        self.lib.oracle_round_bf16(_ptr(v), _ptr(out), v.size)
        return out

    def replay_init(self, ck, W, keep_lo=True):
        """A replay representation starting at state ck (n_slots, D, N): a dict
        with the checkpoint, its bf16 copy (or None), empty buffers and lengths."""
        ck = _f64(ck).copy()
        n_slots, D, N = ck.shape
        return {"ck": ck, "ck_lo": self.round_bf16(ck) if keep_lo else None, "W": int(W),
                "bd": np.zeros((n_slots, W, D)), "bx": np.zeros((n_slots, W, D)),
                "bB": np.zeros((n_slots, W, N)), "len": np.zeros(n_slots, np.int64)}

    def replay_state(self, rep, A):
        """The state each slot of a replay representation stands for (n_slots, D, N)."""
        ck = rep["ck"]
        n_slots, D, N = ck.shape
        h = np.zeros_like(ck)
        self.lib.oracle_replay_state(_ptr(ck), _ptr(rep["bd"]), _ptr(rep["bx"]), _ptr(rep["bB"]),
                                     _iptr(rep["len"]), _ptr(_f64(A)), n_slots, rep["W"], D, N,
                                     _ptr(h))
        return h

    def replay_step(self, conv_state, rep, x, dt, B, C, z, conv_w, conv_b, A, Dskip, dt_bias,
                    delta_softplus=True, state_indices=None, y_init=None):
        """One replay decode step. Returns (y, conv_state', rep'); inputs are not modified."""
        cs = _f64(conv_state).copy()
        lo = rep["ck_lo"]
        new = {"ck": rep["ck"].copy(), "ck_lo": None if lo is None else lo.copy(),
               "W": rep["W"], "bd": rep["bd"].copy(), "bx": rep["bx"].copy(),
               "bB": rep["bB"].copy(), "len": rep["len"].copy()}
        x = _f64(x)
        Bt, D = x.shape
        A = _f64(A)
        N = A.shape[1]
        K = cs.shape[2] + 1
        idx = None if state_indices is None else np.ascontiguousarray(state_indices, np.int64)
        y = np.zeros((Bt, D)) if y_init is None else _f64(y_init).copy()
        args = [_f64(a) for a in (dt, B, C, z, conv_w, conv_b, Dskip, dt_bias)]
        self.lib.oracle_replay_step(
            _ptr(cs), _ptr(new["ck"]), _ptr(new["ck_lo"]), _ptr(new["bd"]), _ptr(new["bx"]),
            _ptr(new["bB"]), _iptr(new["len"]), new["W"], _ptr(x), _ptr(args[0]), _ptr(args[1]),
            _ptr(args[2]), _ptr(args[3]), _ptr(args[4]), _ptr(args[5]), _ptr(A), _ptr(args[6]),
            _ptr(args[7]), int(delta_softplus), _iptr(idx), cs.shape[0], _ptr(y), Bt, D, N, K)
        return y, cs, new


_DEFAULT = None


def load(path: str | None = None) -> Oracle:
    """Return the oracle, compiling it first if the library is missing or stale."""
    global _DEFAULT
    if path is not None:
        return Oracle(path)
    if _DEFAULT is None:
        if _stale(LIBRARY, SOURCE):
            compile_oracle()
        _DEFAULT = Oracle(LIBRARY)
    return _DEFAULT
