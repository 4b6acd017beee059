"""Checks that pin the fp64 oracle to facts other than itself.

Each ``check_*`` function takes an ``oracle.Oracle`` handle and raises
AssertionError when the oracle disagrees with the fact it is pinned to:

* closed form: constant inputs turn the recurrence into a geometric series;
* brute force: the unrolled sum y_t = sum_s C_t (prod_{r=s+1..t} exp(D_r A)) D_s B_s x_s
  + C_t (prod_{r=s0..t} exp(D_r A)) h0 + Dskip x_t, gated, on tiny random inputs;
* library routines: numpy.correlate for the depthwise causal conv, numpy.logaddexp
  and scipy.special.expit for softplus and silu;
* spot values: softplus(0) = ln 2, softplus(1) = ln(1 + e), silu(1) = sigmoid(1), ...;
* invariants: a packed batch equals its sequences run one by one; a prefill cut
  in two with the state carried equals the one-shot prefill; prefill followed
  by k decode steps equals prefill over the extended sequence; permuted state
  indices with -1 padding touch exactly the named slots;
* a hand-worked dyadic example stored under tests/golden/;
* replay decode (checkpoint plus buffered inputs) against eager decode: equal
  outputs and states, the bf16 checkpoint copy entering exactly the outputs
  of non-checkpoint steps (a linearity identity), and bf16 rounding against a
  bit-level round-to-nearest-even of float32 values and torch's conversion.

The same checks run against deliberately broken copies of the oracle in
test_oracle_mutants.py, which shows that each plausible slip is caught.
"""

from __future__ import annotations

import os

import numpy as np
from scipy.special import expit

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rel_err(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    scale = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / scale) if a.size else 0.0


def _softplus_lib(v):
    return np.logaddexp(0.0, v)


def _silu_lib(v):
    return v * expit(v)


# ---------------------------------------------------------------------------
# spot values
# ---------------------------------------------------------------------------

def check_softplus_spot(orc):
    """N=1, A=0 (dA=1), h0=0, B=C=u=1, no skip, no gate: y equals Delta."""
    vals = np.array([0.0, 1.0, -30.0, 30.0, 2.5], dtype=np.float64)
    want = np.array([0.6931471805599453, 1.3132616875182228, 9.357622968840175e-14,
                     30.000000000000092, np.logaddexp(0.0, 2.5)])
    for v, w in zip(vals, want):
        y = orc.selective_scan(u=np.ones((1, 1)), delta=np.full((1, 1), v),
                               A=np.zeros((1, 1)), B=np.ones((1, 1)), C=np.ones((1, 1)),
                               delta_softplus=True)
        assert abs(y[0, 0] - w) <= 1e-15 * max(1.0, abs(w)), (v, y[0, 0], w)
        y = orc.selective_scan(u=np.ones((1, 1)), delta=np.full((1, 1), v),
                               A=np.zeros((1, 1)), B=np.ones((1, 1)), C=np.ones((1, 1)),
                               delta_softplus=False)
        assert y[0, 0] == v


def check_silu_spot(orc):
    """B=0 keeps h at 0; Dskip=1, u=1: y equals silu(z)."""
    z = np.array([[0.0], [1.0], [-1.0], [40.0], [-40.0]])
    want = np.array([0.0, 0.7310585786300049, -0.2689414213699951, 40.0, -40.0 * expit(-40.0)])
    y = orc.selective_scan(u=np.ones((5, 1)), delta=np.full((5, 1), 0.1), A=-np.ones((1, 1)),
                           B=np.zeros((5, 1)), C=np.ones((5, 1)), Dskip=np.ones(1), z=z,
                           delta_softplus=False)
    assert np.max(np.abs(y[:, 0] - want)) <= 1e-15, (y[:, 0], want)


def check_conv_identity_tap(orc):
    """w = e_{K-1} and zero bias: the conv returns silu(x) exactly (library expit)."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((37, 5)) * 3
    K = 4
    w = np.zeros((5, K))
    w[:, K - 1] = 1.0
    xc = orc.causal_conv1d(x, w, bias=np.zeros(5), cu_seqlens=[0, 10, 37])
    assert _rel_err(xc, _silu_lib(x)) <= 1e-15


# ---------------------------------------------------------------------------
# closed form
# ---------------------------------------------------------------------------

def check_closed_form(orc, L=4096, D=3, N=5):
    """Constant Delta, A, B, C, x per channel: with a = exp(Delta A), b = Delta B x,
    h_t = a^{t+1} h0 + b (1 - a^{t+1}) / (1 - a) and y_t = sum_n C_n h_t + Dskip x."""
    rng = np.random.default_rng(5)
    delta = np.array([1e-3, 3e-2, 0.1])[:D]
    A = -np.exp(rng.uniform(np.log(0.1), np.log(8.0), (D, N)))
    xs = rng.standard_normal(D)
    Bv = rng.standard_normal(N)
    Cv = rng.standard_normal(N)
    Dsk = rng.standard_normal(D)
    h0 = rng.standard_normal((1, D, N))
    u = np.tile(xs, (L, 1))
    y, hf = orc.selective_scan(u=u, delta=np.tile(delta, (L, 1)), A=A, B=np.tile(Bv, (L, 1)),
                               C=np.tile(Cv, (L, 1)), Dskip=Dsk, h0=h0, delta_softplus=False,
                               want_state=True)
    t = np.arange(L, dtype=np.float64)[:, None, None] + 1.0  # t + 1
    lna = (delta[:, None] * A)[None]  # log a, (1, D, N)
    a_pow = np.exp(lna * t)
    b = (delta[:, None] * xs[:, None]) * Bv[None, :]
    geo = -np.expm1(lna * t) / -np.expm1(lna)  # (1 - a^{t+1}) / (1 - a)
    h = a_pow * h0 + b[None] * geo
    y_want = np.einsum("tdn,n->td", h, Cv) + Dsk[None] * xs[None]
    assert _rel_err(y, y_want) <= 1e-11, _rel_err(y, y_want)
    assert _rel_err(hf[0], h[-1]) <= 1e-11, _rel_err(hf[0], h[-1])


# ---------------------------------------------------------------------------
# brute force
# ---------------------------------------------------------------------------

def brute_force_scan(u, dt, A, B, C, Dskip, z, dt_bias, h0, cu):
    """O(L^2 N) unrolled sum per token; returns (y, h_final)."""
    tok, D = u.shape
    N = A.shape[1]
    S = len(cu) - 1
    y = np.zeros((tok, D))
    hf = np.zeros((S, D, N))
    delta = _softplus_lib(dt + dt_bias[None, :])
    for s in range(S):
        s0, s1 = cu[s], cu[s + 1]
        for c in range(D):
            for t in range(s0, s1 + 1):  # t == s1 gives the final state
                last = t if t < s1 else s1 - 1
                hsum = np.zeros(N)
                for q in range(s0, last + 1):
                    decay = np.ones(N)
                    for r in range(q + 1, last + 1):
                        decay *= np.exp(delta[r, c] * A[c])
                    hsum += decay * delta[q, c] * B[q] * u[q, c]
                decay0 = np.ones(N)
                for r in range(s0, last + 1):
                    decay0 *= np.exp(delta[r, c] * A[c])
                hsum += decay0 * h0[s, c]
                if t < s1:
                    yt = np.dot(C[t], hsum) + Dskip[c] * u[t, c]
                    y[t, c] = yt * _silu_lib(z[t, c])
                else:
                    hf[s, c] = hsum
    return y, hf


def check_bruteforce(orc):
    rng = np.random.default_rng(7)
    lens = [6, 0, 1, 11, 3]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    tok, D, N = int(cu[-1]), 3, 4
    u = rng.standard_normal((tok, D))
    dt = 0.5 * rng.standard_normal((tok, D))
    A = -np.exp(rng.uniform(-2, 1.5, (D, N)))
    B = rng.standard_normal((tok, N))
    C = rng.standard_normal((tok, N))
    Dsk = rng.standard_normal(D)
    z = rng.standard_normal((tok, D))
    dtb = 0.3 * rng.standard_normal(D)
    h0 = rng.standard_normal((len(lens), D, N))
    y, hf = orc.selective_scan(u, dt, A, B, C, Dskip=Dsk, z=z, dt_bias=dtb, delta_softplus=True,
                               h0=h0, cu_seqlens=cu, want_state=True)
    yb, hb = brute_force_scan(u, dt, A, B, C, Dsk, z, dtb, h0, cu)
    assert _rel_err(y, yb) <= 1e-12, _rel_err(y, yb)
    assert _rel_err(hf, hb) <= 1e-12, _rel_err(hf, hb)


# ---------------------------------------------------------------------------
# convolution against numpy.correlate
# ---------------------------------------------------------------------------

def check_conv_correlate(orc):
    rng = np.random.default_rng(3)
    K, D = 4, 6
    lens = [7, 0, 1, 2, 3, 13]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    tok, S = int(cu[-1]), len(lens)
    x = rng.standard_normal((tok, D))
    w = 0.5 * rng.standard_normal((D, K))
    bias = rng.standard_normal(D)
    st = rng.standard_normal((S, D, K - 1))
    for with_state in (False, True):
        st_in = st if with_state else None
        xc, so = orc.causal_conv1d(x, w, bias=bias, cu_seqlens=cu, state_in=st_in,
                                   want_state=True, apply_silu=False)
        for s in range(S):
            s0, s1 = cu[s], cu[s + 1]
            for c in range(D):
                head = st[s, c] if with_state else np.zeros(K - 1)
                full = np.concatenate([head, x[s0:s1, c]])
                if s1 > s0:  # (numpy swaps the operands when the signal is shorter)
                    want = np.correlate(full, w[c], mode="valid") + bias[c]
                    assert want.shape[0] == s1 - s0
                    assert _rel_err(xc[s0:s1, c], want) <= 1e-14
                assert np.array_equal(so[s, c], full[-(K - 1):]), (s, c)
        # the activation is silu of the same pre-activation
        xc2 = orc.causal_conv1d(x, w, bias=bias, cu_seqlens=cu, state_in=st_in)
        assert _rel_err(xc2, _silu_lib(xc)) <= 1e-15


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------

def _layer(orc, x, dt, z, B, C, p, cu, conv_state=None, h0=None):
    """conv then scan over a packed batch; returns (y, h_final, conv_state_out)."""
    xc, cs = orc.causal_conv1d(x, p["w"], bias=p["b"], cu_seqlens=cu, state_in=conv_state,
                               want_state=True)
    y, hf = orc.selective_scan(xc, dt, p["A"], B, C, Dskip=p["D"], z=z, dt_bias=p["dtb"],
                               delta_softplus=True, h0=h0, cu_seqlens=cu, want_state=True)
    return y, hf, cs


def _rand_layer(seed, tok, D, N, K):
    rng = np.random.default_rng(seed)
    p = {"w": 0.5 * rng.standard_normal((D, K)), "b": 0.5 * rng.standard_normal(D),
         "A": -np.exp(rng.uniform(-2, 2, (D, N))), "D": rng.standard_normal(D),
         "dtb": rng.uniform(-5, -1, D)}
    acts = {"x": rng.standard_normal((tok, D)), "dt": 0.3 * rng.standard_normal((tok, D)),
            "z": rng.standard_normal((tok, D)), "B": rng.standard_normal((tok, N)),
            "C": rng.standard_normal((tok, N))}
    return p, acts


def check_pack_equals_separate(orc):
    lens = [5, 1, 0, 17, 2, 9]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    tok, D, N, K = int(cu[-1]), 4, 8, 4
    p, a = _rand_layer(21, tok, D, N, K)
    rng = np.random.default_rng(22)
    cs0 = rng.standard_normal((len(lens), D, K - 1))
    h0 = rng.standard_normal((len(lens), D, N))
    y, hf, cs = _layer(orc, a["x"], a["dt"], a["z"], a["B"], a["C"], p, cu, cs0, h0)
    for s in range(len(lens)):
        s0, s1 = cu[s], cu[s + 1]
        one = np.array([0, s1 - s0], dtype=np.int64)
        ys, hs, css = _layer(orc, a["x"][s0:s1], a["dt"][s0:s1], a["z"][s0:s1], a["B"][s0:s1],
                             a["C"][s0:s1], p, one, cs0[s:s + 1], h0[s:s + 1])
        assert np.array_equal(y[s0:s1], ys), s
        assert np.array_equal(hf[s], hs[0]), s
        assert np.array_equal(cs[s], css[0]), s


def check_chunked_equals_oneshot(orc):
    L, D, N, K = 29, 3, 6, 4
    p, a = _rand_layer(31, L, D, N, K)
    one = np.array([0, L], dtype=np.int64)
    y, hf, cs = _layer(orc, a["x"], a["dt"], a["z"], a["B"], a["C"], p, one)
    for L1 in (0, 1, 2, 3, 4, 13, L):
        c1 = np.array([0, L1], dtype=np.int64)
        c2 = np.array([0, L - L1], dtype=np.int64)
        y1, h1, s1 = _layer(orc, a["x"][:L1], a["dt"][:L1], a["z"][:L1], a["B"][:L1],
                            a["C"][:L1], p, c1)
        y2, h2, s2 = _layer(orc, a["x"][L1:], a["dt"][L1:], a["z"][L1:], a["B"][L1:],
                            a["C"][L1:], p, c2, conv_state=s1, h0=h1)
        assert np.array_equal(np.concatenate([y1, y2]), y), L1
        assert np.array_equal(h2, hf), L1
        assert np.array_equal(s2, cs), L1


def check_decode_invariant(orc, k_steps=(1, 7)):
    D, N, K = 5, 4, 4
    for k in k_steps:
        L0 = 9
        L = L0 + k
        p, a = _rand_layer(41 + k, L, D, N, K)
        y, hf, cs = _layer(orc, a["x"], a["dt"], a["z"], a["B"], a["C"], p,
                           np.array([0, L], dtype=np.int64))
        y0, h, c = _layer(orc, a["x"][:L0], a["dt"][:L0], a["z"][:L0], a["B"][:L0],
                          a["C"][:L0], p, np.array([0, L0], dtype=np.int64))
        for t in range(L0, L):
            sl = slice(t, t + 1)
            yt, c, h = orc.state_update(c, h, a["x"][sl], a["dt"][sl], a["B"][sl], a["C"][sl],
                                        a["z"][sl], p["w"], p["b"], p["A"], p["D"], p["dtb"],
                                        delta_softplus=True)
            assert np.array_equal(yt[0], y[t]), (k, t)
        assert np.array_equal(h, hf), k
        assert np.array_equal(c, cs), k


def check_state_indices(orc):
    n_slots, Bt, D, N, K = 7, 4, 3, 4, 4
    rng = np.random.default_rng(51)
    p, a = _rand_layer(52, Bt, D, N, K)
    cs = rng.standard_normal((n_slots, D, K - 1))
    ss = rng.standard_normal((n_slots, D, N))
    idx = np.array([5, -1, 0, 3], dtype=np.int64)
    sentinel = np.full((Bt, D), 123.5)
    y, cs2, ss2 = orc.state_update(cs, ss, a["x"], a["dt"], a["B"], a["C"], a["z"], p["w"],
                                   p["b"], p["A"], p["D"], p["dtb"], state_indices=idx,
                                   y_init=sentinel)
    untouched = [s for s in range(n_slots) if s not in idx]
    assert np.array_equal(cs2[untouched], cs[untouched])
    assert np.array_equal(ss2[untouched], ss[untouched])
    assert np.array_equal(y[1], sentinel[1])
    # the touched slots equal a dense run over the gathered states
    rows = [0, 2, 3]
    slots = idx[rows]
    yd, csd, ssd = orc.state_update(cs[slots], ss[slots], a["x"][rows], a["dt"][rows],
                                    a["B"][rows], a["C"][rows], a["z"][rows], p["w"], p["b"],
                                    p["A"], p["D"], p["dtb"])
    assert np.array_equal(y[rows], yd)
    assert np.array_equal(cs2[slots], csd)
    assert np.array_equal(ss2[slots], ssd)


# ---------------------------------------------------------------------------
# hand-worked dyadic example (tests/golden/dyadic_scan.txt)
# ---------------------------------------------------------------------------

def load_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, rest = line.split("=", 1)
            vals[key.strip()] = np.array([float(v) for v in rest.split()], dtype=np.float64)
    return vals


def check_golden_dyadic(orc):
    g = load_golden("dyadic_scan.txt")
    L, N = 3, 2
    y, hf = orc.selective_scan(u=g["u"].reshape(L, 1), delta=g["delta"].reshape(L, 1),
                               A=np.log(g["dA"]).reshape(1, N), B=g["B"].reshape(L, N),
                               C=g["C"].reshape(L, N), Dskip=g["Dskip"],
                               h0=g["h0"].reshape(1, 1, N), delta_softplus=False,
                               want_state=True)
    assert np.max(np.abs(y[:, 0] - g["y"])) <= 1e-14, (y[:, 0], g["y"])
    assert np.max(np.abs(hf.reshape(-1) - g["h_final"])) <= 1e-14
    gc = load_golden("dyadic_conv.txt")
    xc, so = orc.causal_conv1d(gc["x"].reshape(-1, 1), gc["w"].reshape(1, -1), bias=gc["bias"],
                               state_in=gc["state_in"].reshape(1, 1, -1), want_state=True,
                               apply_silu=False)
    assert np.array_equal(xc[:, 0], gc["xc"]), (xc[:, 0], gc["xc"])
    assert np.array_equal(so.reshape(-1), gc["state_out"])


# ---------------------------------------------------------------------------
# replay decode ("ReplaySSM: Cache SSM Inputs, Not State", abstract)
# ---------------------------------------------------------------------------

def _bf16_bits_rne(v32):
    """Round float32 values to bf16 on their bit patterns (round to nearest, ties to even)."""
    bits = np.asarray(v32, np.float32).view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    out = ((bits + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return out.view(np.float32).astype(np.float64)


def check_round_bf16(orc):
    import torch

    rng = np.random.default_rng(71)
    v = (rng.standard_normal(4000) * np.exp(rng.uniform(-30, 30, 4000))).astype(np.float32)
    # exact ties between two bf16 values: the even neighbour wins
    ties = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 3 * 2.0 ** -9 + 2.0 ** -9,
                     (1 + 2.0 ** -7 + 2.0 ** -8) * 2.0 ** 20], dtype=np.float32)
    v = np.concatenate([v, ties, np.float32([0.0, 1.0, -2.5, 65280.0, 1e-30])])
    got = orc.round_bf16(v.astype(np.float64))
    assert np.array_equal(got, _bf16_bits_rne(v))
    lib = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(got, lib)
    assert got[4000] == 1.0 and got[4001] == 1 + 2.0 ** -6


def _replay_setup(seed, n_slots, D, N, K):
    rng = np.random.default_rng(seed)
    p, _ = _rand_layer(seed + 1, 1, D, N, K)
    cs = rng.standard_normal((n_slots, D, K - 1))
    h = rng.standard_normal((n_slots, D, N))
    return p, cs, h, rng


def _step_inputs(rng, Bt, D, N):
    return {"x": rng.standard_normal((Bt, D)), "dt": 0.3 * rng.standard_normal((Bt, D)),
            "z": rng.standard_normal((Bt, D)), "B": rng.standard_normal((Bt, N)),
            "C": rng.standard_normal((Bt, N))}


def check_replay_equals_eager(orc):
    n_slots, D, N, K = 3, 5, 4, 4
    for W in (1, 2, 3, 5):
        p, cs0, h0, rng = _replay_setup(81 + W, n_slots, D, N, K)
        rep = orc.replay_init(h0, W, keep_lo=False)
        cs_e, h_e, cs_r = cs0, h0, cs0
        for t in range(11):
            a = _step_inputs(rng, n_slots, D, N)
            args = (a["x"], a["dt"], a["B"], a["C"], a["z"], p["w"], p["b"], p["A"], p["D"],
                    p["dtb"])
            y_e, cs_e, h_e = orc.state_update(cs_e, h_e, *args)
            y_r, cs_r, rep = orc.replay_step(cs_r, rep, *args)
            assert _rel_err(y_r, y_e) <= 1e-12, (W, t)
            assert np.array_equal(cs_r, cs_e), (W, t)
            assert np.all(rep["len"] == (t + 1) % W), (W, t, rep["len"])
            assert _rel_err(orc.replay_state(rep, p["A"]), h_e) <= 1e-12, (W, t)
            if (t + 1) % W == 0:
                assert _rel_err(rep["ck"], h_e) <= 1e-12, (W, t)


def check_replay_low_precision(orc):
    """With a bf16 copy, a non-checkpoint step's output differs from eager by
    exactly the copy's rounding carried through the decay of the buffered
    tokens (the output is linear in the checkpoint); checkpoint steps use the
    fp64 checkpoint and match eager."""
    from scipy.special import expit

    n_slots, D, N, K, W = 2, 6, 5, 4, 4
    p, cs0, h0, rng = _replay_setup(91, n_slots, D, N, K)
    rep = orc.replay_init(h0, W, keep_lo=True)
    assert np.array_equal(rep["ck_lo"], orc.round_bf16(h0))
    cs_e, h_e, cs_r = cs0, h0, cs0
    dsum = np.zeros((n_slots, D))
    for t in range(10):
        a = _step_inputs(rng, n_slots, D, N)
        args = (a["x"], a["dt"], a["B"], a["C"], a["z"], p["w"], p["b"], p["A"], p["D"], p["dtb"])
        ck_before, lo_before = rep["ck"].copy(), rep["ck_lo"].copy()
        y_e, cs_e, h_e = orc.state_update(cs_e, h_e, *args)
        y_r, cs_r, rep = orc.replay_step(cs_r, rep, *args)
        dsum += np.logaddexp(0.0, a["dt"] + p["dtb"][None, :])
        if (t + 1) % W == 0:
            assert _rel_err(y_r, y_e) <= 1e-12, t
            assert _rel_err(rep["ck"], h_e) <= 1e-12, t
            assert np.array_equal(rep["ck_lo"], orc.round_bf16(rep["ck"])), t
            dsum[:] = 0.0
        else:
            decay = np.exp(p["A"][None, :, :] * dsum[:, :, None])
            corr = np.sum(a["C"][:, None, :] * decay * (lo_before - ck_before), axis=2)
            want = y_e + corr * a["z"] * expit(a["z"])
            assert _rel_err(y_r, want) <= 1e-12, t
            assert not np.allclose(y_r, y_e, rtol=0, atol=1e-9 * np.abs(y_e).max()), t
            assert np.array_equal(rep["ck"], ck_before) and np.array_equal(rep["ck_lo"], lo_before)


def check_replay_state_indices(orc):
    n_slots, Bt, D, N, K, W = 7, 4, 3, 4, 4, 3
    p, cs, h, rng = _replay_setup(101, n_slots, D, N, K)
    rep = orc.replay_init(h, W, keep_lo=True)
    rep["len"][:] = [0, 1, 2, 1, 0, 2, 1]  # slots at different points of their windows
    rep["bd"][:] = np.abs(rng.standard_normal(rep["bd"].shape)) * 0.05
    rep["bx"][:] = rng.standard_normal(rep["bx"].shape)
    rep["bB"][:] = rng.standard_normal(rep["bB"].shape)
    a = _step_inputs(rng, Bt, D, N)
    idx = np.array([5, -1, 0, 3], dtype=np.int64)
    sentinel = np.full((Bt, D), 123.5)
    args = (a["x"], a["dt"], a["B"], a["C"], a["z"], p["w"], p["b"], p["A"], p["D"], p["dtb"])
    y, cs2, rep2 = orc.replay_step(cs, rep, *args, state_indices=idx, y_init=sentinel)
    untouched = [s for s in range(n_slots) if s not in idx]
    for key in ("ck", "ck_lo", "bd", "bx", "bB", "len"):
        assert np.array_equal(rep2[key][untouched], rep[key][untouched]), key
    assert np.array_equal(cs2[untouched], cs[untouched])
    assert np.array_equal(y[1], sentinel[1])
    assert list(rep2["len"][[5, 0, 3]]) == [0, 1, 2]  # slot 5 reached W tokens: checkpoint step
    # the touched slots equal a run over the gathered slots, and eager decode of
    # their materialised states
    rows, slots = [0, 2, 3], idx[[0, 2, 3]]
    sub = {k: (v[slots] if isinstance(v, np.ndarray) else v) for k, v in rep.items()}
    sub_args = tuple(v[rows] for v in args[:5]) + args[5:]
    yd, csd, repd = orc.replay_step(cs[slots], sub, *sub_args)
    assert np.array_equal(y[rows], yd)
    assert np.array_equal(cs2[slots], csd)
    for key in ("ck", "ck_lo", "bd", "bx", "bB", "len"):
        assert np.array_equal(rep2[key][slots], repd[key]), key
    h_now = orc.replay_state(rep, p["A"])[slots]
    ye, _, he = orc.state_update(cs[slots], h_now, *sub_args)
    nolo = dict(sub, ck_lo=None)
    yn, _, repn = orc.replay_step(cs[slots], nolo, *sub_args)
    assert _rel_err(yn, ye) <= 1e-12
    assert _rel_err(orc.replay_state(repn, p["A"]), he) <= 1e-12


def check_replay_after_prefill(orc):
    """Prefill, then k replay steps from its final state, equals prefill over
    the extended sequence (outputs and state)."""
    D, N, K, L0, k, W = 4, 4, 4, 9, 7, 3
    L = L0 + k
    p, a = _rand_layer(111, L, D, N, K)
    y, hf, cs = _layer(orc, a["x"], a["dt"], a["z"], a["B"], a["C"], p,
                       np.array([0, L], dtype=np.int64))
    _, h, c = _layer(orc, a["x"][:L0], a["dt"][:L0], a["z"][:L0], a["B"][:L0], a["C"][:L0], p,
                     np.array([0, L0], dtype=np.int64))
    rep = orc.replay_init(h, W, keep_lo=False)
    for t in range(L0, L):
        sl = slice(t, t + 1)
        yt, c, rep = orc.replay_step(c, rep, a["x"][sl], a["dt"][sl], a["B"][sl], a["C"][sl],
                                     a["z"][sl], p["w"], p["b"], p["A"], p["D"], p["dtb"])
        assert _rel_err(yt[0], y[t]) <= 1e-12, t
    assert _rel_err(orc.replay_state(rep, p["A"]), hf) <= 1e-12
    assert np.array_equal(c, cs)


# ---------------------------------------------------------------------------
# backward scan (training): chain rule against finite differences
# ---------------------------------------------------------------------------

def _bwd_case(seed, lens, D, N, gate=True, softplus=True):
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    tok, S = int(cu[-1]), len(lens)
    # the step size must stay positive: raw values through the softplus, or
    # positive values directly when it is off
    delta = 0.4 * rng.standard_normal((tok, D)) if softplus else 0.1 * np.abs(
        rng.standard_normal((tok, D)))
    f = {"u": rng.standard_normal((tok, D)), "delta": delta,
         "A": -np.exp(rng.uniform(-1, 1, (D, N))), "B": rng.standard_normal((tok, N)),
         "C": rng.standard_normal((tok, N)), "Dskip": rng.standard_normal(D),
         "z": rng.standard_normal((tok, D)) if gate else None,
         "dt_bias": rng.uniform(-2, -0.5, D) if softplus else rng.uniform(0.05, 0.3, D),
         "h0": rng.standard_normal((S, D, N))}
    w = {"dy": rng.standard_normal((tok, D)), "dh_final": rng.standard_normal((S, D, N))}
    return f, w, cu, softplus


def _loss(orc, f, w, cu, softplus):
    y, hf = orc.selective_scan(f["u"], f["delta"], f["A"], f["B"], f["C"], Dskip=f["Dskip"],
                               z=f["z"], dt_bias=f["dt_bias"], delta_softplus=softplus,
                               h0=f["h0"], cu_seqlens=cu, want_state=True)
    return float(np.sum(w["dy"] * y) + np.sum(w["dh_final"] * hf))


def check_bwd_finite_differences(orc):
    """Every gradient of the backward scan equals the central difference of the
    forward scan's loss sum(dy*y) + sum(dh_final*h_final), element by element."""
    names = {"u": "du", "delta": "ddt", "z": "dz", "B": "dB", "C": "dC", "A": "dA",
             "Dskip": "dDskip", "dt_bias": "ddt_bias", "h0": "dh0"}
    for gate, softplus, lens in ((True, True, [3, 0, 5]), (False, False, [4, 2])):
        f, w, cu, sp = _bwd_case(121 + len(lens), lens, 2, 3, gate, softplus)
        g = orc.selective_scan_bwd(f["u"], f["delta"], f["A"], f["B"], f["C"], w["dy"],
                                   Dskip=f["Dskip"], z=f["z"], dt_bias=f["dt_bias"],
                                   delta_softplus=sp, h0=f["h0"], cu_seqlens=cu,
                                   dh_final=w["dh_final"])
        eps = 1e-6
        for name, gname in names.items():
            if f[name] is None:
                assert g[gname] is None
                continue
            arr = f[name]
            num = np.zeros(arr.shape)
            for idx in np.ndindex(arr.shape):
                keep = arr[idx]
                arr[idx] = keep + eps
                lp = _loss(orc, f, w, cu, sp)
                arr[idx] = keep - eps
                lm = _loss(orc, f, w, cu, sp)
                arr[idx] = keep
                num[idx] = (lp - lm) / (2 * eps)
            scale = max(np.max(np.abs(num)), 1.0)
            err = np.max(np.abs(g[gname] - num)) / scale
            assert err <= 1e-6, (name, gate, softplus, err)


def check_bwd_pack_equals_separate(orc):
    """A packed backward equals its sequences' backwards: per-token gradients
    and dh0 exactly, the per-channel sums (dA, dDskip, ddt_bias) as the sum of
    the separate runs."""
    lens = [5, 1, 0, 7]
    f, w, cu, sp = _bwd_case(131, lens, 3, 4)
    g = orc.selective_scan_bwd(f["u"], f["delta"], f["A"], f["B"], f["C"], w["dy"],
                               Dskip=f["Dskip"], z=f["z"], dt_bias=f["dt_bias"], h0=f["h0"],
                               cu_seqlens=cu, dh_final=w["dh_final"])
    tot = {k: np.zeros_like(g[k]) for k in ("dA", "dDskip", "ddt_bias")}
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        gs = orc.selective_scan_bwd(f["u"][a:b], f["delta"][a:b], f["A"], f["B"][a:b],
                                    f["C"][a:b], w["dy"][a:b], Dskip=f["Dskip"],
                                    z=f["z"][a:b], dt_bias=f["dt_bias"], h0=f["h0"][s:s + 1],
                                    cu_seqlens=np.array([0, b - a]),
                                    dh_final=w["dh_final"][s:s + 1])
        for k in ("du", "ddt", "dz", "dB", "dC"):
            assert np.array_equal(g[k][a:b], gs[k]), (s, k)
        assert np.array_equal(g["dh0"][s], gs["dh0"][0]), s
        for k in tot:
            tot[k] += gs[k]
    for k in tot:
        assert _rel_err(g[k], tot[k]) <= 1e-14, k


ALL_CHECKS = [
    check_softplus_spot, check_silu_spot, check_conv_identity_tap, check_closed_form,
    check_bruteforce, check_conv_correlate, check_pack_equals_separate,
    check_chunked_equals_oneshot, check_decode_invariant, check_state_indices,
    check_golden_dyadic, check_round_bf16, check_replay_equals_eager,
    check_replay_low_precision, check_replay_state_indices, check_replay_after_prefill,
    check_bwd_finite_differences, check_bwd_pack_equals_separate,
]
