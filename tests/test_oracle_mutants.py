"""Planted mistakes in the oracle must fail at least one pin (CPU only).

Each case copies the oracle's C source, plants one plausible slip (a dropped
term, a wrong sign or index, a swapped operand), compiles the copy into a
temporary directory and runs every pin from oracle_pins against it. Every
mutant keeps all memory accesses in bounds.
"""

import os

import pytest

import oracle
import oracle_pins as pins

MUTANTS = {
    "dropped_decay": ("h[n] = dA * h[n] + d * ut * B[t * N + n];",
                      "h[n] = h[n] + d * ut * B[t * N + n];", 0),
    "wrong_sign_of_A": ("const double dA = exp(d * A[c * N + n]);",
                        "const double dA = exp(-d * A[c * N + n]);", 0),
    "C_in_place_of_B": ("d * ut * B[t * N + n]", "d * ut * C[t * N + n]", 0),
    "B_in_place_of_C": ("acc += C[t * N + n] * h[n];", "acc += B[t * N + n] * h[n];", 0),
    "dropped_skip": ("double yt = acc + (Dskip ? Dskip[c] : 0.0) * ut;", "double yt = acc;", 0),
    "readout_before_update": ("h[n] = dA * h[n] + d * ut * B[t * N + n];\n"
                              "                    acc += C[t * N + n] * h[n];",
                              "acc += C[t * N + n] * h[n];\n"
                              "                    h[n] = dA * h[n] + d * ut * B[t * N + n];", 0),
    "input_decayed_by_own_step": ("h[n] = dA * h[n] + d * ut * B[t * N + n];",
                                  "h[n] = dA * (h[n] + d * ut * B[t * N + n]);", 0),
    "gate_without_silu": ("yt *= silu(z[t * D + c]);", "yt *= z[t * D + c];", 0),
    "silu_sign": ("return v / (1.0 + exp(-v));", "return v / (1.0 + exp(v));", 0),
    "softplus_missing_linear_part": ("return (v > 0.0 ? v : 0.0) + log1p(exp(-fabs(v)));",
                                     "return log1p(exp(-fabs(v)));", 0),
    "dropped_dt_bias": ("double d = delta[t * D + c] + (dt_bias ? dt_bias[c] : 0.0);",
                        "double d = delta[t * D + c];", 0),
    "ignored_h0": ("for (int n = 0; n < N; ++n) h[n] = h0 ? h0[(s * D + c) * N + n] : 0.0;",
                   "for (int n = 0; n < N; ++n) h[n] = 0.0;", 0),
    "reversed_taps": ("acc += w[c * K + k] * window_value(",
                      "acc += w[c * K + (K - 1 - k)] * window_value(", 0),
    "reversed_state_order": ("return state_in[(s * D + c) * (K - 1) + (K - 1) + p];",
                             "return state_in[(s * D + c) * (K - 1) + (-1 - p)];", 0),
    "window_leaks_across_sequences": ("if (p >= 0) return x[(start + p) * D + c];",
                                      "if (start + p >= 0) return x[(start + p) * D + c];", 0),
    "state_out_ignores_carried_state": ("window_value(x, state_in, D, K, start, s, c, p);",
                                        "window_value(x, NULL, D, K, start, s, c, p);", 0),
    "decode_no_shift": ("conv_state[(s * D + c) * (K - 1) + j] = win[j + 1];",
                        "conv_state[(s * D + c) * (K - 1) + j] = win[j];", 0),
    "decode_uses_preconv_input": ("h[n] = dA * h[n] + d * xcv * B[b * N + n];",
                                  "h[n] = dA * h[n] + d * x[b * D + c] * B[b * N + n];", 0),
    "decode_skip_on_raw_input": ("double yt = sum + (Dskip ? Dskip[c] : 0.0) * xcv;",
                                 "double yt = sum + (Dskip ? Dskip[c] : 0.0) * x[b * D + c];", 0),
    "decode_wrong_slot": ("const int64_t s = idx ? idx[b] : b;",
                          "const int64_t s = b < n_slots ? b : -1;", 0),
    "replay_base_not_decayed": ("double h = exp(a * total) * base[c * N + n];",
                                "double h = base[c * N + n];", 0),
    "replay_input_decayed_by_own_step": ("for (int64_t r = i + 1; r < len; ++r)",
                                         "for (int64_t r = i; r < len; ++r)", 0),
    "replay_B_of_newest_token": ("* bx[i * D + c] * bB[i * N + n];",
                                 "* bx[i * D + c] * bB[(len - 1) * N + n];", 0),
    "replay_checkpoint_step_reads_low_copy": (
        "const double *base = (flush || ck_lo == NULL) ? ck : ck_lo;",
        "const double *base = (ck_lo == NULL) ? ck : ck_lo;", 0),
    "replay_never_reads_low_copy": ("const double *base = (flush || ck_lo == NULL) ? ck : ck_lo;",
                                    "const double *base = ck;", 0),
    "replay_length_not_reset": ("len[s] = flush ? 0 : j + 1;", "len[s] = flush ? j : j + 1;", 0),
    "replay_checkpoint_every_step": ("const int flush = (j + 1 == W);", "const int flush = 1;", 0),
    "replay_low_copy_not_refreshed": ("if (ck_lo) ck_lo[(s * D + c) * N + n] = round_bf16(h[n]);",
                                      "(void)0;", 0),
    "round_bf16_truncates": ("ldexp(nearbyint(ldexp(m, 8)), e - 8)",
                             "ldexp(trunc(ldexp(m, 8)), e - 8)", 0),
    "round_bf16_seven_bits": ("ldexp(nearbyint(ldexp(m, 8)), e - 8)",
                              "ldexp(nearbyint(ldexp(m, 7)), e - 7)", 0),
    "bwd_gradient_not_decayed": ("G[n] *= a;", "G[n] *= 1.0;", 0),
    "bwd_readout_term_dropped": ("G[n] += dq * C[t * N + n];", "G[n] += 0.0 * C[t * N + n];", 0),
    "bwd_softplus_derivative_dropped": (
        "const double dsp = delta_softplus ? 1.0 / (1.0 + exp(-v)) : 1.0;",
        "const double dsp = 1.0;", 0),
    "bwd_dA_with_current_state": ("dA[c * N + n] += G[n] * d * a * hp[n];",
                                  "dA[c * N + n] += G[n] * d * a * h[n];", 0),
    "bwd_dB_without_u": ("dB[t * N + n] += G[n] * d * ut;", "dB[t * N + n] += G[n] * d;", 0),
    "bwd_gate_derivative_wrong": ("dg = sg * (1.0 + zt * (1.0 - sg));", "dg = sg;", 0),
    "bwd_skip_term_dropped": ("double dut = dq * (Dskip ? Dskip[c] : 0.0), dd = 0.0;",
                              "double dut = 0.0, dd = 0.0;", 0),
    "bwd_ddelta_state_term_dropped": (
        "dd += G[n] * (ut * B[t * N + n] + A[c * N + n] * a * hp[n]);",
        "dd += G[n] * (ut * B[t * N + n]);", 0),
    "bwd_dC_with_state_gradient": ("dC[t * N + n] += dq * h[n];", "dC[t * N + n] += G[n] * h[n];",
                                   0),
}


def _replace_nth(text, old, new, nth):
    pos = -1
    for _ in range(nth + 1):
        pos = text.find(old, pos + 1)
        assert pos >= 0, f"pattern not found: {old!r}"
    return text[:pos] + new + text[pos + len(old):]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new, nth = MUTANTS[name]
    src = open(oracle.SOURCE).read()
    mutated = _replace_nth(src, old, new, nth)
    assert mutated != src
    c_path = os.path.join(tmp_path, "mutant.c")
    so_path = os.path.join(tmp_path, "libmutant.so")
    with open(c_path, "w") as f:
        f.write(mutated)
    oracle.compile_oracle(c_path, so_path)
    mut = oracle.load(so_path)
    caught = []
    for check in pins.ALL_CHECKS:
        try:
            check(mut)
        except AssertionError:
            caught.append(check.__name__)
    assert caught, f"mutant {name} passed every pin"
