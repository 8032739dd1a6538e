"""Plant plausible mistakes in copies of the oracle (on the CPU) and require
that at least one pin catches each.  This shows the pins constrain every part
of the oracle: the readout index, skip and gate order, discretisation, bias,
operand indexing, checkpoint placement, decode step and every adjoint term.
"""
import multiprocessing as mp
import os

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ss_oracle.c")

# (name, exact text in ss_oracle.c, replacement).  Each mutant stays in bounds.
MUTANTS = [
    ("readout_before_update",
     "h[n] = abar * h[n] + dt * Bm[bi] * u[i];        /* Euler for B    */\n"
     "          ys += Cm[bi] * h[n];                            /* readout, h_t   */",
     "ys += Cm[bi] * h[n];\n          h[n] = abar * h[n] + dt * Bm[bi] * u[i];"),
    ("skip_dropped",
     "double out = ys + at(Dskip, (size_t)d, 0.0) * u[i]; /* D skip       */",
     "double out = ys;"),
    ("gate_before_skip",
     "y[i] = z ? out * z[i] * sg(z[i]) : out;            /* SiLU(z) gate */",
     "y[i] = z ? ys * z[i] * sg(z[i]) + (out - ys) : out;"),
    ("decay_sign", "double abar = exp(dt * A[d * N + n]);          /* ZOH for A      */",
     "double abar = exp(-dt * A[d * N + n]);"),
    ("bias_dropped_fwd",
     "double x = delta[i] + at(bias, (size_t)d, 0.0);\n        double dt = softplus ? sp(x) : x;\n"
     "        double ys = 0.0;\n        for (int64_t n = 0; n < N; ++n) {\n"
     "          size_t bi = ((size_t)b * N + n) * (size_t)L + (size_t)t;\n"
     "          double abar",
     "double x = delta[i];\n        double dt = softplus ? sp(x) : x;\n"
     "        double ys = 0.0;\n        for (int64_t n = 0; n < N; ++n) {\n"
     "          size_t bi = ((size_t)b * N + n) * (size_t)L + (size_t)t;\n"
     "          double abar"),
    ("B_time_reversed",
     "size_t bi = ((size_t)b * N + n) * (size_t)L + (size_t)t;\n          double abar",
     "size_t bi = ((size_t)b * N + n) * (size_t)L + (size_t)(L - 1 - t);\n          double abar"),
    ("zoh_for_B", "h[n] = abar * h[n] + dt * Bm[bi] * u[i];        /* Euler for B    */",
     "h[n] = abar * h[n] + (abar - 1.0) / A[d * N + n] * Bm[bi] * u[i];"),
    ("softplus_no_abs", "return (x > 0 ? x : 0.0) + log1p(exp(-fabs(x)));",
     "return (x > 0 ? x : 0.0) + log1p(exp(-x));"),
    ("checkpoint_off_by_one", "t % chunk == chunk - 1", "t % chunk == 0"),
    ("bwd_drop_dA_term_in_dDelta", "double dDelta = u[i] * sgb + sga;",
     "double dDelta = u[i] * sgb;"),
    ("bwd_dz_sign", "(1.0 + z[i] * (1.0 - s))", "(1.0 - z[i] * (1.0 - s))"),
    ("bwd_double_decay", "g[n] += dout * Cm[bi];",
     "g[n] = g[n] * Ab[(size_t)t * N + n] + dout * Cm[bi];"),
    ("bwd_dA_uses_h_t", "double q = g[n] * a * hp[n];", "double q = g[n] * a * ht[n];"),
    ("bwd_no_softplus_chain", "double dx = softplus ? dDelta * sg(x) : dDelta;",
     "double dx = dDelta;"),
    ("bwd_du_no_skip", "du[i] = dout * Dd + dt * sgb;", "du[i] = dt * sgb;"),
    ("bwd_dC_uses_h_prev", "dC[bi] += dout * ht[n];", "dC[bi] += dout * hp[n];"),
    ("bwd_dB_missing_u", "dB[bi] += g[n] * dt * u[i];", "dB[bi] += g[n] * dt;"),
    ("bwd_dfinal_ignored", "g[n] = dfinal ? dfinal[row * N + n] : 0.0;", "g[n] = 0.0;"),
    ("conv_taps_reversed",
     "pre += w[d * W + k] * conv_in(x, state_in, W, row, L, t - (W - 1) + k);\n        u[row",
     "pre += w[d * W + (W - 1 - k)] * conv_in(x, state_in, W, row, L, t - (W - 1) + k);\n        u[row"),
    ("conv_state_out_shifted", "? conv_in(x, state_in, W, row, L, L - (W - 1) + j) : 0.0;",
     "? conv_in(x, state_in, W, row, L, L - W + j + (L - W + j < -(W - 1) ? 1 : 0)) : 0.0;"),
    ("conv_bwd_silu_derivative", "g *= s * (1.0 + pre * (1.0 - s));", "g *= s;"),
    ("conv_bwd_dx_taps_reversed", "same_doc(seq_idx, b, L, s, t)) g += w[d * W + k] * dp[t];",
     "same_doc(seq_idx, b, L, s, t)) g += w[d * W + (W - 1 - k)] * dp[t];"),
    ("conv_step_window_not_shifted", "if (W > 1) st[W - 2] = x[i];", "if (W > 1) st[0] = x[i];"),
    ("seq_reset_ignored_fwd", "if (reset_before(seq_idx, b, L, t))\n          for (int64_t n = 0; n < N; ++n) h[n] = 0.0;",
     "if (0 && reset_before(seq_idx, b, L, t))\n          for (int64_t n = 0; n < N; ++n) h[n] = 0.0;"),
    ("seq_reset_ignored_bwd", "double a = rst ? 0.0 : exp(dt * A[d * N + n]);",
     "double a = exp(dt * A[d * N + n]); (void)rst;"),
    ("ssd_group_index", "int64_t g = h / hpg;", "int64_t g = h % ng;"),
    ("ssd_decay_sign", "double a = exp(Dt * A[h]);", "double a = exp(-Dt * A[h]);"),
    ("ssd_B_C_swapped", "acc += *hp * Ct[n];", "acc += *hp * Bt[n];"),
    ("ssd_no_dt_in_input", "*hp = a * *hp + Dt * xp * Bt[n];", "*hp = a * *hp + xp * Bt[n];"),
    ("ssd_bwd_dB_missing_dt", "dB[bo + n] += Dt * *gp * x[xo + p];", "dB[bo + n] += *gp * x[xo + p];"),
    ("ssd_bwd_dC_uses_prev_state", "dC[bo + n] += Ht[p * N + n] * dout[p];",
     "dC[bo + n] += Hp[p * N + n] * dout[p];"),
    ("ssd_bwd_drop_decay_term", "double dDelta = gbx + A[h] * q;", "double dDelta = gbx;"),
    ("ssd_bwd_dx_no_skip", "dx[xo + p] = Dt * gb + Dh * dout[p];", "dx[xo + p] = Dt * gb;"),
    ("ssd_bwd_carry_not_decayed", "for (int64_t i = 0; i < PN; ++i) G[i] *= a;", "(void)a;"),
    ("ssd_bwd_dz_sign", "(1.0 + zz * (1.0 - s))", "(1.0 - zz * (1.0 - s))"),
    ("ssd_bwd_dfinal_ignored", "G[i] = dfinal ? dfinal[sidx + i] : 0.0;", "G[i] = 0.0;"),
    ("ssd_bwd_dA_uses_H_t", "q += *gp * a * Hp[p * N + n];", "q += *gp * Ht[p * N + n];"),
    ("ssd_bwd_group_index", "const int64_t grp = h / hpg;", "const int64_t grp = h % ng;"),
    ("conv_seq_ignored_dx", "if (t >= 0 && t < L && same_doc(seq_idx, b, L, s, t))",
     "if (t >= 0 && t < L && (1 || same_doc(seq_idx, b, L, s, t)))"),
    ("update_uses_C_for_B", "*h = a * *h + dt * Bm[b * N + n] * u[i];",
     "*h = a * *h + dt * Cm[b * N + n] * u[i];"),
    ("update_no_skip", "double out = ys + at(Dskip, (size_t)d, 0.0) * u[i];\n      y[i]",
     "double out = ys;\n      y[i]"),
]


def _run_pins(so_path, q):
    orc = oracle.Oracle(so_path)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
        except Exception as e:  # a crash inside a pin also counts as caught
            caught.append(f"{pin.__name__}:{type(e).__name__}")
    q.put(caught)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique/present"
    mpath = tmp_path / f"{name}.c"
    mpath.write_text(src.replace(old, new))
    so = oracle.build(force=True, src=str(mpath), out=str(tmp_path / f"{name}.so"))
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_run_pins, args=(so, q))
    p.start()
    p.join(300)
    assert p.exitcode is not None, "pin run hung"
    caught = q.get(timeout=5) if p.exitcode == 0 else ["process crashed"]
    assert caught, f"no pin caught mutant {name}"


def test_unmutated_copy_passes_every_pin(tmp_path):
    """Control: the same harness on an unmodified copy catches nothing."""
    mpath = tmp_path / "control.c"
    mpath.write_text(open(SRC).read())
    so = oracle.build(force=True, src=str(mpath), out=str(tmp_path / "control.so"))
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_run_pins, args=(so, q))
    p.start()
    p.join(300)
    assert p.exitcode == 0
    assert q.get(timeout=5) == []
