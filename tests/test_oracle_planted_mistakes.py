"""Planted mistakes in a copy of the oracle must each fail a pin.

Each mutation below is a plausible slip in writing the recurrence (a wrong
sign, a dropped term, a transposed operand, a wrong index).  The test
compiles a mutated copy of oracle.c into a temporary library and checks that
at least one pin in tests/pins.py rejects it.  The real oracle is untouched.
"""
import os
import tempfile

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTATIONS = {
    "combine_transposed": ("*b_out = a2 * b1 + b2;", "*b_out = a1 * b2 + b1;"),
    "fade_applied_to_input": ("hp[n] = abar * hp[n] + bbar_u;",
                              "hp[n] = hp[n] + abar * bbar_u;"),
    "readout_uses_B": ("after the update. */\n        acc += Cb[n * seqlen + t] * hp[n];",
                       "after the update. */\n        acc += Bb[n * seqlen + t] * hp[n];"),
    "skip_dropped": ("double yt = acc + dskip * ut;", "double yt = acc;"),
    "decay_sign": ("exp(dt * A[d * dstate + n])", "exp(-dt * A[d * dstate + n])"),
    "B_index_transposed": ("dt * Bb[n * seqlen + t] * ut",
                           "dt * Bb[t * dstate + n] * ut"),
    "softplus_sign": ("log1p(exp(-ax))", "log1p(exp(ax))"),
    "softplus_no_max": ("(x > 0.0 ? x : 0.0) + log1p", "0.0 + log1p"),
    "silu_sign": ("z / (1.0 + exp(-z))", "z / (1.0 + exp(z))"),
    "bias_ignored": ("double x = delta + bias;", "double x = delta;"),
    "h0_ignored": ("hp[n] = h0 ? h0[(b * dim + d) * dstate + n] : 0.0;",
                   "hp[n] = 0.0;"),
    "input_without_step": ("const double bbar_u = dt * Bb[n * seqlen + t] * ut;",
                           "const double bbar_u = Bb[n * seqlen + t] * ut;"),
    "gate_before_skip": ("double yt = acc + dskip * ut;\n      if (zrow) yt *= oracle_silu_f64(zrow[t]);",
                         "double yt = acc;\n      if (zrow) yt *= oracle_silu_f64(zrow[t]);\n      yt += dskip * ut;"),
    "readout_before_update": (
        "        hp[n] = abar * hp[n] + bbar_u;\n        /* [eq]: y_t = C_t h_t, with the state after the update. */\n        acc += Cb[n * seqlen + t] * hp[n];",
        "        acc += Cb[n * seqlen + t] * hp[n];\n        hp[n] = abar * hp[n] + bbar_u;"),
    "reset_dropped": ("          for (int64_t n = 0; n < dstate; ++n) hp[n] = wprev[n] = 0.0;",
                      "          ;"),
    "reset_one_step_late": ("cu_seqlens[next] == t)", "cu_seqlens[next] == t - 1)"),
    "bwd_adjoint_not_decayed": ("          lam[n] *= a;\n", "\n"),
    "bwd_dA_without_step": ("pA[(b * dim + d) * N + n] += lam[n] * dt * a * hprev;",
                            "pA[(b * dim + d) * N + n] += lam[n] * a * hprev;"),
    "bwd_dC_uses_previous_state": ("dCb[n * L + t] += ds * H[(t + 1) * N + n];",
                                   "dCb[n * L + t] += ds * H[t * N + n];"),
    "bwd_gate_derivative_wrong": ("return sg * (1.0 + z * (1.0 - sg));", "return sg;"),
    "bwd_softplus_derivative_dropped": ("? dDelta / (1.0 + exp(-x)) : dDelta;", "? dDelta : dDelta;"),
    "bwd_packed_adjoint_flows_back": ("const double a = starts[t] ? 0.0 : exp(dt * an);",
                                      "const double a = exp(dt * an);"),
    "bwd_packed_state_not_reset": ("const double hin = starts[t] ? 0.0 : H[t * N + n];",
                                   "const double hin = H[t * N + n];"),
    "trap_previous_input_not_decayed": ("0.5 * dt * (abar * wprev[n] + w)", "0.5 * dt * (wprev[n] + w)"),
    "trap_full_step_weights": ("0.5 * dt * (abar * wprev[n] + w)", "dt * (abar * wprev[n] + w)"),
    "trap_previous_input_not_kept": ("          wprev[n] = w;\n", "\n"),
    "ssd_group_index": ("const int64_t g = h / heads_per_group;",
                        "const int64_t g = h % ngroups;"),
    "ssd_decay_sign": ("exp(step * A[h])", "exp(-step * A[h])"),
    "ssd_readout_uses_B": ("acc += Ct[n] * S[p * dstate + n];",
                           "acc += Bt[n] * S[p * dstate + n];"),
    "ssd_skip_dropped": ("double yp = acc + dskip * xp;", "double yp = acc;"),
    "ssd_input_without_step": ("step * Bt[n] * xp", "Bt[n] * xp"),
    "ssd_h0_transposed": ("h0[((b * nheads + h) * headdim + p) * dstate + n]",
                          "h0[((b * nheads + h) * dstate + n) * headdim + p]"),
    "ssd_dt_of_head_zero": ("dt[(b * seqlen + t) * nheads + h]", "dt[(b * seqlen + t) * nheads]"),
    "update_step_uses_input_twice": (
        "step * B[b * dstate + n] * x[ch];", "step * B[b * dstate + n] * x[ch] * x[ch];"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique/found"
    with tempfile.TemporaryDirectory() as tmp:
        path = os.path.join(tmp, "mutant.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        so = oracle.build(force=True, src=path,
                          out=os.path.join(tmp, "libmutant.so"), openmp=False)
        lib = oracle.load(path=so)
        failed = []
        for pin in pins.ALL_PINS:
            try:
                pin(lib)
            except AssertionError:
                failed.append(pin.__name__)
        assert failed, f"no pin caught the planted mistake {name}"
