"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that
at least one pin catches each of them.  This shows the pins are strong enough
that a dropped term, a wrong sign, a wrong index or a transposed operand in
the oracle would not go unnoticed."""
import os

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "s6_oracle.c")

MUTATIONS = {
    "euler_instead_of_zoh": ("const double Bbar = Delta * psi(x) * Bm[n * L + t];",
                             "const double Bbar = Delta * Bm[n * L + t];"),
    "wrong_sign_in_Abar": ("      const double Abar = exp(x);\n      const double Bbar",
                           "      const double Abar = exp(-x);\n      const double Bbar"),
    "exp_instead_of_softplus": ("    const double Delta = softplus(dl[t] + bias);\n    double y0 = 0.0;\n    for (i64 n = 0; n < N; ++n) {\n      const double x",
                                "    const double Delta = exp(dl[t] + bias);\n    double y0 = 0.0;\n    for (i64 n = 0; n < N; ++n) {\n      const double x"),
    "readout_before_update": ("      h[n] = Abar * h[n] + Bbar * u[t];\n      y0 += Cm[n * L + t] * h[n];",
                              "      y0 += Cm[n * L + t] * h[n];\n      h[n] = Abar * h[n] + Bbar * u[t];"),
    "B_read_transposed": ("const double Bbar = Delta * psi(x) * Bm[n * L + t];",
                          "const double Bbar = Delta * psi(x) * Bm[t * N + n];"),
    "dropped_D_skip": ("    if (j->D) y0 += Dd * u[t];\n    if (z) y0 *= z[t] * sigmoid(z[t]);",
                       "    if (z) y0 *= z[t] * sigmoid(z[t]);"),
    "sigmoid_gate_not_silu": ("if (z) y0 *= z[t] * sigmoid(z[t]);", "if (z) y0 *= sigmoid(z[t]);"),
    "bias_ignored": ("const double bias = j->bias ? j->bias[d] : 0.0;\n  const double Dd = j->D ? j->D[d] : 0.0;\n  double *y",
                     "const double bias = 0.0;\n  const double Dd = j->D ? j->D[d] : 0.0;\n  double *y"),
    "initial_state_ignored": ("h[n] = j->h0 ? j->h0[(b * dim + d) * N + n] : 0.0;",
                              "h[n] = 0.0;"),
    "bwd_dropped_phi_term": ("Bt * u[t] * Delta * Delta * phi(x)", "0.0"),
    "bwd_adjoint_uses_current_Abar": ("Abar_next[n] * G[n];", "Abar * G[n];"),
    "bwd_dz_missing_factor": ("s * (1.0 + z[t] * (1.0 - s))", "s"),
    "bwd_dDelta_sign": ("(A[n] * hprev + Bt * u[t])", "(A[n] * hprev - Bt * u[t])"),
    "conv_weight_reversed": ("if (s >= 0) p += w[d * W + k] * x[off + s];",
                             "if (s >= 0) p += w[d * W + (W - 1 - k)] * x[off + s];"),
    "conv_silu_dropped": ("u[off + t] = p * sigmoid(p);", "u[off + t] = p;"),
    "conv_bias_ignored": ("double p = cb ? cb[d] : 0.0;", "double p = 0.0;"),
    "bwd_conv_dx_wrong_weight": ("dx[off + src] += conv_w[d * W + k] * dpre;",
                                 "dx[off + src] += conv_w[d * W + (W - 1 - k)] * dpre;"),
    "bwd_conv_silu_derivative": ("s * (1.0 + pre[off + t] * (1.0 - s))", "s"),
    "bwd_conv_dw_uses_output_step": ("dconv_w[d * W + k] += dpre * x[off + src];",
                                     "dconv_w[d * W + k] += dpre * x[off + t];"),
    "dtproj_W_transposed": ("s += W[d * R + r] * dt_low[(b * R + r) * L + t];",
                            "s += W[r * dim + d] * dt_low[(b * R + r) * L + t];"),
    "bwd_dtproj_dW_wrong_input": ("dW_dt[d * R + r] += g * dt_low[(b * R + r) * L + t];",
                                  "dW_dt[d * R + r] += g * W_dt[d * R + r];"),
    "bwd_dtproj_ddt_low_missing_W": ("d_dt_low[(b * R + r) * L + t] += W_dt[d * R + r] * g;",
                                     "d_dt_low[(b * R + r) * L + t] += g;"),
    "cplx_readout_drops_imaginary_product": (
        "y0 += creal(cget(Cm + t, n, N, L) * h[n]);",
        "y0 += creal(cget(Cm + t, n, N, L)) * creal(h[n]);"),
    "cplx_bwd_adjoint_without_conjugates": (
        "G[n] = conj(Cn) * dy0 + conj(Anext[n]) * G[n];", "G[n] = Cn * dy0 + Anext[n] * G[n];"),
    "cplx_bwd_dA_without_conjugate": (
        "gA[n] += conj(Delta * Abar * hprev + Delta * Delta * cphi(x) * Bn * ut) * G[n];",
        "gA[n] += (Delta * Abar * hprev + Delta * Delta * cphi(x) * Bn * ut) * G[n];"),
    "bwd_dC_uses_prev_state": ("dCacc[(b * N + n) * L + t] += dy0 * H[(t + 1) * N + n];",
                               "dCacc[(b * N + n) * L + t] += dy0 * H[t * N + n];"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique/found"
    mutant_src = tmp_path / "mutant.c"
    mutant_src.write_text(src.replace(old, new))
    lib = oracle.load_library(oracle.compile_source(str(mutant_src), str(tmp_path / "m.so")))
    results = oracle_pins.run_all(lib)
    caught = [k for k, v in results.items() if not (v[0] <= v[1])]
    assert caught, f"no pin caught the planted mistake {name}: {results}"
