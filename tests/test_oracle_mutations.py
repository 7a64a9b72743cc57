"""Plant plausible mistakes in copies of the oracle (CPU only) and check that each one
breaks at least one pin.  The planted copies live in a temporary directory; the real
oracle source is never modified."""
import os

import pytest

import oracle
import pins

_SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

# (name, [(old, new, occurrence index)])
MUTATIONS = [
    ("erase_dropped", [("+= -beta * ki * kS[j] + beta * ki * (double)v[j];", "+= beta * ki * (double)v[j];", 0)]),
    ("erase_sign", [("-beta * ki * kS[j]", "+beta * ki * kS[j]", 0)]),
    ("write_without_beta", [("+ beta * ki * (double)v[j]", "+ ki * (double)v[j]", 0)]),
    ("decay_after_update", [
        ("                    S[(int64_t)i * dv + j] *= decay[i];\n", "                    ;\n", 0),
        ("            /* o_t = S_t^T q_t */",
         "            for (int i = 0; i < dk; ++i) for (int j = 0; j < dv; ++j) S[(int64_t)i * dv + j] *= decay[i];\n"
         "            /* o_t = S_t^T q_t */", 0)]),
    ("output_reads_key", [("const double qi = (double)q[i];", "const double qi = (double)k[i];", 0)]),
    ("output_transposed", [("o[j] += S[(int64_t)i * dv + j] * qi;", "o[j] += S[(int64_t)j * dv + i] * qi;", 0)]),
    ("output_before_update", [
        ("            /* o_t = S_t^T q_t */", "            /* o_t = S_t^T q_t */ if (0)", 0),
        ("            /* S_t = (I - beta k k^T) S_dec + beta k v^T, term by term. */",
         "            for (int j = 0; j < dv; ++j) { o[j] = 0.0; for (int i = 0; i < dk; ++i) o[j] += S[(int64_t)i * dv + j] * (double)q[i]; }\n", 0)]),
    ("gate_sign", [("return g_min / (1.0 + exp(-a));", "return g_min / (1.0 + exp(a));", 0)]),
    ("gate_unscaled", [("return g_min / (1.0 + exp(-a));", "return -1.0 / (1.0 + exp(-a));", 0)]),
    ("decay_inverted", [("decay[i] = exp(gate_f64(", "decay[i] = exp(-gate_f64(", 0)]),
    ("logsigmoid_branch", [("return a - log1p(exp(a));", "return -log1p(exp(a));", 0)]),
    ("initial_state_ignored", [("if (J->S0)\n            memcpy(S, J->S0 + s_off", "if (0)\n            memcpy(S, J->S0 + s_off", 0)]),
    ("chunk_A_without_beta", [("A_rs *= br;", ";", 0)]),
    ("chunk_P_strict", [("for (int s = 0; s <= r; ++s) {", "for (int s = 0; s < r; ++s) {", 0)]),
    ("chunk_state_decay_sign", [("exp(Gl[c] - G[(int64_t)s * dk + c])", "exp(G[(int64_t)s * dk + c] - Gl[c])", 0)]),
    ("chunk_rhs_undecayed", [("const double kb = (double)kr[c] * exp(G[(int64_t)r * dk + c]);", "const double kb = (double)kr[c];", 0)]),
    ("chunk_cumsum_exclusive", [("G[(int64_t)r * dk + c] = (r ? G[(int64_t)(r - 1) * dk + c] : 0.0) + gv;",
                                 "G[(int64_t)r * dk + c] = (r ? G[(int64_t)(r - 1) * dk + c] + gv : 0.0);", 0)]),
    ("chunk_pair_transposed", [("exp(G[(int64_t)r * dk + c] - G[(int64_t)s * dk + c]);\n                    A_rs",
                                "exp(G[(int64_t)s * dk + c] - G[(int64_t)r * dk + c]);\n                    A_rs", 0)]),
    ("tile_col_factor_sign", [("expf(Gf - Gr);", "expf(Gr - Gf);", 0)]),
    ("head_scale_ignored", [("const double scale = exp((double)A_log[h]);", "const double scale = 1.0;", 0)]),
    ("bwd_erase_path_dropped", [("                               - Sd[(int64_t)i * dv + j] * beta * du[j];", "                               ;", 0)]),
    ("bwd_dq_from_previous_state", [("acc += S_t[(int64_t)i * dv + j] * (double)dO[j];", "acc += S_prev[(int64_t)i * dv + j] * (double)dO[j];", 0)]),
    ("bwd_state_grad_undecayed", [("dS[(int64_t)i * dv + j] = decay[i] * d;", "dS[(int64_t)i * dv + j] = d;", 0)]),
    ("bwd_dg_uses_dS", [("dg += d * Sd[(int64_t)i * dv + j];", "dg += dS[(int64_t)i * dv + j] * Sd[(int64_t)i * dv + j];", 0)]),
    ("bwd_dbeta_sign", [("db += du[j] * r[j];", "db -= du[j] * r[j];", 0)]),
    ("bwd_dv_without_beta", [("dvv[j] = beta * du[j];", "dvv[j] = du[j];", 0)]),
    ("bwd_gate_grad_missing_factor", [("return g_min * s * (1.0 - s);", "return g_min * s;", 0)]),
    ("bwd_logsig_grad", [("    return 1.0 - s;\n}", "    return s;\n}", 0)]),
    ("bwd_output_grad_transposed", [("dS[(int64_t)i * dv + j] += (double)q[i] * (double)dO[j];", "dS[(int64_t)i * dv + j] += (double)q[j] * (double)dO[i];", 0)]),
    ("head_scale_wrong_head", [("const double scale = exp((double)A_log[h]);",
                                "const double scale = exp((double)A_log[0]);", 0)]),
]


def _nth_replace(s, old, new, n):
    idx = -1
    for _ in range(n + 1):
        idx = s.index(old, idx + 1)
    return s[:idx] + new + s[idx + len(old):]


@pytest.mark.parametrize("name,edits", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(name, edits, tmp_path):
    src = open(_SRC).read()
    for old, new, n in edits:
        assert src.count(old) > n, f"mutation {name}: pattern not found"
        src = _nth_replace(src, old, new, n)
    mpath = tmp_path / f"{name}.c"
    mpath.write_text(src)
    lib = oracle.load(oracle.build(str(mpath), str(tmp_path / f"lib{name}.so"), extra_flags=("-O1",)))
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
            break
    assert failed, f"planted mistake {name} passed every pin"
