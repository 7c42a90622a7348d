"""Plant mistakes in copies of the oracle and require the pins to catch each.

Every mutant is a one-line textual change to a temporary copy of
oracle/moe_oracle.c (never to the file itself), compiled with the same flags
as the real oracle and loaded through oracle.use_library.  A mutant passes the
test only if at least one pin in tests/oracle_pins.py fails on it.  The
unmutated copy, built the same way, must pass every pin.
"""
import os
import subprocess

import pytest

import oracle
import oracle_pins as P
from oracle import build as obuild

SRC = os.path.join(os.path.dirname(obuild.__file__), "moe_oracle.c")

# (name, original text, mistaken text)
MUTANTS = [
    ("sigmoid_sign", "return 1.0 / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(z));"),
    ("silu_drops_z", "return z / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(-z));"),
    ("router_no_accumulate",
     "acc += oracle_bf16_to_f64(xt[i]) * oracle_bf16_to_f64(we[i]);",
     "acc = oracle_bf16_to_f64(xt[i]) * oracle_bf16_to_f64(we[i]);"),
    ("bias_dropped_from_selection", "b[e] = s[e] + (double)c->bias[e];", "b[e] = s[e];"),
    ("weights_from_biased_scores", "if (taken[e]) sum += s[e];", "if (taken[e]) sum += b[e];"),
    ("no_renormalisation", "c->scale * (s[e] / sum)", "c->scale * s[e]"),
    ("no_scaling_factor", "c->scale * (s[e] / sum)", "(s[e] / sum)"),
    ("ties_to_higher_index", "if (best < 0 || b[e] > b[best]) best = e;",
     "if (best < 0 || b[e] >= b[best]) best = e;"),
    ("topk_smallest", "if (best < 0 || b[e] > b[best]) best = e;",
     "if (best < 0 || b[e] < b[best]) best = e;"),
    ("gap_wrong_sign", "c->gap[t] = (k < E) ? (kth - next) : INFINITY;",
     "c->gap[t] = (k < E) ? (next - kth) : INFINITY;"),
    ("gate_up_swapped", "a[n] = oracle_silu(g) * u;", "a[n] = oracle_silu(u) * g;"),
    ("no_silu", "a[n] = oracle_silu(g) * u;", "a[n] = g * u;"),
    ("down_transposed", "acc += oracle_bf16_to_f64(wd[n]) * a[n];",
     "acc += oracle_bf16_to_f64(w_down[(size_t)n * d + o]) * a[n];"),
    ("shared_expert_dropped", "oracle_swiglu_row(xt, c->sgu, c->sdn, d, c->inter, o, NULL);",
     "for (int i = 0; i < d; ++i) o[i] = 0.0;"),
    ("routed_weight_dropped", "for (int i = 0; i < d; ++i) o[i] += w * y[i];",
     "for (int i = 0; i < d; ++i) o[i] += y[i];"),
    ("permute_unstable",
     "        for (int t = 0; t < T; ++t)\n            for (int j = 0; j < k; ++j)\n"
     "                if (topk_idx[(size_t)t * k + j] == e) {",
     "        for (int t = T - 1; t >= 0; --t)\n            for (int j = 0; j < k; ++j)\n"
     "                if (topk_idx[(size_t)t * k + j] == e) {"),
    ("row_token_wrong_index", "row_token[row] = t;", "row_token[row] = j;"),
    ("slot_row_local_rank", "slot_row[(size_t)t * k + j] = row;",
     "slot_row[(size_t)t * k + j] = row - offsets[e];"),
    ("combine_drops_shared", "o[i] = y_shared ? y_shared[(size_t)t * d + i] : 0.0;", "o[i] = 0.0;"),
    ("bf16_truncates", "r = ldexp(rint(ldexp(m, 8)), e - 8);",
     "r = ldexp(trunc(ldexp(m, 8)), e - 8);"),
    ("e4m3_truncates", "double m = rint(ldexp(a, 3 - e));", "double m = trunc(ldexp(a, 3 - e));"),
    ("e4m3_bias_off_by_one", "ldexp(1.0 + man / 8.0, ex - 7)", "ldexp(1.0 + man / 8.0, ex - 8)"),
    ("e4m3_subnormal_step", "const double m = rint(a * 0x1p9);", "const double m = rint(a * 0x1p8);"),
    ("fp8_exponent_one_low", "if (amax > ldexp(448.0, s)) s += 1;",
     "if (amax > ldexp(448.0, s)) s += 0;"),
    ("fp8_scale_applied_twice",
     "q[r * cols + c] = oracle_e4m3_encode(ldexp(oracle_bf16_to_f64(w[r * cols + c]), -s));",
     "q[r * cols + c] = oracle_e4m3_encode(ldexp(oracle_bf16_to_f64(w[r * cols + c]), -2 * s));"),
    ("fp8_dequant_block_transposed", "sexp[(r / 128) * bc + c / 128]",
     "sexp[(r / 128) + (c / 128) * (rows / 128)]"),
    ("bias_update_sign_flipped", "b = b - gamma;                                    /* over-loaded: lower */",
     "b = b + gamma;                                    /* over-loaded: lower */"),
    ("bias_update_truncated_mean",
     "        else if (scaled < total)\n            b = b + gamma;",
     "        else if ((long long)counts[e] < total / E)\n            b = b + gamma;"),
    ("seq_aux_unnormalized", "pb[i] += scores[(size_t)t * E + i] / tot;", "pb[i] += scores[(size_t)t * E + i];"),
    ("seq_aux_no_f_scale", "fb[i] *= (double)E / ((double)k * S);", "fb[i] *= 1.0;"),
    ("fp8c_drops_x_exponent", "g = ldexp(g, s_gu[n] + sx);", "g = ldexp(g, s_gu[n]);"),
    ("fp8c_up_uses_gate_exponent", "u = ldexp(u, s_gu[inter + n] + sx);",
     "u = ldexp(u, s_gu[n] + sx);"),
    ("fp8c_x_exponent_sign", "g = ldexp(g, s_gu[n] + sx);", "g = ldexp(g, s_gu[n] - sx);"),
    ("fp8c_h_not_rounded",
     "h[n] = oracle_bf16_to_f64(oracle_f64_to_bf16(oracle_silu(g) * u));",
     "h[n] = oracle_silu(g) * u;"),
    ("fp8c_down_exponent_dropped", "y[o] = ldexp(acc, s_dn[o] + sh);", "y[o] = ldexp(acc, sh);"),
    ("fp8c_activation_exponent_dropped", "y[o] = ldexp(acc, s_dn[o] + sh);",
     "y[o] = ldexp(acc, s_dn[o]);"),
    ("fp8c_shared_dropped",
     "oracle_swiglu_row_fp8(xt, c->sgq, c->sgs, c->sdq, c->sds, d, c->inter, o);",
     "for (int i = 0; i < d; ++i) o[i] = 0.0;"),
    ("fp8c_expert_by_slot",
     "oracle_swiglu_row_fp8(xt, c->egq[e], c->egs[e], c->edq[e], c->eds[e], d, c->inter, y);",
     "oracle_swiglu_row_fp8(xt, c->egq[j], c->egs[j], c->edq[j], c->eds[j], d, c->inter, y);"),
    ("fp8c_routed_weight_dropped", "for (int i = 0; i < d; ++i) o[i] += y[i] * w;",
     "for (int i = 0; i < d; ++i) o[i] += y[i];"),
    ("int4_scale_over_8", "const uint16_t sb = oracle_f64_to_bf16(amax / 7.0);",
     "const uint16_t sb = oracle_f64_to_bf16(amax / 8.0);"),
    ("int4_truncates", "n = rint(oracle_bf16_to_f64(wg[i]) / sv);",
     "n = trunc(oracle_bf16_to_f64(wg[i]) / sv);"),
    ("int4_signed_max", "const double v = fabs(oracle_bf16_to_f64(wg[i]));",
     "const double v = oracle_bf16_to_f64(wg[i]);"),
    ("int4_scale_transposed", "scale[r * groups + g] = sb;", "scale[g * rows + r] = sb;"),
    ("int4_dequant_wrong_group", "oracle_bf16_to_f64(scale[r * groups + c / 32])",
     "oracle_bf16_to_f64(scale[r * groups + c / 64])"),
    ("fp8_rows_signed_max", "if (fabs(v[i]) > amax) amax = fabs(v[i]);",
     "if (v[i] > amax) amax = v[i];"),
]


def _build_variant(tmpdir, name, text):
    src = os.path.join(tmpdir, f"{name}.c")
    hdr_dir = os.path.dirname(SRC)
    with open(src, "w") as f:
        f.write(text)
    lib = os.path.join(tmpdir, f"lib{name}.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                    "-ffp-contract=off", "-fno-fast-math", "-I", hdr_dir, "-o", lib, src,
                    "-lm"], check=True)
    return lib


def test_unmutated_copy_passes(tmp_path):
    text = open(SRC).read()
    lib = _build_variant(str(tmp_path), "clean", text)
    with oracle.use_library(lib):
        assert P.failing_pins() == []


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site for {name} not unique"
    lib = _build_variant(str(tmp_path), name, text.replace(old, new))
    with oracle.use_library(lib):
        caught = P.failing_pins()
    assert caught, f"no pin catches the planted mistake {name}"
