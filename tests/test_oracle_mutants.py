"""Plant one mistake at a time in a copy of the oracle source and check that the pins
catch it (CPU only). The mistakes are the plausible ones: a flipped sign, a dropped term,
a wrong index or operand, an off-by-one mask, a wrong scale."""
import os

import pytest

import oracle
import oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "diffattn_oracle.c")

MUTANTS = {
    "subtract_sign": ("double w = a1[j] - lam * a2[j];", "double w = a1[j] + lam * a2[j];"),
    "branch2_reads_k1": ("a2[j] = dot(q2, k2 + (long)j * ks, d)", "a2[j] = dot(q2, k1 + (long)j * ks, d)"),
    "scale_1_over_d": ("double inv_sqrt_d = 1.0 / sqrt((double)d);\n  for (int j = 0; j < n_keys",
                       "double inv_sqrt_d = 1.0 / (double)d;\n  for (int j = 0; j < n_keys"),
    "causal_off_by_one_v1": ("int hi = jb->causal ? i + (jb->Nk - N) : jb->Nk - 1; /* last visible key */\n    int lo = (jb->causal && jb->window > 0 && hi - jb->window + 1 > 0) ? hi - jb->window + 1 : 0;\n    double* o = jb->out + (((long)b * n_rows + r) * H",
                             "int hi = jb->causal ? i - 1 + (jb->Nk - N) : jb->Nk - 1; /* last visible key */\n    int lo = (jb->causal && jb->window > 0 && hi - jb->window + 1 > 0) ? hi - jb->window + 1 : 0;\n    double* o = jb->out + (((long)b * n_rows + r) * H"),
    "causal_off_by_one_v2": ("int hi = jb->causal ? i + (jb->Nk - N) : jb->Nk - 1; /* last visible key */\n    int lo = (jb->causal && jb->window > 0 && hi - jb->window + 1 > 0) ? hi - jb->window + 1 : 0;\n    double* o = jb->out + (((long)b * n_rows + r) * P",
                             "int hi = jb->causal ? i - 1 + (jb->Nk - N) : jb->Nk - 1; /* last visible key */\n    int lo = (jb->causal && jb->window > 0 && hi - jb->window + 1 > 0) ? hi - jb->window + 1 : 0;\n    double* o = jb->out + (((long)b * n_rows + r) * P"),
    "chunk_offset_dropped_v1": ("int hi = jb->causal ? i + (jb->Nk - N) : jb->Nk - 1; /* last visible key */\n    int lo = (jb->causal && jb->window > 0 && hi - jb->window + 1 > 0) ? hi - jb->window + 1 : 0;\n    double* o = jb->out + (((long)b * n_rows + r) * H",
                                "int hi = jb->causal ? i : jb->Nk - 1; /* last visible key */\n    int lo = (jb->causal && jb->window > 0 && hi - jb->window + 1 > 0) ? hi - jb->window + 1 : 0;\n    double* o = jb->out + (((long)b * n_rows + r) * H"),
    "window_off_by_one_v1": ("int lo = (jb->causal && jb->window > 0 && hi - jb->window + 1 > 0) ? hi - jb->window + 1 : 0;\n    double* o = jb->out + (((long)b * n_rows + r) * H",
                             "int lo = (jb->causal && jb->window > 0 && hi - jb->window > 0) ? hi - jb->window : 0;\n    double* o = jb->out + (((long)b * n_rows + r) * H"),
    "window_ignored_v2": ("int lo = (jb->causal && jb->window > 0 && hi - jb->window + 1 > 0) ? hi - jb->window + 1 : 0;\n    double* o = jb->out + (((long)b * n_rows + r) * P",
                          "int lo = 0;\n    double* o = jb->out + (((long)b * n_rows + r) * P"),
    "branch2_no_softmax": ("softmax_row(a2, n_keys);", ""),
    "norm_drops_scale": ("o[c] = o[c] / r * (1.0 - lambda_init);", "o[c] = o[c] / r;"),
    "norm_drops_eps": ("double r = sqrt(ss / (double)n + eps);", "double r = sqrt(ss / (double)n);"),
    "norm_mean_over_half": ("double r = sqrt(ss / (double)n + eps);", "double r = sqrt(ss / (double)(n / 2) + eps);"),
    "lambda_init_sign": ("lambda_out[h] = exp(d1) - exp(d2) + li;", "lambda_out[h] = exp(d1) - exp(d2) - li;"),
    "lambda_cross_pairing": ("d2 += lq2[(long)h * dim + c] * lk2[(long)h * dim + c];",
                             "d2 += lq2[(long)h * dim + c] * lk1[(long)h * dim + c];"),
    "lambda_init_rate": ("return 0.8 - 0.6 * exp(-0.3 * (double)(depth - 1));",
                         "return 0.8 - 0.6 * exp(-0.3 * (double)depth);"),
    "lambda_init_rate_constant": ("return 0.8 - 0.6 * exp(-0.3 * (double)(depth - 1));",
                                  "return 0.8 - 0.6 * exp(-0.25 * (double)(depth - 1));"),
    "lambda_init_amplitude": ("return 0.8 - 0.6 * exp(-0.3 * (double)(depth - 1));",
                              "return 0.8 - 0.5 * exp(-0.3 * (double)(depth - 1));"),
    "v1_q2_is_q1": ("const double* q2 = q1 + d;\n    int hi = jb->causal", "const double* q2 = q1;\n    int hi = jb->causal"),
    "v1_decode_q2_is_q1": ("const double* q2 = q1 + d;\n  int n_keys = jb->kv_len", "const double* q2 = q1;\n  int n_keys = jb->kv_len"),
    "v1_value_of_other_head": ("const double* vb = jb->v + (long)b * jb->Nk * tok_v + (long)h * dv;",
                               "const double* vb = jb->v + (long)b * jb->Nk * tok_v + (long)((h + 1) % H) * dv;"),
    "v2_gqa_modulo": ("int g1 = h1 / group, g2 = h2 / group;\n  long tok_q",
                      "int g1 = h1 % jb->Hkv, g2 = h2 % jb->Hkv;\n  long tok_q"),
    "v2_pairing_halves": ("int h1 = 2 * p, h2 = 2 * p + 1;\n  int g1 = h1 / group, g2 = h2 / group;\n  long tok_q",
                          "int h1 = p, h2 = p + P;\n  int g1 = h1 / group, g2 = h2 / group;\n  long tok_q"),
    "decode_drops_last_key": ("int n_keys = jb->kv_len ? jb->kv_len[b] : L;\n  double* o = jb->out + ((long)b * P + p) * d;",
                              "int n_keys = jb->kv_len ? jb->kv_len[b] - 1 : L;\n  double* o = jb->out + ((long)b * P + p) * d;"),
    "v1_decode_drops_last_key": ("int n_keys = jb->kv_len ? jb->kv_len[b] : L;\n  double* o = jb->out + ((long)b * H + h) * dv;",
                                 "int n_keys = jb->kv_len ? jb->kv_len[b] - 1 : L;\n  double* o = jb->out + ((long)b * H + h) * dv;"),
    "v1_decode_branch2_reads_k1": ("diff_row(q1, q2, kb, kb + d, tok_k, vb, tok_v",
                                   "diff_row(q1, q2, kb, kb, tok_k, vb, tok_v"),
    "v1_decode_drops_norm": ("  if (jb->apply_norm) rmsnorm_scale(o, dv, jb->eps, jb->lambda_init);\n}\n\nint oracle_decode_v1",
                             "}\n\nint oracle_decode_v1"),
    "v1_decode_key_of_other_head": ("const double* kb = jb->k + (long)b * L * tok_k + (long)h * 2 * d;",
                                    "const double* kb = jb->k + (long)b * L * tok_k + (long)((h + 1) % H) * 2 * d;"),
    "value_channel_shift": ("for (int c = 0; c < dv; ++c) o[c] += w * vj[c];",
                               "for (int c = 0; c < dv; ++c) o[c] += w * vj[(c + 1) % dv];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/found"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = oracle.compile_source(str(path), str(tmp_path / f"lib_{name}.so"))
    caught = None
    with oracle.use_library(lib):
        for pin in P.ALL_PINS:
            try:
                pin()
            except (AssertionError, ValueError) as e:
                caught = f"{pin.__name__}: {e}"
                break
    assert caught is not None, f"no pin caught mutant {name}"
