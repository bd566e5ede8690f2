"""The oracle's pins catch planted mistakes.

Each case copies oracle.c, plants one plausible mistake in the copy (a dropped
scale, a flipped sign, a transposed operand, an off-by-one mask, a dropped term),
builds it with gcc into a temporary library and runs the pin tests against it
in a child process.  The pins must fail for every mutant.  Nothing here touches
the real oracle build.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "dk_scale_dropped": ("dk[(size_t)j * d + x] = c->scale * acc;", "dk[(size_t)j * d + x] = acc;"),
    "ds_sign_flipped": ("(dP[(size_t)i * Nk + j] - D[i])", "(D[i] - dP[(size_t)i * Nk + j])"),
    "causal_off_by_one": ("if ((sp->flags & ORACLE_CAUSAL) && j > i + off) return 0;",
                          "if ((sp->flags & ORACLE_CAUSAL) && j >= i + off) return 0;"),
    "dv_operand_transposed": ("acc += P[(size_t)i * Nk + j] * dout[(size_t)i * d + x];",
                              "acc += P[(size_t)j * Nk + i] * dout[(size_t)i * d + x];"),
    "lse_max_dropped": ("double lse = m + log(l);", "double lse = log(l);"),
    "mask_index_transposed": ("!sp->mask[(size_t)(i / sp->blk) * sp->nbk + (j / sp->blk)]",
                              "!sp->mask[(size_t)(j / sp->blk) * sp->nbk + (i / sp->blk)]"),
    "scale_dropped_in_scores": ("srow[j] = scale * acc + bias(sp, h, i, j);", "srow[j] = acc + bias(sp, h, i, j);"),
    # extended modes (Nq != Nk, sliding window, ALiBi)
    "alignment_offset_dropped": ("const long off = (long)sp->Nk - sp->Nq;", "const long off = 0;"),
    "window_left_off_by_one": ("if (sp->left >= 0 && j < i + off - sp->left) return 0;",
                               "if (sp->left >= 0 && j <= i + off - sp->left) return 0;"),
    "window_right_ignored": ("if (sp->right >= 0 && j > i + off + sp->right) return 0;", ""),
    "alibi_sign_flipped": ("return -sp->slopes[h % sp->H] * dist;", "return sp->slopes[h % sp->H] * dist;"),
    "alibi_offset_dropped": ("const double dist = fabs((double)i + ((double)sp->Nk - sp->Nq) - (double)j);",
                             "const double dist = fabs((double)i - (double)j);"),
    "alibi_head_ignored": ("return -sp->slopes[h % sp->H] * dist;", "return -sp->slopes[0] * dist;"),
    # the remaining products and statistics of the definition, the online recurrence, the sampled path
    "dq_scale_dropped": ("dq[(size_t)i * d + x] = c->scale * acc;", "dq[(size_t)i * d + x] = acc;"),
    "delta_dropped": ("D[i] = acc;", "D[i] = 0.0;"),
    "o_wrong_value_row": ("acc += P[(size_t)i * Nk + j] * v[(size_t)j * d + x];",
                          "acc += P[(size_t)i * Nk + j] * v[(size_t)(Nk - 1 - j) * d + x];"),
    "p_normalisation_dropped": ("for (int j = 0; j < N; ++j) srow[j] = exp(srow[j] - lse);",
                                "for (int j = 0; j < N; ++j) srow[j] = exp(srow[j] - m);"),
    "online_sum_rescale_dropped": ("            l *= corr;\n", ""),
    "sampled_cols_wrong_lse_row": ("double p = exp(c->scale * s + bias(&c->sp, h, i, j) - lse[i]);",
                                   "double p = exp(c->scale * s + bias(&c->sp, h, i, j) - lse[0]);"),
    "sampled_cols_dv_uses_ds": ("dvj[x] += p * dout", "dvj[x] += ds * dout"),
    "sampled_rows_ds_sign_flipped": ("double ds = prow[j] * (dp - D);", "double ds = prow[j] * (D - dp);"),
    "sampled_rows_dq_scale_dropped": ("for (int x = 0; x < d; ++x) dqi[x] *= c->scale;", ""),
    "empty_row_made_uniform": ("for (int j = 0; j < N; ++j) srow[j] = 0.0;",
                               "for (int j = 0; j < N; ++j) srow[j] = 1.0 / N;"),
}

# FP8 forward (E4M3, rotation, block quantiser, FP8 attention): checked by its own pins
FP8_MUTANTS = {
    "e4m3_bias_off_by_one": ("else v = ldexp(1.0 + m / 8.0, e - 7);", "else v = ldexp(1.0 + m / 8.0, e - 6);"),
    "e4m3_ties_to_odd": ("(dd == bd && (c & 1) == 0)", "(dd == bd && (c & 1) == 1)"),
    "rotation_butterfly_sign": ("x[c + h] = a - b;", "x[c + h] = b - a;"),
    "quantiser_scale_inverted": ("const float inv = amax > 0.0f ? 448.0f / amax : 1.0f;",
                                 "const float inv = amax > 0.0f ? amax / 448.0f : 1.0f;"),
    "fp8_v_scale_dropped": ("const double f = (double)c->sv[h] / l8;", "const double f = 1.0 / l8;"),
    "fp8_key_scale_uses_query_block": ("(double)c->sk[h * nb + j / c->rows]", "(double)c->sk[h * nb + i / c->rows]"),
    "rotation_normalisation_dropped": ("for (int c = 0; c < d; ++c) x[c] = x[c] * r;", ""),
    "fp8_p_left_unrounded": ("p8[j] = c->quant_p ? oracle_e4m3_value(oracle_e4m3_round(pj)) : pj;", "p8[j] = pj;"),
    "fp8_o_normalised_by_unrounded_sum": ("const double f = (double)c->sv[h] / l8;",
                                          "const double f = (double)c->sv[h] / l;"),
    "quantiser_amax_of_first_row_only": ("for (size_t e = 0; e < n; ++e) amax = fmaxf(amax, fabsf(t[e]));",
                                         "for (size_t e = 0; e < (size_t)d; ++e) amax = fmaxf(amax, fabsf(t[e]));"),
    "e4m3_overflow_to_nan": ("if (a >= 448.0) return s | 0x7e;", "if (a >= 448.0) return s | 0x7f;"),
    "rotation_signs_not_applied": ("for (int c = 0; c < d; ++c) x[c] = x[c] * signs[c];", ""),
    "fp8_p_rounded_before_the_max": (
        "p8[j] = c->quant_p ? oracle_e4m3_value(oracle_e4m3_round(pj)) : pj;",
        "p8[j] = c->quant_p ? oracle_e4m3_value(oracle_e4m3_round(exp(s[j]))) * exp(-m) : pj;"),
}

PIN_FILES = ["test_oracle_pins.py", "test_oracle_modes.py"]
FP8_PIN_FILES = ["test_oracle_fp8.py"]
ALL = sorted(MUTANTS) + sorted(FP8_MUTANTS)


@pytest.fixture(scope="module")
def mutant_runs(tmp_path_factory):
    """Builds every mutant and runs its pins, all mutants at once (child
    processes); returns {name: (returncode, tail of the output)}."""
    src = open(SRC).read()
    procs = {}
    for name in ALL:
        old, new = MUTANTS[name] if name in MUTANTS else FP8_MUTANTS[name]
        files = PIN_FILES if name in MUTANTS else FP8_PIN_FILES
        assert src.count(old) >= 1, f"mutation anchor not found for {name}"
        d = tmp_path_factory.mktemp(name)
        cfile = d / "oracle_mut.c"
        cfile.write_text(src.replace(old, new))
        lib = d / "liboracle_mut.so"
        subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-I", os.path.join(ROOT, "oracle"),
                        "-o", str(lib), str(cfile), "-lm", "-lpthread"], check=True)
        # a few oracle threads per child: the children run side by side
        env = dict(os.environ, ORACLE_LIB=str(lib), ORACLE_THREADS="2")
        procs[name] = subprocess.Popen([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                                        *[os.path.join(ROOT, "tests", f) for f in files]],
                                       cwd=ROOT, env=env, stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                       text=True)
    out = {}
    for name, pr in procs.items():
        text, _ = pr.communicate(timeout=900)
        out[name] = (pr.returncode, text[-2000:])
    return out


@pytest.mark.parametrize("name", ALL)
def test_pins_catch_mutant(name, mutant_runs):
    rc, tail = mutant_runs[name]
    assert rc != 0, f"mutant {name} survived the pins:\n{tail}"
