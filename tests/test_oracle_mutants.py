"""Plant plausible mistakes in copies of the oracle and check that its pins
(tests/test_oracle.py) reject every one of them.  Runs on the CPU only."""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "hils_oracle.c")

MUTANTS = {
    "summary_without_scale": ("z[j] = tau * dot_fd(lq, kc + j * d, d);", "z[j] = dot_fd(lq, kc + j * d, d);"),
    "entropy_sign_flipped": ("bp[bh * nc + c] = lse - pz;", "bp[bh * nc + c] = pz - lse;"),
    "score_without_bias": ("(c < own) ? tau * dot_fdd(q, kp + (bh * nc + c) * d, d) + bp[bh * nc + c]",
                           "(c < own) ? tau * dot_fdd(q, kp + (bh * nc + c) * d, d)"),
    "select_without_bias": ("cand[c].s = tau * dot_fdd(q, kp + (bh * nc + c) * d, d) + bp[bh * nc + c];",
                            "cand[c].s = tau * dot_fdd(q, kp + (bh * nc + c) * d, d);"),
    "fusion_without_bias": ("(score_mode == 0) ? tau * dot_fdd(qs, kp + (bh * nc + c) * d, d) + bp[bh * nc + c]",
                            "(score_mode == 0) ? tau * dot_fdd(qs, kp + (bh * nc + c) * d, d)"),
    "fusion_surrogate_unscaled": ("(score_mode == 0) ? tau * dot_fdd(", "(score_mode == 0) ? dot_fdd("),
    "compressed_key_wrong_index": ("out[t] += p * (double)kc[j * d + t];", "out[t] += p * (double)kc[t * d + j % d];"),
    "causal_mask_off_by_one": ("w0, i + 1, d, tau", "w0, i, d, tau"),
    "kv_head_mapping_modulo": ("const int64_t bh = (int64_t)rb[r] * D->Hkv + rhq[r] / G;\n    const int64_t i = rpos[r]",
                               "const int64_t bh = (int64_t)rb[r] * D->Hkv + rhq[r] % D->Hkv;\n    const int64_t i = rpos[r]"),
    "select_ascending": ("if (a->s > b->s) return -1;\n  if (a->s < b->s) return 1;",
                         "if (a->s < b->s) return -1;\n  if (a->s > b->s) return 1;"),
    "own_chunk_is_candidate": ("const int64_t n_cand = n_candidates(D, rpos[r]);",
                               "const int64_t n_cand = n_candidates(D, rpos[r]) + 1;"),
    "window_starts_a_chunk_late": ("int64_t w0 = (own - (window_chunks(D) - 1)) * C;",
                                   "int64_t w0 = (own - (window_chunks(D) - 2)) * C;"),
    "window_candidates_overlap": ("const int64_t n = i / D->C - (window_chunks(D) - 1);",
                                  "const int64_t n = i / D->C - (window_chunks(D) - 2);"),
    "fusion_uniform_weights": ("const double w = exp(u[t] - M) / Z;", "const double w = 1.0 / (double)m_used;"),
    "fusion_drops_own_chunk": ("u[m_used] = lo;", "u[m_used] = -INFINITY;"),
    "qcal_not_residual": ("double acc = (double)x[t];", "double acc = 0.0;"),
    "qcal_up_transposed": ("acc += (double)Wu[t * r + a] * z[a];", "acc += (double)Wu[a * d + t] * z[a];"),
    "qcal_down_transposed": ("acc += (double)Wd[a * d + t] * (double)x[t];",
                             "acc += (double)Wd[t * r + a] * (double)x[t];"),
    "qcal_one_head_for_all": ("const float* Wd = w_down + (int64_t)rhq[row] * r * d;", "const float* Wd = w_down;"),
    "fusion_ignores_scoring_query": ("const float* qs = qscore ? qscore + r * d : q;", "const float* qs = q;"),
    "select_ties_to_higher_id": ("if (a->s < b->s) return 1;\n  return (a->c < b->c) ? -1 : (a->c > b->c);",
                                 "if (a->s < b->s) return 1;\n  return (a->c > b->c) ? -1 : (a->c < b->c);"),
    "summary_of_the_next_chunk": ("const float* kc = K + (bh * D->N + c * C) * d;",
                                  "const float* kc = K + (bh * D->N + ((c + 1) % (D->N / C)) * C) * d;"),
    "compressed_key_unnormalised": ("const double p = exp(z[j] - m) / Z;", "const double p = exp(z[j] - m);"),
    "chunk_values_are_keys": ("attend_keys(q, Kbh, Vbh, c * C, (c + 1) * C, d, tau, s, oc + m_used * d);",
                              "attend_keys(q, Kbh, Kbh, c * C, (c + 1) * C, d, tau, s, oc + m_used * d);"),
    "chunk_attention_drops_first_key": ("attend_keys(q, Kbh, Vbh, c * C, (c + 1) * C, d, tau, s, oc + m_used * d);",
                                        "attend_keys(q, Kbh, Vbh, c * C + 1, (c + 1) * C, d, tau, s, oc + m_used * d);"),
    "attention_logits_unscaled": ("s[j - j0] = tau * dot_fd(q, Kbh + j * d, d);",
                                  "s[j - j0] = dot_fd(q, Kbh + j * d, d);"),
}

# mistakes in the backward pass, rejected by tests/test_oracle_backward.py
BWD_MUTANTS = {
    "bwd_no_compressed_key_gradient": ("dkp[(bh * nc + cc) * d + t] += tau * du * (double)qs[t];",
                                       "dkp[(bh * nc + cc) * d + t] += 0.0;"),
    "bwd_no_bias_gradient": ("dbp[bh * nc + cc] += du;", "dbp[bh * nc + cc] += 0.0;"),
    "bwd_window_without_score_term": ("if (br[c].chunk < 0) dz += du * pj;", "(void)du;"),
    "bwd_entropy_sign": ("const double dz = pj * proj - dbpc * pj * (zl[j] - zbar);",
                         "const double dz = pj * proj + dbpc * pj * (zl[j] - zbar);"),
    "bwd_summary_value_path": ("dkj[t] += tau * dz * (double)lq[t] + pj * dkpc[t];",
                               "dkj[t] += tau * dz * (double)lq[t];"),
    "bwd_score_uses_attention_query": ("dqs[t] += tau * du * kp[(bh * nc + cc) * d + t];",
                                       "dqs[t] += tau * du * (double)Kbh[cc * C * d + t];"),
    "bwd_value_weight_unfused": ("dvj[t] += a * pj * (double)gr[t];", "dvj[t] += pj * (double)gr[t];"),
    "bwd_softmax_without_row_term": ("double dz = a * pj * (dP - X);", "double dz = a * pj * dP;"),
    "bwd_fusion_without_output_term": ("const double du = a * (X - Dg);", "const double du = a * X;"),
    "bwd_query_gradient_unscaled": ("dq[t] += tau * dz * (double)Kbh[j * d + t];",
                                    "dq[t] += dz * (double)Kbh[j * d + t];"),
    "bwd_landmark_gradient_from_the_summary": ("dlq[t] += tau * dz * (double)kc[j * d + t];",
                                               "dlq[t] += tau * dz * kpc[t];"),
}


def run_pins_on_mutant(old, new, pin_file):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not unique: {old[:60]}"
    with tempfile.TemporaryDirectory() as tmp:
        cfile = os.path.join(tmp, "mutant.c")
        lib = os.path.join(tmp, "libmutant.so")
        open(cfile, "w").write(src.replace(old, new))
        subprocess.check_call(["gcc", "-O1", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-std=c11",
                               cfile, "-o", lib, "-lm"])
        env = dict(os.environ, HILS_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
        r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                            os.path.join(ROOT, "tests", pin_file)],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
        return r


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name):
    r = run_pins_on_mutant(*MUTANTS[name], "test_oracle.py")
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_backward_pins_reject_mutant(name):
    r = run_pins_on_mutant(*BWD_MUTANTS[name], "test_oracle_backward.py")
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
