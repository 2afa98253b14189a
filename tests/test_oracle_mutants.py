"""Planted mistakes: each test copies the oracle's C source, plants one
plausible mistake (a dropped term, a wrong sign or index, a transposed
operand, a reversed tie rule), compiles the copy on the CPU and checks that
the pin suite fails on it.  This shows the pins constrain every step of the
oracle, not only the ones they were written for."""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = [os.path.join(ROOT, "tests", "test_oracle_pins.py"),
        os.path.join(ROOT, "tests", "test_oracle_snapkv_pins.py"),
        os.path.join(ROOT, "tests", "test_oracle_sampling_pins.py"),
        os.path.join(ROOT, "tests", "test_oracle_group_pins.py"),
        os.path.join(ROOT, "tests", "test_oracle_vprune_pins.py"),
        os.path.join(ROOT, "tests", "test_oracle_think_pins.py"),
        os.path.join(ROOT, "tests", "test_oracle_topp_pins.py"),
        os.path.join(ROOT, "tests", "test_oracle_pyramid_pins.py")]

MUTANTS = {
    "tie_rule_reversed": ("return (a->j > b->j) - (a->j < b->j);",
                          "return (a->j < b->j) - (a->j > b->j);"),
    "qnorm_one_group_head": ("for (int g = 0; g < G; ++g)\n                for (int t = 0; t < W; ++t)",
                             "for (int g = 0; g < 1; ++g)\n                for (int t = 0; t < W; ++t)"),
    "qnorm_drops_window": ("for (int t = 0; t < W; ++t) {\n                    double x",
                           "for (int t = 0; t < 1; ++t) {\n                    double x"),
    "saliency_no_abs": ("float a = fabsf(k_tj);", "float a = k_tj;"),
    "recovery_no_division": ("? mu / qj : 0.0;", "? mu : 0.0;"),
    "recovery_sign_flip": ("? mu / qj : 0.0;", "? -mu / qj : 0.0;"),
    "stats_over_kept": ("} else {\n                    double x = (double)w[j];",
                        "}\n                {\n                    double x = (double)w[j];"),
    "mean_wrong_denominator": ("? sw / n : 0.0;", "? sw / (n + 1.0) : 0.0;"),
    "keeps_one_less": ("for (int r = 0; r < T; ++r)", "for (int r = 0; r < T - 1; ++r)"),
    "vals_reversed": ("vrow[pos++] = krow[j];", "vrow[T - 1 - pos++] = krow[j];"),
    "score_scale_1_over_D": ("const double scale = 1.0 / sqrt((double)D);\n    for (long bh = 0; bh < BH; ++bh) {\n        oracle_recover_keys(mask",
                             "const double scale = 1.0 / (double)D;\n    for (long bh = 0; bh < BH; ++bh) {\n        oracle_recover_keys(mask"),
    # SnapKV pre-pass (readings R11-R13)
    "snapkv_normaliser_not_causal": ("for (long t = 0; t <= p; ++t)\n                    l += exp(logit[t] - m);",
                                     "for (long t = 0; t < S; ++t)\n                    l += exp(logit[t] - m);"),
    "snapkv_one_head": ("for (int g = 0; g < G; ++g)\n            for (int w = 0; w < W; ++w) {\n                const float *q = q_obs",
                        "for (int g = 0; g < 1; ++g)\n            for (int w = 0; w < W; ++w) {\n                const float *q = q_obs"),
    "snapkv_unnormalised": ("sc[t] += exp(logit[t] - m) / l;", "sc[t] += exp(logit[t] - m);"),
    "snapkv_pool_narrow": ("for (long u = t - h; u <= t + h; ++u)", "for (long u = t - h + 1; u <= t + h; ++u)"),
    "snapkv_ties_reversed": ("return (a->t > b->t) - (a->t < b->t);", "return (a->t < b->t) - (a->t > b->t);"),
    "snapkv_drops_window": ("out[kp + w] = P + w;", "out[kp + w] = P + w - 1;"),
    # sampling recoveries (reading R14)
    "philox_nine_rounds": ("for (int r = 0; r < 10; ++r) {", "for (int r = 0; r < 9; ++r) {"),
    "philox_key_not_bumped": ("k[1] += 0xBB67AE85u;", "k[1] += 0u;"),
    "gaussian_variance_as_sd": ("return mu + sqrt(var) * sqrt(-2.0 * log(u1)) * cos(2.0 * M_PI * u2);",
                                "return mu + var * sqrt(-2.0 * log(u1)) * cos(2.0 * M_PI * u2);"),
    "gaussian_angle_from_radius_draw": ("cos(2.0 * M_PI * u2)", "cos(2.0 * M_PI * u1)"),
    "exponential_unit_mean": ("return -mu * log(u1);", "return -log(u1);"),
    "sampled_key_not_back_solved": ("Kt[t * D + j] = (qj > 0.0) ? w / qj : 0.0;", "Kt[t * D + j] = w;"),
    "gqa_transposed": ("const float *qrow = q + (bh * G + g) * (long)D;",
                       "const float *qrow = q + ((long)g * BH + bh) * (long)D;"),
    "tail_keys_from_values": ("(double)k_tail[(bh * tail_cap + t) * D + j];",
                              "(double)v_tail[(bh * tail_cap + t) * D + j];"),
    # SparK-g (reading R15)
    "group_order_ascending": ("if (a->q > b->q) return -1;\n    if (a->q < b->q) return 1;",
                              "if (a->q < b->q) return -1;\n    if (a->q > b->q) return 1;"),
    "group_norm_ties_reversed": ("return a->j < b->j ? -1 : (a->j > b->j);",
                                 "return a->j > b->j ? -1 : (a->j < b->j);"),
    "group_budget_truncates": ("Tg[k] = (int)llround((1.0 - (double)rates[k]) * (double)size);",
                               "Tg[k] = (int)((1.0 - (double)rates[k]) * (double)size);"),
    "group_budget_of_whole_head": ("Tg[k] = (int)llround((1.0 - (double)rates[k]) * (double)size);",
                                   "Tg[k] = (int)llround((1.0 - (double)rates[k]) * (double)D / 4);"),
    "group_keeps_one_less": ("for (int r = 0; r < Tg[grp] && r < m; ++r)",
                             "for (int r = 0; r < Tg[grp] - 1 && r < m; ++r)"),
    # V-channel pruning (reading R16)
    "values_pruned_not_dropped": ("? (double)vrow[pos++] : 0.0;", "? (double)vrow[pos++] : 1e-3;"),
    "values_index_not_advanced": ("? (double)vrow[pos++] : 0.0;", "? (double)vrow[pos] : 0.0;"),
    # ThinK comparator (reading R18)
    "think_no_query_norm": ("ord[j].s = (double)qn[bh * D + j] * sqrt(ss);", "ord[j].s = sqrt(ss);"),
    "think_sum_not_squared": ("ss += x * x;", "ss += fabs(x);"),
    "think_ties_reversed": ("return (a->j < b->j) ? -1 : ((a->j > b->j) ? 1 : 0);",
                            "return (a->j > b->j) ? -1 : ((a->j < b->j) ? 1 : 0);"),
    "think_recovers_mean": ("stats[bh * 4 + 3] = 0.0;\n    }\n    free(ord);",
                            "stats[bh * 4 + 3] = 1.0;\n    }\n    free(ord);"),
    # SparK-p (reading R19)
    "topp_reach_strict": ("while (n < D && cum < target) {", "while (n < D && cum <= target) {"),
    "topp_p_ignored": ("const double target = (double)p * total;", "const double target = total;"),
    "topp_fp32_cumulative": ("            double cum = 0.0;\n", "            float cum = 0.0f;\n"),
    "topp_channel_order": ("                cum += (double)order[n].w;", "                cum += (double)w[n];"),
    "topp_cap_off_by_one": ("const int n_keep = n < Tcap ? n : Tcap;", "const int n_keep = n < Tcap ? n : Tcap - 1;"),
    "topp_padding_not_zero": ("vrow[r] = 0.0f;", "vrow[r] = 1.0f;"),
    # PyramidKV budgets (reading R20)
    "pyramid_increasing": ("frac = 1.0 - 2.0 * (double)l / (double)(L - 1);",
                           "frac = 2.0 * (double)l / (double)(L - 1) - 1.0;"),
    "pyramid_denominator_L": ("frac = 1.0 - 2.0 * (double)l / (double)(L - 1);",
                              "frac = 1.0 - 2.0 * (double)l / (double)L;"),
    "pyramid_truncates": ("long r = (long)floor(fabs(x) + 0.5);", "long r = (long)floor(fabs(x));"),
    "lambda_truncates": ("return (int)llround((1.0 - (double)lambda) * (double)D);",
                         "return (int)((1.0 - (double)lambda) * (double)D);"),
}


def _run_mutant(name, workdir):
    """Build the oracle with one planted mistake and run the pin suite on it;
    returns (pin-suite exit code, the tail of its output)."""
    before, after = MUTANTS[name]
    src = open(os.path.join(ROOT, "oracle", "spark_oracle.c")).read()
    if src.count(before) != 1:
        return None, f"mutation site for {name} not unique"
    d = os.path.join(workdir, name)
    os.makedirs(d, exist_ok=True)
    mutant_c = os.path.join(d, "mutant.c")
    with open(mutant_c, "w") as f:
        f.write(src.replace(before, after))
    lib = oracle.build(force=True, src=mutant_c, out=os.path.join(d, "libmutant.so"))
    env = dict(os.environ, ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    """All mutants at once, one pin-suite process per mutant on the host's
    cores (each builds its own copy of the oracle)."""
    import concurrent.futures as cf
    work = str(tmp_path_factory.mktemp("mutants"))
    workers = max(1, min(len(MUTANTS), os.cpu_count() or 1))
    with cf.ThreadPoolExecutor(max_workers=workers) as ex:
        futs = {name: ex.submit(_run_mutant, name, work) for name in MUTANTS}
        return {name: f.result() for name, f in futs.items()}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(mutant_results, name):
    rc, out = mutant_results[name]
    assert rc is not None, out
    assert rc != 0, f"pins did not catch mutant {name}:\n{out}"
