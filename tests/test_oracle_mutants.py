"""Mutation check of the oracle pins (no GPU).

Each case plants one plausible mistake in a private copy of the oracle's C source (a
dropped term, a wrong sign, slot, index or bound), builds it, runs the pin suite against
the mutant and requires at least one pin to fail.  The mistakes are planted in the oracle
only, on the CPU; the real oracle is untouched.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "hcl_oracle.c")

MUTANTS = {
    "csa_window_not_overlapped": ("long first = overlap ? (long)m * (i - 1) : (long)m * i;",
                                  "long first = overlap ? (long)m * i : (long)m * i;"),
    "softmax_sign_flipped": ("double e = exp(z - zmax);", "double e = exp(zmax - z);"),
    "bias_slots_reversed": ("double z = or_bf16_to_f64(g[(b * L + t) * d + ch]) + (double)bias[j];\n"
                            "                    double e",
                            "double z = or_bf16_to_f64(g[(b * L + t) * d + ch]) + (double)bias[span - 1 - j];\n"
                            "                    double e"),
    "relu_dropped": ("(dot > 0.0 ? dot : 0.0)", "dot"),
    "visibility_off_by_one": ("long v = (p + 1) / m;", "long v = (p + 2) / m;"),
    "topk_ties_to_higher_index": ("return (a->i < b->i) ? -1 : (a->i > b->i);",
                                  "return (a->i > b->i) ? -1 : (a->i < b->i);"),
    "attn_scale_dropped": ("z[j] = scale * dot;", "z[j] = dot;"),
    "window_one_too_long": ("long lo = p - W + 1;", "long lo = p - W;"),
    "window_excludes_current": ("for (long t = lo; t <= p; t++, n++)", "for (long t = lo; t < p; t++, n++)"),
    "lse_missing_max": ("*lse = zmax + log(den);", "*lse = log(den);"),
    "sink_ignored": ("double den = has_sink ? exp(sink - zmax) : 0.0;", "double den = 0.0;"),
    "index_key_batch_ignored": ("index_vec(fmt, kI, kI_sf, b * Nc + i, dI, k);",
                                "index_vec(fmt, kI, kI_sf, i, dI, k);"),
    "head_weight_index_transposed": ("acc += (double)w[row * HI + h]", "acc += (double)w[h * B + (row % B)]"),
    "fp8_scale_wrong_max": ("amax / 448.0f", "amax / 240.0f"),
    "e4m3_subnormal_quantum": ("double r = nearbyint(ldexp(a, 9));", "double r = nearbyint(ldexp(a, 10));"),
    "e2m1_ties_to_odd": ("(dlt == bestd && (c & 1) == 0)", "(dlt == bestd && (c & 1) == 1)"),
    "mxfp4_exponent_off": ("ilogb(amax) - 2", "ilogb(amax) - 1"),
    # (Swapping the nibble order in the decoder alone is an equivalent mutant: it permutes
    # q_I and k_I alike inside each pair, so every dot product is unchanged.)
    "mxfp4_pack_order": ("(uint8_t)(lo | (hi << 4))", "(uint8_t)(hi | (lo << 4))"),
    "bf16_round_truncates": ("double r = nearbyint(ldexp(a, -qexp));", "double r = floor(ldexp(a, -qexp));"),
    "split_row_scale_dropped": ("out[c] = or_e4m3_to_f64(n[c]) * sc;", "out[c] = or_e4m3_to_f64(n[c]);"),
    "ring_slot_ignored": ("long slot = b * kv->cap + (t % kv->cap);", "long slot = b * kv->cap + t;"),
    "hca_uses_overlap_visibility": ("long nvis = or_num_visible(q_pos[row], mh, Nh);",
                                    "long nvis = or_num_visible(q_pos[row] + mh, mh, Nh);"),
    "value_weights_unnormalised": ("double p = exp(z[j] - zmax) / den;", "double p = exp(z[j] - zmax);"),
    "compress_pools_gate_not_value": ("num += e * or_bf16_to_f64(x[(b * L + t) * d + ch]);",
                                      "num += e * or_bf16_to_f64(g[(b * L + t) * d + ch]);"),
    "compress_unnormalised": ("o[ch] = (den > 0.0) ? num / den : 0.0;", "o[ch] = num;"),
    "compress_bias_dropped": (" + (double)bias[j];", ";"),
    "index_abs_instead_of_relu": ("(dot > 0.0 ? dot : 0.0)", "(dot > 0.0 ? dot : -dot)"),
    "visibility_counts_incomplete_entry": ("long v = (p + 1) / m;", "long v = (p + m) / m;"),
    "topk_output_in_score_order": ("qsort(out, take, sizeof(int), by_index);", "(void)by_index;"),
    "topk_takes_lowest_scores": ("if (a->s > b->s) return -1;\n    if (a->s < b->s) return 1;",
                                 "if (a->s > b->s) return 1;\n    if (a->s < b->s) return -1;"),
    "topk_pads_with_zero": ("for (long j = take; j < k; j++) out[j] = -1;",
                            "for (long j = take; j < k; j++) out[j] = 0;"),
    "csa_drops_last_selected": ("for (int j = 0; j < k; j++) {\n                    int e = idx[row * k + j];",
                                "for (int j = 0; j < k - 1; j++) {\n                    int e = idx[row * k + j];"),
    "hca_drops_last_visible": ("for (long i = 0; i < nvis; i++, n++) {", "for (long i = 1; i < nvis; i++, n++) {"),
    "fp8_rope_half_from_nope_dims": ("rope[r * h + c] = x[h + c];", "rope[r * h + c] = x[c];"),
    "fp8_amax_over_all_dims": ("for (int c = 0; c < h; c++) {\n            float v = fabsf(",
                               "for (int c = 0; c < 2 * h; c++) {\n            float v = fabsf("),
    "mxfp4_amax_signed": ("double a = fabs(or_bf16_to_f64(v[c]));", "double a = or_bf16_to_f64(v[c]);"),
    "rmsnorm_eps_outside_sqrt": ("double inv = 1.0 / sqrt(ss / d + eps);",
                                 "double inv = 1.0 / (sqrt(ss / d) + eps);"),
    "rmsnorm_sum_not_mean": ("double inv = 1.0 / sqrt(ss / d + eps);", "double inv = 1.0 / sqrt(ss + eps);"),
    "rmsnorm_gamma_ignored": ("(gamma ? (double)gamma[c] : 1.0)", "1.0"),
}


def _run_mutant(name, workdir):
    """Build the oracle with mutant `name` planted and run the pin suite against it; returns
    (pytest exit code, end of its output)."""
    old, new = MUTANTS[name]
    src = open(SRC).read()
    if src.count(old) < 1:
        return None, f"mutation site for {name} not found"
    csrc = os.path.join(workdir, name + ".c")
    with open(csrc, "w") as fh:
        fh.write(src.replace(old, new))
    so = os.path.join(workdir, "lib" + name + ".so")
    from oracle.build import build_oracle
    build_oracle(force=True, src=csrc, out=so)
    env = dict(os.environ, HCL_ORACLE_LIB=so, PYTHONPATH=ROOT, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    """Every mutant's pin run, several at a time (each run is a separate process)."""
    sys.path.insert(0, ROOT)
    workdir = str(tmp_path_factory.mktemp("mutants"))
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        futs = {name: ex.submit(_run_mutant, name, workdir) for name in sorted(MUTANTS)}
        return {name: f.result() for name, f in futs.items()}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, mutant_results):
    code, out = mutant_results[name]
    assert code is not None, out
    assert code != 0, f"no pin caught mutant {name}:\n{out}"
