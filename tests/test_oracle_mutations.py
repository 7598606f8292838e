"""Planted mistakes: each mutation below plants one plausible bug in a copy of
the CPU oracle (on the CPU, never in the CUDA path) and checks that at least
one pin of tests/test_oracle_pins.py catches it.  This is the evidence that the
pins constrain every part of the oracle they claim to."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "hqmq_oracle.c")
PINS = "tests/test_oracle_pins.py"

MUTATIONS = [
    # (id, original text, planted text, pins expected to fail)
    ("hamilton_sign", "double x = a[0] * b[1] + a[1] * b[0] + a[2] * b[3] - a[3] * b[2];",
     "double x = a[0] * b[1] + a[1] * b[0] - a[2] * b[3] + a[3] * b[2];",
     ["test_hamilton_defining_relations"]),
    ("codeword_term_order", "t = a0 * b1; t = t + a1 * b0; t = t + a2 * b3; t = t - a3 * b2; c[1] = t;",
     "t = a0 * b1; t = t + a1 * b0; t = t - a2 * b3; t = t + a3 * b2; c[1] = t;",
     ["test_codeword_f32_is_the_rounded_product", "test_search_matches_independent_brute_force"]),
    ("2t_half_sign", "q[c] = ((m >> c) & 1) ? -0.5 : 0.5;", "q[c] = ((m >> (c ^ 1)) & 1) ? -0.5 : 0.5;",
     ["test_2t_enumeration_convention"]),
    ("median_rank", "uint32_t k = keys[n / 2 - 1];", "uint32_t k = keys[n / 2];",
     ["test_lower_median_worked_example", "test_median_matches_numpy_partition"]),
    ("ties_to_highest", "if (sc > best) { second = best; best = sc; bi = i; }",
     "if (sc >= best) { second = best; best = sc; bi = i; }",
     ["test_ties_go_to_lowest_index"]),
    ("pack_msb_first", "idx |= ((w[bit / 32] >> (bit % 32)) & 1u) << i;",
     "idx |= ((w[bit / 32] >> (bit % 32)) & 1u) << (b - 1 - i);",
     ["test_packing_worked_example_b8", "test_packing_worked_example_b10"]),
    ("box_muller_angle", "double th0 = two_pi * u[1];", "double th0 = 3.141592653589793 * u[1];",
     ["test_codebook_is_haar_uniform_on_s3"]),
    ("philox_swap", "uint32_t n0 = hi_b ^ c1 ^ k0;", "uint32_t n0 = hi_a ^ c1 ^ k0;",
     ["test_philox4x32_10_known_answers"]),
    ("f16_truncate", "double q = rint((m - 1.0) * 1024.0);", "double q = floor((m - 1.0) * 1024.0);",
     ["test_f16_matches_numpy_round_to_nearest_even"]),
    ("norm_drop_term", "r2 = fmaf(x[3], x[3], r2);", "r2 = r2;",
     ["test_chunk_norm_error_bound"]),
    ("outlier_keeps_value", "if (r > *thr_h) { c[0] = c[1] = c[2] = c[3] = 0.0f; return 1; }",
     "if (r > *thr_h) { return 1; }",
     ["test_extract_finds_planted_outliers_in_order"]),
    ("decode_drops_radius", "for (int i = 0; i < 4; ++i) acc[4 * j + i] = r * c[i];",
     "for (int i = 0; i < 4; ++i) acc[4 * j + i] = c[i];",
     ["test_decode_is_radius_times_codeword"]),
    # the near-tie arbiter (score of a given codeword, best / second) and the
    # sampled encode used by the full-size parity checks
    ("score_wrong_head", "out[q] = oracle_score(c, codebook + (size_t)h * S * 4, S, idx[q]);",
     "out[q] = oracle_score(c, codebook, S, idx[q]);",
     ["test_score_chunks_matches_independent_fp64_scores"]),
    ("score_secondary_zero", "oracle_codeword_f32((int)(idx % 24u), qs_head + (size_t)(idx / 24u) * 4, c);",
     "oracle_codeword_f32((int)(idx % 24u), qs_head, c);",
     ["test_score_chunks_matches_independent_fp64_scores"]),
    ("score_returns_best", "    return dot4_f32(u, c);\n}",
     "    float bb = -INFINITY;\n"
     "    for (uint32_t i2 = 0; i2 < 24u * S; ++i2) {\n"
     "        float c2[4];\n"
     "        oracle_codeword_f32((int)(i2 % 24u), qs_head + (size_t)(i2 / 24u) * 4, c2);\n"
     "        float v2 = dot4_f32(u, c2);\n"
     "        if (v2 > bb) bb = v2;\n"
     "    }\n"
     "    (void)c;\n"
     "    return bb;\n}",
     ["test_score_chunks_matches_independent_fp64_scores"]),
    ("score_skips_zeroing", "load_chunk(x, dtype, j, thr ? thr + h : NULL, gran, c);\n        out[q]",
     "load_chunk(x, dtype, j, NULL, gran, c);\n        out[q]",
     ["test_score_chunks_matches_independent_fp64_scores"]),
    ("second_not_tracked", "else if (sc > second) second = sc;", ";",
     ["test_best_and_second_are_the_top_two_scores"]),
    ("chunks_head0", "if (h != cur_h) { build_table(codebook + (size_t)h * S * 4, S, table); cur_h = h; }",
     "if (h != cur_h) { build_table(codebook, S, table); cur_h = h; }",
     ["test_encode_chunks_equals_the_whole_call_encode"]),
    ("chunks_skip_zeroing",
     "load_chunk(x, dtype, j, thr ? thr + h : NULL, gran, c);\n        float r, bs, sc;\n"
     "        uint32_t idx = search_chunk(c, table, S",
     "load_chunk(x, dtype, j, NULL, gran, c);\n        float r, bs, sc;\n"
     "        uint32_t idx = search_chunk(c, table, S",
     ["test_encode_chunks_equals_the_whole_call_encode"]),
    # the joint (index, radius level) code and the outlier flags
    ("joint_most_significant_first", "                v += d * p;\n", "                v = v * m + d;\n",
     ["test_pack_equals_the_big_integer_definition"], "tests/test_oracle_joint.py"),
    ("joint_base_L", "uint64_t m = (uint64_t)(24u * S) * (uint64_t)(24u * S);   /* L^2 */",
     "uint64_t m = (uint64_t)(24u * S);   /* L^2 */",
     ["test_block_size_is_the_largest_that_fits_64_bits"], "tests/test_oracle_joint.py"),
    ("flags_msb_first", "if (j < n_chunks) flags[j / 32] |= 1u << (j % 32);",
     "if (j < n_chunks) flags[j / 32] |= 1u << (31 - j % 32);",
     ["test_flags_are_the_list_as_a_bitmap"], "tests/test_oracle_joint.py"),
    ("qradius_rounds_down", "float t = q + 0.5f;", "float t = q;",
     ["test_level_is_the_nearest_grid_point"], "tests/test_oracle_qradius.py"),
    ("qradius_levels_pow2", "uint32_t b = oracle_index_bits(S), L = 24u * S;\n    float *acc",
     "uint32_t b = oracle_index_bits(S), L = 1u << oracle_index_bits(S);\n    float *acc",
     ["test_decode_on_the_grid_equals_the_fp16_radius_decode"], "tests/test_oracle_qradius.py"),
]
MUTATIONS = [m if len(m) == 5 else m + (PINS,) for m in MUTATIONS]


@pytest.mark.parametrize("mid,old,new,pins,pin_file", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(tmp_path, mid, old, new, pins, pin_file):
    src = open(SRC).read()
    assert src.count(old) == 1, mid
    mutant = tmp_path / ("mut_%s.c" % mid)
    mutant.write_text(src.replace(old, new))
    so = tmp_path / ("libmut_%s.so" % mid)
    sys.path.insert(0, ROOT)
    from oracle import hqmq_oracle
    subprocess.check_call(["gcc", *hqmq_oracle.CFLAGS, "-o", str(so), str(mutant), "-lm"])
    env = dict(os.environ, HQMQ_ORACLE_LIB=str(so))
    sel = " or ".join(pins)
    r = subprocess.run([sys.executable, "-m", "pytest", pin_file, "-q", "-x", "-k", sel, "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert "passed" in r.stdout or "failed" in r.stdout, r.stdout + r.stderr
    assert r.returncode != 0, "mutation %s was not caught:\n%s" % (mid, r.stdout[-2000:])
