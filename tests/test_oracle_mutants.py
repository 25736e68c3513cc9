"""The oracle's pins must catch plausible mistakes in the oracle.

Each entry below plants one mistake in a copy of the oracle (a dropped term,
a wrong sign or index, a transposed operand, an off-by-one boundary, a tie
broken the other way), on the CPU, in a temporary directory: the committed
oracle is never touched.  The pin file named beside the mistake is then run
against the mutated copy and must fail.  A mistake that every pin lets through
would mean the oracle is pinned only to itself there.

A control run first checks that the unmutated copy passes every pin file, so
that a failure below is the planted mistake and not the harness.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
C = "oracle/lsa_oracle.c"
P = "oracle/__init__.py"
NUM = "test_oracle_numerics.py"
WARD = "test_oracle_ward.py"
SEL = "test_oracle_select_attn.py"
PCA = "test_oracle_pca.py"
BWD = "test_oracle_backward.py"
FP8 = "test_oracle_fp8.py"

# (name, file, original text, mutated text, pin file that must fail)
MUTANTS = [
    # key / query latent (essay ch. 2, tutorial section 二)
    ("latent_not_normalised", C, "z[c] = (nrm > 0.0) ? v[c] / nrm : 0.0;", "z[c] = v[c];", NUM),
    ("latent_W_transposed", C, "bf(x[e]) * (double)W[(int64_t)e * dl + c]",
     "bf(x[e]) * (double)W[(int64_t)c * d + e]", NUM),
    ("pool_divides_by_pool_on_ragged_unit", C, "u[c] = acc[c] / (double)n;",
     "u[c] = acc[c] / (double)pool;", NUM),
    ("pool_renormalised", C, "for (int32_t c = 0; c < dl; ++c) u[c] = acc[c] / (double)n;",
     "{ double q = 0.0; for (int32_t c = 0; c < dl; ++c) q = q + acc[c] * acc[c]; q = sqrt(q);"
     " for (int32_t c = 0; c < dl; ++c) u[c] = q > 0.0 ? acc[c] / q : 0.0; }", NUM),
    ("query_group_strided", C, "latent_of(Q + (t * hq + g * G + i) * (int64_t)d",
     "latent_of(Q + (t * hq + g + i * hkv) * (int64_t)d", NUM),
    ("query_mean_not_divided", C, "lsao_bf16_rne(acc[c] / (double)G)", "lsao_bf16_rne(acc[c])", NUM),
    ("latent_norm_not_square_rooted", C,
     "    double nrm = sqrt(n2);\n    for (int32_t c = 0; c < dl; ++c) z[c] = (nrm > 0.0) ? v[c] / nrm : 0.0;",
     "    double nrm = n2;\n    for (int32_t c = 0; c < dl; ++c) z[c] = (nrm > 0.0) ? v[c] / nrm : 0.0;", NUM),
    # bf16 rounding
    ("bf16_truncates", C, "double r = nearbyint(ldexp(a, -ulp_exp));",
     "double r = floor(ldexp(a, -ulp_exp));", NUM),
    ("bf16_ties_away_from_zero", C, "double r = nearbyint(ldexp(a, -ulp_exp));",
     "double r = round(ldexp(a, -ulp_exp));", NUM),
    # Ward (essay ch. 2; Ward 1963)
    ("ward_no_size_factor", C, "double f = (double)(nA * nB) / (double)(nA + nB);", "double f = 1.0;", WARD),
    ("ward_sums_not_means", C, "double df = sA[c] / (double)nA - sB[c] / (double)nB;",
     "double df = sA[c] - sB[c];", WARD),
    ("ward_cap_off_by_one", C, "if (w->size[a] + w->size[b] > w->max_units) return INFINITY;",
     "if (w->size[a] + w->size[b] >= w->max_units) return INFINITY;", WARD),
    ("ward_naive_tie_to_later_pair", C, "if (dd < d1) { d2 = d1; d1 = dd; ba = a; bb = b; }",
     "if (dd <= d1) { d2 = d1; d1 = dd; ba = a; bb = b; }", WARD),
    ("ward_nn_tie_to_later_pair", C,
     "if (nnd[r] < bd || (nnd[r] == bd && (lo < ba || (lo == ba && hi < bb)))) {",
     "if (nnd[r] <= bd) {", WARD),
    ("ward_buckets_numbered_descending", C,
     "int32_t rank = 0;\n        for (int32_t a = 0; a < n; ++a) {",
     "int32_t rank = 0;\n        for (int32_t a = n - 1; a >= 0; --a) {", WARD),
    ("cluster_sum_skips_first_member", C, "    for (int32_t i = 0; i < w->size[a]; ++i) {",
     "    for (int32_t i = 1; i < w->size[a]; ++i) {", WARD),
    ("merge_loses_a_member", C, "w->size[a] = na + nb;", "w->size[a] = na + nb - 1;", WARD),
    # bucket cache (essay ch. 2-3)
    ("ragged_block_bucket_count_floored", C,
     "int32_t m = (int32_t)(((int64_t)n * bpb + bu - 1) / bu);",
     "int32_t m = (int32_t)(((int64_t)n * bpb) / bu); if (m < 1) m = 1;", WARD),
    ("last_sink_counted_long_range", C,
     "if (p >= sinks) { ++c_lr; if (p < mlr) mlr = (int32_t)p; }",
     "if (p > sinks) { ++c_lr; if (p < mlr) mlr = (int32_t)p; }", SEL),
    ("minlr_is_the_last_key", C,
     "if (p >= sinks) { ++c_lr; if (p < mlr) mlr = (int32_t)p; }",
     "if (p >= sinks) { ++c_lr; mlr = (int32_t)p; }", SEL),
    ("centroid_not_normalised", C,
     "cent[hb * dl + c] = lsao_bf16_rne(nrm > 0.0 ? s[c] / nrm : 0.0);",
     "cent[hb * dl + c] = lsao_bf16_rne(s[c]);", WARD),
    # tree (essay ch. 4)
    ("tree_node_keeps_left_child_only", C,
     "S[node * dl + c] = has_b ? S[a * dl + c] + S[b * dl + c] : S[a * dl + c];",
     "S[node * dl + c] = S[a * dl + c];", SEL),
    ("tree_minlr_is_max", C, "M[node] = (has_b && M[b] < M[a]) ? M[b] : M[a];",
     "M[node] = (has_b && M[b] > M[a]) ? M[b] : M[a];", SEL),
    ("tree_stop_level_off_by_one", C, "((int64_t)1 << Lstar) < k && Lstar < 62) ++Lstar;",
     "((int64_t)1 << Lstar) <= k && Lstar < 62) ++Lstar;", SEL),
    ("tree_leaf_range_one_short", C, "int64_t b0 = bm2[i] << Lstar, b1 = (bm2[i] + 1) << Lstar;",
     "int64_t b0 = bm2[i] << Lstar, b1 = ((bm2[i] + 1) << Lstar) - 1;", SEL),
    ("tree_beam_keeps_one_fewer", C, "int32_t keep = nl < beam ? nl : beam;",
     "int32_t keep = nl < beam ? nl : (beam > 1 ? beam - 1 : 1);", SEL),
    # selection and index assembly (essay ch. 3, 5)
    ("equal_scores_take_higher_id", C, "return (a->id < b->id) ? -1 : (a->id > b->id);",
     "return (a->id > b->id) ? -1 : (a->id < b->id);", SEL),
    ("scores_ranked_ascending", C, "if (a->s > b->s) return -1;\n    if (a->s < b->s) return 1;",
     "if (a->s < b->s) return -1;\n    if (a->s > b->s) return 1;", SEL),
    ("score_reversed_operand_index", C, "s = s + bf(y[i]) * bf(c[i]);",
     "s = s + bf(y[i]) * bf(c[dl - 1 - i]);", SEL),
    ("native_takes_last_head", C, "if (v > best) best = v;", "best = v;", SEL),
    ("native_takes_min_over_heads", C,
     "double best = -INFINITY;\n    for (int32_t g = 0; g < ng; ++g) {\n"
     "        double v = score1(yq + (int64_t)g * dl, c, dl);\n        if (v > best) best = v;",
     "double best = INFINITY;\n    for (int32_t g = 0; g < ng; ++g) {\n"
     "        double v = score1(yq + (int64_t)g * dl, c, dl);\n        if (v < best) best = v;", SEL),
    ("eligibility_off_by_one", C,
     "if ((int64_t)mlr[b] > lim) continue;\n                    cand[ncand].s = node_score(yq, ng, dl, C + b * dl, &nc);\n"
     "                    cand[ncand].id = b;\n                    ++ncand;\n                }\n            } else {",
     "if ((int64_t)mlr[b] >= lim) continue;\n                    cand[ncand].s = node_score(yq, ng, dl, C + b * dl, &nc);\n"
     "                    cand[ncand].id = b;\n                    ++ncand;\n                }\n            } else {", SEL),
    ("long_range_overlaps_window", C, "int64_t lim = t - W;   /* last long-range key position */",
     "int64_t lim = t - W + 1;", SEL),
    ("window_one_short", C, "int64_t w0 = t - W + 1 > S ? t - W + 1 : S;",
     "int64_t w0 = t - W + 2 > S ? t - W + 2 : S;", SEL),
    ("window_excludes_t", C, "for (int64_t p = w0; p <= t; ++p) out[o2++] = (int32_t)p;",
     "for (int64_t p = w0; p < t; ++p) out[o2++] = (int32_t)p;", SEL),
    ("sinks_exclude_t", C, "for (int32_t i = 0; i < S && i <= t; ++i) out[i] = i;",
     "for (int32_t i = 0; i < S && i < t; ++i) out[i] = i;", SEL),
    ("partial_weight_counts_sinks", C, "if (p >= S && p <= lim) ++w;", "if (p <= lim) ++w;", SEL),
    ("truncated_bucket_skipped", C, "int32_t tk = (int32_t)(w < need ? w : need);",
     "if (w > need) continue;\n                int32_t tk = (int32_t)w;", SEL),
    ("truncation_keeps_a_wrong_key", C,
     "if (p >= S && p <= lim) { out[o++] = (int32_t)p; --rem; }",
     "if (p >= S && p <= lim && rem > 1) { out[o++] = (int32_t)p; --rem; }"
     " else if (p >= S && p <= lim) { out[o++] = (int32_t)(lim); --rem; }", SEL),
    # attention (tutorial section 二)
    ("attention_scale_1_over_d", C,
     "double* lg = (double*)malloc(sizeof(double) * (n_idx > 0 ? n_idx : 1));\n    double sc = 1.0 / sqrt((double)d);",
     "double* lg = (double*)malloc(sizeof(double) * (n_idx > 0 ? n_idx : 1));\n    double sc = 1.0 / (double)d;", SEL),
    ("attention_list_of_wrong_group", C,
     "const int32_t* list = idx + (q * hkv + h / G) * (int64_t)n_idx;",
     "const int32_t* list = idx + (q * hkv + h % hkv) * (int64_t)n_idx;", SEL),
    ("attention_kv_head_of_wrong_group", C,
     "const uint16_t* kv = K + ((int64_t)list[i] * hkv + h / G) * d;",
     "const uint16_t* kv = K + ((int64_t)list[i] * hkv + h % hkv) * d;", SEL),
    ("attention_not_normalised", C, "for (int32_t e = 0; e < d; ++e) o[e] = o[e] / den;",
     "for (int32_t e = 0; e < d; ++e) o[e] = o[e];", SEL),
    ("attention_values_from_keys", C,
     "const uint16_t* vv = V + ((int64_t)list[i] * hkv + h / G) * d;",
     "const uint16_t* vv = K + ((int64_t)list[i] * hkv + h / G) * d;", SEL),
    # sparse-attention backward
    ("backward_scale_1_over_d", C,
     "double* o = (double*)malloc(sizeof(double) * d);\n    double sc = 1.0 / sqrt((double)d);",
     "double* o = (double*)malloc(sizeof(double) * d);\n    double sc = 1.0 / (double)d;", BWD),
    ("backward_drops_D", C, "double ds = p[i] * (dp - D);", "double ds = p[i] * dp;", BWD),
    ("backward_dK_unscaled", C, "dK[r + e] = dK[r + e] + (sc * ds) * qv[e];",
     "dK[r + e] = dK[r + e] + ds * qv[e];", BWD),
    ("backward_dQ_unscaled", C, "for (int32_t e = 0; e < d; ++e) dq[e] = sc * dq[e];",
     "for (int32_t e = 0; e < d; ++e) dq[e] = dq[e];", BWD),
    ("backward_dQ_from_values", C, "dq[e] = dq[e] + ds * K[r + e];", "dq[e] = dq[e] + ds * V[r + e];", BWD),
    ("backward_dV_unweighted", C, "dV[r + e] = dV[r + e] + p[i] * gv[e];", "dV[r + e] = dV[r + e] + gv[e];", BWD),
    ("backward_wrong_group", C, "int32_t g = h / G;\n            const int32_t* list",
     "int32_t g = h % hkv;\n            const int32_t* list", BWD),
    ("backward_D_from_gradient_only", C, "for (int32_t e = 0; e < d; ++e) D = D + gv[e] * o[e];",
     "for (int32_t e = 0; e < d; ++e) D = D + gv[e];", BWD),
    # training-free PCA projection
    ("pca_uncentred", P, "    Xc = X - mean\n", "    Xc = X\n", PCA),
    ("pca_mean_over_wrong_count", P, "mean = X.sum(axis=0) / N", "mean = X.sum(axis=0) / (N + 1)", PCA),
    ("pca_smallest_first", P, 'order = np.argsort(-lam, kind="stable")',
     'order = np.argsort(lam, kind="stable")', PCA),
    ("pca_directions_as_rows", P,
     "return np.ascontiguousarray(V[:, :d_latent], dtype=np.float32), lam, V",
     "return np.ascontiguousarray(V.T[:, :d_latent], dtype=np.float32), lam, V", PCA),
    ("pca_sign_flipped", P, "        if V[i, j] < 0:\n", "        if V[i, j] > 0:\n", PCA),
    ("pca_divides_by_n_minus_1", P, "C = (Xc.T @ Xc) / N", "C = (Xc.T @ Xc) / (N - 1)", PCA),
    # FP8 centroid cache (essay ch. 8)
    ("e4m3_ties_away_from_zero", C, "double r = nearbyint(ldexp(a, -ulp_exp)) ;",
     "double r = round(ldexp(a, -ulp_exp)) ;", FP8),
    ("e4m3_exponent_bias_8", C, "int E = ye - 1 + 7;", "int E = ye - 1 + 8;", FP8),
    ("e4m3_subnormal_range_one_short", C, "if (e - 1 < -6) ulp_exp = -9;", "if (e - 1 < -7) ulp_exp = -9;", FP8),
    ("e4m3_no_saturation", C, "if (y > 448.0) y = 448.0;", "if (y > 480.0) y = 480.0;", FP8),
    ("fp8_scale_2_7", C, "ldexp(s[c] / nrm, 8)", "ldexp(s[c] / nrm, 7)", FP8),
    ("fp8_centroid_not_normalised", C, "lsao_e4m3_rne(nrm > 0.0 ? ldexp(s[c] / nrm, 8) : 0.0)",
     "lsao_e4m3_rne(nrm > 0.0 ? ldexp(s[c], 8) : 0.0)", FP8),
    ("fp8_decoded_without_scale", P, "bf16_rne(np.ldexp(e4m3_to_f64(codes), -FP8_SCALE_EXP))",
     "bf16_rne(e4m3_to_f64(codes))", FP8),
]

PIN_FILES = (NUM, WARD, SEL, PCA, BWD, FP8)


def _copy(dst):
    """A copy of the oracle, the input generators and the pin files."""
    skip = shutil.ignore_patterns("*.so", "*.so.tmp*", "__pycache__")
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"), ignore=skip)
    shutil.copytree(os.path.join(ROOT, "synth"), os.path.join(dst, "synth"), ignore=skip)
    os.makedirs(os.path.join(dst, "tests"))
    for f in ("conftest.py",) + PIN_FILES:
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(dst, "tests", f))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), dst)


def _env():
    e = dict(os.environ)
    for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        e[k] = "1"
    e.pop("PYTHONPATH", None)
    return e


def _run(dst, files):
    """Build the copy's oracle, then run the given pin files in the copy.
    Returns (build return code, pytest return code, last output line)."""
    b = subprocess.run([sys.executable, "-c", "import oracle; oracle.build(force=True)"],
                       cwd=dst, env=_env(), capture_output=True, text=True, timeout=300)
    if b.returncode:
        return b.returncode, None, b.stderr.strip().splitlines()[-1:]
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "not gpu"]
                       + [os.path.join("tests", f) for f in files],
                       cwd=dst, env=_env(), capture_output=True, text=True, timeout=900)
    lines = r.stdout.strip().splitlines()
    return 0, r.returncode, [l for l in lines if l.startswith("FAILED")][:1] or lines[-1:]


def _mutant(tmp, m):
    name, f, old, new, pin = m
    dst = os.path.join(tmp, name)
    _copy(dst)
    path = os.path.join(dst, f)
    with open(path) as fh:
        src = fh.read()
    n = src.count(old)
    if n != 1:
        return name, f"the original text occurs {n} times in {f}"
    with open(path, "w") as fh:
        fh.write(src.replace(old, new))
    brc, rc, tail = _run(dst, [pin])
    shutil.rmtree(dst, ignore_errors=True)
    if brc:
        return name, f"mutated oracle does not build: {tail}"
    if rc != 1:  # 1: tests ran and some failed
        return name, f"{pin} did not fail (pytest rc {rc}): {tail}"
    return name, None


def test_unmutated_copy_passes_every_pin(tmp_path):
    _copy(str(tmp_path))
    brc, rc, tail = _run(str(tmp_path), PIN_FILES)
    assert brc == 0 and rc == 0, tail


def test_every_planted_mistake_fails_a_pin(tmp_path):
    assert len({m[0] for m in MUTANTS}) == len(MUTANTS)
    workers = max(2, min(8, os.cpu_count() or 2))
    with ThreadPoolExecutor(workers) as ex:
        res = list(ex.map(lambda m: _mutant(str(tmp_path), m), MUTANTS))
    survivors = [(n, why) for n, why in res if why]
    assert not survivors, survivors
