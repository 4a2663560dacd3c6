"""The oracle's pins catch plausible mistakes in the oracle.

Each mutant below copies the oracle package into a temporary folder, changes
one thing in it (a dropped term, a wrong sign, an index or an off-by-one), and
runs the pin tests (test_oracle_pins.py) against that copy.  The pins must fail
on every mutant and pass on an unchanged copy.  Nothing here touches the CUDA
library; the mistakes are planted in copies of the oracle, on the CPU.

Every mutant's snippet must occur exactly once in the current source, so a
change to the oracle that moves a snippet fails here instead of silently
testing nothing.
"""
import concurrent.futures
import os
import re
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")
C_SRC = "lcx_oracle.c"
PY_SRC = "__init__.py"

# name: (what the mistake is and which passage it breaks, file, [(old, new), ...])
MUTANTS = {
    "theta_exponent": (
        "theta_i = b^(-i/D) instead of b^(-2i/D) (RoPE frequencies, 2.1)", C_SRC,
        [("double theta = pow(base, -2.0 * (double)i / (double)D);",
          "double theta = pow(base, -1.0 * (double)i / (double)D);")]),
    "pi_multiplies": (
        "PI multiplies theta by s instead of dividing (4.2)", C_SRC,
        [("tp = theta / s;", "tp = theta * s;")]),
    "ntk_base_no_exponent": (
        "NTK-aware base b s instead of b s^(D/(D-2)) (5.2)", C_SRC,
        [("double new_base = base * pow(s, (double)D / (double)(D - 2));",
          "double new_base = base * s;")]),
    "ntk_exponent_inverted": (
        "NTK-aware exponent (D-2)/D instead of D/(D-2) (5.2)", C_SRC,
        [("double new_base = base * pow(s, (double)D / (double)(D - 2));",
          "double new_base = base * pow(s, (double)(D - 2) / (double)D);")]),
    "yarn_ramp_roles_swapped": (
        "YaRN interpolates the high-frequency pairs and keeps the low ones (6.2)", C_SRC,
        [("tp = (1.0 - ramp) * (theta / s) + ramp * theta;",
          "tp = ramp * (theta / s) + (1.0 - ramp) * theta;")]),
    "yarn_wavelength_no_2pi": (
        "YaRN wavelength 1/theta instead of 2 pi/theta (6.2)", C_SRC,
        [("double wavelength = 2.0 * ORC_PI_D / theta;", "double wavelength = 1.0 / theta;")]),
    "yarn_ramp_denominator": (
        "YaRN ramp (r - alpha)/beta instead of (r - alpha)/(beta - alpha) (6.2)", C_SRC,
        [("double ramp = (r - alpha) / (beta - alpha);", "double ramp = (r - alpha) / beta;")]),
    "mscale_one_over_t": (
        "attention scale 1/t instead of sqrt(1/t) = 0.1 ln s + 1 (6.3)", C_SRC,
        [("? (0.1 * log(s) + 1.0) : 1.0;", "? (0.1 * log(s) + 1.0) * (0.1 * log(s) + 1.0) : 1.0;")]),
    "mscale_log2": (
        "attention scale with log2 s instead of ln s (6.3)", C_SRC,
        [("? (0.1 * log(s) + 1.0) : 1.0;", "? (0.1 * log2(s) + 1.0) : 1.0;")]),
    "rotation_first_sign": (
        "first rotated component x_p cos + x_q sin (2.2)", C_SRC,
        [("y[p] = ms * (xp * c - xq * sn);", "y[p] = ms * (xp * c + xq * sn);")]),
    "rotation_second_sign": (
        "second rotated component -x_p sin + x_q cos (2.2)", C_SRC,
        [("y[q] = ms * (xp * sn + xq * c);", "y[q] = ms * (-xp * sn + xq * c);")]),
    "rotation_mscale_one_component": (
        "mscale applied to the first component of a pair only (6.3)", C_SRC,
        [("y[q] = ms * (xp * sn + xq * c);", "y[q] = (xp * sn + xq * c);")]),
    "half_pairing_mirrored": (
        "half pairing (i, D-1-i) instead of (i, i + D/2) (2.4)", C_SRC,
        [("int q = (pairing == ORC_PAIR_HALF) ? i + half : 2 * i + 1;",
          "int q = (pairing == ORC_PAIR_HALF) ? D - 1 - i : 2 * i + 1;")]),
    "interleaved_pair_reversed": (
        "interleaved pairing (2i+1, 2i) instead of (2i, 2i+1) (2.1)", C_SRC,
        [("int p = (pairing == ORC_PAIR_HALF) ? i : 2 * i;",
          "int p = (pairing == ORC_PAIR_HALF) ? i : 2 * i + 1;"),
         ("int q = (pairing == ORC_PAIR_HALF) ? i + half : 2 * i + 1;",
          "int q = (pairing == ORC_PAIR_HALF) ? i + half : 2 * i;")]),
    "position_plus_one": (
        "angle (m + 1) theta instead of m theta (2.2)", C_SRC,
        [("double phi = (double)m * (double)table[i];",
          "double phi = (double)(m + 1) * (double)table[i];")]),
    "causal_sees_next_key": (
        "causal mask lets query i see key i + 1 (2.4)", C_SRC,
        [("if (j > i) return 0;", "if (j > i + 1) return 0;")]),
    "causal_hides_diagonal": (
        "causal mask hides the query's own key (2.4)", C_SRC,
        [("if (j > i) return 0;", "if (j >= i) return 0;")]),
    "window_one_too_wide": (
        "sliding window of W + 1 keys (10.1)", C_SRC,
        [("if (i - j < window) return 1;", "if (i - j <= window) return 1;")]),
    "sinks_one_too_many": (
        "S + 1 sink keys (10.2)", C_SRC,
        [("if (j < sinks) return 1;", "if (j <= sinks) return 1;")]),
    "noncausal_hides_future": (
        "attention without the causal mask still hides later keys (2.4)", C_SRC,
        [("if (!causal) return 1;", "if (!causal) return j <= i;")]),
    "sinks_seen_by_earlier_queries": (
        "sink keys visible to queries before them (10.2: sinks are earlier tokens)", C_SRC,
        [("    if (j > i) return 0;\n    if (window <= 0) return 1;",
          "    if (window > 0 && j < sinks) return 1;\n    if (j > i) return 0;\n"
          "    if (window <= 0) return 1;")]),
    "table_truncated": (
        "the fp32 table truncated toward zero instead of rounded to nearest", C_SRC,
        [("table[i] = (float)tp[i];",
          "{ float f_ = (float)tp[i]; if ((double)f_ > tp[i]) f_ = nextafterf(f_, 0.0f); "
          "table[i] = f_; }")]),
    "midpoint_never_flags": (
        "the midpoint flag never set, so a table entry on an fp32 rounding midpoint "
        "would still be compared bit for bit", C_SRC,
        [("return (fabs(v - mid_up) < tol || fabs(v - mid_dn) < tol) ? 1 : 0;",
          "return 0 * ((fabs(v - mid_up) < tol || fabs(v - mid_dn) < tol) ? 1 : 0);")]),
    "midpoint_flags_everything": (
        "the midpoint tolerance far too wide (2^-20), flagging ordinary entries", C_SRC,
        [("double tol = fabs(v) * ldexp(1.0, -40);", "double tol = fabs(v) * ldexp(1.0, -20);")]),
    "gqa_heads_interleaved": (
        "query head h reads kv head h mod Hkv instead of floor(h / G)", C_SRC,
        [("if (row_b[r] == b && row_h[r] / G == g) sel[ns++] = r;",
          "if (row_b[r] == b && row_h[r] % Hkv == g) sel[ns++] = r;")]),
    "key_offset_ignored": (
        "keys rotated at index j instead of position offset + j", C_SRC,
        [("(int)c->D, c->pos_offset + j,", "(int)c->D, j,")]),
    "query_offset_ignored": (
        "queries rotated at index i instead of position offset + i", C_SRC,
        [("rotate_row(x, qr, (int)D, c->pos_offset + i,", "rotate_row(x, qr, (int)D, i,")]),
    "lse_without_max": (
        "lse = ln Z without the row max (online softmax statistics, 8.3.4)", C_SRC,
        [("o[d] /= Z;\n    c->lse[r] = mx + log(Z);\n    free(s);\n}\n\n/*\n * Attention outputs",
          "o[d] /= Z;\n    c->lse[r] = log(Z);\n    free(s);\n}\n\n/*\n * Attention outputs")]),
    "output_not_normalised": (
        "weighted sum of V not divided by the softmax denominator (2.4)", C_SRC,
        [("for (int64_t d = 0; d < D; d++) o[d] /= Z;\n    c->lse[r] = mx + log(Z);",
          "c->lse[r] = mx + log(Z);")]),
    "key_range_start_ignored": (
        "a partial result over keys [k_begin, k_end) that also takes keys before k_begin",
        C_SRC,
        [("if (j < c->k_begin || j >= c->k_end ||", "if (j >= c->k_end ||")]),
    "key_range_end_ignored": (
        "a partial result over keys [k_begin, k_end) that also takes keys from k_end on",
        C_SRC,
        [("if (j < c->k_begin || j >= c->k_end ||", "if (j < c->k_begin ||")]),
    "merge_equal_weights": (
        "merge averages the partial outputs instead of weighting by e^lse (8.3.4)", C_SRC,
        [("double w = exp(l - m);", "double w = 1.0;")]),
    "merge_lse_without_max": (
        "merged lse = ln sum e^(lse_s - m) without adding m back (8.3.4)", C_SRC,
        [("lse[r] = m + log(z);", "lse[r] = log(z);")]),
    "merge_not_normalised": (
        "merged output not divided by the sum of the weights (8.3.4)", C_SRC,
        [("for (int64_t d = 0; d < D; d++) orow[d] /= z;", "")]),
    "dynamic_ntk_rescales_short": (
        "dynamic NTK changes the base for sequences shorter than the training length",
        C_SRC,
        [("double se = (seq_len > L_train) ? (double)seq_len / (double)L_train : 1.0;",
          "double se = (double)seq_len / (double)L_train;")]),
    "dynamic_ntk_as_pi": (
        "dynamic scaling by position interpolation instead of the NTK-aware base", C_SRC,
        [("return orc_rope_theta_fp64(ORC_NTK, D, base, se,",
          "return orc_rope_theta_fp64(ORC_PI, D, base, se,")]),
    "factors_multiply": (
        "per-pair factors multiply theta instead of dividing it (7.3)", C_SRC,
        [("(double)i / (double)D) / lam[i];", "(double)i / (double)D) * lam[i];")]),
    "short_factors_inverted": (
        "the short factor table used for long sequences and the long one for short (7.4)",
        C_SRC,
        [("(factors_short && seq_len <= L_train)", "(factors_short && seq_len > L_train)")]),
    "short_factors_threshold": (
        "the short factor table dropped at seq_len = L_train already (7.4: it holds up to "
        "the training length)", C_SRC,
        [("(factors_short && seq_len <= L_train)", "(factors_short && seq_len < L_train)")]),
    "mla_rope_slice_first": (
        "decoupled RoPE takes q_R from the front of the query row (9.5)", C_SRC,
        [("xr[d] = (double)c->q[r * Dq + c->Dc + d];", "xr[d] = (double)c->q[r * Dq + d];")]),
    "mla_key_without_mscale": (
        "decoupled RoPE rotates the shared key without the attention scale (9.7, 6.3)", C_SRC,
        [("pos_offset + t % L, table, (double)mscale,", "pos_offset + t % L, table, 1.0,")]),
    "mla_key_positions_across_batch": (
        "the shared rotary key of batch b > 0 rotated at b L + j instead of j", C_SRC,
        [("pos_offset + t % L, table,", "pos_offset + t, table,")]),
    "mla_heads_interleaved": (
        "decoupled RoPE: query head h reads kv head h mod Hkv", C_SRC,
        [("const int64_t g = h / (c->Hq / c->Hkv), Dq", "const int64_t g = h % c->Hkv, Dq")]),
    "mla_lse_without_max": (
        "decoupled RoPE: lse without the row max", C_SRC,
        [("o[d] /= Z;\n    c->lse[r] = mx + log(Z);\n    free(s);\n}\n\n/*\n * Attention rows with",
          "o[d] /= Z;\n    c->lse[r] = log(Z);\n    free(s);\n}\n\n/*\n * Attention rows with")]),
    "default_scale_one_over_d": (
        "default score scale 1/D instead of 1/sqrt(D) (2.4)", PY_SRC,
        [("scale = 1.0 / np.sqrt(D)\n", "scale = 1.0 / D\n")]),
    "mla_default_scale_rope_dims": (
        "decoupled RoPE default scale 1/sqrt(d_R) instead of 1/sqrt(d_C + d_R) (9.5)", PY_SRC,
        [("scale = 1.0 / np.sqrt(Dc + Dr)", "scale = 1.0 / np.sqrt(Dr)")]),
}


def _copy_oracle(dst, edits, file):
    pkg = os.path.join(dst, "oracle")
    os.makedirs(pkg)
    for f in (C_SRC, PY_SRC, "build.py"):
        shutil.copy(os.path.join(ROOT, "oracle", f), os.path.join(pkg, f))
    path = os.path.join(pkg, file)
    with open(path, encoding="utf-8") as fh:
        src = fh.read()
    for old, new in edits:
        n = src.count(old)
        if n != 1:
            return "snippet occurs %d times in oracle/%s: %r" % (n, file, old[:60])
        src = src.replace(old, new)
    with open(path, "w", encoding="utf-8") as fh:
        fh.write(src)
    return None


def _run_pins(dst):
    """Build the copy's library, then run the pins against it.  Returns (exit
    code, first failing test, the copy's oracle path as imported)."""
    env = dict(os.environ)
    env["PYTHONPATH"] = os.pathsep.join([dst, ROOT] + [p for p in
                                        env.get("PYTHONPATH", "").split(os.pathsep) if p])
    env["OMP_NUM_THREADS"] = "1"
    where = subprocess.run([sys.executable, "-c",
                            "import oracle, oracle.build as b; b.build(force=True); "
                            "print(oracle.__file__)"],
                           cwd=dst, env=env, capture_output=True, text=True, timeout=300)
    if where.returncode != 0:
        return -1, where.stderr[-400:], None
    r = subprocess.run([sys.executable, "-m", "pytest", PINS, "-x", "-q", "-m", "not gpu",
                        "-p", "no:cacheprovider", "-rf"],
                       cwd=dst, env=env, capture_output=True, text=True, timeout=600)
    failed = re.findall(r"^FAILED (\S+)", r.stdout, re.M)
    return r.returncode, (failed[0] if failed else r.stdout[-400:]), where.stdout.strip()


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    jobs = {"unchanged": ("no change", C_SRC, [])}
    jobs.update(MUTANTS)
    dirs, res = {}, {}
    for name, (_, file, edits) in jobs.items():
        d = str(tmp_path_factory.mktemp(name))
        err = _copy_oracle(d, edits, file)
        if err:
            res[name] = ("bad snippet", err, None)
        else:
            dirs[name] = d
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        futs = {name: ex.submit(_run_pins, d) for name, d in dirs.items()}
        for name, f in futs.items():
            res[name] = f.result() + (dirs[name],)
    return res


def test_unchanged_copy_passes(outcomes):
    rc, detail, imported, dst = outcomes["unchanged"]
    assert imported is not None and imported.startswith(dst), (imported, dst)
    assert rc == 0, detail


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(outcomes, name):
    res = outcomes[name]
    assert res[0] != "bad snippet", res[1]
    rc, detail, imported, dst = res
    assert imported is not None and imported.startswith(dst), (name, imported, detail)
    # 1 = tests failed (a pin caught it); anything else is a harness problem
    assert rc == 1, "pins did not catch %r (%s): rc=%d %s" % (name, MUTANTS[name][0], rc,
                                                              detail)
