"""The oracle's pins catch plausible mistakes.

Each case copies the oracle into a temporary directory, plants one mistake
in the copy's C source (a dropped term, a wrong sign, a transposed operand,
a wrong index), and runs the pin suite against the copy in a subprocess.
The suite must fail for every planted mistake and pass for the unmodified
copy.  Nothing here touches the real oracle or any GPU.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

MUTATIONS = {
    "no_softmax_scale": ("s[j] = scale * dot;", "s[j] = dot;"),
    "no_softmax_normalisation": ("o[c] /= l;", "o[c] /= 1.0;"),
    "value_row_index": ("const double* vj = v + IDX4(b, j, h, 0, L, H, d);",
                        "const double* vj = v + IDX4(b, i, h, 0, L, H, d);"),
    "phi_q_transposed": ("acc += qi[a] * Wq[(size_t)a * d + c];",
                         "acc += qi[a] * Wq[(size_t)c * d + a];"),
    "read_state_transposed": ("acc += qp[c] * S[(size_t)c * d + n];",
                              "acc += qp[c] * S[(size_t)n * d + c];"),
    "phi_kv_transposed": ("for (int a = 0; a < d; ++a) acc += xr[a] * W[(size_t)a * d + c];",
                          "for (int a = 0; a < d; ++a) acc += xr[a] * W[(size_t)c * d + a];"),
    "no_key_normalisation": ("if (l2norm) {", "if (0) {"),
    "residual_sign": ("r[(size_t)t * d + n] = vp[(size_t)t * d + n] - acc;",
                      "r[(size_t)t * d + n] = vp[(size_t)t * d + n] + acc;"),
    "residual_dropped": ("r[(size_t)t * d + n] = vp[(size_t)t * d + n] - acc;",
                         "r[(size_t)t * d + n] = vp[(size_t)t * d + n];"),
    "alpha_dropped": ("S[(size_t)c * d + n] = a * S[(size_t)c * d + n] + dS[(size_t)c * d + n];",
                      "S[(size_t)c * d + n] = S[(size_t)c * d + n] + dS[(size_t)c * d + n];"),
    "beta_dropped": ("acc += bt[t] * kp[(size_t)t * d + c] * r[(size_t)t * d + n];",
                     "acc += kp[(size_t)t * d + c] * r[(size_t)t * d + n];"),
    "update_outer_product_transposed": (
        "acc += bt[t] * kp[(size_t)t * d + c] * r[(size_t)t * d + n];",
        "acc += bt[t] * kp[(size_t)t * d + n] * r[(size_t)t * d + c];"),
    "update_on_every_pass": ("if (clean) return arl2_oracle_state_update(",
                             "if (1) return arl2_oracle_state_update("),
    "elementwise_gate_on_value_features": (
        "S[(size_t)c * d + n] = a * S[(size_t)c * d + n] + dS[(size_t)c * d + n];",
        "S[(size_t)c * d + n] = (alpha_per_key ? alpha[((size_t)b * H + h) * d + n] : a)"
        " * S[(size_t)c * d + n] + dS[(size_t)c * d + n];"),
    "elementwise_gate_one_value": ("const double a = alpha_per_key ? alpha[((size_t)b * H + h) * d + c]",
                                   "const double a = alpha_per_key ? alpha[((size_t)b * H + h) * d]"),
    "token_level_reads_frame_state": (
        "for (int c = 0; c < d; ++c) acc += qp[(size_t)i * d + c] * St[(size_t)c * d + n];",
        "for (int c = 0; c < d; ++c) acc += qp[(size_t)i * d + c] * S[(size_t)c * d + n];"),
    "token_level_residual_against_frame_state": (
        "for (int c = 0; c < d; ++c) acc += kp[(size_t)i * d + c] * St[(size_t)c * d + n];",
        "for (int c = 0; c < d; ++c) acc += kp[(size_t)i * d + c] * S[(size_t)c * d + n];"),
    "token_level_gate_every_token": ("if (i == 0) g = alpha_per_key", "if (1) g = alpha_per_key"),
    "gate_alpha_mean_of_sigmoids": ("a_sum += a;", "a_sum += sigmoid(a) - 0.5;"),
    "gate_alpha_sum_not_mean": ("alpha[(size_t)b * H + h] = sigmoid(a_sum / L);",
                                "alpha[(size_t)b * H + h] = sigmoid(a_sum);"),
    "gate_weight_transposed": ("a += xi[e] * w[(size_t)e * 2 * H + h];",
                               "a += xi[e] * w[(size_t)h * D + e];"),
    "gate_beta_bias_dropped": ("double a = bias[h], g = bias[H + h];", "double a = bias[h], g = 0.0;"),
    "gate_alpha_from_beta_column": ("a += xi[e] * w[(size_t)e * 2 * H + h];",
                                    "a += xi[e] * w[(size_t)e * 2 * H + H + h];"),
    "teacher_scale_dropped": ("s[j] = dot * scale;", "s[j] = dot;"),
    "teacher_cached_values_from_keys": ("const double* vj = j < Lc ? vc + IDX4(b, j, h, 0, Lc, H, d)",
                                        "const double* vj = j < Lc ? kc + IDX4(b, j, h, 0, Lc, H, d)"),
    "teacher_cache_stride_of_a_frame": ("const double* kj = j < Lc ? kc + IDX4(b, j, h, 0, Lc, H, d)",
                                        "const double* kj = j < Lc ? kc + IDX4(b, j, h, 0, L, H, d)"),
    "teacher_frame_key_head_dropped": (": k + IDX4(b, j - Lc, h, 0, L, H, d);",
                                       ": k + IDX4(b, j - Lc, 0, 0, L, H, d);"),
    "teacher_normaliser_without_cache": (
        "for (int j = 0; j < n; ++j) {\n        s[j] = exp(s[j] - m);\n        l += s[j];",
        "for (int j = 0; j < n; ++j) {\n        s[j] = exp(s[j] - m);\n        l += j < Lc ? 0.0 : s[j];"),
}


def _run_pins_on_copy(tmp_path, mutation):
    dst = tmp_path / "oracle"
    shutil.copytree(os.path.join(ROOT, "oracle"), dst,
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    src = dst / "arl2_oracle.c"
    text = src.read_text()
    if mutation is not None:
        old, new = mutation
        assert text.count(old) == 1, f"mutation anchor not unique: {old!r}"
        src.write_text(text.replace(old, new))
    env = dict(os.environ)
    env["PYTHONPATH"] = str(tmp_path) + os.pathsep + env.get("PYTHONPATH", "")
    env["OMP_NUM_THREADS"] = "2"
    cmd = [sys.executable, "-c",
           "import sys, pytest; import oracle; assert oracle.__file__.startswith(sys.argv[1]); "
           "sys.exit(pytest.main(['-q', '-x', '-p', 'no:cacheprovider', sys.argv[2]]))",
           str(tmp_path), PINS]
    return subprocess.run(cmd, env=env, cwd=str(tmp_path), capture_output=True, text=True,
                          timeout=300)


def test_unmodified_copy_passes(tmp_path):
    r = _run_pins_on_copy(tmp_path, None)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    r = _run_pins_on_copy(tmp_path, MUTATIONS[name])
    assert r.returncode != 0, f"pins did not catch mutation {name}"
