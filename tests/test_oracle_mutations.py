"""The oracle's pins catch planted mistakes.

Each case copies the oracle into a scratch directory, plants one mistake in its C source (a
generator constant, a sign, a dropped term, a tie rule, a scale factor, a bit position), builds
it there and runs the pin suite against it: every planted mistake must make a pin fail (pytest
exit status 1, a failed test, not a build or collection error).  CPU only.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = "gradient_quantization_communication_b200"

# (name, text of the oracle that is replaced, replacement)
MUTATIONS = [
    ("philox_multiplier", "0xD2511F53u", "0xD2511F55u"),
    ("philox_key_bump", "k1 += 0xBB67AE85u;", "k1 += 0xBB67AE84u;"),
    ("orq_variance_sign", "tot += (__int128)(b - pos[i]) * (__int128)(pos[i] - a);",
     "tot += (__int128)(b - pos[i]) * (__int128)(pos[i] + a);"),
    ("orq_bracket_edge", "while (k + 2 < nl && lv[k + 1] <= c) ++k;", "while (k + 2 < nl && lv[k + 1] < c) ++k;"),
    ("orq_tie_rule", "if (best_c < 0 || v < best_v) {", "if (best_c < 0 || v <= best_v) {"),
    ("orq_probability", "float p = sat01((u[i] - a) * rinv);", "float p = sat01((b - u[i]) * rinv);"),
    ("qsgd_half_span", "float h = (float)(s - 1) * 0.5f;", "float h = (float)(s - 1) * 0.25f;"),
    ("qsgd_level_ratio", "return (float)(2 * code - (s - 1)) / (float)(s - 1);",
     "return (float)(2 * code - (s - 1)) / (float)(s);"),
    ("bingrad_b_dropped_term", "double j = l * l / (double)k + r * r / (double)(n - k);",
     "double j = l * l / (double)k + r * r;"),
    ("bingrad_b_equal_values", "if (!(srt[k - 1] < srt[k])) continue;", "if (0) continue;"),
    ("bingrad_pb_clamp_term", "if (x < a) e += (__int128)(a - x) * (a - x);", "if (x < a) e += (__int128)(a - x);"),
    ("bingrad_pb_inner_term", "else e += (__int128)(b - x) * (x - a);", "else e += (__int128)(b - x) * (b - x);"),
    ("clip_mean", "double var = (double)sxx / (double)n - mean * mean;", "double var = (double)sxx / (double)n;"),
    ("grid_step", "gi->step = range / 63.0f;", "gi->step = range / 64.0f;"),
    ("average_scale", "or_message_layout(cfg, &bytes, &coff, &loff);\n    float inv_w = 1.0f / (float)nmsgs;",
     "or_message_layout(cfg, &bytes, &coff, &loff);\n    float inv_w = 1.0f / (float)(nmsgs + 1);"),
    ("tg_layer_average_scale", "int64_t words = (int64_t)d * 2 / 32;\n    float inv_w = 1.0f / (float)nmsgs;",
     "int64_t words = (int64_t)d * 2 / 32;\n    float inv_w = 1.0f / (float)(nmsgs + 1);"),
    ("residual_sign", "r[base + i] = v[i] - q[i];", "r[base + i] = q[i] - v[i];"),
    ("uniform_bits", "if (len > 24) word &= ~((1u << (len - 24)) - 1u);", "if (len > 23) word &= ~((1u << (len - 23)) - 1u);"),
    ("pack_padding", "memset(words, 0, sizeof(uint32_t) * (size_t)(d * b / 32));",
     "memset(words, 0xff, sizeof(uint32_t) * (size_t)(d * b / 32));"),
    ("pack_bit_order", "if ((code[e] >> j) & 1) words[k / 32] |= 1u << (k % 32);",
     "if ((code[e] >> j) & 1) words[k / 32] |= 1u << (31 - k % 32);"),
    ("bingrad_b_tie_rule", "if (best < 0 || j > best_j) {", "if (best < 0 || j >= best_j) {"),
    ("bingrad_pb_tie_rule", "if (bestA < 0 || e < best_e) {", "if (bestA < 0 || e <= best_e) {"),
    ("bingrad_pb_lower_limit", "*Amax = am;", "*Amax = OR_GRIDPTS - 2;"),
    ("bingrad_pb_upper_limit", "if (gi->grid[j] >= b) bm = j;", "if (gi->grid[j] >= a) bm = j;"),
    ("quant_error_term", "e += P * dh * dh + (1.0 - P) * dl * dl;", "e += P * dh * dh + P * dl * dl;"),
    ("entropy_digit_order", "for (int k = g - 1; k >= 0; --k) {", "for (int k = 0; k < g; ++k) {"),
    ("entropy_group_bits", "case 9: *g = 5; *B = 16; return 1;", "case 9: *g = 5; *B = 17; return 1;"),
    ("entropy_unpack_radix", "v /= (uint32_t)s;", "v /= (uint32_t)(s + 1);"),
    ("qsgd_nearest_tie", "up = p >= 0.5f;", "up = p > 0.5f;"),
    ("sign_zero_up", "int up = u[i] >= 0.0f;", "int up = u[i] > 0.0f;"),
    ("sign_mean_divisor", "return (float)(ldexp((double)S, -E) / (double)n);",
     "return (float)(ldexp((double)S, -E) / (double)(n + 1));"),
    ("sign_table_order", "table[0] = -m1;", "table[0] = m1;"),
    ("elias_zigzag", "return z >= 0 ? (uint32_t)(2 * z + 1) : (uint32_t)(-2 * z);",
     "return z >= 0 ? (uint32_t)(2 * z + 1) : (uint32_t)(-2 * z + 1);"),
    ("elias_bit_order", "for (int j = N; j >= 0; --j, ++k)", "for (int j = 0; j <= N; ++j, ++k)"),
    ("elias_offsets", "offs[bk] = k;", "offs[bk] = k + 1;"),
    ("l2_sqrt", "return (float)ldexp(sqrt((double)sxx), -e);", "return (float)ldexp((double)sxx, -e);"),
    ("tg_layer_segment_edge", "while (t + 1 < nseg && off[t + 1] <= i) ++t;",
     "while (t + 1 < nseg && off[t + 1] < i) ++t;"),
    ("tg_layer_scale_range", "for (int64_t i = off[t]; i < off[t + 1]; ++i) {",
     "for (int64_t i = off[t]; i + 1 < off[t + 1]; ++i) {"),
    ("tg_layer_no_draw", "(uint32_t)worker, i);\n            int c = k + (U < p ? 1 : 0);",
     "(uint32_t)worker, i);\n            int c = k + (p >= 0.5f ? 1 : 0);"),
    ("fused_bucket_sum", "for (int i = 0; i < n; ++i) acc[i] = acc[i] + q[i];",
     "for (int i = 0; i < n; ++i) acc[i] = acc[i] + v[i];"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new):
    src = open(os.path.join(ROOT, "oracle", "gq_oracle.c")).read()
    assert src.count(old) == 1, "anchor of %s not found once in the oracle" % name
    ignore = shutil.ignore_patterns("*.so", "__pycache__")
    shutil.copytree(os.path.join(ROOT, "oracle"), tmp_path / "oracle", ignore=ignore)
    shutil.copytree(os.path.join(ROOT, "tests"), tmp_path / "tests", ignore=ignore)
    os.makedirs(tmp_path / PKG)
    for f in ("__init__.py", "gq.py", "synth.py", "build.py"):
        shutil.copy2(os.path.join(ROOT, PKG, f), tmp_path / PKG / f)
    shutil.copy2(os.path.join(ROOT, "pytest.ini"), tmp_path / "pytest.ini")
    (tmp_path / "oracle" / "gq_oracle.c").write_text(src.replace(old, new))
    env = dict(os.environ, GQ_SKIP_CUDA_BUILD="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-q", "-x"], cwd=tmp_path,
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 1, "%s survived the pins (exit %d):\n%s" % (name, r.returncode, r.stdout[-3000:])
