"""Plants plausible mistakes in a copy of the CPU oracle and checks that the
oracle's pins catch each one. Everything runs on the CPU; the shipped oracle
is never modified."""
import concurrent.futures as cf
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.cpp")
PIN_TESTS = ["tests/test_oracle_layout.py", "tests/test_oracle_quant.py",
             "tests/test_oracle_combine.py", "tests/test_oracle_special_bwd.py",
             "tests/test_oracle_quant_bwd.py"]

# (name, text in oracle.cpp, replacement)
MUTATIONS = [
    ("drop_shared_add",
     "if (shared_x) acc = acc + load16(shared_x",
     "if (false) acc = acc + load16(shared_x"),
    ("const_sign",
     "m = p1 + p2;\n        }\n        float prod", "m = p1 - p2;\n        }\n        float prod"),
    ("const_operand_swapped",
     "float p1 = load16(alpha1, q * h + j, dtype) *\n                     load16(ori_x",
     "float p1 = load16(alpha2, q * h + j, dtype) *\n                     load16(ori_x"),
    ("unstable_segment_order",
     "[](const Pair& a, const Pair& b) { return a.e < b.e; }",
     "[](const Pair& a, const Pair& b) { return a.e < b.e || (a.e == b.e && a.t > b.t); }"),
    ("round_half_away",
     "float r = std::nearbyint(load16(xr, j, dtype) / scale);",
     "float r = std::round(load16(xr, j, dtype) / scale);"),
    ("amax_without_abs",
     "amax = std::max(amax, std::fabs(load16(xr, j, dtype)));",
     "amax = std::max(amax, load16(xr, j, dtype));"),
    ("k_order_reversed",
     "      for (int k = 0; k < K; ++k) {\n        if (pair_problem(row, k, n_ids)) continue;",
     "      for (int k = K - 1; k >= 0; --k) {\n        if (pair_problem(row, k, n_ids)) continue;"),
    ("grad_w_weighted",
     "static_cast<double>(load16(xr, j, dtype));\n        dot += term;",
     "static_cast<double>(load16(xr, j, dtype));\n        dot += w * term;"),
    ("scan_off_by_one",
     "ep_send_counts[e + 1] = ep_send_counts[e] + expert_token_nums[e];",
     "ep_send_counts[e + 1] = ep_send_counts[e] + expert_token_nums[e] + (e == 0);"),
    ("special_weight_dropped",
     "float prod = topk_weights[static_cast<size_t>(t) * K + k] * m;",
     "float prod = id < num_experts ? topk_weights[static_cast<size_t>(t) * K + k] * m : m;"),
    ("mask_ignored_in_layout",
     "      if (!pair_active(mask, mask_ndim, t, k, K)) continue;\n      if (row[k] >= num_experts)",
     "      if (row[k] >= num_experts)"),
    ("int8_roundtrip_skipped",
     "  if (amax == 0.0f) return 0.0f;\n  const float scale = amax / 127.0f;",
     "  if (amax >= 0.0f) return y;\n  const float scale = amax / 127.0f;"),
    ("special_bwd_alpha1_dropped",
     "          acc = acc + c * load16(alpha1, q * h + j, dtype);",
     "          acc = acc + c;"),
    ("special_bwd_v_grad_operand",
     "          gv[q * h + j] += c * load16(alpha2, q * h + j, dtype);",
     "          gv[q * h + j] += c * load16(const_v, q * h + j, dtype);"),
    ("smooth_expert_of_first_k",
     "const int32_t e = topk_idx[static_cast<size_t>(t) * K + k];\n      const float* se",
     "const int32_t e = topk_idx[static_cast<size_t>(t) * K];\n      const float* se"),
    ("smooth_amax_unscaled",
     "        amax = std::max(amax, std::fabs(y[j]));",
     "        amax = std::max(amax, std::fabs(load16(xr, j, dtype)));"),
    ("duplicate_ids_accepted",
     "    if (row[j] == id) return ST_DUP_ID;", "    if (false) return ST_DUP_ID;"),
    ("quant_bwd_roundtrip_dropped",
     "const float d = int8_roundtrip(load16(yr, j, dtype), amax);",
     "const float d = load16(yr, j, dtype);"),
    ("quant_bwd_scale_of_grad_row",
     "const float amax = row_amax(yr, h, dtype);", "const float amax = row_amax(g, h, dtype);"),
]


def _run(mut, tmp):
    name, old, new = mut
    src = open(SRC).read()
    assert src.count(old) == 1, name
    path = os.path.join(tmp, name + ".cpp")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(tmp, name + ".so")
    subprocess.check_call(["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fPIC", "-shared",
                           path, "-o", so])
    env = dict(os.environ, ORACLE_LIB=so)
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        *PIN_TESTS], cwd=ROOT, env=env, capture_output=True, text=True)
    return name, p.returncode


def test_every_planted_mistake_is_caught():
    with tempfile.TemporaryDirectory() as tmp:
        with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 2)) as ex:
            results = list(ex.map(lambda m: _run(m, tmp), MUTATIONS))
    survived = [n for n, rc in results if rc == 0]
    assert not survived, f"pins did not catch: {survived}"
