"""The pins must catch plausible mistakes: each mutant below is a copy of the
oracle with one planted error (a dropped term, a wrong sign or index, a
transposed operand, a wrong mask), built on the CPU and run against the pin
suite in a child process, which must fail."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "top_left_causal": ("return j <= i + (n_kv - n_q);", "return j <= i;"),
    "causal_off_by_one": ("return j <= i + (n_kv - n_q);", "return j < i + (n_kv - n_q);"),
    "no_max_subtraction": ("double e = std::exp(s[j] - m);", "double e = std::exp(s[j]);"),
    "sign_flip": ("double e = std::exp(s[j] - m);", "double e = std::exp(m - s[j]);"),
    "lse_drops_max": ("*lse = m + std::log(l);", "*lse = std::log(l);"),
    "scale_dropped": ("s[j] = scale * dot;", "s[j] = dot;"),
    "dot_drops_last_term": ("for (int c = 0; c < d_k; ++c) dot +=", "for (int c = 0; c + 1 < d_k; ++c) dot +="),
    "no_normalisation": ("for (int c = 0; c < d_v; ++c) o[c] /= l;", ""),
    "v_row_index_wrong": ("const float* v = V + j * d_v;", "const float* v = V + (n_kv - 1 - j) * d_v;"),
    "q_k_swapped_rows": ("const float* k = K + j * d_k;", "const float* k = K + (j % (i + 1)) * d_k;"),
    "window_left_off_by_one": ("if (left >= 0 && j < pos - left) return false;", "if (left >= 0 && j <= pos - left) return false;"),
    "window_right_ignored": ("if (right >= 0 && j > pos + right) return false;", ""),
    "window_position_top_left": ("const int64_t pos = i + (n_kv - n_q);", "const int64_t pos = i;"),
    "gqa_heads_interleaved": ("const int64_t kv = b * H_kv + h / group;", "const int64_t kv = b * H_kv + h % H_kv;"),
    "bwd_drops_jacobian_row_term": ("const double dsij = pij * (dp[(size_t)j] - rowdot);", "const double dsij = pij * dp[(size_t)j];"),
    "bwd_dk_without_scale": ("dKb[kj_slot * d_k + c] += scale * dsij * (double)qi_row[c];", "dKb[kj_slot * d_k + c] += dsij * (double)qi_row[c];"),
    "bwd_dv_uses_transposed_index": ("dVb[kj_slot * d_v + c] += pij * (double)dOi[c];", "dVb[kj_slot * d_v + c] += pij * (double)dOb[(n_q - 1 - i) * d_v + c];"),
    "gqa_v_head_interleaved": ("attend_row(s.data(), V + kv * n_cap * d_v,", "attend_row(s.data(), V + (b * H_kv + h % H_kv) * n_cap * d_v,"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(os.path.join(ROOT, "oracle", "oracle.cpp")).read()
    assert src.count(old) == 1, "mutation site not found: " + name
    (tmp_path / "oracle.cpp").write_text(src.replace(old, new))
    shutil.copy(os.path.join(ROOT, "oracle", "oracle.h"), tmp_path / "oracle.h")
    so = str(tmp_path / "liboracle_mutant.so")
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
                           str(tmp_path / "oracle.cpp"), "-o", so])
    env = dict(os.environ, SDPA_ORACLE_LIBRARY=so)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, "mutant %s passed every pin:\n%s" % (name, r.stdout[-2000:])
