"""The oracle's pins must catch plausible mistakes (CPU only).

Each case plants one mistake in a temporary copy of the oracle source (a
dropped term, a wrong sign, index or offset, a broken convention), builds it
into a separate library, and runs the pin suite against that library in a
child process. The suite must fail for every mutant. The committed oracle
itself is never modified.
"""
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "mla_oracle.cpp")

# (name, [(original text, replacement)]) -- every original must occur exactly once.
MUTANTS = [
    ("drop_rope_term", [("for (int i = 0; i < dr; ++i) dot += bf16_value(qv[dn + i]) * bf16_value(kpe[i]);", "")]),
    ("no_softmax_scale", [("z[a] = p->scale * dot;", "z[a] = dot;")]),
    ("causal_off_by_one", [("t <= s) mark[t] = 1;", "t < s) mark[t] = 1;")]),
    ("causal_only_off_by_one", [("for (int t = 0; t <= s; ++t) sel[n].push_back(t);\n      continue;",
                                 "for (int t = 0; t < s; ++t) sel[n].push_back(t);\n      continue;")]),
    ("value_reads_key_half", [("static_cast<size_t>(b * T + A[a]) * per_head + dn;",
                               "static_cast<size_t>(b * T + A[a]) * per_head;")]),
    ("wrong_head_stride", [("static_cast<int64_t>(h) * per_head + r, j);", "static_cast<int64_t>(h) * dn + r, j);")]),
    ("q_rope_reads_nope", [("bf16_value(qv[dn + i]) * bf16_value(kpe[i])", "bf16_value(qv[i]) * bf16_value(kpe[i])")]),
    ("softmax_sign", [("w[a] = std::exp(z[a] - m);", "w[a] = std::exp(m - z[a]);")]),
    ("missing_normalisation", [("for (int d = 0; d < dv; ++d) o[d] /= l;", "")]),
    ("duplicates_counted", [("mark[t] = 1;  // index mask", "mark[t] += 1;  // index mask"),
                            ("if (mark[t]) sel[n].push_back(t);",
                             "for (int c = 0; c < mark[t]; ++c) sel[n].push_back(t);")]),
    ("out_of_range_wraps", [("if (t >= 0 && t < T && t <= s) mark[t] = 1;",
                             "if (t <= s) mark[((t % T) + T) % T] = 1;")]),
    ("wo_row_reversed", [("const double ak = rows_in[static_cast<size_t>(n) * K + k];",
                          "const double ak = rows_in[static_cast<size_t>(n) * K + K - 1 - k];")]),
    ("e4m3_bias", [("ex - 7);", "ex - 8);")]),
    ("e4m3_subnormal_exponent", [("static_cast<double>(man) / 8.0, -6);", "static_cast<double>(man) / 8.0, -7);")]),
    ("bf16_shift", [("static_cast<uint32_t>(bits) << 16;", "static_cast<uint32_t>(bits) << 15;")]),
    ("fp8_scale_transposed", [("sc[(r / 128) * sc_cols + (c / 128)]", "sc[(c / 128) % sc_cols + (r / 128) % 2]")]),
    ("empty_row_not_zero", [("if (A.empty()) continue;  // no surviving key: attn = 0", "")]),
    # dynamic FP8 activations
    ("act_scale_447", [("const float s = amax / 448.0f;", "const float s = amax / 447.0f;")]),
    ("act_ties_away", [("double v = std::nearbyint(a / quantum) * quantum;",
                        "double v = std::round(a / quantum) * quantum;")]),
    ("act_no_saturation", [("if (v > 448.0) v = 448.0;", "")]),
    ("act_subnormal_quantum", [("if (e < -6) e = -6;", "if (e < -7) e = -7;")]),
    ("act_group_64", [("const int w = n - g < 128 ? n - g : 128;", "const int w = n - g < 64 ? n - g : 64;"),
                      ("for (int g = 0; g < n; g += 128) {", "for (int g = 0; g < n; g += 64) {")]),
    ("act_latent_not_quantized", [("  if (!p->act_e4m3) {\n    for (int j = 0; j < L; ++j) out[j] = bf16_value(lat[j]);",
                                   "  if (true) {\n    for (int j = 0; j < L; ++j) out[j] = bf16_value(lat[j]);")]),
    ("act_attn_not_rounded", [("xb[k] = static_cast<float>(bf16_value(bf16_bits_nearest(a[k])));",
                               "xb[k] = static_cast<float>(a[k]);")]),
    ("bf16_round_quantum", [("const double quantum = std::ldexp(1.0, e - 7);",
                             "const double quantum = std::ldexp(1.0, e - 8);")]),
]


def _build_mutant(tmp, name, edits):
    src = open(SRC).read()
    for old, new in edits:
        assert src.count(old) == 1, f"{name}: pattern not unique/present: {old!r}"
        src = src.replace(old, new)
    cpp = os.path.join(tmp, f"{name}.cpp")
    so = os.path.join(tmp, f"{name}.so")
    with open(cpp, "w") as f:
        f.write(src)
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-fPIC", "-shared", "-o", so, cpp])
    return so


def _run_pins(so):
    env = dict(os.environ, MLA_ORACLE_LIB=so)
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
           os.path.join(ROOT, "tests", "test_oracle_pins.py"), "-k", "not weight_shapes"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode


# Scratch for the mutant builds, inside the repository's ignored build folder.
SCRATCH = os.path.join(ROOT, "_build")


def _scratch():
    os.makedirs(SCRATCH, exist_ok=True)
    return tempfile.mkdtemp(prefix="mla_mutants_", dir=SCRATCH)


def test_every_mutant_is_caught():
    tmp = _scratch()
    try:
        libs = [(n, _build_mutant(tmp, n, e)) for n, e in MUTANTS]
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            codes = list(ex.map(lambda nl: _run_pins(nl[1]), libs))
        survivors = [n for (n, _), c in zip(libs, codes) if c == 0]
        assert not survivors, f"pins did not catch: {survivors}"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


def test_unmutated_copy_passes():
    tmp = _scratch()
    try:
        so = _build_mutant(tmp, "identity", [])
        assert _run_pins(so) == 0
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


if __name__ == "__main__":  # pragma: no cover
    sys.exit(pytest.main([__file__, "-q"]))
