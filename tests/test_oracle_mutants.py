"""The oracle's pins must catch plausible mistakes.

Each case below plants one slip in a copy of oracle.cpp (on the CPU, in a
temporary directory), builds it, and runs the pin suite against that copy in
a child process: the suite has to fail."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.cpp")

MUTANTS = {
    "scale dropped": ("s[j] = sc * dot;", "s[j] = dot;"),
    "no max shift in normaliser": ("Z += std::exp(s[j] - m);", "Z += std::exp(s[j]);"),
    "no max shift in weights": ("double p = std::exp(s[j] - m);", "double p = std::exp(s[j]);"),
    "lse in base 2": ("*lse = m + std::log(Z);", "*lse = m + std::log2(Z);"),
    "lse without max": ("*lse = m + std::log(Z);", "*lse = std::log(Z);"),
    "output not normalised": ("for (int d = 0; d < D; ++d) out[d] /= Z;",
                              "for (int d = 0; d < D; ++d) out[d] /= (Z + 1.0);"),
    "value read from keys": ("out[d] += p * load(v, j * ld + d);",
                             "out[d] += p * load(k, j * ld + d);"),
    "key read from values": ("dot += load(q, d) * load(k, j * ld + d);",
                             "dot += load(q, d) * load(v, j * ld + d);"),
    "GQA interleaved mapping": ("kv = h / G;", "kv = h % Hkv;"),
    "chunk end off by one": ("long end = (s + 1) * C < n ? (s + 1) * C : n;",
                             "long end = (s + 1) * C - 1 < n ? (s + 1) * C - 1 : n;"),
    "combine unweighted": ("double w = std::exp(l_s[s] - M);", "double w = 1.0;"),
    "combine lse drops max": ("*lse = M + std::log(W);", "*lse = std::log(W);"),
    "max is first element": ("for (long j = 0; j < n; ++j) m = s[j] > m ? s[j] : m;",
                             "m = s[0];"),
    "lengths not clamped to max_len": ("    if (n > max_len) n = max_len;\n", ""),
    "batch base counts query heads": ("const long base = (b * Hkv + kv) * max_len * D;",
                                      "const long base = (b * Hq + kv) * max_len * D;"),
    "every head reads the first query": ("attend_one_head(n, D, q + i * D, k + base",
                                         "attend_one_head(n, D, q + b * Hq * D, k + base"),
    "empty split lse zero": ("part_lse[s] = s < S ? l_s[s] : ninf;",
                             "part_lse[s] = s < S ? l_s[s] : 0.0;"),
    "empty sequence lse zero": ("    *lse = ninf;\n    return;\n  }\n  std::vector<double> s(",
                                "    *lse = 0.0;\n    return;\n  }\n  std::vector<double> s("),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for '{name}' not found"
    mutated = src.replace(old, new)
    path = tmp_path / "oracle_mutant.cpp"
    path.write_text(mutated)
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread",
                           str(path), "-o", str(lib)])
    env = dict(os.environ, FD_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"pins did not catch mutant '{name}':\n{r.stdout[-2000:]}"
