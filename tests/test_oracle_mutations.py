"""The oracle's pins catch plausible mistakes.  Each case below plants one mistake in a copy
of oracle.c (a dropped term, a wrong sign or index, a swapped operand, a skipped step),
compiles it, and runs the pin tests of that function against the broken copy: at least one
pin must fail.  The intact oracle passes the same pins (they are part of this suite)."""
import concurrent.futures
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

ATTN = ["tests/test_oracle_attention.py"]
WALK = ["tests/test_golden.py", "tests/test_oracle_accept.py"]

# (name, pin tests, [(text in oracle.c, replacement), ...])
MUTATIONS = [
    ("O1 a node does not attend to itself", ATTN,
     [("for (int a = i; a >= 0; a = parents[(size_t)b * N + a]) path[np++] = a;",
       "for (int a = parents[(size_t)b * N + i]; a >= 0; a = parents[(size_t)b * N + a]) path[np++] = a;")]),
    ("O1 query head mapped to the wrong kv head", ATTN,
     [("const int g = h / G;", "const int g = h % Hkv;")]),
    ("O1 softmax scale dropped", ATTN, [("        s *= scale;\n", "        s *= 1.0;\n")]),
    ("O2 last hidden element dropped", ["tests/test_oracle_lm_head.py"],
     [("for (int k = 0; k < H; ++k)", "for (int k = 0; k < H - 1; ++k)")]),
    ("O3 accept test reversed", WALK, [("if (u < ratio) {", "if (u > ratio) {")]),
    ("O3 residual with the wrong sign", WALK,
     [("const double d = p[v] - (double)p_hat[v];", "const double d = (double)p_hat[v] - p[v];")]),
    ("O3 residual not renormalised", WALK,
     [("for (int v = 0; v < V; ++v) p[v] = r[v] / mass;", "for (int v = 0; v < V; ++v) p[v] = r[v];")]),
    ("O3 greedy ties to the higher index", WALK,
     [("if (logit_row[v] > logit_row[m]) m = v;", "if (logit_row[v] >= logit_row[m]) m = v;")]),
    ("O3 temperature ignored", WALK,
     [("p[v] = exp(logit_row[v] / T - mx);", "p[v] = exp(logit_row[v] - mx * T);")]),
    ("race key multiplied by the weight", ["tests/test_oracle_sampler.py"],
     [("const double key = e / weight[v];", "const double key = e * weight[v];")]),
    ("O4 committed rows in reverse order", ["tests/test_oracle_commit.py"],
     [("const size_t node = (size_t)b * N + path[t];", "const size_t node = (size_t)b * N + path[n - 1 - t];")]),
    ("O4 V rows copied into the K cache", ["tests/test_oracle_commit.py"],
     [("memcpy((char *)k_prefix + dst, (const char *)k_tree + src, row);",
       "memcpy((char *)k_prefix + dst, (const char *)v_tree + src, row);")]),
    ("O5 lowest values kept", ["tests/test_oracle_rerank.py"],
     [("if (x->value > y->value) return -1;\n    if (x->value < y->value) return 1;",
       "if (x->value < y->value) return -1;\n    if (x->value > y->value) return 1;")]),
    ("O5 confidences not clamped", ["tests/test_oracle_rerank.py"],
     [("const float ci = c[i] > 0.0f ? (c[i] < 1.0f ? c[i] : 1.0f) : 0.0f;", "const float ci = c[i];")]),
    ("O5 masks without the node itself", ["tests/test_oracle_rerank.py"],
     [("for (int32_t a = i; a >= 0; a = par[a]) mask |= 1ull << newidx[a];",
       "for (int32_t a = par[i]; a >= 0; a = par[a]) mask |= 1ull << newidx[a];")]),
    ("O6 temperature ignored", ["tests/test_oracle_draft.py"],
     [("const double Tp = T > 0.0 ? T : 1.0;", "const double Tp = 1.0;")]),
    ("O6 one Philox purpose shared by the k races", ["tests/test_oracle_draft.py"],
     [("arg = orc_race_purpose(V, p, seed, offset, b, f, 2 + j, &gap);",
       "arg = orc_race_purpose(V, p, seed, offset, b, f, 2, &gap);")]),
    ("O7 clock E * p instead of E / p", ["tests/test_oracle_distinct.py"],
     [("clk[2 * n] = -log(orc_uniform(seed, offset, b, f, v, 2)) / p[v];",
       "clk[2 * n] = -log(orc_uniform(seed, offset, b, f, v, 2)) * p[v];")]),
    ("O7 child rows not renormalised", ["tests/test_oracle_distinct.py"],
     [("q[v] = (!dead && !gone[v] && R > 0.0) ? p[v] / R : 0.0;",
       "q[v] = (!dead && !gone[v] && R > 0.0) ? p[v] : 0.0;")]),
    ("O7 remaining mass as 1 minus the removed mass", ["tests/test_oracle_distinct.py"],
     [("            double R = 0.0;\n", "            double R = 1.0;\n"),
      ("if (!gone[v]) R += p[v];", "if (gone[v]) R -= p[v];")]),
]


def _run(case, tmpdir):
    name, tests, edits = case
    src = open(SRC).read()
    for old, new in edits:
        assert src.count(old) >= 1, f"{name}: text not found in oracle.c: {old!r}"
        src = src.replace(old, new)
    tag = "".join(c if c.isalnum() else "_" for c in name)
    c_path = os.path.join(tmpdir, f"{tag}.c")
    so_path = os.path.join(tmpdir, f"{tag}.so")
    with open(c_path, "w") as f:
        f.write(src)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-w", c_path, "-o",
                           so_path, "-lm"])
    env = dict(os.environ, EAGLE_ORACLE_LIB=so_path, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu",
                        *tests], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return name, r.returncode, r.stdout[-600:]


def test_every_planted_mistake_fails_a_pin(tmp_path):
    workers = max(1, min(len(MUTATIONS), (os.cpu_count() or 2) - 1))
    with concurrent.futures.ThreadPoolExecutor(workers) as pool:
        results = list(pool.map(lambda c: _run(c, str(tmp_path)), MUTATIONS))
    survived = [(name, out) for name, rc, out in results if rc == 0]
    assert not survived, "mistakes no pin caught:\n" + "\n".join(f"{n}\n{o}" for n, o in survived)
    # rc 1 is a failing test; anything else (2..5) would be a broken run, not a caught mistake
    broken = [(name, rc, out) for name, rc, out in results if rc != 1]
    assert not broken, broken
