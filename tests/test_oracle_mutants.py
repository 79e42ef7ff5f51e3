"""The oracle's pins catch planted mistakes (no GPU needed).

Each case copies the oracle source to a temporary folder, plants one plausible
mistake there by a textual edit (a dropped term, a wrong comparison, order,
constant or rounding), builds that copy, and runs the pin suite
(tests/test_oracle_pins.py) against it in a subprocess.  The suite must fail
for every mutant.  The oracle in oracle/ itself is never modified.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "mpzch_oracle.cpp")
HDR = os.path.join(ROOT, "oracle", "mpzch_oracle.h")

# (name, text in the oracle, replacement)
MUTANTS = [
    ("hash: final xor-shift dropped", "return z ^ (z >> 31);", "return z;"),
    ("lookup: window one slot short",
     "  for (int32_t j = 0; j < t->P; ++j) {\n    int64_t s = window_slot(t, key, j);\n    if (t->keys[s] == key && found < 0) found = s;",
     "  for (int32_t j = 0; j + 1 < t->P; ++j) {\n    int64_t s = window_slot(t, key, j);\n    if (t->keys[s] == key && found < 0) found = s;"),
    ("lookup: stops at the first empty slot",
     "if (t->keys[s] == key && found < 0) found = s;",
     "if (t->keys[s] == -1) break;\n    if (t->keys[s] == key && found < 0) found = s;"),
    ("victim: ties broken by probe order, not row index",
     "(t->last[s] == t->last[best] && s < best)", "false"),
    ("victim: most recently used instead of least",
     "t->last[s] < t->last[best] ||", "t->last[s] > t->last[best] ||"),
    ("resident ids not refreshed", "      t->last[r] = step;\n", "\n"),
    ("missing ids inserted in descending key order",
     "return uniq[a] < uniq[b];", "return uniq[a] > uniq[b];"),
    ("evictions not counted", "if (t->keys[best] != -1) ++n_evicted;", ""),
    ("Writeback stores e instead of e_hat - (e_hat - e)",
     "m[d] = e_hat - step_d;", "m[d] = ek[d];"),
    ("learning rate ignored", "float step_d = t->eta * g;", "float step_d = g;"),
    ("Writeback sign flipped", "float g = e_hat - ek[d];", "float g = ek[d] - e_hat;"),
    ("dedup keeps the last occurrence",
     "    if (first.emplace(ids[i], i).second) {\n      uniq[u] = ids[i];\n      pos[u] = i;\n      ++u;\n    }",
     "    auto it = first.find(ids[i]);\n    if (it == first.end()) {\n      first.emplace(ids[i], u);\n      uniq[u] = ids[i];\n      pos[u] = i;\n      ++u;\n    } else {\n      pos[it->second] = i;\n    }"),
    ("miss feature is -0.0", "o[d] = 0.0f;", "o[d] = -0.0f;"),
    ("select uses > instead of >=", "t->last[r] >= since", "t->last[r] > since"),
    ("int8 scale divides by 128", "const float s = a / 127.0f;", "const float s = a / 128.0f;"),
    ("int8 rounds by truncation", "float v = std::nearbyint(x[d] / s);",
     "float v = std::trunc(x[d] / s);"),
    ("owner taken from the low hash bits",
     "(int32_t)((orc_splitmix64((uint64_t)key) >> 32) % (uint64_t)n_owners)",
     "(int32_t)(orc_splitmix64((uint64_t)key) % (uint64_t)n_owners)"),
    ("serving divides by the scale",
     "(float)snap_q[r * (int64_t)dim + d] * snap_scale[r]",
     "(float)snap_q[r * (int64_t)dim + d] / snap_scale[r]"),
]


# Mistakes in the sharded oracle (Python, oracle/__init__.py): (name, text, replacement)
PY_MUTANTS = [
    ("owner receives ranks in reverse order",
     "for ids, e in zip(rank_ids, rank_e):  # ranks in order",
     "for ids, e in list(zip(rank_ids, rank_e))[::-1]:"),
    ("first dedup sends the e row at the distinct id's index, not its batch position",
     "recv_e[s].append(_c(e, np.float32)[pos[sel]])",
     "recv_e[s].append(_c(e, np.float32)[np.nonzero(sel)[0]])"),
    ("global row misses the shard offset", "rows[at] = np.where(h != 0, r + s * self.Cs, -1)",
     "rows[at] = np.where(h != 0, r, -1)"),
]
PKG = os.path.join(ROOT, "oracle")


def build_mutant(tmp, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not unique: {old!r}"
    with open(os.path.join(tmp, "mpzch_oracle.cpp"), "w") as f:
        f.write(src.replace(old, new))
    shutil.copy(HDR, os.path.join(tmp, "mpzch_oracle.h"))
    lib = os.path.join(tmp, "libmutant.so")
    subprocess.run(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                    "-shared", os.path.join(tmp, "mpzch_oracle.cpp"), "-o", lib], check=True)
    return lib


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new):
    lib = build_mutant(str(tmp_path), old, new)
    env = dict(os.environ, MPZCH_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join("tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode != 0, f"planted mistake survived every pin: {name}\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout, r.stdout[-2000:]


def run_pins_on_py_copy(tmp_path, old, new):
    import oracle
    lib = oracle.lib()._name  # the real C++ oracle, already built
    dst = tmp_path / "oracle"
    dst.mkdir()
    src = open(os.path.join(PKG, "__init__.py")).read()
    assert src.count(old) == 1, f"mutation site not unique: {old!r}"
    (dst / "__init__.py").write_text(src.replace(old, new))
    shutil.copy(os.path.join(PKG, "build.py"), dst / "build.py")
    env = dict(os.environ, MPZCH_ORACLE_LIB=lib, MPZCH_ORACLE_PKG_PARENT=str(tmp_path))
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           os.path.join("tests", "test_oracle_pins.py"), "-k",
                           "owner or shard or exchange"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)


def test_unmutated_copy_of_the_sharded_oracle_passes(tmp_path):
    """Control: the copy mechanism itself breaks nothing."""
    r = run_pins_on_py_copy(tmp_path, "class ShardedOracle:", "class ShardedOracle:")
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name,old,new", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_pins_catch_planted_mistake_in_sharded_oracle(tmp_path, name, old, new):
    r = run_pins_on_py_copy(tmp_path, old, new)
    assert r.returncode != 0, f"planted mistake survived every pin: {name}\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout, r.stdout[-2000:]
