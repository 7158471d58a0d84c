"""CPU: the oracle's pins catch plausible mistakes.

Each case plants one mistake in a private copy of oracle/dash_oracle.c (a dropped term, a
wrong index, a transposed root, ...), builds that copy and runs tests/test_oracle_pins.py
against it; at least one pin must fail.  The unmodified copy must pass, so that a broken
harness cannot make every mutant look caught.  Nothing under the repository's oracle/
is modified.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, text in dash_oracle.c, replacement, replace every occurrence: the fine logits and
# the GQA index appear in the forward and the backward routines alike)
MUTATIONS = [
    ("dropped log prior in the fine logits", "lbuf[i] = dot * isd + lw;", "lbuf[i] = dot * isd;", True),
    ("unscaled fine logits (no 1/sqrt(d))", "lbuf[i] = dot * isd + lw;", "lbuf[i] = dot + lw;", True),
    ("block sum instead of block mean", "for (long long c = 0; c < d; ++c) o[c] /= (double)blk;", "", False),
    ("coarse score without 1/sqrt(d)", "x[j] = (P->alpha - 1.0) * P->cs * dot * isd;",
     "x[j] = (P->alpha - 1.0) * P->cs * dot;", False),
    ("coarse score without (alpha - 1)", "x[j] = (P->alpha - 1.0) * P->cs * dot * isd;",
     "x[j] = P->cs * dot * isd;", False),
    ("wrong GQA head-to-KV-head index", "long long g = h / G;", "long long g = h % Hkv;", True),
    ("own block with prior 1/2 instead of 1", "row_fine(&P, r, b, g, t, p, lp, 1.0, lbuf, out + r * d);",
     "row_fine(&P, r, b, g, t, p, lp, 0.5, lbuf, out + r * d);", False),
    ("log p without the 1/(alpha - 1) power", "lp[j] = p[j] > 0.0 ? log(x[j] - tau) / (alpha - 1.0) : -INFINITY;",
     "lp[j] = p[j] > 0.0 ? log(x[j] - tau) : -INFINITY;", False),
    ("larger root of the alpha = 1.5 quadratic", "tau = mu - sqrt(disc);", "tau = mu + sqrt(disc);", False),
]


def _workdir(base, name, mutation):
    """A private tree: oracle/ (possibly mutated), tests/ with the pins, conftest and golden
    data.  The pins import only the oracle."""
    wd = os.path.join(base, name)
    os.makedirs(os.path.join(wd, "oracle"))
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), os.path.join(wd, "oracle"))
    with open(os.path.join(ROOT, "oracle", "dash_oracle.c")) as f:
        src = f.read()
    if mutation is not None:
        old, new, every = mutation
        n = src.count(old)
        assert n >= 1 and (every or n == 1), f"mutation site not unique: {old!r} occurs {n} times"
        src = src.replace(old, new)
    with open(os.path.join(wd, "oracle", "dash_oracle.c"), "w") as f:
        f.write(src)
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(wd, "tests", "golden"))
    for fn in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", fn), os.path.join(wd, "tests"))
    with open(os.path.join(wd, "pytest.ini"), "w") as f:
        f.write("[pytest]\n")
    return wd


def _run_pins(wd):
    env = dict(os.environ)
    env.pop("PYTHONPATH", None)
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x", "-q",
                        "-p", "no:cacheprovider"], cwd=wd, env=env, capture_output=True, text=True,
                       timeout=600)
    tail = (r.stdout + r.stderr).strip().splitlines()[-1:] or [""]
    return r.returncode, tail[0]


@pytest.mark.slow
def test_pins_catch_every_planted_mistake(tmp_path):
    cases = [("control", None)] + [(f"m{i}", (old, new, every)) for i, (_, old, new, every) in enumerate(MUTATIONS)]
    dirs = {name: _workdir(str(tmp_path), name, mut) for name, mut in cases}
    with ThreadPoolExecutor(max_workers=min(len(cases), max(2, (os.cpu_count() or 2) // 2))) as pool:
        results = dict(zip(dirs, pool.map(_run_pins, dirs.values())))
    rc, tail = results.pop("control")
    assert rc == 0, f"the unmodified oracle copy fails its pins: {tail}"
    # caught = a pin assertion failed (not a build or collection error of the copy)
    missed = [MUTATIONS[int(k[1:])][0] for k, (rc, tail) in results.items() if rc == 0 or "failed" not in tail]
    assert not missed, f"planted mistakes no pin catches: {missed}"
    for k, (rc, tail) in sorted(results.items()):
        print(f"{MUTATIONS[int(k[1:])][0]}: {tail}")
