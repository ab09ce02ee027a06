"""The oracle's pins catch plausible mistakes: each mistake of
``_oracle_mutants`` is planted in the oracle (on the CPU, in a child pytest
process) and the independent pins (tests/test_oracle_*.py, not the golden
fixture, which the oracle itself wrote) must fail on it."""
import concurrent.futures as cf
import os
import re
import subprocess
import sys

import _oracle_mutants

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = [os.path.join("tests", f) for f in ("test_oracle_fp4.py", "test_oracle_routing.py", "test_oracle_layer.py",
                                           "test_oracle_lru.py", "test_oracle_formats.py",
                                           "test_oracle_nvfp4_act.py")]


def run_pins(mutant):
    env = dict(os.environ, FT_ORACLE_MUTANT=mutant)
    p = subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    failed = re.findall(r"^FAILED (\S+)(.*)$", p.stdout, re.M)
    return p.returncode, failed, p.stdout[-3000:] + p.stderr[-2000:]


def test_every_planted_mistake_fails_a_pin():
    names = sorted(_oracle_mutants.MUTANTS)
    with cf.ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
        res = dict(zip(names, ex.map(run_pins, names)))
    survivors = [n for n, (rc, _, _) in res.items() if rc == 0]
    broken = {n: out for n, (rc, failed, out) in res.items() if rc != 0 and (rc != 1 or not failed)}
    assert not broken, broken
    assert not survivors, f"pins do not catch: {survivors}"


def test_mutant_helpers_are_not_shadowed():
    """A second top-level definition with the same name would silently replace
    the first and plant a different mistake than the one named."""
    import ast
    with open(_oracle_mutants.__file__) as f:
        names = [n.name for n in ast.parse(f.read()).body if isinstance(n, ast.FunctionDef)]
    assert len(names) == len(set(names)), sorted(n for n in set(names) if names.count(n) > 1)


def test_an_unknown_mutant_is_refused():
    rc, _, out = run_pins("no_such_mistake")
    assert rc not in (0, 1) and "unknown oracle mutant" in out
