"""Mutation test of the oracle's pins.

Every mutant in tests/oracle_mutants.py is the oracle with one planted mistake (a dropped
term, a wrong sign, bias or index, a transposed operand, an off-by-one range, a reversed
order).  The oracle pins (tests/test_oracle_*.py) must fail against each: they are then
strong enough that a plausible slip anywhere in the oracle cannot pass them unnoticed.
The mutants run in one child process (the nested pytest runs stay out of this session),
next to an unmutated copy built and loaded the same way, which must pass: a failure is
then the mutant's doing.
"""
import json
import os
import subprocess
import sys

import oracle_mutants

HERE = os.path.dirname(os.path.abspath(__file__))


def test_every_planted_mistake_fails_a_pin(tmp_path):
    out = tmp_path / "codes.json"
    r = subprocess.run([sys.executable, os.path.join(HERE, "oracle_mutants.py"), str(out)],
                       cwd=os.path.dirname(HERE), capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    codes = json.loads(out.read_text())
    assert codes.pop(oracle_mutants.CONTROL) == 0, "the unmutated copy must pass the pins"
    assert set(codes) == {m[0] for m in oracle_mutants.MUTANTS}
    survivors = sorted(name for name, code in codes.items() if code == 0)
    assert not survivors, f"mutants that pass every pin: {survivors}"
    # exit code 1 = tests failed; anything else (2 interrupted, 3 internal, 4 usage,
    # 5 nothing collected) would mean the pins did not run
    assert all(code == 1 for code in codes.values()), codes


def test_unmutated_oracle_passes_the_pins():
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "not gpu",
                        *oracle_mutants.PIN_FILES], cwd=os.path.dirname(HERE), capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:]
