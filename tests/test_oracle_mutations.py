"""The oracle's pins must catch a plausible mistake anywhere in it: each mutation of
tests/oracle_mutations.py (a flipped sign, a dropped term or scale, a wrong index or
operand) is planted in memory in a child pytest run of tests/test_oracle_pins.py, which
must then fail.  The unmutated run must pass."""
import concurrent.futures
import os
import pathlib
import subprocess
import sys

import pytest

import oracle_mutations

TESTS = pathlib.Path(__file__).resolve().parent


def _run_pins(index):
    env = dict(os.environ)
    if index is None:
        env.pop("HRA_ORACLE_MUTATION", None)
    else:
        env["HRA_ORACLE_MUTATION"] = str(index)
    r = subprocess.run([sys.executable, "-m", "pytest", str(TESTS / "test_oracle_pins.py"), "-x", "-q",
                        "-p", "no:cacheprovider"], cwd=TESTS.parent, env=env, capture_output=True, text=True,
                       timeout=600)
    return index, r.returncode, r.stdout[-400:]


def test_every_planted_mistake_fails_a_pin():
    indices = [None] + list(range(len(oracle_mutations.MUTATIONS)))
    with concurrent.futures.ThreadPoolExecutor(max_workers=4) as pool:
        results = dict((i, (rc, out)) for i, rc, out in pool.map(_run_pins, indices))
    rc, out = results[None]
    assert rc == 0, f"pins fail on the unmutated oracle:\n{out}"
    missed = [oracle_mutations.MUTATIONS[i][3] for i in indices[1:] if results[i][0] == 0]
    assert not missed, f"mistakes no pin catches: {missed}"
    crashed = [oracle_mutations.MUTATIONS[i][3] for i in indices[1:] if results[i][0] not in (0, 1)]
    assert not crashed, f"mutations that did not run cleanly: {crashed}"
