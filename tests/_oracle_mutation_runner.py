"""Runs the oracle's pin tests against several builds of oracle.c in one process.

    python tests/_oracle_mutation_runner.py <dir> <name> [<name> ...]

For each name, ``<dir>/<name>.so`` is loaded as the oracle library and the pin
files (tests/test_oracle_*.py, minus the mutation check itself) run with
``-x``. The last line printed is ``RESULTS {"name": pytest exit code, ...}``:
0 when every pin passed, 1 when a pin failed. Used by
tests/test_oracle_mutations.py; importing torch and the test modules once
keeps each run to a couple of seconds.
"""
import contextlib
import io
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import pytest  # noqa: E402

import oracle  # noqa: E402

PIN_FILES = [os.path.join(ROOT, "tests", f) for f in (
    "test_oracle_geometry.py", "test_oracle_layout.py", "test_oracle_pixels.py", "test_oracle_tables.py",
    "test_oracle_video.py")]


def main(lib_dir: str, names: list[str]) -> dict:
    results = {}
    for name in names:
        oracle.load_build(os.path.join(lib_dir, name + ".so"))
        log = io.StringIO()
        with contextlib.redirect_stdout(log):
            code = pytest.main(["-x", "-q", "-p", "no:cacheprovider", *PIN_FILES])
        results[name] = int(code)
    oracle.load_build(None)
    return results


if __name__ == "__main__":
    print("RESULTS " + json.dumps(main(sys.argv[1], sys.argv[2:])), flush=True)
