"""Runs the oracle's pin tests against several builds of oracle.c in one process.

    python tests/_oracle_mutation_runner.py <dir> <name> [<name> ...]

For a name ``n``, ``<dir>/n.so`` is loaded as the oracle library (a build of
a changed oracle.c). For a name ``pymod_n``, ``<dir>/pymod_n/oracle`` is imported as
the whole oracle package instead (a changed oracle/__init__.py). Either way the
pin files (tests/test_oracle_*.py, minus the mutation check itself) run with
``-x``. The last line printed is ``RESULTS {"name": pytest exit code, ...}``:
0 when every pin passed, 1 when a pin failed. Used by
tests/test_oracle_mutations.py; importing torch once keeps each run to a
couple of seconds.
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

PY_PREFIX = "pymod_"  # names of Python-package mutants

PIN_FILES = [os.path.join(ROOT, "tests", f) for f in (
    "test_oracle_geometry.py", "test_oracle_layout.py", "test_oracle_pixels.py", "test_oracle_tables.py",
    "test_oracle_video.py", "test_oracle_library_pins.py")]


def run_pins() -> int:
    log = io.StringIO()
    with contextlib.redirect_stdout(log):
        return int(pytest.main(["-x", "-q", "-p", "no:cacheprovider", *PIN_FILES]))


def _swapped_modules():
    return [k for k in sys.modules if k == "oracle" or k.startswith("oracle.") or k.startswith("test_oracle_")]


def run_with_package(pkg_parent: str) -> int:
    """The pins against the oracle package under ``pkg_parent``: the cached oracle and pin modules are set
    aside so that the pin files import the other package, then put back."""
    saved_path = list(sys.path)
    saved = {k: sys.modules.pop(k) for k in _swapped_modules()}
    sys.path.insert(0, pkg_parent)
    try:
        return run_pins()
    finally:
        for k in _swapped_modules():
            sys.modules.pop(k)
        sys.modules.update(saved)
        sys.path[:] = saved_path


def main(lib_dir: str, names: list[str]) -> dict:
    results = {}
    for name in names:
        if name.startswith(PY_PREFIX):
            results[name] = run_with_package(os.path.join(lib_dir, name))
        else:
            oracle.load_build(os.path.join(lib_dir, name + ".so"))
            results[name] = run_pins()
    oracle.load_build(None)
    return results


if __name__ == "__main__":
    print("RESULTS " + json.dumps(main(sys.argv[1], sys.argv[2:])), flush=True)
