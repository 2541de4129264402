"""The synthetic inputs are reproducible: every generated buffer hashes to the
SHA-256 committed in tests/golden/workload_digests.json (written by
tests/golden/make_workload_digests.py, which calls only workloads.py)."""
import importlib.util
import json
import os

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden", "workload_digests.json")


def _maker():
    spec = importlib.util.spec_from_file_location("make_workload_digests",
                                                  os.path.join(HERE, "golden", "make_workload_digests.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


MAKER = _maker()
with open(GOLDEN) as _f:
    EXPECTED = json.load(_f)
CASES = dict(MAKER.cases())


def test_every_workload_has_a_digest():
    assert set(CASES) == set(EXPECTED)


@pytest.mark.parametrize("name", sorted(CASES))
def test_workload_digest(name):
    got = MAKER.digest(CASES[name]())
    assert got == EXPECTED[name], f"{name}: generated buffers differ from the committed digests"
