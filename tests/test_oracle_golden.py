"""The oracle against its stored fixtures in tests/golden/: the generator's published
known-answer vectors live in test_oracle_philox_rht.py; here the oracle's quantizers are
re-run on the small edge-case input of oracle_small.json (written by make_golden.py from
oracle/ only) and must reproduce every stored byte, so any change to the oracle's arithmetic
shows up as a diff of that file."""
import importlib.util
import json
import os

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _make_golden():
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "make_golden.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_oracle_reproduces_stored_fixture():
    stored = json.load(open(os.path.join(HERE, "oracle_small.json")))
    fresh = json.loads(json.dumps(_make_golden().build()))
    assert stored.keys() == fresh.keys()
    for k in stored:
        assert stored[k] == fresh[k], f"oracle output changed: {k}"


def test_fixture_input_has_its_edge_cases():
    stored = json.load(open(os.path.join(HERE, "oracle_small.json")))
    rows = stored["x_bf16"]
    assert len(rows) == 16 and all(len(r) == 128 * 4 for r in rows)
    assert set(rows[0]) == {"0"}                                  # all-zero row
    assert rows[1][17 * 4:18 * 4] == "7f62"                       # 3e38 in BF16
    assert all(int(rows[2][4 * i:4 * i + 4], 16) & 0x7F80 == 0 for i in range(128))   # subnormals
    assert {rows[3][4 * i:4 * i + 4] for i in range(128)} == {"0000", "8000"}         # signed zeros
