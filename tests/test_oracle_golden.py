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


def _bytes(hex_rows):
    return [int(h[i:i + 2], 16) for h in hex_rows for i in range(0, len(h), 2)]


def test_fixture_nvfp4_entries_make_real_decisions():
    """The NVFP4 entries use an input without the near-maximum value, so their block scales
    are non-zero outside the zero, subnormal and signed-zero rows, and the stochastic-rounding
    entries hold codes of several magnitudes (not only signed zeros)."""
    stored = json.load(open(os.path.join(HERE, "oracle_small.json")))
    x4 = stored["x_nvfp4_bf16"]
    assert x4[1][17 * 4:18 * 4] == "42c0"                         # 96.0 in BF16
    assert [r for i, r in enumerate(x4) if i != 1] == [r for i, r in enumerate(stored["x_bf16"]) if i != 1]
    for k in ("nvfp4_rowwise_rne", "nvfp4_rowwise_rht5_sr6"):
        sf = _bytes(stored[k]["sf"])
        assert sum(b != 0 for b in sf) == 128 - 3 * 8, k          # rows 0, 2, 3 have zero scales
    assert all(b != 0 for b in _bytes(stored["nvfp4_colwise_rht5_sr6"]["sf"]))
    for k in ("nvfp4_rowwise_rht5_sr6", "nvfp4_colwise_rht5_sr6"):
        nib = {b & 7 for b in _bytes(stored[k]["q"])} | {(b >> 4) & 7 for b in _bytes(stored[k]["q"])}
        assert len(nib) >= 6, (k, nib)
