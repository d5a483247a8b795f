"""The calibrated threshold table: keys, exact round trip through JSON (CPU)."""
import math

import pytest

from sparse_input_gemv_b200.thresholds import ThresholdTable


def test_round_trip_is_exact(tmp_path):
    path = str(tmp_path / "t.json")
    tab = ThresholdTable(path)
    values = {("l70", "gate_up-in", 0.5, 7): 0.6953125,            # a bf16 value
              ("l70", "down-in", 0.5, 7): 0.5397616028785706,      # an fp32 value
              ("l70", "gate_up-in", 0.0, 7): -math.inf,            # p = 0 keeps everything
              ("8b", "qkv-in", 0.65, "a"): 1.0498046875}
    for (c, s, p, seed), t in values.items():
        tab.put(c, s, p, seed, t)
    tab.save()
    back = ThresholdTable(path)
    for (c, s, p, seed), t in values.items():
        got = back.get(c, s, p, seed)
        assert got == t and math.copysign(1, got) == math.copysign(1, t)
    assert back.get("l70", "gate_up-in", 0.4, 7) is None        # another p
    assert back.get("l70", "gate_up-in", 0.5, 8) is None        # another seed


def test_rejects_unknown_version(tmp_path):
    path = tmp_path / "t.json"
    path.write_text('{"version": 99, "entries": []}')
    with pytest.raises(ValueError):
        ThresholdTable(str(path))
