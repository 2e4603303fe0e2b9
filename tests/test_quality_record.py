"""The stored OAM / SAM selection-quality record reproduces from the oracle (CPU).

The record (tests/golden/oam_sam_gqa8k.json, written by tests/golden/oam_sam_record.py) says how
much of dense attention each scoring metric's block selection keeps.  It is a measurement, not
a claim this build asserts: the test only checks that the stored numbers are what the oracle
computes today, and that they are sane.
"""
import json
from pathlib import Path

import pytest

GOLDEN = Path(__file__).resolve().parent / "golden"


def test_oam_sam_record_reproduces(orc):
    import importlib.util
    spec = importlib.util.spec_from_file_location("oam_sam_record", GOLDEN / "oam_sam_record.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    stored = json.loads((GOLDEN / "oam_sam_gqa8k.json").read_text())
    for dist, rec in mod.compute_all().items():
        for name, vals in rec["metrics"].items():
            for key, x in vals.items():
                assert x == pytest.approx(stored[dist]["metrics"][name][key], rel=1e-9, abs=1e-15), (dist, name, key)
                assert 0.0 <= x < 10.0
