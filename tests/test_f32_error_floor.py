"""The record the f32 elementwise parity guard is derived from
(tests/golden/f32_error_floor.json) is what its committed script computes:
the plain f32 evaluation of the recurrences against the f64 oracle, on the
seeded inputs of the f32 parity cases.  The evaluation is recomputed here on
the host and each recorded error must match it (float32 library routines may
round differently on another host, hence the factor of two)."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.join(ROOT, "tests", "golden"))

import f32_error_floor as F  # noqa: E402


def test_record_matches_its_script(tmp_path, monkeypatch):
    with open(F.OUT) as f:
        rec = json.load(f)
    out = tmp_path / "floor.json"
    monkeypatch.setattr(F, "OUT", str(out))
    F.main()
    with open(out) as f:
        new = json.load(f)
    for fam in ("m1", "m3"):
        assert set(new[fam]) == set(rec[fam])
        for case, ts in rec[fam].items():
            for tensor, ent in ts.items():
                e, got = ent["elem"], new[fam][case][tensor]["elem"]
                assert got <= 2 * e + 1e-12 and e <= 2 * got + 1e-12, (fam, case, tensor, e, got)


def test_guard_is_the_stated_multiple():
    """The guard of tests/_util.py is F32_ELEM_FACTOR times the record, per
    tensor, and the family's largest for tensors outside the record."""
    sys.path.insert(0, ROOT)
    from tests import _util as U
    with open(F.OUT) as f:
        rec = json.load(f)
    worst = max(e["elem"] for ts in rec["m3"].values() for e in ts.values())
    dal = max(ts["dalpha"]["elem"] for ts in rec["m3"].values() if "dalpha" in ts)
    assert U.f32_elem_tol("m3", "dalpha") == U.F32_ELEM_FACTOR * dal
    assert U.f32_elem_tol("m3", "no_such_tensor") == U.F32_ELEM_FACTOR * worst
    assert U.f32_elem_tol("m1", "out@7") == U.f32_elem_tol("m1", "out")
