"""The magnitude-versus-slicing diagnostic (oracle/retention_diagnostic.py) on a
small synthetic case: it runs, every loss lies in [0, 1] (energy) or is finite
(output), and magnitude selection never loses more query energy than slicing
(the k largest magnitudes maximise the kept squared norm).  CPU only."""
import math

from oracle import retention_diagnostic as RD


def test_retention_diagnostic_small_case():
    res = RD.run(T=256, kv_heads=1, group=4, ks=(96, 32))
    assert [r["k"] for r in res["rows"]] == [96, 32]
    for r in res["rows"]:
        for m in ("magnitude", "slicing"):
            assert 0.0 <= r[f"{m}_energy"] <= 1.0
            assert math.isfinite(r[f"{m}_output"]) and r[f"{m}_output"] >= 0.0
        assert r["magnitude_energy"] <= r["slicing_energy"]
