"""The benchmark's CPU-baseline helpers for the extra legs run on the host alone and report
positive, extrapolated times in the legs' own units."""
import bench


def test_oracle_extras_small_samples():
    out = bench.oracle_extras(rows_w4=2, tokens_rot=64, rows_obq=1)
    assert set(out) == {"w4a16", "rotation", "obq"}
    for v in out.values():
        assert v["kind"] == "oracle" and v["value"] > 0 and v["cores"] >= 1
        assert "of" in v["sample"]
