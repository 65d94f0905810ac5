"""Host arithmetic of bench.py's roofline on CPU: which ceiling binds a
kernel class, and the achieved/peak figures of each case."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

INT_S, FP_S, HBM = 1.0e12, 3.0e12, 6000.0  # products/s, products/s, GB/s


def test_hbm_bound_class():
    # 12 GB take 2 ms at 6 TB/s, 1e9 integer products 1 ms at 1e12/s: bytes bind
    ms, launches, nbytes, mults, mults_fp = 2.0, 1, 12e9, 1e9, 0.0
    r = bench.roofline_for("x", (ms, launches, nbytes, mults, mults_fp), INT_S, FP_S, HBM, "measured")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(12e9 / 2e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / HBM)
    assert r["traffic"] is None


def test_alu_bound_class_weights_the_two_pipes():
    # 3e9 products, 2e9 of them FP64: ideal 1e9/1e12 + 2e9/3e12 = 1.667 ms; bytes small
    ms, launches, nbytes, mults, mults_fp = 4.0, 2, 1e6, 6e9, 4e9  # per launch: 2 ms, 3e9 products
    r = bench.roofline_for("x", (ms, launches, nbytes, mults, mults_fp), INT_S, FP_S, HBM, "measured")
    assert r["bound"] == "alu" and r["unit"] == "Gmodmul/s"
    ideal = 1e9 / INT_S + 2e9 / FP_S
    assert r["peak"] == pytest.approx(3e9 / ideal / 1e9)
    assert r["achieved"] == pytest.approx(3e9 / 2e-3 / 1e9)
    assert r["frac"] == pytest.approx(ideal / 2e-3)
    assert r["fp64_share"] == pytest.approx(2.0 / 3.0)


def test_traffic_is_scaled_from_a_capture_of_unchanged_sources(tmp_path, monkeypatch):
    """A stored ratio is used only while the digest of its kernel's sources
    matches the one recorded with the capture."""
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    table = {"x": {"ratio": 0.91, "sources": ["k.cu"], "sha256": bench.source_digest(["k.cu"])}}
    monkeypatch.setattr(bench, "NCU_TRAFFIC", table)
    r = bench.roofline_for("x", (1.0, 1, 1e9, 1.0, 0.0), INT_S, FP_S, HBM, "measured")
    assert r["traffic"] == pytest.approx(0.91e9)
    src.write_text("kernel v2")  # the kernel changed after the capture
    r = bench.roofline_for("x", (1.0, 1, 1e9, 1.0, 0.0), INT_S, FP_S, HBM, "measured")
    assert r["traffic"] is None
    assert bench.traffic_ratio("y") is None


def test_stored_traffic_ratios_are_current():
    """Every committed ratio still matches its kernel's sources and lies near
    the algorithmic bytes (no class is re-reading what it should not)."""
    for name, e in bench.NCU_TRAFFIC.items():
        assert bench.traffic_ratio(name) is not None, name
        assert 0.8 < e["ratio"] < 1.3, name


def test_attention_sum_steps_agree_with_the_oracle():
    """The rotation keys the attention benchmark uploads for the feature sum
    are the oracle's schedule's non-zero steps."""
    import bench
    from oracle import ckks as C

    for n_tok, d in [(256, 64), (32, 16), (8, 2), (4, 128), (16, 1)]:
        want = sorted({x for st in C.attention_sum_steps(n_tok, d) for x in st if x})
        assert sorted(bench.attention_sum_steps(n_tok, d)) == want
