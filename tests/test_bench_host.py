"""Host-side logic of bench.py that needs no GPU: the code digest that ties an ncu summary to
the sources it was captured on, and the traffic lookup that depends on it."""

import os

import bench


def test_code_digest_ignores_comments_and_blank_lines():
    a = "int f(int x) {  // first\n    /* a block\n       comment */\n    return x + 1;\n}\n"
    b = "int f(int x) {\n\n    return x + 1;   \n}\n// trailing note\n"
    c = "int f(int x) {\n    return x + 2;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def _fake_tree(tmp_path, source_text):
    src = tmp_path / "block_scaled_precision_sm_b200" / "csrc"
    src.mkdir(parents=True)
    for rel in bench.KERNEL_SOURCES["quantize"]:
        (tmp_path / rel).write_text(source_text)
    (tmp_path / "profiles").mkdir()
    return tmp_path


def test_traffic_only_while_the_digest_matches(tmp_path, monkeypatch):
    root = _fake_tree(tmp_path, "int k() { return 1; }\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    digest = bench.sources_digest("quantize")
    (root / "profiles" / "quantize_x.md").write_text(f"traffic_bytes_per_launch: 12345\nsources_digest: {digest}\n")
    assert bench.profiled_traffic("quantize_x.md") == 12345.0
    # a comment edit keeps it; a code edit makes it stale
    for rel in bench.KERNEL_SOURCES["quantize"]:
        (root / rel).write_text("int k() { return 1; }  // note\n")
    assert bench.profiled_traffic("quantize_x.md") == 12345.0
    for rel in bench.KERNEL_SOURCES["quantize"]:
        (root / rel).write_text("int k() { return 2; }\n")
    assert bench.profiled_traffic("quantize_x.md") is None
    assert bench.profiled_traffic("missing.md") is None


def test_committed_summaries_name_their_command_and_digest():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for name in os.listdir(os.path.join(root, "profiles")):
        text = open(os.path.join(root, "profiles", name)).read()
        assert "ncu " in text and "--clock-control none" in text, name
        assert "sources_digest:" in text, name


def test_spread_reports_median_and_percentiles():
    import numpy as np

    d = bench.spread(np.array([1.0, 2.0, 3.0, 4.0, 100.0]))
    assert d["median_ms"] == 3.0 and d["samples"] == 5
    assert d["p10_ms"] < d["median_ms"] < d["p90_ms"] and d["mean_ms"] == 22.0


def test_peak_fractions_against_spec_and_clock():
    # 148 SMs x 16384 FP8 flops per clock at 1965 MHz = 4765 TFLOP/s
    f = bench.peak_fractions(2382.5, "fp8", 148, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0})
    assert abs(f["clock_peak_tflops_at_sampled_clock"] - 4764.9) < 0.2
    assert abs(f["frac_of_clock_peak_at_sampled_clock"] - 0.5) < 1e-3
    assert f["frac_of_spec"] == round(2382.5 / 4500.0, 4)
    assert "frac_of_clock_peak_at_sampled_clock" not in bench.peak_fractions(1.0, "bf16", 148, {"sm_mhz": None})


def test_clock_window_selects_the_timed_samples(monkeypatch):
    s = bench.ClockSampler(0)
    s.max_mhz = 1965.0
    sw_power_cap = 0x4
    s.samples = [(0.0, 1000.0, 100.0, 0), (1.0, 1965.0, 500.0, 0), (1.001, 1950.0, 600.0, sw_power_cap),
                 (1.002, 1965.0, 550.0, 0), (2.0, 900.0, 90.0, 0)]
    w = s.window(0.9, 1.1)
    assert w["samples"] == 3 and w["sm_mhz"] == 1965.0 and w["sm_mhz_min"] == 1950.0
    assert w["reasons"] == ["sw_power_cap"]
    # a window shorter than the sampling period takes the samples on either side
    assert s.window(1.5, 1.6)["samples"] == 2
    assert bench.ClockSampler(0).window()["samples"] == 0


def test_every_profile_the_bench_reads_is_committed_with_its_figures():
    # the summaries bench.py looks up for its traffic figures, and the ones its --profile cases write
    import re

    text = open(os.path.join(os.path.dirname(bench.__file__), "bench.py")).read()
    names = set(re.findall(r'profiled_traffic\("([^"]+\.md)"', text))
    names |= {"gemm_fp8_1024x7168x7168.md", "gemm_fp8_4096x7168x7168.md", "sf_transform_fp32_36864x56.md",
              "sf_transform_fp32_64x36864x56.md", "sf_transform_fp32_7168x512.md",
              "quantize_fp8_fp32_4096x16384_1x128.md", "quantize_fp8_bf16_7168x16384_128x128.md"}
    for name in sorted(names):
        path = os.path.join(bench.ROOT, "profiles", name)
        assert os.path.exists(path), name
        body = open(path).read()
        assert re.search(r"traffic_bytes_per_launch:\s*[0-9]+", body), name
        assert re.search(r"sources_digest:\s*[0-9a-f]{16}", body), name
        assert "--clock-control none" in body and "python bench.py --profile" in body, name
