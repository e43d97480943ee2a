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
