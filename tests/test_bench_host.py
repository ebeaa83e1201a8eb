"""Host-side helpers of bench.py (no GPU): the source digest that decides whether
committed DRAM-traffic counters still describe the kernels being timed."""
import bench


def test_strip_comments_keeps_code_and_literals():
    src = 'int a = 1; // trailing\n/* block\n comment */ const char *s = "// not a comment";\n\n  b = a / 2;\n'
    out = bench.strip_comments(src)
    assert "trailing" not in out and "block" not in out
    assert '"// not a comment"' in out and "b = a / 2;" in out
    assert bench.strip_comments("x = '/'; // c") == "x = '/';"


def test_digest_ignores_comments_but_tracks_code(tmp_path, monkeypatch):
    csrc = tmp_path / "ternary_weight_fwd_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "include").mkdir()
    (tmp_path / "include" / "bitnet.h").write_text("int f(void);\n")
    for name in {n for files in bench.KIND_SOURCES.values() for n in files}:
        (csrc / name).write_text(f"// {name}\nint {name.split('.')[0]}_v = 1;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d0 = bench.source_digest("decode_sequence")
    p0 = bench.source_digest("prefill_q_o")
    (csrc / "decode_tasks.cuh").write_text("// a different comment\nint decode_tasks_v = 1;  /* and another */\n")
    assert bench.source_digest("decode_sequence") == d0          # comments only
    (csrc / "decode_tasks.cuh").write_text("int decode_tasks_v = 2;\n")
    assert bench.source_digest("decode_sequence") != d0          # code changed
    assert bench.source_digest("prefill_gate_up") == p0          # not a prefill source
    (csrc / "bitnet.cu").write_text("int bitnet_v = 3;\n")
    assert bench.source_digest("prefill_down") != p0             # the shared host code is tracked
