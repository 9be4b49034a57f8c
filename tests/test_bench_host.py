"""Host logic of bench.py that needs no GPU: the kernel-source hash that ties the
committed ncu summaries under profiles/ to the code they were taken on."""
import bench


def test_code_tokens_drops_comments_and_layout_only():
    src = 'int a = 1;  // note\n/* block\n comment */ char *s = "x // y /* z */";\nchar q = \'\\\'\';\n'
    got = bench._code_tokens(src)
    assert got == 'int a = 1; char *s = "x // y /* z */"; char q = \'\\\'\';'
    # a code change shows; a comment or layout change does not
    assert bench._code_tokens(src.replace("a = 1", "a = 2")) != got
    assert bench._code_tokens(src.replace("// note", "// other note")) == got
    assert bench._code_tokens(src.replace("int a", "int   a")) == got


def test_recorded_traffic_matches_current_source():
    h = bench.kernel_source_hash()
    assert len(h) == 12
    for wl in ("gtr640_b1h16_40x40", "hires_b1h16_128x128"):
        t = bench.recorded_traffic(wl)
        # either the summary was taken on this code (a positive byte count) or it is
        # reported as unknown; never a stale number
        assert t is None or t > 0
