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
    for k in bench.KERNEL_FILES:
        assert len(bench.kernel_source_hash(k)) == 12
    # the host section of gtr_gla.cu is not part of any kernel's hash
    assert bench.kernel_source_hash("gla_fwd_span_kernel") != bench.kernel_source_hash("gla_fwd_pipe_kernel")
    for wl in ("gtr640_b1h16_40x40", "hires_b1h16_128x128", "stress_b4h12_37x53_dk128", "gtr640_b1h16_40x40+z"):
        t = bench.recorded_traffic(wl)
        # either the summary was taken on this code (a positive byte count) or it is
        # reported as unknown; never a stale number
        assert t is None or t > 0


def test_backward_bytes_alg():
    # read q, k, g, v, d_out in fp16 and write the four gradients in fp32: 1664 B per
    # token-head at dk = dv = 64, plus the fp32 states (init_state, d_final_state read,
    # grad_init_state written)
    w = bench.WORKLOADS["hires_b1h16_128x128"]
    th = w.B * w.N * w.heads
    assert bench.bwd_bytes_alg(w) == th * 1664 + 3 * w.B * w.heads * 64 * 64 * 4
    w2 = bench.WORKLOADS["gtr640_b1h16_40x40"]   # no initial state: d_final_state and grad_init_state
    assert bench.bwd_bytes_alg(w2) == w2.B * w2.N * w2.heads * 1664 + 2 * w2.B * w2.heads * 64 * 64 * 4
