"""Host-side helpers of bench.py (no GPU): the staleness check of recorded
ncu traffic ignores comments but not code."""

import bench


def test_strip_comments_keeps_code_and_strings():
    src = 'int a = 1; // note\n/* block\n comment */ const char* s = "// kept";\n'
    assert bench._strip_comments(src) == 'int a = 1; const char* s = "// kept";'


def test_comment_edits_do_not_change_the_code_view():
    a = "x = f(y);  // one reason\n"
    b = "/* another reason */\nx = f(y);\n"
    c = "x = f(z);\n"
    assert bench._strip_comments(a) == bench._strip_comments(b)
    assert bench._strip_comments(a) != bench._strip_comments(c)


def test_recorded_traffic_matches_current_forward_sources():
    import json
    import os
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "attn_fwd_traffic.json")))
    e = rec["striped_causal_N262144_H16_d128_P16_qk3x"]
    assert e["kernel_hash"] == bench.kernel_source_hash()
    assert bench.recorded_traffic("striped_causal_N262144_H16_d128_P16_qk3x") == \
        e["dram_bytes_per_launch"]
