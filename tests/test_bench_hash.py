"""bench.py reports a profile's DRAM traffic only for the kernel code the
capture ran: the hash over the GEMM sources ignores comments and layout but
not code."""
import bench


def test_comments_and_whitespace_do_not_count():
    a = "int f(int x) {\n  return x + 1;  // one more\n}\n"
    b = "/* add one */ int f(int x) { return x + 1; }"
    assert bench.strip_c_comments(a) == bench.strip_c_comments(b)


def test_code_and_literals_count():
    base = bench.strip_c_comments('asm("add.u32 %0, %1, 1; // not a comment");')
    assert "// not a comment" in base
    assert bench.strip_c_comments("x = a + 1;") != bench.strip_c_comments("x = a + 2;")
    assert bench.strip_c_comments("c = '/';") == "c = '/';"
    assert bench.strip_c_comments('s = "a\\"b // c";') == 's = "a\\"b // c";'


def test_committed_profile_matches_or_is_reported_stale():
    traffic, src = bench.profiled_traffic("qkv_1024")
    assert (traffic is None) == (src in ("no ncu summary", "kernel changed since the ncu capture",
                                         "no traffic line"))
