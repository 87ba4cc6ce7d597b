"""The bench reports the captured DRAM traffic only while the kernel's code is
the code it was captured on: the hash ignores comments and layout, and sees
any change to code."""
import bench


def test_comments_and_layout_do_not_change_the_code_text():
    a = "int f(int x) {  // doubles x\n  return 2 * x; /* no overflow\n check */\n}\n"
    b = "/* header */\nint f(int x) {\n\treturn 2 * x;\n}  // end\n"
    assert bench._code_only(a) == bench._code_only(b)


def test_code_changes_are_seen():
    a = "int f(int x) { return 2 * x; }"
    for b in ("int f(int x) { return 3 * x; }", "int f(int y) { return 2 * y; }",
              "int f(int x) { return 2 * x; } int g;"):
        assert bench._code_only(a) != bench._code_only(b)



def test_hash_covers_every_build_input():
    names = {__import__("os").path.basename(p) for p in bench.kernel_sources()}
    for must in ("tm_attn.cu", "tm_api.cu", "tm_sm100.cuh", "tm_tiles.cuh", "tm.h", "build.py"):
        assert must in names, must
