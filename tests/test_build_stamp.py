"""The in-tree libraries are rebuilt from a digest of their sources and build
command, not from file times (a copied tree can reorder those)."""
import os

from long_context_prefill_trianglemix_b200 import build


def test_stamp_follows_content_not_time(tmp_path):
    src = tmp_path / "a.cu"
    lib = tmp_path / "liba.so"
    src.write_text("int x;\n")
    lib.write_bytes(b"lib")
    cmd = ["-O3"]
    assert build._stale(str(lib), [str(src)], cmd)            # no stamp yet
    build._write_stamp(str(lib), [str(src)], cmd)
    assert not build._stale(str(lib), [str(src)], cmd)
    os.utime(lib, (0, 0))                                       # library "older" than its source
    assert not build._stale(str(lib), [str(src)], cmd)
    assert build._stale(str(lib), [str(src)], ["-O2"])         # another command
    src.write_text("int y;\n")                                  # another source
    assert build._stale(str(lib), [str(src)], cmd)


def test_in_tree_library_matches_its_stamp():
    build.build_lib()
    _, deps, flags = build.lib_inputs()
    assert not build._stale(build.LIBTM, deps, flags)
