"""The library is tied to its sources by a compiled-in build id, not by
file modification times: a library whose id differs from the hash of the
sources beside it is rebuilt (CPU only; fake libraries built with gcc)."""
import os
import subprocess

import pytest

from rotated_int8_quantized_b200 import build


def _fake_lib(tmp_path, name, build_id):
    src = tmp_path / (name + ".c")
    src.write_text('const char *convrot_build_id(void) { return "%s"; }\n' % build_id)
    lib = tmp_path / (name + ".so")
    subprocess.check_call(["gcc", "-shared", "-fPIC", "-o", str(lib), str(src)])
    return str(lib)


def test_library_build_id_is_read_from_the_library(tmp_path):
    lib = _fake_lib(tmp_path, "a", "0123456789abcdef")
    assert build.library_build_id(lib) == "0123456789abcdef"
    assert build.library_build_id(str(tmp_path / "missing.so")) is None


def test_mismatch_means_rebuild_and_mtime_does_not_matter(tmp_path):
    lib = _fake_lib(tmp_path, "b", "feedfacefeedface")
    # newer than every source, but built from other sources: rebuild
    future = max(os.path.getmtime(s) for s in build.sources()) + 3600
    os.utime(lib, (future, future))
    assert build.needs_build(lib, expected="0000000000000000")
    assert not build.needs_build(lib, expected="feedfacefeedface")
    assert build.needs_build(str(tmp_path / "missing.so"))


def test_source_hash_covers_contents_and_flags(tmp_path):
    a = tmp_path / "x.cu"
    a.write_text("int a;\n")
    h1 = build.source_hash([str(a)])
    a.write_text("int b;\n")
    h2 = build.source_hash([str(a)])
    assert h1 != h2 and len(h1) == 16
    assert build.source_hash([str(a)], flags=["-O2"]) != build.source_hash([str(a)], flags=["-O3"])


def test_in_tree_library_carries_its_sources_hash():
    build.build()
    assert build.library_build_id() == build.source_hash()
    import rotated_int8_quantized_b200 as cr
    assert cr.build_id() == build.source_hash()
