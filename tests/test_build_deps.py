"""The library build's staleness check covers every file the build reads: a
newer copy of any csrc header (or of include/sru.h) makes the build stale."""
import os
import shutil

from parallelizable_recurrence_b200 import build as libbuild


def test_every_header_is_a_dependency():
    names = {os.path.basename(p) for p in libbuild.deps()}
    on_disk = {f for f in os.listdir(libbuild.CSRC) if f.endswith((".cu", ".cuh"))}
    assert on_disk <= names, on_disk - names
    assert "sru.h" in names


def test_touching_any_header_makes_the_build_stale(tmp_path):
    pkg = tmp_path / "pkg"
    shutil.copytree(libbuild.CSRC, pkg / "csrc")
    shutil.copytree(os.path.join(libbuild.ROOT, "include"), tmp_path / "include")
    lib = pkg / "libsru.so"
    lib.write_bytes(b"")
    csrc = str(pkg / "csrc")
    files = libbuild.deps(csrc)
    assert len(files) >= 8
    t0 = 1_000_000_000
    for f in files:
        os.utime(f, (t0, t0))
    os.utime(lib, (t0 + 10, t0 + 10))
    assert not libbuild._stale(str(lib), csrc)
    for f in files:
        os.utime(f, (t0 + 20, t0 + 20))
        assert libbuild._stale(str(lib), csrc), f
        os.utime(f, (t0, t0))
    assert not libbuild._stale(str(lib), csrc)
