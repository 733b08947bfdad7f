"""The build step's staleness rule (CPU): the library is rebuilt whenever the
recorded sha256 of its inputs (CUDA sources and headers, the public header,
the peak microbenchmark, the build script, the flags) differs from the
current one, whatever the files' modification times say."""
import os
import shutil

from sparse_activation_quantization_b200 import build as B


def test_hash_covers_flags():
    assert B.source_hash() == B.source_hash()
    assert B.source_hash() != B.source_hash(extra=("-DSHARQ_TRACE",))


def test_hash_covers_every_cuda_source(tmp_path, monkeypatch):
    csrc = tmp_path / "csrc"
    shutil.copytree(B.CSRC, csrc, ignore=shutil.ignore_patterns("*.o", "*.so"))
    monkeypatch.setattr(B, "CSRC", str(csrc))
    h0 = B.source_hash()
    for name in sorted(os.listdir(csrc)):
        if not name.endswith((".cu", ".cuh", ".h")):
            continue
        p = csrc / name
        text = p.read_bytes()
        p.write_bytes(text + b"\n")          # a one-byte edit
        assert B.source_hash() != h0, name
        p.write_bytes(text)
        assert B.source_hash() == h0, name


def test_stale_unless_the_stamp_matches(tmp_path, monkeypatch):
    lib, peak, stamp = tmp_path / "libsharq.so", tmp_path / "libsharq_peak.so", tmp_path / "libsharq.so.sha256"
    monkeypatch.setattr(B, "LIB", str(lib))
    monkeypatch.setattr(B, "PEAK_LIB", str(peak))
    monkeypatch.setattr(B, "STAMP", str(stamp))
    digest = B.source_hash()
    assert B._stale(digest)                  # nothing built yet
    lib.write_bytes(b"x")
    peak.write_bytes(b"x")
    assert B._stale(digest)                  # a library with no stamp (e.g. copied in) is not trusted
    stamp.write_text(digest + "\n")
    assert not B._stale(digest)
    assert B._stale(B.source_hash(extra=("-G",)))
    stamp.write_text("0" * 64 + "\n")        # built from other sources, even if newer on disk
    os.utime(lib, None)
    assert B._stale(digest)
    peak.unlink()
    stamp.write_text(digest + "\n")
    assert B._stale(digest)                  # the peak library is part of the build
