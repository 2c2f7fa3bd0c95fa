"""Host-side logic of bench.py that needs no GPU."""
import os
import shutil

import bench

SOURCES = ("kv_cache_early_art_b200/csrc/art_kernels.cuh", "kv_cache_early_art_b200/csrc/art_ptx.cuh",
           "kv_cache_early_art_b200/csrc/art_api.cu")


def _copy_sources(tmp_path):
    for rel in SOURCES:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(bench.ROOT, rel), dst)


def test_kernel_hash_ignores_comments_not_code(tmp_path, monkeypatch):
    """An ncu record stays valid across comment edits and is voided by a code edit."""
    _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    k = tmp_path / SOURCES[0]
    src = k.read_text()
    k.write_text("// a new comment line\n\n/* and a block\n   comment */\n" + src.replace("\n", "  // trailing\n", 3))
    assert bench.kernel_source_hash() == h0
    k.write_text(src.replace("kMinWindow = 8", "kMinWindow = 9", 1))
    assert bench.kernel_source_hash() != h0
