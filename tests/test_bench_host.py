"""Host-side logic of bench.py that needs no GPU."""
import os
import shutil

import bench

SOURCES = ("kv_cache_early_art_b200/csrc/art_kernels.cuh", "kv_cache_early_art_b200/csrc/art_ptx.cuh",
           "kv_cache_early_art_b200/csrc/art_api.cu", "kv_cache_early_art_b200/csrc/art_host.h",
           "kv_cache_early_art_b200/build.py", "kv_cache_early_art_b200/csrc/art_walk.h",
           "kv_cache_early_art_b200/csrc/art_walk_dl.cuh", "kv_cache_early_art_b200/csrc/art_walk_gr.cuh",
           "kv_cache_early_art_b200/csrc/art_walk_f32.cu", "kv_cache_early_art_b200/csrc/art_walk_bf16.cu",
           "kv_cache_early_art_b200/csrc/art_walk_mma.cu", "kv_cache_early_art_b200/csrc/art_walk_multi.cu")


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


def test_kernel_hash_covers_build_flags_and_host_header(tmp_path, monkeypatch):
    """A different nvcc flag or a change of the host header the walk is built
    with voids the record; a docstring or comment edit in the build script
    does not."""
    _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    b = tmp_path / SOURCES[4]
    src = b.read_text()
    b.write_text('"""another docstring"""\n# a comment\n' + src)
    assert bench.kernel_source_hash() == h0
    b.write_text(src.replace('"-O3"', '"-O2"', 1))
    assert bench.kernel_source_hash() != h0
    b.write_text(src)
    hh = tmp_path / SOURCES[3]
    hh.write_text(hh.read_text() + "\ninline int extra_helper() { return 1; }\n")
    assert bench.kernel_source_hash() != h0


def test_oracle_sample_is_bounded():
    """The CPU baseline times groups of sequences until its budget passes,
    never a whole large batch at once."""
    from kv_cache_early_art_b200.workloads import make_custom
    w = make_custom(B=5, Hq=8, Hkv=2, d=32, page=8, dtype="f32", seq_lens=[40, 9, 64, 1, 30], seed=3)
    qps, used, done, el = bench.time_oracle(w, 0.05, ncores=3)
    assert used == 3 and done >= 2 and qps > 0
    g = bench.sequences(w, [1, 3])
    assert g.B == 2 and g.seq_lens.tolist() == [9, 1]


def test_seq_len_override_keeps_the_shape():
    """bench.py --seq-len builds a smaller case of the same workload (for
    profiling): the same batch, heads, page size and parameters, the new
    length, its own name; a ragged workload refuses it."""
    import pytest
    from kv_cache_early_art_b200.workloads import make_workload
    w = make_workload("tiny_fp32")
    s = make_workload("tiny_fp32", seq_len=256)
    assert (s.B, s.Hq, s.Hkv, s.d, s.page) == (w.B, w.Hq, w.Hkv, w.d, w.page)
    assert s.name == "tiny_fp32_L256" and int(s.seq_lens.max()) == 256
    assert int(s.n_blocks().max()) == 256 // s.page
    assert w.uniform_params() == s.uniform_params()
    with pytest.raises(ValueError):
        make_workload("mistral7b_b128", seq_len=1024)
