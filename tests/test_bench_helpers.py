"""CPU checks of the measurement helpers behind the bench line: the DRAM traffic of
the dominant kernel is reported only when the committed ncu record was taken on the
same kernel code and the same workload, and the code hash ignores comments."""

import json
import os

import pytest

import bench


def _fake_tree(tmp_path, kernel_src):
    csrc = tmp_path / "h2o_kv_cache_attn_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "include").mkdir()
    (csrc / "k.cu").write_text(kernel_src)
    (tmp_path / "include" / "h.h").write_text("int f(void);\n")
    (tmp_path / "profiles").mkdir()
    return ["k.cu", "../../include/h.h"]


def test_strip_comments():
    src = "int a; // one\n/* two\n three */ int b;\n\n   int c;  /* four */\n"
    assert bench.strip_comments(src) == "int a;\nint b;\nint c;"


def test_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    files = _fake_tree(tmp_path, "__global__ void k() { int x = 1; }\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash(files)
    (tmp_path / "h2o_kv_cache_attn_b200" / "csrc" / "k.cu").write_text(
        "// a kernel\n/* its\n   description */\n__global__ void k() { int x = 1; }  // one\n\n")
    assert bench.kernel_source_hash(files) == h0
    (tmp_path / "h2o_kv_cache_attn_b200" / "csrc" / "k.cu").write_text(
        "__global__ void k() { int x = 2; }\n")
    assert bench.kernel_source_hash(files) != h0


def test_recorded_traffic_requires_same_code_and_workload(tmp_path, monkeypatch):
    files = _fake_tree(tmp_path, "__global__ void k() {}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = {"k": {"bytes_per_launch": 1234, "config": "128k", "sources": files,
                 "source_hash": bench.kernel_source_hash(files)}}
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("k", "128k") == 1234
    assert bench.recorded_traffic("k", "64k") is None        # another workload
    assert bench.recorded_traffic("other", "128k") is None   # no record
    (tmp_path / "h2o_kv_cache_attn_b200" / "csrc" / "k.cu").write_text("__global__ void k() { }\n;")
    assert bench.recorded_traffic("k", "128k") is None       # the kernel's code changed


def test_committed_traffic_record_is_well_formed():
    """Each committed record names its workload and sources; its bytes are the read and
    write counts of one launch (the bench reports it only while the code matches)."""
    with open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        rec = json.load(f)
    assert "attn_fwd_kernel" in rec
    for name, e in rec.items():
        assert e["config"] in bench.SHORT, name
        assert e["sources"] and e["source_hash"], name
        assert e["bytes_per_launch"] == e["dram_bytes_read"] + e["dram_bytes_write"]


@pytest.mark.parametrize("config", ["128k", "64k"])
def test_algorithmic_flops(config):
    wl = bench.SHORT[config]
    n = wl.capacity
    assert bench.alg_flops_chunk(wl, n, wl.chunk) == 4.0 * wl.B * wl.Hq * wl.chunk * n * wl.d
    assert bench.exec_flops_chunk(wl, n, wl.chunk) == 1.5 * bench.alg_flops_chunk(wl, n, wl.chunk)


def test_launch_counts_follow_the_library_rules():
    from h2o_kv_cache_attn_b200.configs import SHORT
    assert bench.evict_launches(0, 0, 100) == 1          # fold only
    assert bench.evict_launches(0, 64, 100) == 2         # filling: fold + rows
    assert bench.evict_launches(64, 64, 100) == 3        # choosing: fold + choose + rows
    wl = SHORT["128k"]
    assert bench.attention_launches(wl, 1024, 32768, 148) == 3  # 128 pairs fill 86 % of a wave
    assert bench.attention_launches(SHORT["tiny"], 128, 256, 148) == 2  # CUDA-core path


def test_stack_flops_and_bytes_scale_with_layers():
    from h2o_kv_cache_attn_b200.configs import SHORT
    wl = SHORT["int4stack"]
    one = bench.evict_bytes_chunk(wl, wl.chunk)
    # per (b, h_k): 12 N_C + 4 S d + 2 S (row + scale) + 8 S bytes
    per = 12 * 32768 + 4 * 2048 * 128 + 2 * 2048 * (64 + 2) + 8 * 2048
    assert one == per * 4 * 8
    assert bench.alg_flops_chunk(wl, 32768, 2048) == 4.0 * 4 * 32 * 2048 * 32768 * 128


def test_eviction_bytes_of_the_named_layers():
    from h2o_kv_cache_attn_b200.configs import SHORT
    # the 128K bf16 layer: 8 groups of 12 N_C + 4 S d + 2 S row + 8 S bytes = 11.6 MB per chunk
    one = bench.evict_bytes_chunk(SHORT["128k"], 1024)
    assert one == (12 * 32768 + 4 * 1024 * 128 + 2 * 1024 * 256 + 8 * 1024) * 8
    assert round(one / 1e6, 1) == 11.6
    # the 36-layer int4 stack: 1152 groups, about 1.99 GB per chunk
    wl = SHORT["int4stack"]
    assert round(bench.evict_bytes_chunk(wl, wl.chunk) * wl.layers / 1e9, 2) == 1.99

