"""bench.py reports an ncu summary's DRAM traffic only while the summary was
taken on the current sources of that workload's kernel (CPU, no GPU)."""
import os
import shutil

import bench


def test_each_workload_maps_to_its_kernel_sources():
    assert bench.kernel_sources("prefill_T8189") == bench.WIDE_SOURCES
    assert bench.kernel_sources("decode_T16") == bench.SKINNY_SOURCES
    # the wide kernel does not include the skinny one's files
    assert not set(bench.WIDE_SOURCES) & {"expert_ffn_skinny.cuh", "fp8.cuh", "fp4.cuh"}


def test_traffic_only_for_a_matching_source_sha(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    csrc = tmp_path / "group_limited_routed_moe_b200" / "csrc"
    shutil.copytree(os.path.join(bench.ROOT, "group_limited_routed_moe_b200", "csrc"), csrc,
                    ignore=shutil.ignore_patterns("*.so", "*.o"))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.kernel_source_sha(bench.SKINNY_SOURCES)
    (prof / "expert_ffn_decode_T16.md").write_text(
        f"# x\n\nsource_sha: {sha}\ntraffic_bytes_per_launch: 123456\n")
    assert bench.profiled_traffic("expert_ffn", "decode_T16") == 123456.0
    # a wide-kernel profile is judged against the wide kernel's sources only
    (prof / "expert_ffn_prefill_T8189.md").write_text(
        f"source_sha: {sha}\ntraffic_bytes_per_launch: 1\n")
    assert bench.profiled_traffic("expert_ffn", "prefill_T8189") is None
    # any change to one of the kernel's sources makes the summary stale
    with open(csrc / "fp4.cuh", "a") as f:
        f.write("\n")
    assert bench.profiled_traffic("expert_ffn", "decode_T16") is None
    assert bench.profiled_traffic("expert_ffn_nvfp4", "decode_T16") is None  # no such file


def test_committed_profiles_name_a_sha_and_traffic():
    d = os.path.join(bench.ROOT, "profiles")
    for name in os.listdir(d):
        if not name.startswith("expert_ffn"):
            continue
        text = open(os.path.join(d, name)).read()
        assert "source_sha:" in text and "traffic_bytes_per_launch:" in text, name
