"""bench.py reports a kernel's DRAM traffic from profiles/traffic.json only
while the recorded hash of that kernel's sources matches the current files
(its .cu file and the shared headers); otherwise the traffic is null."""
import json
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

CSRC = os.path.join("diffusion_transformer_joint_attn_b200", "csrc")


def _copy_tree(tmp_path):
    """A copy of the kernel sources under tmp_path with a traffic record whose
    hashes match them (whether or not the committed record is current)."""
    shutil.copytree(os.path.join(ROOT, CSRC), tmp_path / CSRC)
    (tmp_path / "profiles").mkdir()
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for kernel in bench.KERNEL_SOURCES:
        rec["kernels"][kernel]["source_sha"] = bench.kernel_source_sha(kernel)
    with open(tmp_path / "profiles" / "traffic.json", "w") as f:
        json.dump(rec, f)
    return tmp_path


def test_record_is_consistent_and_reported_only_for_its_sources():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    assert rec["workload"] == bench.WORKLOAD
    for kernel in bench.KERNEL_SOURCES:
        entry = rec["kernels"][kernel]
        assert entry["dram_bytes_per_launch"] == entry["dram_bytes_read_per_launch"] + entry["dram_bytes_write_per_launch"]
        current = entry["source_sha"] == bench.kernel_source_sha(kernel)
        assert bench.profile_traffic(kernel) == (entry["dram_bytes_per_launch"] if current else None), kernel


def test_a_changed_kernel_source_voids_only_its_own_counters(tmp_path, monkeypatch):
    root = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    before = {k: bench.profile_traffic(k) for k in bench.KERNEL_SOURCES}
    assert all(v is not None for v in before.values())
    with open(root / CSRC / "merge.cu", "a") as f:
        f.write("\n// changed\n")
    assert bench.profile_traffic("merge_kernel") is None
    assert bench.profile_traffic("attn_fwd_bf16_kernel") == before["attn_fwd_bf16_kernel"]
    assert bench.profile_traffic("attn_fwd_fp8_kernel") == before["attn_fwd_fp8_kernel"]
    with open(root / CSRC / "quant_fp8.cu", "a") as f:    # not a profiled kernel's file
        f.write("\n// changed\n")
    assert bench.profile_traffic("attn_fwd_bf16_kernel") == before["attn_fwd_bf16_kernel"]


def test_a_changed_shared_header_voids_every_kernel(tmp_path, monkeypatch):
    root = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    with open(root / CSRC / "ptx.cuh", "a") as f:
        f.write("\n// changed\n")
    assert all(bench.profile_traffic(k) is None for k in bench.KERNEL_SOURCES)
