"""Host-side logic of bench.py: which sources each stored DRAM-traffic figure
depends on, and that a figure is withheld once those sources change."""

import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_source_groups_name_existing_files():
    for files in bench.SOURCE_GROUPS.values():
        for f in files:
            assert os.path.exists(os.path.join(ROOT, "full_vocabulary_reverse_b200", "csrc", f)), f


def test_kernel_group_matches_the_defining_file():
    where = {"tc": "tc_kernels.cu", "small": "small_kernels.cu", "topk": "topk_kernels.cu"}
    with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as fh:
        kernels = [k.split("@")[0] for k in json.load(fh)["kernels"]]
    for k in set(kernels):
        src = open(os.path.join(ROOT, "full_vocabulary_reverse_b200", "csrc", where[bench.kernel_group(k)])).read()
        # the library names kernels by role; the tensor-core roles are the
        # fused / gradient kernels, the others are named after their function
        if bench.kernel_group(k) != "tc":
            assert (k + "_kernel") in src, k
        assert where[bench.kernel_group(k)] in bench.SOURCE_GROUPS[bench.kernel_group(k)]


def test_traffic_withheld_when_sources_change(monkeypatch):
    with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as fh:
        d = json.load(fh)
    key = next(iter(d["kernels"]))
    kernel, workload = key.split("@")
    group = bench.kernel_group(kernel)
    monkeypatch.setattr(bench, "source_sha", lambda g: d["source_sha"][g])
    assert bench.traffic_for(kernel, workload) == d["kernels"][key]["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "source_sha", lambda g: "changed" if g == group else d["source_sha"][g])
    assert bench.traffic_for(kernel, workload) is None


def test_every_workload_takes_one_path():
    expected = {"tiny_fp32": "hidden", "qwen_hidden": "hidden", "self_distill": "hidden", "long_prompt": "hidden",
                "teacher_logits": "logits", "logits_pair": "pair", "logits_pair_topk": "topk_pair",
                "topk_hidden": "topk_hidden", "topk_logits": "topk_logits", "multi_teacher": "multi",
                "qwen_hidden_stats": "stats"}
    assert set(expected) == set(bench.WORKLOADS)
    for name, cfg in bench.WORKLOADS.items():
        path = bench.path_of(cfg)
        assert path in bench.PATHS and path == expected[name], (name, path)
        # sampled tokens are drawn exactly for the paths that read them
        assert (cfg.get("targets") is not None) == (path in ("topk_pair", "topk_hidden", "topk_logits", "stats")), name
