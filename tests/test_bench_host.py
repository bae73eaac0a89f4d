"""Host-side bookkeeping of bench.py (CPU): the byte counts behind the roofline and
the rule that a stored ncu traffic figure is reported only for the kernel sources it
was taken on."""
import json
import os

import torch

import bench
import kimi_delta_attention_28_b200 as kda

BF16 = torch.bfloat16


def test_record_bytes_match_the_library_workspace():
    # one more chunk per sequence adds one record per (sequence, head)
    grow = kda.workspace_size(2, 4096 + 64, 8, 128, 128, 0, BF16) - \
        kda.workspace_size(2, 4096, 8, 128, 128, 0, BF16)
    assert grow == 2 * 8 * bench.record_bytes()


def _tree(root, code):
    src = os.path.join(root, "kimi_delta_attention_28_b200", "csrc")
    os.makedirs(src, exist_ok=True)
    with open(os.path.join(src, "k.cu"), "w") as f:
        f.write(code)
    return src


def test_traffic_is_reported_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    root = str(tmp_path)
    monkeypatch.setattr(bench, "ROOT", root)
    src = _tree(root, "// a kernel\n__global__ void k(int *p) { p[0] = 1; }\n")
    sha = bench.kernel_source_sha()
    os.makedirs(os.path.join(root, "profiles"))
    with open(os.path.join(root, "profiles", "traffic.json"), "w") as f:
        json.dump({"kernel_source_sha256": sha, "per_launch_dram_bytes": {"intra": 123.0}}, f)
    assert bench.load_traffic("intra") == 123.0
    assert bench.load_traffic("decode") is None
    # a comment-only edit keeps the figure ...
    _tree(root, "/* the same kernel */\n__global__ void k(int *p) { p[0] = 1; }  // store\n")
    assert bench.kernel_source_sha() == sha
    assert bench.load_traffic("intra") == 123.0
    # ... a code edit drops it
    _tree(root, "__global__ void k(int *p) { p[0] = 2; }\n")
    assert bench.kernel_source_sha() != sha
    assert bench.load_traffic("intra") is None
    assert os.path.isdir(src)
