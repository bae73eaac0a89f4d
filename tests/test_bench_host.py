"""Host-side bookkeeping of bench.py (CPU): the byte counts behind the roofline and
the rule that a stored ncu traffic figure is reported only for the kernel sources it
was taken on."""
import json
import os

import pytest
import torch

import bench
import kimi_delta_attention_28_b200 as kda

BF16 = torch.bfloat16


def test_record_bytes_match_the_library_workspace():
    # one more chunk per sequence adds one record and one 4-byte ready flag per
    # (sequence, head)
    grow = kda.workspace_size(2, 4096 + 64, 8, 128, 128, 0, BF16) - \
        kda.workspace_size(2, 4096, 8, 128, 128, 0, BF16)
    assert grow == 2 * 8 * (bench.record_bytes() + 4)


def _tree(root, code, name="k.cuh"):
    src = os.path.join(root, "kimi_delta_attention_28_b200", "csrc")
    os.makedirs(src, exist_ok=True)
    with open(os.path.join(src, name), "w") as f:
        f.write(code)
    return src


def test_traffic_is_reported_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    root = str(tmp_path)
    monkeypatch.setattr(bench, "ROOT", root)
    monkeypatch.setattr(bench, "KERNEL_SOURCES", {"prep": ("k.cuh", "c.cuh"),
                                                  "decode": ("d.cuh", "c.cuh")})
    src = _tree(root, "// a kernel\n__global__ void k(int *p) { p[0] = 1; }\n")
    _tree(root, "__device__ int c() { return 0; }\n", name="c.cuh")
    _tree(root, "__global__ void d(int *p) { p[0] = 3; }\n", name="d.cuh")
    sha, sha_d = bench.kernel_source_sha("prep"), bench.kernel_source_sha("decode")
    os.makedirs(os.path.join(root, "profiles"))
    with open(os.path.join(root, "profiles", "traffic.json"), "w") as f:
        json.dump({"source_sha256": {"prep": sha, "decode": sha_d},
                   "dram_bytes_per_unit": {"prep": 1.5, "decode": 4.0}}, f)
    assert bench.load_traffic("prep", 100) == 150.0      # per-unit figure x units
    assert bench.load_traffic("decode", 10) == 40.0
    assert bench.load_traffic("other", 100) is None
    # a comment-only edit keeps the figure ...
    _tree(root, "/* the same kernel */\n__global__ void k(int *p) { p[0] = 1; }  // store\n")
    assert bench.kernel_source_sha("prep") == sha
    assert bench.load_traffic("prep", 2) == 3.0
    # ... so does host-side code (launch policy) beside the kernels ...
    _tree(root, "int policy() { return 2; }\n", name="api.cu")
    assert bench.kernel_source_sha("prep") == sha
    # ... a code edit of one kernel's header drops its figure, not the other's ...
    _tree(root, "__global__ void k(int *p) { p[0] = 2; }\n")
    assert bench.kernel_source_sha("prep") != sha
    assert bench.load_traffic("prep", 2) is None
    assert bench.load_traffic("decode", 10) == 40.0
    # ... and an edit of the shared header drops both
    _tree(root, "__device__ int c() { return 1; }\n", name="c.cuh")
    assert bench.load_traffic("decode", 10) is None
    assert os.path.isdir(src)


def test_compulsory_bytes_follow_the_method_not_the_records():
    """1,540 B per token-head (q, k, v bf16, g fp32, beta, o bf16) plus each state once
    (read if given, written always); the records are counted apart."""
    from kimi_delta_attention_28_b200 import workloads as W
    inp = W.make_prefill_inputs(2, 128, 3, 128, 128, BF16, True, seed=1)
    A = bench.algorithmic(W.PREFILL, inp)
    units = 2 * 128 * 3
    assert A["units"] == units and A["per_unit_compulsory"] == 1540
    assert A["compulsory"] == units * 1540 + 2 * (2 * 3 * 128 * 128 * 4)
    assert A["prep_compulsory"] + A["state_compulsory"] == A["compulsory"]
    assert A["intermediate"] == 2 * units * bench.record_bytes() / 64
    inp0 = W.make_prefill_inputs(1, 64, 2, 128, 128, BF16, False, seed=1)
    A0 = bench.algorithmic(W.LONG, inp0)
    assert A0["compulsory"] == 64 * 2 * 1540 + 2 * 128 * 128 * 4     # final states only


def test_headline_workload_is_the_largest_single_gpu_prefill():
    from kimi_delta_attention_28_b200 import workloads as W
    assert bench.HEADLINE == "long" and bench.workload_of(bench.HEADLINE) is W.LONG
    assert bench.default_steps("long") >= 3


@pytest.mark.parametrize("name", ["prefill", "profile"])
def test_reference_arm_config_from_shapes_alone(name):
    """The reference arm reports the whole workload's config from shape-only (meta)
    tensors, drawing only its sample: the config must equal the GPU arm's."""
    import bench
    from kimi_delta_attention_28_b200 import workloads as W
    w = bench.workload_of(name)
    real = W.make_workload(w, "cpu")
    assert bench.prefill_config(w, bench.workload_shapes(w), 1) == bench.prefill_config(w, real, 1)
    shapes = bench.workload_shapes(bench.workload_of("long"))
    assert tuple(shapes["q"].shape) == (1, 1 << 20, 16, 128) and shapes["q"].device.type == "meta"
