"""bench.py's host-side bookkeeping (no GPU): which kernel a workload runs on,
and the source hash that ties a committed ncu summary to the kernel code (a
summary's DRAM traffic is reported only while that hash matches)."""
import bench
from neighborhood_attention_na2d_b200.inputs import WORKLOADS


def test_code_only_ignores_comments_and_blank_lines():
    a = "int f(int x) {  // doubles x\n\n    return 2 * x; /* plain */\n}\n"
    b = "/* a block\n   comment */\nint f(int x) {\n    return 2 * x;\n}\n"
    assert bench.code_only(a) == bench.code_only(b)
    assert bench.code_only(a) != bench.code_only(a.replace("2 * x", "3 * x"))


def test_dominant_kernel_per_workload():
    assert bench.dominant_kernel(WORKLOADS["nat_tiny_s1_fp16"]) == "fwd_stream_kernel"
    assert bench.dominant_kernel(WORKLOADS["dinat_s1_bf16"]) == "fwd_umma_kernel"
