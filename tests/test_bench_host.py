"""bench.py's host-side bookkeeping (no GPU): which kernel a workload runs on,
and the source hash that ties a committed ncu summary to the kernel code (a
summary's DRAM traffic is reported only while that hash matches)."""
import pytest

import bench
from neighborhood_attention_na2d_b200.inputs import WORKLOADS


def test_code_only_ignores_comments_and_blank_lines():
    a = "int f(int x) {  // doubles x\n\n    return 2 * x; /* plain */\n}\n"
    b = "/* a block\n   comment */\nint f(int x) {\n    return 2 * x;\n}\n"
    assert bench.code_only(a) == bench.code_only(b)
    assert bench.code_only(a) != bench.code_only(a.replace("2 * x", "3 * x"))


@pytest.mark.parametrize("K", [1, 3, 20, 199, 200, 201, 450, 20000])
def test_graph_plan_times_exactly_k_steps(K):
    """A timed run replays graphs covering exactly --steps steps, at least one
    graph replay (the driver's --steps 20 must replay a graph, not launch
    eagerly)."""
    G, full, rest = bench.graph_plan(K)
    assert 1 <= G <= 200 and 0 <= rest < G
    assert full * G + rest == K
    assert full >= 1


def test_roofline_picks_the_slower_limit():
    wl = WORKLOADS["nat_tiny_s1_fp16"]
    r = bench.roofline(wl, 0.010, None)
    assert r["bound"] == "hbm" and r["t_hbm_us"] > r["t_tensor_us"]
    assert abs(r["achieved"] - wl.shapes[0].algorithmic_bytes() / 1e-5 / 1e9) < 1e-6 * r["achieved"]


def _profile_summaries():
    out = []
    for f in sorted(bench.PROFILES.glob("*.md")):
        kernel = next((k for k in bench.KERNEL_SOURCES if f.stem.startswith(k + "_")), None)
        if kernel is not None:
            out.append((kernel, f.stem[len(kernel) + 1:]))
    return out


@pytest.mark.parametrize("kernel,workload", _profile_summaries(), ids=lambda x: x)
def test_committed_profile_matches_the_kernel_source(kernel, workload):
    """Every committed ncu summary that records a traffic figure was taken on
    the current source of its kernel, so the bench line reports it (a kernel
    change without a new capture would turn the line's traffic to null)."""
    text = (bench.PROFILES / f"{kernel}_{workload}.md").read_text()
    if "traffic_per_launch_bytes" not in text:
        pytest.skip("summary without a traffic figure")
    assert bench.recorded_traffic(kernel, workload) is not None, \
        f"{kernel}_{workload}.md was captured on another source (sha now {bench.kernel_sha(kernel)})"
