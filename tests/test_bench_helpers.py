"""Host-side helpers of bench.py (no GPU)."""
import pytest

import bench
from self_sparse_speculative_b200.workloads import algorithmic_bytes
from self_sparse_speculative_b200.workloads import Workload, spec


def test_profiled_traffic_is_reported_only_for_the_profiled_workload():
    t = bench.verify_traffic()
    if t is None:
        pytest.skip("the committed verify summary was taken on other kernel sources")
    assert bench.verify_traffic(spec(1).name) == t
    # workload 3 moves the same verify bytes, but its launch was not profiled
    assert algorithmic_bytes(Workload(spec(3), seed=0))["verify"] == \
        algorithmic_bytes(Workload(spec(1), seed=0))["verify"]
    for w in (0, 2, 3, 4):
        assert bench.verify_traffic(spec(w).name) is None


def test_launch_count_per_step():
    # drafter draws, gamma x (select, attention), verify, statistics + normalisers + draw
    assert bench.launches_per_step(spec(1)) == 1 + 2 * 4 + 1 + 3
    assert bench.launches_per_step(spec(1), 1) == 1 + 4 + 1 + 3
    assert bench.launches_per_step(spec(4)) == 1 + 2 * 8 + 1 + 3


def test_source_hash_ignores_comments_and_blank_lines():
    code = "int a;\nint b;"
    assert bench._code_only(code) == code
    assert bench._code_only("int a;   // the first\n\n/* a\n   block */\nint b;  \n") == code
    assert bench._code_only("int a; int c;") != code


def test_source_hash_covers_the_attention_device_code():
    import os
    path = os.path.join(os.path.dirname(bench.__file__), "self_sparse_speculative_b200", "csrc", "s3r_attn_tok.cu")
    text = open(path, encoding="utf-8").read()
    assert bench.HOST_SECTION in text                   # the host launch code follows the kernel
    h = bench.verify_source_hash()
    assert len(h) == 16 and int(h, 16) >= 0
