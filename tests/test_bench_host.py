"""The benchmark's host arithmetic, on CPU: algorithmic byte counts, the
launch count it claims, the config object both arms print, and the rule
that reads the combine's DRAM traffic from the committed ncu summary."""

import numpy as np

import bench
import oracle
import workloads as W


def test_v3_byte_counts_follow_from_the_layout():
    w = W.WORKLOADS["v3"]
    inp = W.make_inputs(w, seed=0)
    lay = oracle.layout(inp["topk_idx"], w.E, w.S, w.align)
    V = int(lay["counts"].sum())
    R = int(lay["R"])
    P = R - V
    assert (V, P) == (65536, 15232)            # top-8 of 256 distinct experts, alignment 128
    nb = bench.step_bytes(w, w.T, V, P, R)
    H, k, B = w.H, w.k, w.H // 128
    # read x once + the slot map; write every valid and padding row with its scales
    assert nb["dispatch"] == w.T * (H * 2 + k * 4) + (V + P) * (H + 4 * B) == 714_739_712
    # read each valid y row; write each token's output; read slot map and weights
    assert nb["combine"] == V * H * 2 + w.T * (H * 2 + k * 8) == 1_057_488_896


def test_bf16_byte_counts():
    w = W.WORKLOADS["tiny"]
    nb = bench.step_bytes(w, 128, 200, 0, 200)
    assert nb["dispatch"] == 128 * (256 * 2 + 2 * 4) + 200 * 256 * 2


def test_launch_count_rule_matches_the_layout_chunking():
    # one chunk holds 1024 slots of whole tokens: 1024 // k tokens
    assert bench.layout_launches(128, 8) == 1          # decode: T*k = 1024
    assert bench.layout_launches(129, 8) == 2
    assert bench.layout_launches(8192, 8) == 2
    assert bench.layout_launches(341, 3) == 1 and bench.layout_launches(342, 3) == 2


def test_both_arms_print_the_same_config():
    w = W.WORKLOADS["v3"]
    c = bench.step_config(w, w.T, 1)
    assert c["T"] == 8192 and c["hidden"] == 7168 and c["topk"] == 8 and c["alignment"] == 128
    assert c["parallelism"] == "replicas1" and c["dispatch"] == "bf16 -> e4m3 1x128"
    assert bench.step_config(w, w.T, 4)["parallelism"] == "replicas4"


def test_combine_traffic_is_read_only_for_the_profiled_source_and_workload():
    t = bench.combine_traffic("v3", 8192)
    assert t is None or t > 900_000_000         # present while combine.cu is the profiled source
    assert bench.combine_traffic("v3", 2048) is None
    assert bench.combine_traffic("mid", 8192) is None


def test_combine_traffic_comes_from_the_json_record(tmp_path, monkeypatch):
    # the record is machine-readable: read + write bytes, keyed by the kernel
    # source's sha256 prefix, the workload and T
    import hashlib
    import json
    import os
    src = tmp_path / "combine_ep_get_06_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "combine.cu").write_bytes(b"// some kernel\n")
    sha = hashlib.sha256(b"// some kernel\n").hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    rec = {"combine_kernel": {"workload": "v3", "T": 8192, "source_sha16": sha,
                              "dram_read_bytes": 940, "dram_write_bytes": 65}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.combine_traffic("v3", 8192) == 1005
    (src / "combine.cu").write_bytes(b"// changed\n")           # kernel changed since the capture
    assert bench.combine_traffic("v3", 8192) is None
    assert os.path.exists(tmp_path / "profiles" / "traffic.json")


def test_line_labels():
    # the arithmetic the path computes in, not a precision claim
    assert "e4m3" in bench.DTYPE and "f32" in bench.DTYPE


def test_weak_scaling_sums_bytes_over_ranks():
    assert np.isclose(bench.weak_scaling_gbs(1_000_000_000, 4, 2.0), 4 * 1.0 / 2e-3)
