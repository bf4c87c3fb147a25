"""The benchmark's work model (algorithmic FLOPs and bytes per layer call)
against the per-token and per-expert figures the layer's shapes fix."""
import bench
from sigmoid_top_routing_warp_b200 import workloads as W


def test_flops_per_token():
    # 2*k*3*H*I (routed SwiGLU) + 2*3*H*Is (shared) + 2*H*E (router), per token
    d = W.WORKLOADS["decode"]
    per_tok = bench.layer_work(d, touched=100)["flops"] / d.T
    assert abs(per_tok - 427.3e6) / 427.3e6 < 1e-3
    g = W.WORKLOADS["grouped"]
    per_tok = bench.layer_work(g, touched=128)["flops"] / g.T
    assert abs(per_tok - 277.9e6) / 277.9e6 < 1e-3


def test_bytes_per_touched_expert():
    d = W.WORKLOADS["decode"]
    one = bench.layer_work(d, touched=1)["bytes"]
    two = bench.layer_work(d, touched=2)["bytes"]
    assert two - one == 3 * 5120 * 1536 * 2          # 47.19 MB of bf16 weights
    f = W.WORKLOADS["fp8_256"]
    one = bench.layer_work(f, touched=1)["bytes"]
    two = bench.layer_work(f, touched=2)["bytes"]
    # e4m3 codes plus one fp32 scale per 128 x 128 block
    assert abs((two - one) - 3 * 5120 * 1536 * (1 + 4 / 128 ** 2)) < 1e-3


def test_gate_up_share_of_the_stream():
    # the gate/up launch streams two of the three weight matrices of each touched expert
    d = W.WORKLOADS["decode"]
    w1 = bench.layer_work(d, touched=1)["g1_bytes"]
    w2 = bench.layer_work(d, touched=2)["g1_bytes"]
    assert w2 - w1 == 2 * 5120 * 1536 * 2


def test_traffic_record_selection(tmp_path, monkeypatch):
    """profile_traffic: a record counts only while its source hash matches;
    an exact-workload byte count beats a ratio taken on this workload's
    shape, which beats a generic ratio for the kernel."""
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "a.md").write_text(
        "text\n\n    kernel: k1\n    traffic_over_algorithmic: 1.50\n    source_hash: old\n\n"
        "    kernel: k1\n    traffic_over_algorithmic: 1.10\n    source_hash: cur\n")
    (prof / "b.md").write_text(
        "    kernel: k1\n    workload: w2\n    traffic_over_algorithmic: 1.20\n    source_hash: cur\n"
        "\n    kernel: k1\n    workload: w3\n    traffic_bytes_per_launch: 777\n    source_hash: cur\n"
        "\n    kernel: k2\n    traffic_over_algorithmic: 9.0\n    source_hash: cur\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_hash", lambda kind: "cur")
    assert abs(bench.profile_traffic("k1", 100.0, "w1") - 110.0) < 1e-9   # generic ratio
    assert abs(bench.profile_traffic("k1", 100.0, "w2") - 120.0) < 1e-9   # this shape's ratio
    assert bench.profile_traffic("k1", 100.0, "w3") == 777.0               # measured bytes
    assert bench.profile_traffic("k3", 100.0, "w1") is None                # no record
    monkeypatch.setattr(bench, "source_hash", lambda kind: "new")
    assert bench.profile_traffic("k1", 100.0, "w1") is None                # kernel changed


def test_committed_traffic_records_name_known_kernels():
    # every machine-read record under profiles/ names a kernel kind the bench knows
    import os
    import re
    kinds = set(bench.KERNEL_SOURCES)
    for name in os.listdir(os.path.join(bench.ROOT, "profiles")):
        text = open(os.path.join(bench.ROOT, "profiles", name)).read()
        for k in re.findall(r"^    kernel: (\S+)$", text, flags=re.M):
            assert k in kinds, (name, k)
