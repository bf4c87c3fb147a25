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
