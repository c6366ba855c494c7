"""The benchmark's algorithmic work per kernel (the numerators of its roofline
fractions), pinned to the closed forms of the method's steps: FLOPs of the six
expert GEMMs and the bytes each HBM-bound kernel must move at least once."""
import bench
from sparse_mixture_experts_smoe_b200.inputs import WORKLOADS


def test_gemm_flops_are_the_method_s():
    cfg = WORKLOADS["mixtral_bf16_swiglu"]
    T, d, f, k = cfg["T"], cfg["d"], cfg["f"], cfg["k"]
    S = T * k
    flops, _ = bench.kernel_work(cfg)
    assert flops["gemm.fwd_up"] == 2.0 * S * d * 2 * f       # x W1 (gate and up)
    assert flops["gemm.fwd_down"] == 2.0 * S * f * d         # A W2
    assert flops["gemm.bwd_dA"] == 2.0 * S * d * f           # dY W2^T
    assert flops["gemm.bwd_dx"] == 2.0 * S * 2 * f * d       # dH W1^T
    assert flops["gemm.bwd_dW1"] == flops["gemm.fwd_up"]
    assert flops["gemm.bwd_dW2"] == flops["gemm.fwd_down"]
    # fwd + bwd = 3 x fwd (the step's 34.64 TFLOP at this shape)
    fwd = flops["gemm.fwd_up"] + flops["gemm.fwd_down"]
    assert abs(sum(flops.values()) - 3 * fwd) < 1e-6 * fwd
    assert abs(3 * fwd / 1e12 - 34.64) < 0.01


def test_hbm_bytes_follow_the_layer_dtype():
    for name, es in (("mixtral_bf16_swiglu", 2), ("tiny_fp32_gelu", 4)):
        cfg = WORKLOADS[name]
        T, d, E, k = cfg["T"], cfg["d"], cfg["E"], cfg["k"]
        S = T * k
        _, b = bench.kernel_work(cfg)
        # router: x and W_r read once, indices and gates written
        assert b["route"] == T * d * es + d * E * es + S * 8
        # combine: every slot row (layer dtype) and its grouped row index read, y written
        assert b["combine.y"] == S * d * es + S * 4 + T * d * es
        assert b["combine.dx"] == b["combine.y"] + S * 8


def test_measured_traffic_needs_the_captured_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu table only while the kernel source
    is the one the counters were taken on (its SHA-256 in the row); any other source,
    workload or kernel gives null."""
    import hashlib
    src = tmp_path / "gemm_tc.cu"
    src.write_text("// kernels\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    table = tmp_path / "traffic.md"
    table.write_text("| workload | kernel | read bytes | write bytes | sha | algorithmic |\n|---|---|---|---|---|---|\n"
                     f"| wl | gemm.bwd_dW1 | 5000 | 300 | {sha} | x |\n")
    monkeypatch.setattr(bench, "KERNEL_SOURCE", str(src))
    monkeypatch.setattr(bench, "TRAFFIC_TABLE", str(table))
    assert bench.measured_traffic("gemm.bwd_dW1", "wl") == 5300
    assert bench.measured_traffic("gemm.bwd_dW2", "wl") is None
    assert bench.measured_traffic("gemm.bwd_dW1", "other") is None
    src.write_text("// kernels, changed\n")
    assert bench.measured_traffic("gemm.bwd_dW1", "wl") is None

