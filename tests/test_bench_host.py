"""Host-side pieces of bench.py (CPU only): the traffic table and its source guard."""
import bench


def test_traffic_scales_with_layers_and_needs_matching_sources(monkeypatch):
    h = bench.kernel_hash("stack_program_kernel")
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", {"w-stack": (h, 1000, 2), "w-lin": (h, 500, 0),
                                                    "w-old": ("0" * 16, 1000, 2)})
    assert bench.measured_traffic("w-stack", "stack_program_kernel", 80) == 40000
    assert bench.measured_traffic("w-lin", "stack_program_kernel", 0) == 500
    assert bench.measured_traffic("w-old", "stack_program_kernel", 80) is None   # sources changed
    assert bench.measured_traffic("w-none", "stack_program_kernel", 80) is None


def test_recorded_traffic_is_plausible():
    # every recorded figure is within 10% of the workload's algorithmic bytes per launch
    for name, (src, nbytes, layers) in bench.MEASURED_TRAFFIC.items():
        model, bpw, kind = bench.WORKLOADS[name][:3]
        if kind == "stack":
            from binary_rank_linear_lb_b200.configs import MODELS
            algo = MODELS[model].bytes_per_token(bpw, layers)
        else:
            from binary_rank_linear_lb_b200.configs import linear_bytes, rank_for
            (i, o), M = model, bench.WORKLOADS[name][3]
            r = rank_for(bpw, i, o)
            algo = linear_bytes(i, o, r) + M * i * 2 + M * o * 4
        assert 0.8 * algo < nbytes < 1.1 * algo, (name, nbytes, algo)


def test_kernel_hash_covers_the_sources():
    assert bench.kernel_hash("stack_program_kernel") == bench.kernel_hash("linear_program_kernel")
    assert bench.kernel_hash("stack_program_kernel") != bench.kernel_hash("prefill_gemm_kernel")
