"""Host logic of bench.py on the CPU: the algorithmic byte and flop counts behind the roofline
lines, the recorded ncu traffic and its source digests, and the small-case batch override."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench      # noqa: E402
import workload   # noqa: E402


@pytest.fixture(autouse=True)
def no_batch_override():
    bench.BATCH = None
    yield
    bench.BATCH = None


def test_backward_bytes_and_flops_of_the_t4k_workload():
    wl, _ = bench.rank_workload("bwd_t4k", 0)
    units = 8 * 16 * 4096
    # reads: q, k, v, b, w, dO bf16 (2 B x 128 each) and g fp32 (4 B x 128); writes: dq, dk,
    # dv, db, dw bf16 and dg fp32; three fp32 states per head (S0, dS_T, dS0)
    per_tok = (6 * 128 * 2 + 128 * 4) + (5 * 128 * 2 + 128 * 4)
    assert bench.bwd_bytes(wl) == units * per_tok + 8 * 16 * 3 * 128 * 128 * 4
    assert abs(bench.bwd_bytes(wl) - 2.038e9) < 1e6
    # tensor products: 22 d^2 + 40 C d per token-head at C = 64
    assert bench.bwd_flops(wl) == units * (22 * 128 * 128 + 40 * 64 * 128)


def test_forward_flops_and_bytes_of_the_t4k_workload():
    wl, mode = bench.rank_workload("gdn2_t4k", 0)
    assert bench.chunk_flops(wl) == 8 * 16 * 4096 * (6 * 128 * 128 + 10 * 64 * 128)
    assert 1.08e9 < bench.chunk_bytes(wl, mode) < 1.10e9   # every input once, o and S_T written


def test_recorded_traffic_is_tied_to_the_sources_it_was_taken_from():
    for (name, kname), (value, digest) in bench.TRAFFIC.items():
        assert value > 0 and len(digest) == 8
    # a digest that no longer matches the kernel's sources gives no figure
    saved = dict(bench.TRAFFIC)
    try:
        key = ("gdn2_t4k", "chunk_tc")
        bench.TRAFFIC[key] = (saved[key][0], "00000000")
        assert bench.traffic_for("gdn2_t4k", "gdr chunk_tc_kernel (tcgen05)") is None
    finally:
        bench.TRAFFIC.clear()
        bench.TRAFFIC.update(saved)
    # the CUDA-core and split kernels have no recorded figure
    assert bench.traffic_for("gdn2_t4k", "gdr chunk_simt_kernel") is None
    assert bench.traffic_for("gdn2_t16k", "gdr chunk_tc_kernel x2 + split_combine_kernel") is None


def test_batch_override_shrinks_the_workload_and_drops_the_traffic_figure():
    full, _ = bench.rank_workload("bwd_t4k", 0)
    bench.BATCH = 1
    small, _ = bench.rank_workload("bwd_t4k", 0)
    assert (small.B, small.H, small.T) == (1, full.H, full.T)
    assert small.units * full.B == full.units
    assert bench.config_of("bwd_t4k", 1)["B"] == 1
    assert bench.traffic_for("bwd_t4k", "x") is None


def test_backward_line_names_its_roof_and_chunk():
    assert bench.metric_name("bwd_t4k").endswith("% HBM roofline")
    cfg = bench.config_of("bwd_t4k", 1)
    assert cfg["chunk"] == 64 and cfg["workload"] == "bwd_t4k" and cfg["parallelism"] == "replicas1"
    assert workload.CONFIGS["gdn2_t4k"].dk == 128


def test_two_phase_steps_report_their_recorded_traffic():
    k16 = "gdr wy_prep_kernel + wy_exact_kernel + state_pass_kernel x2 + split_combine_kernel (two-phase, 6 segments)"
    k2 = "gdr wy_prep_kernel + wy_exact_kernel + state_pass_kernel (two-phase)"
    assert bench.traffic_for("gdn2_t16k", k16) == bench.TRAFFIC[("gdn2_t16k", "two_phase")][0]
    assert bench.traffic_for("gdn_t2k", k2) == bench.TRAFFIC[("gdn_t2k", "two_phase")][0]
    assert bench.traffic_for("gdn2_t16k_kda", k16) is None   # not captured


def test_clock_sampler_waits_for_its_first_sample(monkeypatch):
    # a stand-in for nvidia-smi that starts slowly, then prints one sample every 100 ms: the
    # sampler returns from its entry only once the first sample is in, and keeps it
    import subprocess
    import time
    fake = [sys.executable, "-c",
            "import time\ntime.sleep(0.3)\nwhile True:\n"
            " print('0, 1965, 1965, 700.0, 0x4, Not Active, Not Active, Not Active, Active', flush=True)\n"
            " time.sleep(0.1)"]
    real = subprocess.Popen
    monkeypatch.setattr(bench.subprocess, "Popen", lambda cmd, **kw: real(fake, **kw))
    t0 = time.time()
    with bench.ClockSampler(0) as clk:
        entered = time.time() - t0
    assert entered >= 0.25
    s = clk.summary()
    assert s["sm_mhz"] == 1965.0 and s["samples"] >= 1 and s["reasons"] == ["sw_power_cap"]
