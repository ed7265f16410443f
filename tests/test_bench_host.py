"""Host-side pieces of bench.py that need no GPU: the CPU baseline of the
parallel-sampling workload stays within the block tables the workload was
sized for (the driver times it with few steps), and both bench arms print
the same config for a workload."""
import bench


def test_cow_cpu_baseline_fits_the_tables_of_a_short_run():
    wl = bench.Workload("cow", "cpu", 0, 3 + 1 + 1)      # --steps 3 --warmup 1
    r = bench.cpu_baseline(wl, 0.3)
    assert r["kind"] == "oracle" and r["value"] > 0


def test_both_arms_share_the_decode_config():
    wl = bench.Workload("13b", "cpu", 0, 5 + 3 + 1)
    a = bench.decode_config(wl, "13b", 1, 5, 3)
    b = bench.decode_config(wl, "13b", 1, 5, 3)
    assert a == b and a["bytes_per_step"] > 0 and "mean_context_len" in a
