"""The bench's `roofline.traffic` comes from the committed ncu summaries: each
decode summary carries the kernel-source hash it was taken on, the DRAM bytes
of the profiled launch and that launch's algorithmic bytes.  Checked here:
the fields parse, the DRAM/algorithmic ratio is a plausible streaming ratio
(no re-reads), scaling is linear in the launch's bytes, and a workload with no
summary (or a stale hash) reports None instead of a number."""
import re

import bench


def _fields(workload):
    text = open(bench.PROFILE_SUMMARIES[workload]).read()
    get = lambda k: re.search(k + r":\s*([0-9a-f.eE+]+)", text).group(1)  # noqa: E731
    return get("kernel_source_sha"), float(get("dram_bytes_per_launch_full_workload")), \
        float(get("algorithmic_bytes_of_profiled_launch"))


def test_summaries_parse_with_streaming_ratios():
    for w in bench.PROFILE_SUMMARIES:
        sha, dram, alg = _fields(w)
        assert len(sha) == 16
        assert 1.0 <= dram / alg <= 1.05, (w, dram / alg)


def test_traffic_scales_with_the_launch_or_is_none():
    for w in bench.PROFILE_SUMMARIES:
        sha, dram, alg = _fields(w)
        t1 = bench.profiled_traffic(alg, w)
        t2 = bench.profiled_traffic(2 * alg, w)
        if sha != bench.kernel_source_sha():
            assert t1 is None and t2 is None      # stale summary: no number
        else:
            assert t1 == round(dram) and abs(t2 - 2 * dram) <= 1
    assert bench.profiled_traffic(1e9, "long") is None
    assert bench.profiled_traffic(1e9, "no-such-workload") is None
