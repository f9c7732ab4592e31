"""bench.py's use of the committed ncu summaries and its L2 flush.

roofline.traffic comes from the summary of the kernel a workload's
attention runs, and only while that kernel's sources hash to the value the
summary records: a missing summary or a changed kernel reports no traffic.
"""

import bench


def _summary(path, sha, dram_bytes):
    path.write_text("# capture\n\n"
                    f"- workload: test workload\n- kernel_source_sha256: `{sha}`\n"
                    f"- dram_bytes_per_launch: {dram_bytes}\n")


def test_traffic_only_while_the_sources_match(tmp_path):
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel v1\n")
    prof = tmp_path / "prof.md"
    _summary(prof, bench.kernel_source_hash([str(src)]), 123456789)
    traffic, note = bench.profiled_traffic(str(prof), [str(src)])
    assert traffic == 123456789.0 and note == "test workload"
    src.write_text("// kernel v2\n")
    traffic, note = bench.profiled_traffic(str(prof), [str(src)])
    assert traffic is None and "changed" in note


def test_missing_capture_reports_no_traffic(tmp_path):
    traffic, note = bench.profiled_traffic(str(tmp_path / "none.md"), [bench.__file__])
    assert traffic is None and note == "no committed capture"


def test_default_workload_summary_is_for_the_kernel_it_times():
    # routed d = 128 launches run the one-query-tile kernel (tm_attn3.cu);
    # the INT8-cache workload the two-query-tile kernel after the expansion
    assert [p.rsplit("/", 1)[-1] for p in bench.KERNEL_SOURCES] == ["tm_attn3.cu", "tm_device.cuh"]
    assert [p.rsplit("/", 1)[-1] for p in bench.CACHE_SOURCES] == ["tm_attn2.cu", "tm_device.cuh",
                                                                  "tm_cache_expand.cu"]


def test_flush_writes_and_reads_back_its_buffer():
    import torch
    buf = torch.full((1 << 12,), 7, dtype=torch.uint8)
    bench.flush_l2(buf)
    assert int(buf.max()) == 0
