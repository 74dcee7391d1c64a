"""Host-side pieces of bench.py: the algorithmic byte count the roofline
divides by, the parser of ncu's raw CSV that records a path's DRAM traffic,
and the rule that a record counts only while its kernels' sources are
unchanged. No GPU."""
import csv
import json
import os

import bench
import ssd_inputs as si


def test_algorithmic_bytes_of_the_130m_shape():
    # per token: x read once and out written once (24 x 64 bf16 each), dt of
    # both directions (2 x 24 bf16), B and C of both directions (4 x 24 x 128
    # bf16): 30 816 bytes; plus A and D (2 x 24 fp32 each)
    w = si.WORKLOADS["mixer130m_b32_L1024"]
    assert bench.algorithmic_bytes(w) == 32 * 1024 * 30816 + 4 * 4 * 24 == 1009779072


def test_every_path_names_existing_sources_and_kernels():
    csrc = os.path.join(bench.ROOT, "bidirectional_mamba_ssd_b200", "csrc")
    for path, files in bench.KERNEL_SOURCE.items():
        for f in files:
            assert os.path.exists(os.path.join(csrc, f)), (path, f)
        assert bench.KERNEL_NAMES[path], path
        assert len(bench.kernel_source_sha(path)) == 16


def _raw_csv(tmp_path, rows):
    p = tmp_path / "raw.csv"
    with open(p, "w", newline="") as f:
        w = csv.writer(f)
        w.writerow(["ID", "Kernel Name", "dram__bytes_read.sum", "dram__bytes_write.sum"])
        w.writerow(["", "", "Mbyte", "Gbyte"])
        for r in rows:
            w.writerow(r)
    return str(p)


def test_record_traffic_sums_one_call_and_expires_with_the_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "traffic.json"))
    # two calls of the segmented path: each launches the fused kernel three
    # times and the segment scan once
    rows = []
    for _ in range(2):
        rows += [[0, "void ssd::tc_fused_kernel<128, 2, 0, 0>(CUtensorMap_st, ...)", "1,202.4", "0.003"],
                 [1, "void ssd::tc_fused_kernel<128, 3, 0, 0>(CUtensorMap_st, ...)", "202.4", "0"],
                 [2, "ssd::seg_scan_kernel(const float *, ...)", "8.4", "0"],
                 [3, "void ssd::tc_fused_kernel<128, 1, 0, 0>(CUtensorMap_st, ...)", "806.1", "0.07"]]
    csv_path = _raw_csv(tmp_path, rows)
    bench.record_traffic(csv_path, "segmented", "long_L16384", "ncu ...", scale=2.0, note="scaled")
    d = json.load(open(bench.TRAFFIC_FILE))
    e = d["long_L16384:segmented"]
    # reads in Mbyte (with a thousands separator), writes in Gbyte
    per_call = 1202.4e6 + 0.003e9 + 202.4e6 + 8.4e6 + 806.1e6 + 0.07e9
    assert e["calls_captured"] == 2
    assert e["dram_bytes_per_launch"] == round(per_call * 2.0)
    assert e["scaled"] == {"factor": 2.0, "note": "scaled"}
    assert bench.traffic_record("segmented", "long_L16384") == e["dram_bytes_per_launch"]
    # a record taken on other sources no longer counts
    e["source_sha"] = "0" * 16
    json.dump(d, open(bench.TRAFFIC_FILE, "w"))
    assert bench.traffic_record("segmented", "long_L16384") is None
    assert bench.traffic_record("fused", "no_such_workload") is None


def test_record_traffic_takes_the_segments_kernel_that_ran(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "traffic.json"))
    # one call whose last step ran the two-CTA kernel
    rows = [[0, "void ssd::tc_fused_kernel<128, 2, 0, 0>(CUtensorMap_st, ...)", "200", "0"],
            [1, "void ssd::tc_fused_kernel<128, 3, 0, 0>(CUtensorMap_st, ...)", "200", "0"],
            [2, "ssd::seg_scan_kernel(const float *, ...)", "8", "0"],
            [3, "void ssd::tc_pair_kernel<128>(CUtensorMap_st, ...)", "800", "0.07"]]
    bench.record_traffic(_raw_csv(tmp_path, rows), "segmented", "long_L65536", "ncu ...")
    e = json.load(open(bench.TRAFFIC_FILE))["long_L65536:segmented"]
    assert e["calls_captured"] == 1
    assert e["kernels"] == ["tc_fused_kernel", "seg_scan_kernel", "tc_pair_kernel"]
    assert e["dram_bytes_per_launch"] == round(1208e6 + 0.07e9)


def test_whole_job_throughput_and_time_at_one_rank():
    assert bench.job_time_ms(3.5, 1) == 3.5
    assert bench.job_throughput(1000, 4, 1, 2.0) == 1000 * 4 / 2e-3


def test_intra_chunk_flops_of_the_130m_shape():
    # per direction, head and 256-token chunk: 256 * 257 / 2 lower-triangle
    # entries, each a d_state (128) and a headdim (64) multiply-add: 2 flops
    w = si.WORKLOADS["mixer130m_b32_L1024"]
    per_chunk = 256 * 257 // 2 * 2 * (128 + 64)
    assert bench.intra_chunk_flops(w) == 2 * 24 * (32 * 4) * per_chunk == 77611401216


def test_roofline_takes_the_slower_bound():
    peaks = {"hbm_gbs": 6451.5, "bf16_tflops": 1713.8, "source": "measured"}
    # per-head B/C: 1.01 GB at the copy bandwidth (156 us) outweighs 77.6
    # GFLOP at the tensor peak (45 us)
    r = bench.roofline_bound(si.WORKLOADS["mixer130m_b32_L1024"], 260e-6, peaks)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["frac"] - 1009779072 / 260e-6 / 1e9 / 6451.5) < 1e-4
    # B/C shared by all heads: 0.238 GB (37 us) is now below the same FLOPs (45 us)
    r = bench.roofline_bound(si.WORKLOADS["mixer130m_b32_L1024_g1"], 292.5e-6, peaks)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["frac"] - 77611401216 / 292.5e-6 / 1e12 / 1713.8) < 1e-4
    assert 0.15 < r["frac"] < 0.16
