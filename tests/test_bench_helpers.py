"""CPU checks of the bench's bookkeeping: the algorithmic FLOP and byte counts, the choice of the
tensor peak that matches the sampled clocks, the roofline's choice of bound, the classification of
ncu kernel names and the DRAM-traffic record that the bench reads back (no GPU needed)."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import moe_workloads as W  # noqa: E402


def test_flop_and_byte_counts_of_the_mixtral_layer():
    w = W.WORKLOADS["mixtral_prefill"]
    fl = bench.flops_of(w)
    assert fl["gemm1"] == 4 * 8192 * 4096 * 14336
    assert fl["gemm2"] == 2 * 8192 * 14336 * 4096
    assert fl["router"] == 2 * 4096 * 4096 * 8
    by = bench.bytes_of(w, e_act=8)
    # gate + up weights of all eight experts, x, h written, out zeroed
    assert by["gemm1"] == 2 * 8 * 4096 * 14336 * 2 + 4096 * 4096 * 2 + 8192 * 14336 * 2 \
        + 4096 * 4096 * 4
    assert by["gemm2"] == 8192 * 14336 * 2 + 8 * 14336 * 4096 * 2 + 2 * 4096 * 4096 * 4
    assert by["sparse_map"] == 12 * 8192 + 17 * 4
    # only active experts' weights stream
    assert bench.bytes_of(w, e_act=4)["gemm1"] < by["gemm1"]


def test_tensor_peak_follows_the_clock(monkeypatch):
    monkeypatch.setattr(bench, "peaks", lambda: ({"hbm_gbs": 6000.0, "bf16_tflops": 1600.0,
                                                 "bf16_tflops_sustained": 1400.0}, "measured"))
    near_max = {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0}
    capped = {"sm_mhz": 1400.0, "sm_max_mhz": 1965.0}
    assert bench.tensor_peak("bf16", near_max, 30.0)[0] == 1600.0
    assert bench.tensor_peak("bf16", capped, 0.05)[0] == 1400.0
    assert bench.tensor_peak("bf16", None, 0.05)[0] == 1600.0
    assert bench.tensor_peak("bf16", None, 5.0)[0] == 1400.0
    assert bench.tensor_peak("f32", near_max, 1.0)[0] == 800.0  # tf32 at half the bf16 rate
    assert "burst" in bench.tensor_peak("bf16", near_max, 1.0)[1]


def test_roofline_bound_is_the_longer_ceiling(monkeypatch):
    monkeypatch.setattr(bench, "peaks", lambda: ({"hbm_gbs": 6549.4, "bf16_tflops": 1642.9,
                                                 "bf16_tflops_sustained": 1392.3}, "measured"))
    monkeypatch.setattr(bench, "recorded_traffic", lambda *a, **k: None)
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}
    stage = {"gemm1": 1.0}
    prefill = bench.roofline(W.WORKLOADS["mixtral_prefill"], stage, 8, clocks, 0.05)
    decode = bench.roofline(W.WORKLOADS["mixtral_decode"], stage, 8, clocks, 0.05)
    assert prefill["bound"] == "tensor" and prefill["unit"] == "TFLOP/s"
    assert decode["bound"] == "hbm" and decode["unit"] == "GB/s"
    assert decode["other"]["bound"] == "tensor"
    assert abs(prefill["achieved"] - prefill["flop"] / 1e-3 / 1e12) < 1e-6
    assert abs(decode["frac"] - decode["algorithmic_bytes"] / 1e-3 / 1e9 / 6549.4) < 1e-9


def test_kernel_names_are_classified():
    c = bench.kernel_class
    assert c("void unnamed>::grouped_gemm_kernel<1, 1, 1, 0, 0>(CUtensorMap_st, ...)") == "gemm1"
    assert c("void unnamed>::grouped_gemm_kernel<1, 0, 0, 1, 0>(CUtensorMap_st, ...)") == "gemm2"
    assert c("void unnamed>::grouped_gemm_kernel<1, 0, 0, 0, 1>(CUtensorMap_st, ...)") == "router"
    assert c("void unnamed>::grouped_gemm_2sm_kernel<1, 1, 1, 0>(CUtensorMap_st, ...)") == "gemm1"
    assert c("void unnamed>::grouped_gemm_2sm_kernel<1, 0, 0, 1>(CUtensorMap_st, ...)") == "gemm2"
    # GEMM1 on x rows copied to slot order, and that copy
    assert c("void unnamed>::grouped_gemm_2sm_kernel<1, 0, 1, 0>(CUtensorMap_st, ...)") == "gemm1"
    assert c("void unnamed>::grouped_gemm_kernel<1, 0, 1, 0, 0, 0, 0>(CUtensorMap_st, ...)") == "gemm1"
    assert c("moe::<unnamed>::gather_rows_kernel(const uint4 *, const int *, int, ...)") == "x_copy"
    assert c("void moe::route_e8_kernel<2>(const __nv_bfloat16 *, ...)") == "router"
    assert c("void moe::map_small_kernel(const int *, long, int, ...)") == "sparse_map"
    # the grid map's passes: both assign forms and both scans
    assert c("void unnamed>::map_assign_lane_kernel<16>(const int *, long, ...)") == "sparse_map"
    assert c("void unnamed>::map_assign_warp_kernel<1>(const int *, long, ...)") == "sparse_map"
    assert c("unnamed>::map_scan_rows_kernel(int *, long, int *)") == "sparse_map"
    assert c("unnamed>::map_scan_kernel(int *, long, int *)") == "sparse_map"
    assert c("void at::native::vectorized_elementwise_kernel<4, ...>") is None


def test_traffic_record_round_trip(tmp_path):
    csv_text = (
        '==PROF== Connected to process 1\n'
        '"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream",'
        '"Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit",'
        '"Metric Value"\n')
    rows = [("0", "void unnamed>::grouped_gemm_2sm_kernel<1, 1, 1, 0>(x)", 100, 10, 5000),
            ("1", "void unnamed>::grouped_gemm_2sm_kernel<1, 0, 0, 1>(x)", 60, 6, 3000),
            ("2", "void unnamed>::grouped_gemm_2sm_kernel<1, 1, 1, 0>(x)", 300, 30, 7000)]
    for i, name, rd, wr, ns in rows:
        for metric, val in (("dram__bytes_read.sum", rd), ("dram__bytes_write.sum", wr),
                            ("gpu__time_duration.sum", ns)):
            csv_text += (f'"{i}","1","python","h","{name}","1","7","(352, 1, 1)","(148, 1, 1)",'
                         f'"0","10.0","Command line profiler metrics","{metric}","x","{val}"\n')
    src = tmp_path / "launches.csv"
    src.write_text(csv_text)
    path = str(tmp_path / "traffic.json")
    out = bench.record_traffic(str(src), "mixtral_prefill", "ncu ...", path=path)
    assert out["gemm1"]["dram_bytes_per_launch"] == 220 and out["gemm1"]["launches"] == 2
    assert out["gemm2"]["dram_bytes_per_launch"] == 66
    assert bench.recorded_traffic("gemm1", "mixtral_prefill", path=path) == 220
    assert bench.recorded_traffic("gemm1", "e128", path=path) is None
    # a figure recorded for other sources is not reported
    doc = json.loads(open(path).read())
    doc["entries"]["gemm1@mixtral_prefill"]["sources_sha16"] = "0" * 16
    open(path, "w").write(json.dumps(doc))
    assert bench.recorded_traffic("gemm1", "mixtral_prefill", path=path) is None


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_workload_config_states_the_l2_handling(name):
    w = W.WORKLOADS[name]
    cfg = bench.workload_config(w, 1)
    assert cfg["workload"] == name and cfg["parallelism"] == "replicas1"
    if bench.input_bytes(w) < 2 * bench.L2_BYTES:
        assert "flush" in cfg["l2"]
    else:
        assert "larger than L2" in cfg["l2"]
        assert bench.n_x_buffers(w) * w.S * w.D * bench.elt_bytes(w) > bench.L2_BYTES
