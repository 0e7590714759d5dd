"""Host logic of bench.py's report (CPU): the algorithmic FLOP and bytes of
each workload, the roofline branch and arithmetic per kernel, and the rule
that a committed ncu traffic record counts only while its kernel source is
unchanged."""

import hashlib
import json

import pytest

import bench
from transposed_convolution_02_b200.workloads import WORKLOADS

PEAKS = dict(hbm_gbs=6541.8, tc_tflops=1662.5, tc_tflops_sustained=1400.0, sm_max_mhz=1965.0,
             source="test")


@pytest.mark.parametrize("wid,flop,mbytes", [
    # effective FLOP 2*N*C*(M/g)*prod(in)*prod(k); bytes of X + W + bias + Y once
    (1, 36864, 0.0073),
    (2, 34.36e9, 51.4),
    (3, 7.248e9, 42.05),
    (4, 137.4e9, 343.9),
    (5, 7.40e9, 257.05),
])
def test_workload_numbers(wid, flop, mbytes):
    f, b = bench.workload_numbers(WORKLOADS[wid])
    assert f == pytest.approx(flop, rel=2e-3)
    assert b / 1e6 == pytest.approx(mbytes, rel=1e-2)


def test_workload_numbers_by_hand():
    # the 2-D decoder: 2 * 8 * 256 * 128 * 64 * 64 * 16 FLOP; fp16 bytes of
    # X[8,256,64,64] + W[256,128,4,4] + bias[128] + Y[8,128,128,128]
    f, b = bench.workload_numbers(WORKLOADS[2])
    assert f == 2 * 8 * 256 * 128 * 64 * 64 * 16
    assert b == 2 * (8 * 256 * 64 * 64 + 256 * 128 * 16 + 128 + 8 * 128 * 128 * 128)


def test_roofline_branches():
    # tensor-bound fp16 dense: achieved = FLOP / time against the fp16 peak
    f2, _ = bench.workload_numbers(WORKLOADS[2])
    r = bench.roofline_for(WORKLOADS[2], 40e-6, PEAKS, 148, "dense_tc_pair")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(f2 / 40e-6 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1662.5)
    # HBM-bound fp16 (3-D and grouped): algorithmic bytes / time against the copy peak
    for wid in (3, 5):
        _, b = bench.workload_numbers(WORKLOADS[wid])
        r = bench.roofline_for(WORKLOADS[wid], 50e-6, PEAKS, 148, "dense_tc")
        assert r["bound"] == "hbm" and r["unit"] == "GB/s"
        assert r["achieved"] == pytest.approx(b / 50e-6 / 1e9)
        assert r["frac"] == pytest.approx(r["achieved"] / 6541.8)
    # fp32 on the 3xTF32 pair kernel: a third of the TF32 peak (measured bf16 x 1.1/2.25)
    r = bench.roofline_for(WORKLOADS[4], 0.65e-3, PEAKS, 148, "dense_tc_pair")
    assert r["bound"] == "tensor"
    assert r["peak"] == pytest.approx(1662.5 * 1.1 / 2.25 / 3)
    # fp32 on an FFMA kernel: SMs x 128 lanes x 2 FLOP x max clock
    r = bench.roofline_for(WORKLOADS[4], 3.3e-3, PEAKS, 148, "fp32_gemm")
    assert r["bound"] == "alu"
    assert r["peak"] == pytest.approx(148 * 128 * 2 * 1965e6 / 1e12)


def test_traffic_record_needs_unchanged_source(tmp_path, monkeypatch):
    src_dir = tmp_path / "transposed_convolution_02_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = src_dir / "k_x.cu"
    src.write_bytes(b"kernel source v1\n")
    h = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    rec = {"2": {"kernel": "dense_tc_pair", "source": "k_x.cu", "sha256_16": h,
                 "dram_read": 100, "dram_write": 23, "bytes_per_launch": 123}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for(2, "dense_tc_pair") == 123
    assert bench.traffic_for(2, "dense_tc") is None           # another kernel
    assert bench.traffic_for(3, "dense_tc_pair") is None      # another workload
    roof = bench.annotate_roofline(dict(frac=0.4), 2, "dense_tc_pair", 2, nbytes=246)
    assert roof["traffic"] == 123
    assert roof["traffic_detail"] == {"dram_read": 100, "dram_write": 23}
    assert roof["traffic_over_algorithmic"] == pytest.approx(0.5)
    src.write_bytes(b"kernel source v2\n")                     # the kernel changed
    assert bench.traffic_for(2, "dense_tc_pair") is None
    roof = bench.annotate_roofline(dict(frac=0.4), 2, "dense_tc_pair", 2)
    assert roof["traffic"] is None and "traffic_detail" not in roof


def test_kernel_roofline_uses_the_kernel_time():
    """achieved/frac come from the main kernel timed alone; the whole call is
    reported beside it, with both fractions for the fp16 workloads."""
    info = dict(kernel="dense_tc_pair", kernel_ms_per_launch=0.030, prepare_ms_per_call=0.008,
                launches_per_step=2)
    f2, b2 = bench.workload_numbers(WORKLOADS[2])
    r = bench.kernel_roofline(WORKLOADS[2], 2, info, 40e-6, PEAKS, 148)
    assert r["achieved"] == pytest.approx(f2 / 30e-6 / 1e12)
    assert r["kernel_us"] == pytest.approx(30.0) and r["prepare_us"] == pytest.approx(8.0)
    assert r["call"]["us"] == pytest.approx(40.0)
    assert r["call"]["frac"] == pytest.approx(f2 / 40e-6 / 1e12 / 1662.5)
    assert r["call"]["hbm_frac"] == pytest.approx(b2 / 40e-6 / 1e9 / 6541.8)
    info3 = dict(info, kernel="dense_tc")
    f3, b3 = bench.workload_numbers(WORKLOADS[3])
    r = bench.kernel_roofline(WORKLOADS[3], 3, info3, 40e-6, PEAKS, 148)
    assert r["bound"] == "hbm"
    assert r["tensor_frac"] == pytest.approx(f3 / 30e-6 / 1e12 / 1662.5)
