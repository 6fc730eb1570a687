"""Host-side logic of bench.py on the CPU: the DRAM-traffic records (ncu CSV
parsing, kernel filter, unit conversion, invalidation when the kernel
sources change), the clock-sample summary over the timed windows, the
algorithmic operation count the TOPS figures divide by, and which forward
launches are grouped."""
import datetime
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparsity_sbl_quantize_b200 import workloads as wl  # noqa: E402

HEADER = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size",'
          '"Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"\n')


def _row(launch, kernel, metric, unit, value):
    return (f'"{launch}","1","python3","host","{kernel}","1","7","(256, 1, 1)","(160, 1, 1)","0","10.0",'
            f'"Command line profiler metrics","{metric}","{unit}","{value}"\n')


def _csv(path, rows):
    with open(path, "w") as f:
        f.write("==PROF== Connected to process 1\n")  # ncu's own lines are skipped
        f.write(HEADER)
        f.writelines(rows)


@pytest.fixture
def traffic_file(tmp_path, monkeypatch):
    path = tmp_path / "roofline_traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    return path


def test_record_traffic_filters_kernels_and_converts_units(tmp_path, traffic_file):
    plain, fused = "void decode_kernel<1, 2, 1, 0, 0>(DecodeArgs)", "void decode_kernel<1, 2, 1, 1, 0>(DecodeArgs)"
    a, b = tmp_path / "a.csv", tmp_path / "b.csv"
    _csv(a, [_row(0, plain, "dram__bytes_read.sum", "Mbyte", "4.4"),
             _row(0, plain, "dram__bytes_write.sum", "Kbyte", "40"),
             _row(1, fused, "dram__bytes_read.sum", "Mbyte", "99"),      # another variant: not counted
             _row(1, fused, "dram__bytes_write.sum", "byte", "1"),
             _row(2, plain, "gpu__time_duration.sum", "nsecond", "3000")])  # not a DRAM metric
    _csv(b, [_row(0, plain, "dram__bytes_read.sum", "byte", "4500000"),  # same ID, other file: own launch
             _row(0, plain, "dram__bytes_write.sum", "byte", "20000")])
    rec = bench.record_traffic([str(a), str(b)], "bitnet2b_decode", r"decode_kernel<\d+, \d+, \d+, 0, 0>", "cmd")
    assert rec["launches"] == 2
    assert rec["bytes_per_launch"] == round(((4.4e6 + 40e3) + (4.5e6 + 20e3)) / 2)
    stored = json.loads(traffic_file.read_text())
    assert stored["bitnet2b_decode"]["command"] == "cmd"
    assert bench.stored_traffic("bitnet2b_decode") == rec["bytes_per_launch"]


def test_record_traffic_refuses_a_capture_without_the_kernel(tmp_path, traffic_file):
    a = tmp_path / "a.csv"
    _csv(a, [_row(0, "void gemm_kernel<1, 256, 0>(...)", "dram__bytes_read.sum", "byte", "5")])
    with pytest.raises(SystemExit):
        bench.record_traffic([str(a)], "qwen3b_train", r"gemm_kernel<0|sp24_pair_kernel", "cmd")


def test_stored_traffic_is_null_once_the_kernel_sources_change(tmp_path, traffic_file, monkeypatch):
    a = tmp_path / "a.csv"
    _csv(a, [_row(0, "void gemm_kernel<0, 256, 0>(...)", "dram__bytes_read.sum", "byte", "100"),
             _row(0, "void gemm_kernel<0, 256, 0>(...)", "dram__bytes_write.sum", "byte", "28")])
    bench.record_traffic([str(a)], "qwen05b_mlp", r"gemm_kernel<0|sp24_pair_kernel", "cmd")
    assert bench.stored_traffic("qwen05b_mlp") == 128
    monkeypatch.setattr(bench, "kernel_source_hash", lambda family: "another source")
    assert bench.stored_traffic("qwen05b_mlp") is None
    assert bench.stored_traffic("single_256x128") is None  # never recorded


def test_kernel_families_cover_the_workloads():
    for name, wk in wl.WORKLOADS.items():
        fam = bench.kernel_family(name)
        assert fam == ("decode" if wk.mode == "decode" else "gemm")
        assert bench.kernel_source_hash(fam) == bench.kernel_source_hash(fam)  # stable
    assert bench.kernel_source_hash("gemm") != bench.kernel_source_hash("decode")


class _Done:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler_with_rows(tmp_path, rows, uuid="GPU-abc"):
    s = bench.ClockSampler(uuid)
    s.path = str(tmp_path / "clocks.csv")
    with open(s.path, "w") as f:
        for ts, sm, smax, reasons in rows:
            stamp = datetime.datetime.fromtimestamp(ts).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
            f.write(f"{stamp}, {uuid}, {sm}, {smax}, 700.0, " + ", ".join(reasons) + "\n")
    s.f = open(s.path)
    s.proc = _Done()
    return s


def test_clock_summary_uses_the_rows_inside_the_windows(tmp_path):
    t0 = 1_700_000_000.0
    idle = ["Not Active"] * 4
    capped = ["Not Active", "Not Active", "Not Active", "Active"]
    rows = [(t0 - 1.0, 600, 1965, idle),          # before: ignored
            (t0 + 0.10, 1900, 1965, idle),
            (t0 + 0.20, 1800, 1965, capped),
            (t0 + 0.30, 1850, 1965, idle),
            (t0 + 5.0, 300, 1965, ["Active", "Not Active", "Not Active", "Not Active"])]  # after: ignored
    summary = _sampler_with_rows(tmp_path, rows).stop((t0, t0 + 0.5))
    assert summary["samples"] == 3 and summary["sm_mhz"] == 1850
    assert summary["sm_max_mhz"] == 1965 and summary["reasons"] == ["sw_power_cap"]
    assert summary["window"] == "timed region"


def test_clock_summary_over_several_windows_and_the_fallback(tmp_path):
    t0 = 1_700_000_000.0
    idle = ["Not Active"] * 4
    rows = [(t0 + 0.1, 1900, 1965, idle), (t0 + 2.1, 1700, 1965, idle), (t0 + 9.0, 100, 1965, idle)]
    two = _sampler_with_rows(tmp_path, rows).stop((t0, t0 + 0.5), (t0 + 2.0, t0 + 2.5))
    assert two["samples"] == 2 and two["sm_mhz"] == 1800
    # a timed region shorter than the sampling period: every row, said so
    none_inside = _sampler_with_rows(tmp_path, rows).stop((t0 + 0.6, t0 + 0.7))
    assert none_inside["samples"] == 3 and "shorter" in none_inside["window"]


def test_clock_rows_of_other_gpus_are_ignored(tmp_path):
    t0 = 1_700_000_000.0
    s = _sampler_with_rows(tmp_path, [(t0 + 0.1, 1900, 1965, ["Not Active"] * 4)], uuid="GPU-abc")
    s.uuid = "GPU-other"
    assert s.stop((t0, t0 + 1.0)) is None


def test_algorithmic_ops_counts_kept_weights_and_the_backward():
    """Forward: 2 T O K n/m per linear and pattern; training adds 4 T O K
    (dX and dW, dense by definition)."""
    single = wl.WORKLOADS["single_256x128"]
    assert bench.algorithmic_ops(single, 64) == 2.0 * 64 * 128 * 256 * 6 / 8
    mlp = wl.WORKLOADS["qwen05b_mlp"]
    per_pattern = sum(2.0 * 4096 * lin.d_out * lin.d_in for lin in mlp.linears)
    assert bench.algorithmic_ops(mlp, 4096) == pytest.approx(per_pattern * (6 / 8 + 2 / 4))
    train = wl.WORKLOADS["qwen3b_train"]
    dense = sum(2.0 * 16384 * lin.d_out * lin.d_in for lin in train.linears)
    assert bench.algorithmic_ops(train, 16384) == pytest.approx(dense * (6 / 8 + 2))


def test_reference_arm_line_on_the_host(capsys, monkeypatch):
    """The oracle arm prints one line in our arm's metric and unit, with the
    cpu_baseline and e2e objects; rank 0 alone prints under torchrun."""
    import argparse
    wk = wl.WORKLOADS["single_256x128"]
    args = argparse.Namespace(steps=2, warmup=1, ref_step_seconds=0.2, cpu_threads=2)
    bench.run_reference(args, wk)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TOPS" and line["value"] > 0
    # the same configuration object as our arm's line
    assert line["metric"] == bench.METRIC and line["config"] == bench.workload_config(wk, 1)
    assert line["steps"] == 2 and line["warmup"] == 1 and line["higher_is_better"] is True
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == min(2, bench.cpu_threads()) and cb["value"] == line["value"]
    assert cb["sample"] and 1 <= line["sampled_tokens"] <= wk.tokens[-1]
    assert line["e2e"] == {"value": line["value"], "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # a step is the bounded sample: its time, at least the sample's budget-sized work
    assert 0 < line["ms_per_step"] < 60_000
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(args, wk)
    assert capsys.readouterr().out == ""


def test_cpu_baseline_training_sample_includes_the_backward(monkeypatch):
    """For the training workload the sample runs the fp64 Dual-STE backward
    too, and its operation count includes 4 T O K for it."""
    import oracle
    calls = []
    real = oracle.backward
    monkeypatch.setattr(oracle, "backward", lambda *a, **k: calls.append(a[0].shape) or real(*a, **k))
    small = wl.Workload(name="tiny_train", seed=5, tokens=[64], linears=[wl.Linear("up", d_in=64, d_out=32)],
                        patterns=[(6, 8)], mode="train")
    cb = bench.cpu_baseline(small, budget_s=0.2)
    assert calls and calls[-1][1] == 32 and "backward" in cb["sample"]
    assert 1 <= cb["sampled_tokens"] <= 64
    assert cb["sampled_ops"] == pytest.approx(cb["sampled_tokens"] * (2 * 32 * 64 * 6 / 8 + 4 * 32 * 64))


def test_cpu_baseline_threads_split_outputs_disjointly():
    """The threaded oracle timing hands disjoint slices covering every output
    to the unchanged oracle calls, and reports the threads it used."""
    assert bench.slices(10, 3) == [(0, 3), (3, 6), (6, 10)]
    assert bench.slices(2, 8) == [(0, 1), (1, 2)]
    small = wl.Workload(name="tiny_train", seed=5, tokens=[64], linears=[wl.Linear("up", d_in=64, d_out=32)],
                        patterns=[(6, 8)], mode="train")
    cb = bench.cpu_baselines(small, 0.4, 2)
    assert cb["cores"] == 2 and cb["single_thread"]["cores"] == 1 and cb["value"] > 0


def _grouping(wk_name, sp24_layers=(), mode=None):
    """bench.Runner.forward_groups on a stub runner: the workload's linears
    with their inputs shared as the Runner shares them (Linear.inp)."""
    import types
    wk = wl.WORKLOADS[wk_name]
    sbl = types.SimpleNamespace(SBL_FMT_I8=1, SBL_FMT_SP24=16, SBL_GROUP_MAX=4)
    inputs, layers = {}, []
    for li, lin in enumerate(wk.linears):
        key = lin.inp or f"#{li}"
        layers.append({"lin": lin, "inp": inputs.setdefault(key, {"name": key})})
    pat = wk.patterns[0]
    fmt = {(li, pat): (sbl.SBL_FMT_SP24 if lin.name in sp24_layers else sbl.SBL_FMT_I8)
           for li, lin in enumerate(wk.linears)}
    stub = types.SimpleNamespace(sbl=sbl, layers=layers, fwd_fmt=fmt,
                                 wk=types.SimpleNamespace(mode=mode or wk.mode))
    return [[wk.linears[li].name for li in g] for g in bench.Runner.forward_groups(stub, pat)]


def test_forward_groups_follow_the_decoder_dataflow():
    # q / k / v read x, o the attention output, gate / up the hidden state, down the activation
    assert _grouping("qwen15b_decoder") == [["q", "k", "v"], ["o"], ["gate", "up"], ["down"]]
    assert _grouping("qwen05b_mlp") == [["gate", "up"], ["down"]]
    # a layer on the sparse operand breaks a group; the rest of the input's layers still group
    assert _grouping("qwen15b_decoder", sp24_layers=("q",)) == [["q"], ["k", "v"], ["o"], ["gate", "up"], ["down"]]
    assert _grouping("qwen15b_decoder", sp24_layers=("k",)) == [["q"], ["k"], ["v"], ["o"], ["gate", "up"], ["down"]]
    # training runs each linear's backward right after its forward: never grouped
    assert _grouping("qwen05b_mlp", mode="train") == [["gate"], ["up"], ["down"]]
    assert _grouping("qwen3b_train") == [["up"], ["down"]]
