"""bench.py's host-side pieces on CPU: the reference arm (the oracle timed on
the host cores) prints one JSON line with the contract's keys, and the ncu
traffic record is used only for the kernel source it was taken on."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    # the workload keys name the same configuration as the CUDA arm's line
    assert d["config"]["name"] == "full" and d["config"]["tokens"] == 640 * 360 and d["config"]["window"] == 64
    assert d["metric"].startswith("windowed RIB attention") and d["unit"] == "TFLOP/s" and d["higher_is_better"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_traffic_record_is_keyed_by_the_kernel_source(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel v1\nint f(int a) { return a + 1; }  /* add one */\n")
    h = bench.source_code_hash(str(src))
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "attention_traffic.json").write_text(json.dumps({"full": {"source_code_sha256_16": h,
                                                                      "dram_bytes_per_launch": 123}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic(str(src), "full") == 123
    assert bench.kernel_traffic(str(src), "train") is None
    # comments and layout edited: the same code, the record still holds
    src.write_text("// kernel v1, reworded\n/* block\n comment */\nint f(int a) {\n  return a + 1;\n}\n")
    assert bench.kernel_traffic(str(src), "full") == 123
    # the code changed since the capture: no traffic figure
    src.write_text("// kernel v1\nint f(int a) { return a + 2; }  /* add one */\n")
    assert bench.kernel_traffic(str(src), "full") is None


def test_traffic_record_is_used_only_for_the_attention_source_it_was_taken_on():
    """The committed record is consistent, and the bench reports its traffic
    only while the attention kernel's code is the code it was captured on
    (a record left behind by a kernel change gives traffic null)."""
    sys.path.insert(0, ROOT)
    import bench
    with open(os.path.join(ROOT, "profiles", "attention_traffic.json")) as fh:
        rec = json.load(fh)["full"]
    assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    src = os.path.join(ROOT, "windowed_attention_b200", "csrc", "window_attention.cu")
    if rec["source_code_sha256_16"] == bench.source_code_hash(src):
        assert bench.kernel_traffic(src, "full") == rec["dram_bytes_per_launch"]
    else:
        assert bench.kernel_traffic(src, "full") is None


def test_flop_accounting_of_the_workloads():
    """The FLOP counts the bench divides by: the attention's 2N^2(dh+R) +
    2N^2 dh per window-head (918 GFLOP at 640x360: 60 windows of 64x64 over
    the map padded to 640x384, 6 heads of dh 30, R 16), its backward's
    2N^2(3(dh+R) + 2dh) (3,229 GFLOP for 16 patches of 96x96), and the layer's
    projection (3 C x C per token), pointwise (C x C) and depthwise (9 taps)."""
    sys.path.insert(0, ROOT)
    import bench
    from windowed_attention_b200.workloads import WORKLOADS
    full = WORKLOADS["full"].layer
    assert (full.Hp, full.Wp, full.n_windows) == (384, 640, 60)
    f = bench.layer_flops(full)
    assert f["attention"] == 918_049_259_520
    T, C = 640 * 360, 180
    assert f["projection"] == 2 * T * C * 3 * C and f["pointwise"] == 2 * T * C * C and f["depthwise"] == 18 * T * C
    assert f["layer"] == 978_515_435_520
    train = WORKLOADS["train"].layer
    assert train.n_windows == 16
    assert train.attention_bwd_flops() == 3_228_875_882_496
    # weak scaling: the job does world x the per-rank work in the slowest rank's time
    assert bench.whole_job_tflops(2, 1e12, 10, 1000.0) == 20.0
    assert abs(bench.whole_job_tflops(1, 918_049_259_520, 50, 50 * 1.85) - 496.2428) < 1e-4   # 1.85 ms/step


def test_reference_arm_under_torchrun_prints_once():
    """Launched as the multi-GPU runs are (torchrun, two ranks), the reference
    arm runs on rank 0 alone and prints one line; the other rank exits 0."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "1"]
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0


def test_measured_peaks_file_is_read_and_a_bad_one_falls_back(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.measured_peaks()
    assert src == "fallback" and peaks["bf16_tflops"] == 1590.0 and peaks["hbm_gbs"] == 6650.0
    f = tmp_path / "MEASURED_PEAKS.json"
    f.write_text(json.dumps({"hbm_gbs": 6451.5, "bf16_tflops": 1713.8, "bf16_tflops_sustained": 1402.0,
                             "clocks": {"sm_mhz": 1965}}))
    peaks, src = bench.measured_peaks()
    assert src == "measured" and peaks["bf16_tflops"] == 1713.8 and peaks["hbm_gbs"] == 6451.5
    f.write_text(json.dumps({"hbm_gbs": 6451.5}))          # no GEMM peak: the fallback denominators
    assert bench.measured_peaks() == ({"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0},
                                      "fallback")
    f.write_text("{not json")
    assert bench.measured_peaks()[1] == "fallback"
