"""The benchmark's reference arm (the fp64 oracle on the host cores) prints one JSON
line with the keys the benchmark contract asks for.  CPU only: the smallest workload,
one timed step."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "vim_tiny_224px_fp32", "--steps", "1", "--warmup", "0"],
                         check=True, capture_output=True, text=True, cwd=ROOT, timeout=300).stdout
    lines = [ln for ln in out.splitlines() if ln.strip()]
    assert len(lines) == 1, out
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["unit"] == "tok*ch/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == "vim_tiny_224px_fp32"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_profiled_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    # the DRAM traffic a line reports comes from a committed capture only while the
    # kernel source it names still has the fingerprint the capture recorded
    import hashlib

    sys.path.insert(0, ROOT)
    import bench
    from vision_mamba_selective_b200 import workloads

    w = workloads.WORKLOADS[2]
    csrc = tmp_path / "vision_mamba_selective_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    for src, body in (("scan_kernels.cuh", b"// scan v1\n"), ("bwd_kernels.cuh", b"// bwd v1\n")):
        (csrc / src).write_bytes(body)
    fp = {s: hashlib.sha256((csrc / s).read_bytes()).hexdigest()[:16] for s in ("scan_kernels.cuh", "bwd_kernels.cuh")}
    (tmp_path / "profiles" / f"ncu_scan_kernels_{w.name}.md").write_text(
        "traffic_bytes_per_launch pair_main: 123\n\nkernel source fingerprint (sha256 of scan_kernels.cuh, "
        f"first 16 hex): {fp['scan_kernels.cuh']}\n")
    (tmp_path / "profiles" / f"ncu_bwd_kernels_{w.name}.md").write_text(
        "traffic_bytes_per_launch adj_carry: 7\ntraffic_bytes_per_launch bwd_main: 456\n\nkernel source "
        f"fingerprint (sha256 of bwd_kernels.cuh, first 16 hex): {fp['bwd_kernels.cuh']}\n")
    (tmp_path / "profiles" / f"ncu_scan_kernels_conv_{w.name}.md").write_text(
        "traffic_bytes_per_launch pair_main: 321\n\nkernel source fingerprint (sha256 of scan_kernels.cuh, "
        f"first 16 hex): {fp['scan_kernels.cuh']}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic(w) == 123
    assert bench.profiled_traffic(w, conv=True) == 321
    assert bench.profiled_traffic(w, zoh=True) is None                # no capture of that mode
    assert bench.profiled_traffic(w, zoh=True, conv=True) is None
    assert bench.profiled_traffic(w, bwd=True) == 456
    assert bench.profiled_traffic(w, bwd=True, zoh=True) is None   # no capture of that mode
    assert bench.profiled_traffic(workloads.WORKLOADS[0]) is None   # nor of that workload
    (csrc / "bwd_kernels.cuh").write_bytes(b"// bwd v2\n")
    assert bench.profiled_traffic(w, bwd=True) is None             # the source changed since
    assert bench.profiled_traffic(w) == 123


def test_mode_combinations_are_checked_before_any_gpu_work():
    # modes that do not combine are refused with a message, on the host, before CUDA
    for args, msg in ((["--block", "--ckpt"], "--ckpt applies"), (["--block", "--zoh"], "--block runs alone"),
                      (["--workload", "vmamba_64x64_bf16", "--conv"], "--conv and --block apply")):
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                           cwd=ROOT, timeout=120)
        assert r.returncode != 0 and msg in r.stderr, (args, r.stderr[-300:])
