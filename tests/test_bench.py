"""Host-side logic of bench.py (no GPU): the algorithmic work and bytes it
credits, the ncu traffic records it reads, and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from causal_gqa_attention_sm_b200.workloads import WORKLOADS  # noqa: E402


def test_flops_follow_the_causal_fa_convention():
    # 7 B Hq T^2 D per causal layer: 22.55 GFLOP for B=4, T=1024, Hq=12, D=64
    w = WORKLOADS["long"]
    assert w.flops() == 7 * 4 * 12 * 1024 * 1024 * 64
    assert abs(w.flops() / 1e9 - 22.55) < 0.01
    assert WORKLOADS["stack"].flops() == 16 * WORKLOADS["layer"].flops()
    assert sum(bench.UNITS.values()) == 7.0


def test_prologue_bytes_count_each_element_once():
    w = WORKLOADS["long"]  # float32 storage: fp32 in, bf16 hi + lo out
    nq, nk = 4 * 1024 * 12 * 64, 4 * 1024 * 4 * 64
    assert bench.prologue_bytes(w, "attn_fwd_prologue") == (nq + 2 * nk) * 8
    tp = 1024
    rowterm = 2 * nq * 4 + 4 * 4 * 12 * 1024 + 8 * 4 * 12 * tp
    # the backward prologue gets the forward's saved planes: dO is read once,
    # for the row terms, and split into its planes in the same pass
    assert bench.prologue_bytes(w, "attn_bwd_prologue") == nq * 4 + rowterm
    b = WORKLOADS["sweep1024"]  # bf16: rotated copies of Q and K only
    nq, nk = 16 * 1024 * 12 * 64, 16 * 1024 * 4 * 64
    assert bench.prologue_bytes(b, "attn_fwd_prologue") == (nq + nk) * 4
    assert bench.prologue_bytes(b, "attn_bwd_prologue") == 2 * nq * 2 + 4 * 16 * 12 * 1024 + 8 * 16 * 12 * 1024


def test_every_kernel_has_its_sources():
    csrc = os.path.join(ROOT, "causal_gqa_attention_sm_b200", "csrc")
    for k in bench.KERNELS + ("attn_decode",):
        for name in bench.KERNEL_SOURCES[k]:
            assert os.path.exists(os.path.join(csrc, name))
        assert len(bench.kernel_source_hash(k)) == 16
    for f in bench.SHARED_SOURCES:
        assert os.path.exists(os.path.join(csrc, f))
    # a kernel's hash does not depend on another kernel's header
    assert bench.kernel_source_hash("attn_fwd") != bench.kernel_source_hash("attn_bwd")
    assert bench.kernel_source_hash("attn_fwd_prologue") == bench.kernel_source_hash("attn_bwd_prologue")


def test_committed_traffic_records_are_consistent():
    prof = os.path.join(ROOT, "profiles")
    recs = [f for f in os.listdir(prof) if f.endswith(".json")]
    assert recs
    for f in recs:
        with open(os.path.join(prof, f)) as fh:
            r = json.load(fh)
        assert f == f"{r['kernel']}_{r['workload']}.json"
        assert r["kernel"] in bench.KERNEL_SOURCES and r["workload"] in WORKLOADS
        assert r["dram_bytes_per_launch"] == r["dram_bytes_read"] + r["dram_bytes_write"]
        assert "--clock-control none" in r["command"]


def test_traffic_is_withheld_when_the_kernel_changed(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    rec = {"kernel": "attn_bwd", "workload": "long", "source_hash": bench.kernel_source_hash("attn_bwd"),
           "dram_bytes_read": 3.0, "dram_bytes_write": 1.0, "dram_bytes_per_launch": 4.0}
    (tmp_path / "profiles" / "attn_bwd_long.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k, h=rec["source_hash"]: h)
    assert bench.ncu_traffic("attn_bwd", "long") == 4.0
    assert bench.ncu_traffic("attn_fwd", "long") is None  # no record
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k: "0" * 16)
    assert bench.ncu_traffic("attn_bwd", "long") is None  # sources changed since the capture


@pytest.mark.parametrize("workload", ["tiny", "decode1024", "block", "ffn"])
def test_reference_arm_prints_the_contract_line(workload):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          workload, "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["warmup"] >= 3 and line["value"] > 0
    assert line["config"]["workload"] == workload
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_clock_sampler_without_nvidia_smi_reports_it(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))  # no nvidia-smi on the path
    c = bench.ClockSampler(0, str(tmp_path / "clocks.csv"))
    with c:
        pass
    assert c.summary()["reasons"] == ["nvidia-smi unavailable"]
    assert c.f.closed
    assert not bench.ClockSampler(3).path.startswith(ROOT)  # raw samples go to a temporary file by default


def test_reference_arm_under_torchrun_prints_once():
    """Launched as the driver launches N > 1 (torchrun, one process per rank),
    the reference arm runs on rank 0 alone: one JSON line, every rank exits 0."""
    import socket

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus",
           "2", "--workload", "tiny", "--steps", "1", "--warmup", "3"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(l) for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1 and lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2
