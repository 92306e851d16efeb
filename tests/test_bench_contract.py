"""The bench's JSON line keeps its contract: the reference arm (the oracle on
the host's cores, no GPU) runs a tiny sample and prints one line with the keys
the driver reads."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0", "--ref-tokens", "8", "--workload", "replay"], capture_output=True,
                         text=True, timeout=600,
                         cwd=ROOT, env={**os.environ, "RANK": "0"})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith("replay: T=4096 D=2048 I=1024 E=64 k=6 L=4")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_reference_arm_other_ranks_exit_quietly():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0", "--ref-tokens", "8"], capture_output=True, text=True, timeout=120,
                         cwd=ROOT, env={**os.environ, "RANK": "1"})
    assert out.returncode == 0 and not [l for l in out.stdout.splitlines() if l.startswith("{")]


def test_default_workload_is_the_largest_single_gpu_configuration():
    """With no flags the bench times the long-sequence prefill chunk (T=131072,
    d_model=6144, I=2048, 32 experts, top-8, skewed routing with empty
    experts), the largest configuration of the layer on one GPU."""
    sys.path.insert(0, ROOT)
    import bench
    from moe_expert_layer_replay_b200.inputs import WORKLOADS
    args = bench.build_parser().parse_args([])
    wl = WORKLOADS[args.workload]
    assert (wl.T, wl.D, wl.I, wl.E, wl.k, wl.empty) == (131072, 6144, 2048, 32, 8, 4)
    assert args.gpus == 1 and args.warmup >= 3 and args.impl == "ours"
    assert bench.default_sample_tokens(wl, 3e11) <= 512
