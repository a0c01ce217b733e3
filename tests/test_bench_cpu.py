"""Host-side arithmetic of bench.py: the roofline numerator and the job rate."""
import bench
from linear_attention_layer_kda_b200 import inputs as I


def test_algorithmic_bytes_per_step():
    # FP8 q/k/v/o + fp32 128x128 scales + bf16 gate weights + fp32 state read and write + x + out
    expect = {1: 102_187_008, 2: 72_654_848, 3: 119_062_528, 4: 558_206_976, 0: 248_352}
    for cfg, n in expect.items():
        s = I.CONFIGS[cfg]
        assert bench.ideal_bytes(s, s.batch) == n, cfg


def test_algorithmic_bytes_by_hand_at_batch_8():
    H, D, nh, r, B = 4096, 4096, 32, 64, 8
    fp8 = 4 * D * H
    scales = 4 * 4 * (D // 128) * (H // 128)
    gates = 2 * (r * H + D * r + nh * H)
    state = 2 * B * nh * 128 * 128 * 4
    assert bench.ideal_bytes(I.CONFIGS[1], B) == fp8 + scales + gates + state + B * H * 2 + B * H * 4


def test_job_rate_counts_every_rank():
    assert bench.job_steps_per_s(0.05, 1) == 20000.0
    assert bench.job_steps_per_s(0.05, 8) == 160000.0
    assert bench.job_steps_per_s(0.05, 8, tp=True) == 20000.0  # the ranks advance one batch together


def test_kernel_revision_ignores_comments(tmp_path, monkeypatch):
    import os
    import shutil
    src = os.path.join(bench.ROOT, "linear_attention_layer_kda_b200", "csrc")
    fake = tmp_path / "linear_attention_layer_kda_b200" / "csrc"
    shutil.copytree(src, fake)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rev = bench.kernel_rev()
    with open(fake / "fused.cu", "a") as f:
        f.write("\n// a comment only\n\n")
    assert bench.kernel_rev() == rev
    with open(fake / "fused.cu", "a") as f:
        f.write("static int kda_extra_symbol_for_the_test = 1;\n")
    rev2 = bench.kernel_rev()
    assert rev2 != rev
    with open(fake / "chunk.cu", "a") as f:  # the prefill kernels are not part of the fused engine
        f.write("static int kda_other_engine_symbol = 1;\n")
    assert bench.kernel_rev() == rev2


def test_step_percentiles():
    med, p10, p90 = bench.step_percentiles([float(i) for i in range(1, 102)])
    assert med == 51.0 and p10 == 11.0 and p90 == 91.0


def test_launcher_starts_one_rank_per_gpu():
    """`--gpus 2` without a torchrun environment starts two ranks of bench.py with RANK and
    WORLD_SIZE set (checked with the launcher self-check flag, which exits before any CUDA)."""
    import json
    import os
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--gpus", "2", "--print-rank",
                        "--launch-limit", "120"], env=env, capture_output=True, text=True, timeout=180)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert sorted(d["rank"] for d in lines) == [0, 1]
    assert all(d["world_size"] == 2 for d in lines)


def test_refuses_a_line_for_a_different_gpu_count(monkeypatch, capsys):
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    assert bench.main(["--gpus", "2", "--print-rank"]) == 2
    assert "refusing" in capsys.readouterr().err


def test_reference_arm_reports_the_same_config_as_ours(capsys):
    """The reference arm's config equals the dictionary the GPU arm prints for the same workload."""
    import json
    shape = I.CONFIGS[0]
    args = bench.parse_args(["--steps", "2", "--warmup", "0"])
    assert bench.run_reference(args, shape, 0, 1) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 1
    assert line["config"] == bench.workload_config(shape, 1, bench.rotation_sets(shape))
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["cpu_model"]
