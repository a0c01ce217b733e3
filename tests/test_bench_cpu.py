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
    assert bench.kernel_rev() != rev
