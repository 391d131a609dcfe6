"""CPU checks of bench.py's arithmetic: the algorithmic bytes and FLOPs behind the roofline
fraction, the job-wide value, and the source hash that ties a stored ncu traffic figure to
the kernel code."""
import os
import shutil

import pytest

import bench
import synth


def test_decode_gate_up_bytes_by_hand():
    # Flash-Next decode, 370 activated experts: each holds gate and up rows [2*640][2560]
    # in bf16; plus the shared expert's, the 64 token rows, and h as a bf16 hi/lo pair for
    # the 640 routed rows and the 64 shared rows.
    cfg = synth.CONFIGS["flash_decode"]
    weights = (370 * 2 * 640 * 2560 + 2 * 640 * 2560) * 2
    x = 64 * 2560 * 2
    h = (640 * 640 + 64 * 640) * 2 * 2
    assert bench.algorithmic_bytes("gate_up", cfg, 370) == weights + x + h == 2433515520


def test_decode_down_bytes_by_hand():
    cfg = synth.CONFIGS["flash_decode"]
    weights = (370 * 2560 * 640 + 2560 * 640) * 2
    h = (640 * 640 + 64 * 640) * 2 * 2
    out = 64 * 2560 * 4
    assert bench.algorithmic_bytes("down", cfg, 370) == weights + h + out == 1218150400


def test_prefill_flops_match_the_layer_count():
    # 6*H*I per routed assignment plus 6*H*Is per token for the shared expert, split 2:1
    # between gate|up and down (805.3 G + 80.5 G for the Flash-Next prefill, counted by hand)
    cfg = synth.CONFIGS["flash_prefill"]
    total = bench.kernel_flops("gate_up", cfg) + bench.kernel_flops("down", cfg)
    assert total == 6 * (cfg.R * cfg.H * cfg.I + cfg.T * cfg.H * cfg.Is)
    assert total == pytest.approx(805.3e9 + 80.5e9, rel=1e-3)
    assert bench.kernel_flops("gate_up", cfg) == 2 * bench.kernel_flops("down", cfg)


def test_job_value_counts_every_rank():
    assert bench.job_value(64, 200, 1, 120.0) == pytest.approx(64 * 200 / 0.12)
    assert bench.job_value(64, 200, 8, 120.0) == pytest.approx(8 * 64 * 200 / 0.12)


def test_source_hash_ignores_comments_not_code(tmp_path, monkeypatch):
    csrc = tmp_path / "sparse_moe_expert_fp32_b200" / "csrc"
    csrc.mkdir(parents=True)
    real = os.path.join(bench.ROOT, "sparse_moe_expert_fp32_b200", "csrc")
    for f in bench.KERNEL_SOURCES["down"]:
        shutil.copy(os.path.join(real, f), csrc / f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.source_hash("down")
    p = csrc / "tc2_gemm.cu"
    src = p.read_text()
    p.write_text("// a new comment line\n" + src.replace("\n", "\n  ", 3) + "\n/* and a block */\n")
    assert bench.source_hash("down") == h0
    p.write_text(src.replace("kSlotCols = 256", "kSlotCols = 255", 1))
    assert bench.source_hash("down") != h0


def test_decode_fp8_bytes_by_hand():
    # the FP8 layer: routed gate|up and down weights at one byte each plus one fp32 scale per
    # weight row; the shared expert, x, h and out as in the bf16 layer
    cfg = synth.CONFIGS["flash_decode"]
    gu = 370 * 2 * 640 * (2560 + 4) + (2 * 640 * 2560 + 64 * 2560) * 2 + (640 * 640 + 64 * 640) * 4
    dn = 370 * 2560 * (640 + 4) + 2560 * 640 * 2 + (640 * 640 + 64 * 640) * 4 + 64 * 2560 * 4
    assert bench.algorithmic_bytes("gate_up", cfg, 370, fp8=True) == gu == 1222993920
    assert bench.algorithmic_bytes("down", cfg, 370, fp8=True) == dn == 615731200


def test_reference_arm_times_the_fp8_oracle():
    import json
    import subprocess
    import sys

    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--fp8", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, cwd=bench.ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference" and line["config"]["variant"] == "fp8"
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]


def test_layer_totals_match_hand_counts():
    # 2.4T-shaped prefill, every expert active: routed 8.246 TFLOP + shared 0.825 TFLOP +
    # router 68.7 GFLOP; 51.54 GB of routed weights + shared expert + router matrix + x + out
    # (fp32) = 52.06 GB
    cfg = synth.CONFIGS["t24_prefill"]
    t = bench.layer_totals(cfg, 512)
    assert t["flops_dense_equivalent"] == t["flops_executed"]
    assert t["flops_dense_equivalent"] == pytest.approx(8.246e12 + 0.825e12 + 68.7e9, rel=1e-3)
    assert t["bytes"] == pytest.approx(52.06e9, rel=1e-3)
    # zero-channel compaction to I_c = 640: executed routed FLOPs scale by 640 / 2048,
    # dense-equivalent FLOPs do not change
    c = bench.layer_totals(synth.CONFIGS["t24_skewed"], 512, I_exec=640)
    full = bench.layer_totals(synth.CONFIGS["t24_skewed"], 512)
    cfg5 = synth.CONFIGS["t24_skewed"]
    routed = 6.0 * cfg5.R * cfg5.H * cfg5.I
    assert c["flops_dense_equivalent"] == full["flops_dense_equivalent"]
    assert full["flops_executed"] - c["flops_executed"] == pytest.approx(routed * (1 - 640 / 2048))


def test_layer_fractions_by_hand():
    tot = {"flops_dense_equivalent": 2e12, "flops_executed": 1e12, "bytes": 4e9}
    peaks = {"bf16_tflops": 1000.0, "bf16_tflops_sustained": 800.0, "hbm_gbs": 2000.0}
    f = bench.layer_fractions(tot, 0.004, peaks)  # 4 ms
    assert f["tc_pct"] == pytest.approx(25.0)      # 1 TFLOP / (1 PFLOP/s x 4 ms)
    assert f["tc_pct_of_sustained"] == pytest.approx(31.25)
    assert f["tc_pct_dense_equivalent"] == pytest.approx(50.0)
    assert f["hbm_pct"] == pytest.approx(50.0)     # 4 GB / (2 TB/s x 4 ms)
    assert f["roofline_pct"] == pytest.approx(50.0) and f["bound"] == "hbm"
    assert f["roofline_us"] == pytest.approx(2000.0)


def test_error_stats_leave_out_differing_id_sets():
    import numpy as np

    ref = {"out": np.array([[1.0, -1.0], [2.0, 2.0], [5.0, 5.0]]),
           "ids": np.array([[0, 1], [2, 3], [4, 5]]), "gap": np.array([1.0, 1.0, 1e-6])}
    gpu = np.array([[1.01, -1.0], [2.0, 2.0], [0.0, 0.0]])
    ids = np.array([[1, 0], [3, 2], [4, 6]])  # last token: a near-tie chose another set
    e = bench.error_stats(gpu, ids, ref, 2)
    rms = np.sqrt((1 + 1 + 4 + 4) / 4)
    assert e["sample_id_sets_differ"] == 1 and e["sample_near_ties_fp64"] == 1
    assert e["max_abs_over_rms"] == pytest.approx(0.01 / rms)
    assert e["mean_rel"] == pytest.approx(0.01 / 6.0)


def test_fp16_down_operands_bytes_by_hand():
    # with the fp16 down operands h is one fp16 value per element: 2 bytes instead of 4
    cfg = synth.CONFIGS["flash_decode"]
    h2 = (640 * 640 + 64 * 640) * 2
    assert bench.algorithmic_bytes("gate_up", cfg, 370, h_bytes=2) == 2433515520 - h2
    assert bench.algorithmic_bytes("down", cfg, 370, h_bytes=2) == 1218150400 - h2
