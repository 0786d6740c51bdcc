"""CPU checks of the benchmark's host logic: the count of attending pairs the
flop figures rest on, the per-workload figures, and the CPU-baseline leg."""
import numpy as np
import pytest

import oracle

import bench
from vision_transformer_windowed_b200.inputs import make_inputs


def _brute_pairs(B, H, W, heads, M, s):
    """(query, key) pairs of one window with equal region labels, counted token
    by token on the grid padded to multiples of M, times B and heads."""
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    lab = oracle.labels(Hp, Wp, M, s)
    n = 0
    for wr in range(Hp // M):
        for wc in range(Wp // M):
            cell = lab[wr * M:(wr + 1) * M, wc * M:(wc + 1) * M].ravel()
            _, counts = np.unique(cell, return_counts=True)
            n += int((counts ** 2).sum())
    return n * B * heads


@pytest.mark.parametrize("shape", [(2, 16, 16, 3, 8, 0), (2, 16, 16, 3, 8, 4), (1, 64, 64, 1, 32, 16),
                                   (1, 20, 13, 2, 8, 4), (1, 40, 36, 1, 16, 8), (3, 24, 40, 2, 8, 0)])
def test_unmasked_pairs_match_brute_force(shape):
    assert bench.unmasked_pairs(*shape) == _brute_pairs(*shape)


def test_workload_flops_count_every_shift():
    wl = dict(B=2, H=16, W=16, heads=3, M=8, shifts=(0, 4), qk_scale=1.0)
    pairs = sum(_brute_pairs(2, 16, 16, 3, 8, s) for s in (0, 4))
    fwd, bwd = bench.workload_flops(wl)
    assert fwd == 4 * 32 * pairs and bwd == 10 * 32 * pairs


def test_config_entry_figures():
    wl = dict(B=1, H=16, W=16, heads=2, M=8, shifts=(0, 4), qk_scale=1.0)
    fwd_f, bwd_f = bench.workload_flops(wl)
    r = {"ms": 2.0, "tflops": (fwd_f + bwd_f) / 2e-3 / 1e12, "tokens_per_s": 1.0, "peak_gb": 0.5,
         "phase_ms": {"fwd": 0.25}, "fwd_flops": fwd_f, "bwd_flops": bwd_f, "ws_bytes": 1000}
    peaks = {"bf16_tflops": 1000.0}
    e = bench.config_entry(wl, r, peaks, 1)
    assert e["fwd_tflops"] == pytest.approx(fwd_f / 0.5e-3 / 1e12)  # two forward calls of 0.25 ms
    assert e["tflops_no_recompute"] == pytest.approx((fwd_f + 0.8 * bwd_f) / 2e-3 / 1e12)
    assert e["pct_bf16_spec"] == pytest.approx(100 * r["tflops"] / bench.SPEC_BF16_TFLOPS)
    assert e["fwd_gbs"] == pytest.approx(260 * 16 * 16 * 2 * 2 / 0.5e-3 / 1e9)
    assert e["bwd_workspace_gb"] == pytest.approx(1e-6)


def test_cpu_baseline_samples_every_unit_of_a_small_workload():
    wl = dict(B=1, H=20, W=13, heads=2, M=8, shifts=(0, 4), qk_scale=1.0)  # padded: 3 x 2 windows
    t = make_inputs(1, 20, 13, 2, 32)
    res = bench.cpu_baseline(t, wl, seconds=2.0)
    n_units = 1 * 3 * 2 * 2
    assert res["kind"] == "oracle" and res["value"] > 0 and res["cores"] >= 1
    assert f"{n_units} of {n_units} at s=0" in res["sample"] and f"{n_units} of {n_units} at s=4" in res["sample"]
    assert res["units_per_s"] == pytest.approx(2 * n_units / res["seconds"])
    assert res["full_step_s_extrapolated"] == pytest.approx(res["seconds"])


def test_four_stage_workload_counts_every_block():
    """The headline step: FlashSwin-T's four stages at p=2, an unshifted and a
    shifted block per stage (stage 4 twice unshifted), flops from the brute-force
    pair count of every block."""
    wl = bench.WORKLOADS["flashswin_t_p2_4stage"]
    blocks = bench.blocks_of(wl)
    assert [(st["H"], st["heads"], st["M"], s) for st, s in blocks] == [
        (128, 3, 32, 0), (128, 3, 32, 16), (64, 6, 32, 0), (64, 6, 32, 16),
        (32, 12, 32, 0), (32, 12, 32, 16), (16, 24, 16, 0), (16, 24, 16, 0)]
    # the pair count of a block is per image and head: brute force on one image, one head
    pairs = sum(_brute_pairs(1, st["H"], st["W"], 1, st["M"], s) * st["B"] * st["heads"] for st, s in blocks)
    fwd, bwd = bench.workload_flops(wl)
    assert fwd == 4 * 32 * pairs and bwd == 10 * 32 * pairs
    assert bench.workload_tokens(wl) == 128 * 2 * (128 ** 2 + 64 ** 2 + 32 ** 2 + 16 ** 2)


def test_roofline_of_the_dominant_kernel():
    wl = dict(stages=[dict(B=1, H=64, W=64, heads=2, M=32, shifts=(0, 16)),
                      dict(B=1, H=16, W=16, heads=4, M=16, shifts=(0,))], qk_scale=1.0)
    blocks = bench.blocks_of(wl)
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "source": "measured"}
    res = {"phase_ms_per_step": {"fwd": 1.0, "bwd_prep": 0.2, "bwd_main": 2.0, "bwd_post": 0.1, "bwd_dtheta": 0.01}}
    roof = bench.roofline(wl, res, peaks, sm_mhz=1900.0)
    fl = sum(10 * 32 * bench.unmasked_pairs(st["B"], st["H"], st["W"], st["heads"], st["M"], s) for st, s in blocks)
    assert roof["kernel"] == "bwd_main" and roof["bound"] == "tensor"
    assert roof["achieved"] == pytest.approx(fl / 2e-3 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 1400.0)
    assert roof["mufu_ceiling_tflops"] == pytest.approx(320 * 16 * 148 * 1900e6 / 1e12)
    # windows inside one tile: HBM-bound, 520 bytes per token-head row for the one-tile backward
    wl8 = dict(B=2, H=16, W=16, heads=3, M=8, shifts=(0, 4), qk_scale=1.0)
    roof8 = bench.roofline(wl8, res, peaks)
    assert roof8["bound"] == "hbm" and roof8["kernel"] == "bwd_main"
    assert roof8["achieved"] == pytest.approx(2 * 520 * 2 * 16 * 16 * 3 / 2e-3 / 1e9)


def test_cpu_baseline_samples_every_stage():
    wl = dict(stages=[dict(B=1, H=16, W=16, heads=2, M=8, shifts=(0, 4)),
                      dict(B=1, H=16, W=16, heads=1, M=16, shifts=(0,))], qk_scale=1.0)
    t = [make_inputs(1, 16, 16, 2, 32), make_inputs(1, 16, 16, 1, 32)]
    res = bench.cpu_baseline(t, wl, seconds=2.0)
    assert "8 of 8 at 16x16/M=8 s=0" in res["sample"] and "8 of 8 at 16x16/M=8 s=4" in res["sample"]
    assert "1 of 1 at 16x16/M=16 s=0" in res["sample"]
    assert res["units_per_s"] == pytest.approx(17 / res["seconds"])


def test_flops_and_bytes_scale_with_the_head_dimension():
    wl = dict(B=1, H=16, W=16, heads=2, M=8, shifts=(4,), qk_scale=1.0, d=64)
    pairs = _brute_pairs(1, 16, 16, 2, 8, 4)
    fwd, bwd = bench.workload_flops(wl)
    assert fwd == 4 * 64 * pairs and bwd == 10 * 64 * pairs
    w = bench.phase_work(bench.stages_of(wl)[0], 4)
    assert w["flops"]["bwd_main"] == 10 * 64 * pairs and not w["hbm_bound"]
    assert w["bytes"]["fwd"] == 516 * 16 * 16 * 2


def test_lrbias_flops_count_the_factor_channels():
    """The bias variant's products contract over d + 16 channels where the factors
    ride along: 4 d + 32 forward and 10 d + 96 backward flops per attending pair."""
    wl = bench.WORKLOADS["flashbias_t_stage1_p2_m32"]
    assert wl["lrbias"]
    pairs = sum(bench.unmasked_pairs(wl["B"], wl["H"], wl["W"], wl["heads"], wl["M"], s) for s in wl["shifts"])
    fwd, bwd = bench.workload_flops(wl)
    assert fwd == 160 * pairs and bwd == 416 * pairs
    st = bench.stages_of(wl)[0]
    w = bench.phase_work(st, 16)
    assert not w["hbm_bound"] and w["flops"]["bwd_main"] == 416 * bench.unmasked_pairs(128, 128, 128, 3, 32, 16)
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "source": "measured"}
    res = {"phase_ms_per_step": {"fwd": 1.0, "bwd_prep": 0.2, "bwd_main": 2.0, "bwd_post": 0.1, "bwd_dtheta": 0.01}}
    roof = bench.roofline(wl, res, peaks, sm_mhz=1900.0)
    assert roof["mufu_ceiling_tflops"] == pytest.approx(416 * 16 * 148 * 1900e6 / 1e12)


def test_cpu_baseline_runs_the_bias_oracle():
    wl = dict(B=1, H=16, W=16, heads=2, M=8, shifts=(4,), qk_scale=1.0, lrbias=True)
    res = bench.cpu_baseline(bench.cpu_stage_inputs(wl), wl, seconds=1.0)
    assert res["value"] > 0 and "8 of 8 at s=4" in res["sample"]


def test_traffic_records_are_reported_only_for_the_sources_they_were_taken_on(monkeypatch):
    """Every stored DRAM-traffic record names a benchmarked workload, an existing
    kernel source and its ncu summary; bench reports its bytes while the
    kernel's sources hash to the stored value and null once they differ."""
    import json
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "profiles", "traffic.json")) as fh:
        recs = json.load(fh)["records"]
    assert recs
    for rec in recs:
        assert rec["workload"] in bench.WORKLOADS
        assert os.path.exists(os.path.join(root, "vision_transformer_windowed_b200", "csrc", rec["source"]))
        assert os.path.exists(os.path.join(root, "profiles", rec["summary"]))
        assert rec["bytes_per_step"] > 0 and len(rec["sources_sha256"]) == 64
        monkeypatch.setattr(bench, "kernel_sources_sha256", lambda tu, h=rec["sources_sha256"]: h)
        assert bench.measured_traffic(rec["phase"], rec["workload"]) == rec["bytes_per_step"]
        monkeypatch.setattr(bench, "kernel_sources_sha256", lambda tu: "0" * 64)
        assert bench.measured_traffic(rec["phase"], rec["workload"]) is None
    assert bench.measured_traffic("bwd_main", "no_such_workload") is None


def _run_reference_arm(rank: int, world: int):
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", str(world),
                          "--workload", "swin_t_stage1_p4_m8", "--steps", "1", "--warmup", "3",
                          "--reference-seconds", "4"], capture_output=True, text=True, env=env, cwd=root, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    return [json.loads(l) for l in out.stdout.splitlines() if l.strip()]


def test_reference_arm_prints_one_line_on_rank_zero_only():
    """The reference arm (the oracle on the host cores) keeps the bench line's
    contract: rank 0 prints one JSON line with the same metric and workload as
    the kernels' arm; the other ranks of a multi-process launch exit 0 silently."""
    assert _run_reference_arm(1, 2) == []
    lines = _run_reference_arm(0, 2)
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["n_gpus"] == 2
    assert line["config"]["workload"] == "swin_t_stage1_p4_m8" and line["steps"] == 1 and line["warmup"] == 3
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
