"""Host logic of bench.py that needs no GPU: the clock/throttle record taken
during the timed region, and the number of rotating weight copies."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _Done:
    """Stands in for the finished nvidia-smi sampler process."""
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _stop(tmp_path, monkeypatch, lines):
    path = tmp_path / "clk.csv"
    path.write_text("".join(ln + "\n" for ln in lines))
    s = bench.ClockSampler(0)
    s.proc, s.path = _Done(), str(path)
    monkeypatch.setattr(bench.time, "sleep", lambda _s: None)
    return s.stop()


NA, ACT = "Not Active", "Active"


def _row(mhz, reasons=(NA, NA, NA, NA), mx=1965):
    return ", ".join(["0", str(mhz), str(mx), "650.1", "0x0"] + list(reasons))


def test_clock_record_takes_the_median_of_the_loaded_samples(tmp_path, monkeypatch):
    r = _stop(tmp_path, monkeypatch, [_row(345), _row(1965), _row(1950), _row(1965), _row(1900), _row(1965)])
    assert r["sm_max_mhz"] == 1965 and r["reasons"] == [] and r["samples"] == 6
    assert r["sm_mhz"] == 1965                     # top half: 1965, 1965, 1965


def test_clock_record_names_every_reason_seen(tmp_path, monkeypatch):
    r = _stop(tmp_path, monkeypatch, [_row(1900, (NA, NA, NA, ACT)), _row(1300, (ACT, NA, NA, ACT)),
                         _row(1800, (NA, NA, ACT, NA))])
    assert r["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]


def test_clock_record_skips_unreadable_fields_and_short_lines(tmp_path, monkeypatch):
    r = _stop(tmp_path, monkeypatch, ["garbage", _row("[N/A]"), _row(1965), "0, 1, 2"])
    assert r["samples"] == 2 and r["sm_mhz"] == 1965
    assert _stop(tmp_path, monkeypatch, [])["reasons"] == ["no samples"]


def test_rotating_copies_exceed_four_l2_and_respect_the_cap():
    l2 = 126 << 20
    for nbytes in (73728, 20971520, 47513600, 655360000):
        r = bench.rotating_copies(nbytes, l2)
        assert r * nbytes >= min(4 * l2, (6 << 30) // nbytes * nbytes) and r >= 1
        assert r * nbytes <= max(6 << 30, nbytes)
    assert bench.rotating_copies(47513600, l2) == 12     # 570 MB for the in_proj headline


def test_replica_throughput_counts_every_rank():
    assert bench.replica_throughput(1000, 10, 1e-6, 1) == 10.0
    assert bench.replica_throughput(1000, 10, 1e-6, 4) == 40.0


def test_all_core_oracle_baseline_covers_disjoint_row_ranges():
    import numpy as np
    from packed_bit_weight_b200 import synth
    rng = np.random.default_rng(0)
    p = synth.gen_fp4(rng, 64, 256)
    x = synth.gen_x(rng, 1, 256)
    r = bench.cpu_oracle_gemv_all_cores(p, x, budget_s=0.05, threads=3)
    assert r["cores"] == 3 and r["value"] > 0 and r["kind"] == "oracle" and r["unit"] == "GB/s"
    assert "48 of 64 rows in 3 disjoint ranges" in r["sample"]
    assert r["cpu"]["nproc"] >= 1 and r["cpu"]["model"]


def test_gemm_oracle_baseline_reports_tflops_of_its_sample():
    r = bench.cpu_oracle_gemm(budget_s=0.01, rows=32, tokens=4)
    assert r["unit"] == "TFLOP/s" and r["value"] > 0 and r["cores"] == 1 and r["kind"] == "oracle"
    assert r["sample"].startswith("32 of 18560 rows x 4 of 2048 tokens, k = 4096")


def test_input_manifest_pins_the_seeded_generators():
    """The bench records the SHA-256 of every generated input buffer; the
    seeded generators must keep drawing the same bytes (an input that changes
    shows up here before it shows up as a different timing)."""
    from packed_bit_weight_b200 import synth
    p, x = synth.make_gemv(synth.IQ4_TINY)
    m = bench.input_manifest(p, x, synth.IQ4_TINY.seed)
    assert m["w_data_sha256"] == "813fb1eda2d42bdad81bb5712c038bfe886fb361cf73a380175e96423c2fd45e"
    assert m["x_sha256"] == "a7fee885ac3cea9ead24bc682ae86dc698fae11aba47f6cafd6f0eb423e63a51"
    assert m["w_scales_sha256"] is None and m["w_data_bytes"] == 256 * 16 * 18 and m["x_bytes"] == 1024
    p, x = synth.make_gemv(synth.FP4_IN_PROJ)
    m = bench.input_manifest(p, x, synth.FP4_IN_PROJ.seed)
    assert m["w_data_bytes"] == 18560 * 4096 // 2 and m["w_scales_bytes"] == 18560 * 4096 // 16 * 2
    assert m["x_bytes"] == 2 * 4096
    # the headline workload's bytes: the hashes its bench lines record
    assert m["w_data_sha256"] == "07e75c9359e62a11bd8c8294416246a722595e0f36c5feec2d61081bf6f967fe"
    assert m["w_scales_sha256"] == "4d534c0f7b8502b73dc8aab103f5c188980a7fed4b67bda941892f97ab8c03d5"
    assert m["x_sha256"] == "12904c048eb2e764a96b57dc6966c304b4da34aeafe420f5e20e7bf9433e9d7a"


def test_config_selection_runs_only_that_configurations_workloads(monkeypatch):
    """`--config N` (extra_workloads(only=N)) measures exactly configuration
    N's workloads; no selection measures every workload."""
    import types

    import numpy as np
    from packed_bit_weight_b200 import synth

    class P:
        n, k = 16, 32

    monkeypatch.setattr(synth, "make_sweep", lambda *a, **k: {"out_proj": (P(), np.zeros((16, 32), np.uint16)),
                                                               "lm_head": (P(), np.zeros((16, 32), np.uint16))})
    monkeypatch.setattr(synth, "make_gemv", lambda *a, **k: (P(), np.zeros((1, 32), np.uint16)))
    fake = {"variant": "v", "gbs": 1.0, "s_per_launch": 1e-6}
    monkeypatch.setattr(bench, "gemv_workload", lambda *a, **k: fake)
    for name in ("gemm_workload", "grouped_workload", "moe_workload", "dequant_workload", "quantize_workload"):
        monkeypatch.setattr(bench, name, lambda *a, **k: {"x": 1})
    args = types.SimpleNamespace(steps=20, warmup=5)
    peaks = {"hbm_gbs": 1.0}
    keys = {n: set(bench.extra_workloads(args, 1, 1 << 27, peaks, only=n)) for n in (1, 3, 4, 5)}
    assert keys[1] == {"iq4nl_gemv_tiny_256x512_m1"}
    assert keys[3] == {"fp4g16_%s_%s_m%d" % (op, mat, m) for mat in ("out_proj", "lm_head")
                       for op, ms in (("gemv", (1, 4, 16)), ("gemm", (32, 64))) for m in ms}
    assert keys[4] == {"iq4nl_grouped_experts_t64_top4", "iq4nl_moe_block_t64_top4", "iq4nl_moe_block_t1_top4"}
    assert keys[5] == {"%s_prefill_gemm_2048x18560x4096" % f for f in ("fp4g16", "fp4g16_e4m3", "mxfp4", "iq4nl")}
    full = set(bench.extra_workloads(args, 1, 1 << 27, peaks))
    assert full >= keys[1] | keys[3] | keys[4] | keys[5]
    assert {"fp4g16_e4m3_gemv_in_proj_m1", "mxfp4_gemv_in_proj_m1", "fp4g16_dequant_in_proj"} <= full


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one
    JSON line with the contract's keys, the headline's config and input
    manifest, and e2e equal to its own value."""
    import json
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3", "--cpu-budget", "0.05"], capture_output=True, text=True, timeout=600,
                       cwd=root, env={k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE")})
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e", "gpu_launches", "inputs"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 3 and line["warmup"] == 3 and line["value"] > 0
    assert line["config"]["workload"] == "fp4g16_gemv_mamba2_8b_in_proj_18560x4096_m1"
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["inputs"]["w_data_sha256"].startswith("07e75c9359e62a11")
