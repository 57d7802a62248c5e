"""Host-side pieces of bench.py that need no GPU: workload accounting, the kernel-source
hash that keys recorded ncu traffic, the shape of the roofline record, and the reference
arm (the oracle timed on the host)."""
import os

import bench


def test_kernel_source_sha_covers_subfolders(tmp_path, monkeypatch):
    sha = bench.kernel_source_sha()
    assert len(sha) == 16 and sha == bench.kernel_source_sha()
    # a file in a subfolder of csrc changes the hash (the device generator lives in one)
    root = tmp_path / "repo"
    (root / "state_space_model_05_b200" / "csrc" / "gen").mkdir(parents=True)
    (root / "state_space_model_05_b200" / "csrc" / "a.cu").write_text("x")
    (root / "state_space_model_05_b200" / "csrc" / "gen" / "b.cu").write_text("y")
    monkeypatch.setattr(bench, "ROOT", str(root))
    h1 = bench.kernel_source_sha()
    (root / "state_space_model_05_b200" / "csrc" / "gen" / "b.cu").write_text("z")
    assert bench.kernel_source_sha() != h1


def test_kernel_source_sha_ignores_comments_not_code(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    (root / "state_space_model_05_b200" / "csrc").mkdir(parents=True)
    src = root / "state_space_model_05_b200" / "csrc" / "k.cu"
    src.write_text("// old note\nint f() { return 1; }  /* block */\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    h1 = bench.kernel_source_sha()
    src.write_text("// a rewritten note\nint f()   {\n  return 1; }\n")
    assert bench.kernel_source_sha() == h1
    src.write_text("int f() { return 2; }\n")
    assert bench.kernel_source_sha() != h1


def test_recorded_traffic_requires_matching_source(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    (root / "state_space_model_05_b200" / "csrc").mkdir(parents=True)
    (root / "state_space_model_05_b200" / "csrc" / "k.cu").write_text("k")
    (root / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(root))
    sha = bench.kernel_source_sha()
    (root / "profiles" / "ncu_traffic.txt").write_text(
        f"kernel=kx workload=wy source_sha={sha} dram_bytes_per_launch=1234\n"
        f"kernel=kx workload=wz source_sha=0000000000000000 dram_bytes_per_launch=99\n")
    assert bench.recorded_traffic("kx", "wy") == 1234
    assert bench.recorded_traffic("kx", "wz") is None
    assert bench.recorded_traffic("other", "wy") is None


def test_prefill_accounting():
    w = bench.WORKLOADS["prefill_2p7b_long"]
    b, T, H, P, N = 4, 16384, 80, 64, 128
    byts = bench.prefill_bytes(w)
    # whole path: x, y bf16; B, C bf16; dt fp32; final state fp32
    assert byts["total"] == b * T * (2 * H * P * 2 + 2 * N * 2 + H * 4) + b * H * P * N * 4
    # the output kernel moves at least x, y and one bf16 state per 128-token block
    assert byts["chunk_output_tc"] > b * T * 2 * H * P * 2 + b * H * (T // 128) * P * N * 2
    f256, f128 = bench.prefill_flops(w)["total"], bench.prefill_flops(w, 128)["total"]
    assert f256 == b * T * ((256 + 1) * N + H * ((256 + 1) * P + 4 * N * P))
    assert f128 < f256
    assert bench.tc_path(w) and not bench.tc_path(dict(w, dtype="f32"))


def test_roofline_prefill_record():
    w = bench.WORKLOADS["prefill_130m"]
    res = {"kernels": {"chunk_cumsum": (1.0, 100), "chunk_state_scan_tc": (4.0, 100),
                       "chunk_output_tc": (5.0, 100)}}
    peaks = {"hbm_gbs": 6545.3, "bf16_tflops": 1651.2}
    r = bench.roofline_prefill(w, res, peaks, "measured", "prefill_130m")
    # the prefill is a dense contraction: measured against the tensor peak, with the dominant
    # kernel's share of the causal-exact FLOPs per launch over its launch duration
    assert r["kernel"] == "chunk_output_tc" and r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    b, T, H, P, N = 8, 2048, 24, 64, 128
    flops = b * T * (257 * N + H * (257 * P + 2 * N * P))      # C B^T, masked X, state -> output
    assert r["kernel_flops"] == flops
    expect = flops / (0.05e-3) / 1e12
    assert abs(r["achieved"] - expect) < 1e-6 * expect
    assert abs(r["frac"] - r["achieved"] / 1651.2) < 1e-12
    # the path's algorithmic bytes: x, dt, B, C read once, y and the final state written once
    assert r["algorithmic_bytes"] == b * T * (2 * H * P * 2 + 2 * N * 2 + H * 4) + b * H * P * N * 4
    assert set(r) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}
    # the fused path's dominant kernel carries every GEMM but C B^T
    fused = bench.roofline_prefill(w, {"kernels": {"chain_prefill_tc": (3.0, 100), "block_gram_tc": (0.5, 100)}},
                                   peaks, "measured", "prefill_130m")
    assert fused["kernel_flops"] == b * T * H * (257 * P + 4 * N * P)


def test_reference_arm_line(monkeypatch, capsys):
    """`bench.py --impl reference`: the oracle timed on the host, one JSON line with the
    contract's keys, on rank 0 only."""
    import json
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    # the oracle's per-step sample is sized from this budget: keep the test to seconds
    monkeypatch.setattr(bench, "oracle_sample_step", _fast_sample(bench.oracle_sample_step))
    assert bench.main(["--impl", "reference", "--workload", "prefill_130m", "--steps", "1", "--warmup", "3"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == "SSD prefill tokens/s"
    assert line["value"] > 0 and line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["steps"] == 1 and line["warmup"] == 3 and line["config"]["workload"] == "prefill_130m"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_decode_line(monkeypatch, capsys):
    """The decode workloads' reference arm: the oracle's decode steps on a sample of units,
    scaled to whole steps."""
    import json
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    real = bench.oracle_decode_rate
    monkeypatch.setattr(bench, "oracle_decode_rate", lambda w, budget, nthreads=0, seed=0: real(w, 0.05, nthreads, seed))
    assert bench.main(["--impl", "reference", "--workload", "decode_2p7b", "--steps", "1", "--warmup", "3"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == "SSD decode steps/s" and line["unit"] == "steps/s"
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["value"] == line["value"] and line["config"]["workload"] == "decode_2p7b"


def test_reference_arm_other_ranks_do_nothing(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(bench, "oracle_sample_step", lambda *a: (_ for _ in ()).throw(AssertionError("ran")))
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""


def _fast_sample(step):
    """The real oracle step on at most two (batch, head) units."""
    def run(w, inp, units, nthreads=0):
        return step(w, inp, list(units)[:2], nthreads)
    return run


def test_oracle_baselines_keep_all_cores_after_a_single_core_run():
    """An OpenMP thread-count setting persists in the process: the all-core oracle timings
    must still use every core after a single-core one."""
    w = bench.WORKLOADS["decode_2p7b"]
    one = bench.oracle_decode_rate(w, 0.02, nthreads=1)
    assert one[4] == 1
    rate, nu, steps, el, cores = bench.oracle_decode_rate(w, 0.02)
    assert cores == bench.host_cores() and rate > 0 and nu >= 64
