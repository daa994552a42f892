"""Host-side arithmetic of bench.py (CPU only): the algorithmic bytes and MUFU
operation counts that the roofline figures divide by, and the sweep schedule
the kernels follow."""
import bench


def test_algorithmic_bytes_per_channel_step():
    N = 8 * 4096 * 1024
    # scans: read A and b, write the state
    assert bench.algorithmic_bytes("scan_diag", False, 8, 4096, 1024) == 12 * N
    assert bench.algorithmic_bytes("scan_block2", False, 8, 4096, 1024) == 32 * N
    # GRU, one sweep: P (3 gates) read once, h written once; h^0 = 0 is not read
    assert bench.algorithmic_bytes("gru", False, 8, 4096, 1024, passes=1) == 16 * N
    assert bench.algorithmic_bytes("gru", True, 8, 4096, 1024, passes=1) == 10 * N
    # a second sweep re-reads P and reads + writes the iterate
    assert bench.algorithmic_bytes("gru", False, 8, 4096, 1024, passes=2) == (16 + 20) * N
    # LSTM: 4 gates, (c, h) state
    assert bench.algorithmic_bytes("lstm", False, 8, 4096, 1024, passes=1) == 24 * N
    assert bench.algorithmic_bytes("lstm", False, 8, 4096, 1024, passes=2) == (24 + 32) * N


def test_sweep_schedule_matches_kernel_defaults():
    # 4 iterations in the first sweep, 2 per later sweep, capped at max_iters + 1
    assert bench.evaluated_iterations(1, 32) == 4
    assert bench.evaluated_iterations(2, 32) == 6
    assert bench.evaluated_iterations(3, 32) == 8
    assert bench.evaluated_iterations(1, 2) == 3
    assert bench.evaluated_iterations(2, 4) == 5


def test_traffic_record_is_tied_to_kernel_sources():
    d1 = bench.kernel_source_digest()
    assert d1 == bench.kernel_source_digest() and len(d1) == 64
    traffic, why = bench.recorded_traffic("no-such-workload")
    assert traffic is None


def test_traffic_record_scaling(tmp_path, monkeypatch):
    """A capture of a shorter sequence is scaled to the full launch; a record
    taken on other sources is refused."""
    import json

    (tmp_path / "profiles").mkdir()
    digest = bench.kernel_source_digest()
    rec = {"kernels": {
        "short": {"dram_bytes_per_launch": 1000, "scale": 8, "capture": "L=1024",
                  "source_sha256": digest},
        "full": {"dram_bytes_per_launch": 1234, "capture": "full", "source_sha256": digest},
        "stale": {"dram_bytes_per_launch": 1, "source_sha256": "0" * 64}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: digest)
    t, src = bench.recorded_traffic("short")
    assert t == 8000 and "x 8" in src
    assert bench.recorded_traffic("full")[0] == 1234
    t, why = bench.recorded_traffic("stale")
    assert t is None and "changed" in why


def test_backward_and_projection_bytes():
    N = 8 * 4096 * 1024
    # backward: read P, the trajectory one step behind and dl/dh (and dl/dc); write dP
    assert bench.algorithmic_bytes("gru_bwd", False, 8, 4096, 1024) == 32 * N
    assert bench.algorithmic_bytes("lstm_bwd", False, 8, 4096, 1024) == 48 * N
    # projection: x [M, K] and W [N, K] in bf16 once, the bias, P once
    M, Nf, K = 8 * 4096, 3 * 1024, 1024
    assert bench.projection_bytes(M, Nf, K, False) == 2 * M * K + 2 * Nf * K + 4 * Nf + 4 * M * Nf
    assert bench.projection_bytes(M, Nf, K, True) == 2 * M * K + 2 * Nf * K + 4 * Nf + 2 * M * Nf
    # multi-head solve: every Newton evaluation streams P and the iterate
    assert bench.algorithmic_bytes("mhgru", False, 8, 4096, 1024, passes=4) == 4 * 20 * N


def test_reference_arm_runs_every_new_workload(capsys):
    """The oracle arm prints one JSON line for the projection and the multi-head
    workloads (bounded samples; no GPU)."""
    import argparse
    import json

    from tests import inputs

    for wl in ("proj", "mhgru", "gru_l"):
        args = argparse.Namespace(workload=wl, steps=1, warmup=1)
        bench.run_reference(args, 1, 0, 0)
        line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
        assert line["impl"] == "reference" and line["value"] > 0
        assert line["e2e"]["h2d_bytes_per_step"] == 0
        # the same config.workload as our arm's line for this workload
        w = inputs.WORKLOADS[wl]
        assert line["config"]["workload"] == bench.workload_name(
            wl, w["B"], w["L"], w["D"], w.get("K"), w.get("G"))
        assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT


def test_cpu_baseline_reports_threaded_and_single_thread():
    """The CPU leg times the oracle's Newton and rollout on the host cores and
    on one thread (a small GRU case, CPU only)."""
    import bench
    import oracle
    from tests import inputs

    x = inputs.gru_inputs(1, 64, 8, seed=5)
    out = bench.cpu_baseline(x, "gru", 1, 64, 8, budget_s=0.05)
    assert out["kind"] == "oracle" and out["cores"] >= 1 and out["value"] > 0
    st = out["single_thread"]
    assert st["newton_channel_steps_per_s"] > 0 and st["rollout_channel_steps_per_s"] > 0
    assert oracle.get_threads() == out["cores"]   # the thread count is restored


def test_cpu_baseline_projected_solve():
    """The CPU leg of the fused projection + solve workload: the oracle's fp64
    projection of a channel sample followed by its serial Newton (small case)."""
    from tests import inputs

    x = inputs.projected_gru_inputs(1, 64, 16, 32, seed=6)
    out = bench.cpu_baseline(x, "proj_solve", 1, 64, 16, budget_s=0.05)
    assert out["kind"] == "oracle" and out["value"] > 0 and out["cores"] >= 1
    assert "projection" in out["sample"]
