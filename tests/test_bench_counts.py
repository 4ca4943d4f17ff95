"""The algorithmic counts bench.py divides by (per token and head, chunk C, head dim d): the
per-kernel FLOP of the tensor-core path sum to the totals of the chunkwise form, and the step's HBM
bytes are the layer's own tensors read and written once."""
import bench


def test_kernel_flops_sum_to_the_chunkwise_totals():
    for C, d in [(64, 128), (16, 32)]:
        Cd, dd = C * d, d * d
        fwd = sum(bench.kernel_flops(k, C, d) for k in ("kda_fwd_prep_tc", "kda_fwd_scan_tc", "kda_fwd_out_tc"))
        bwd = sum(bench.kernel_flops(k, C, d) for k in ("kda_bwd_scan_tc", "kda_bwd_dq_tc",
                                                         "kda_bwd_dkv_tc"))
        assert fwd == 10 * Cd + 6 * dd
        assert bwd == 18 * Cd + 14 * dd
        assert bench.kernel_flops("not_a_kernel", C, d) == 0


def test_step_bytes_are_inputs_and_outputs_once():
    d = 128
    # forward: q, k, v, g (bf16, 2 d each) and beta (2) in, o (2 d) out;
    # backward: those and dO in, dq, dk, dv (bf16) and dg (fp32, 4 d), dbeta (fp32, 4) out
    fwd = 4 * 2 * d + 2 + 2 * d
    bwd = 4 * 2 * d + 2 + 2 * d + 3 * 2 * d + 4 * d + 4
    assert (fwd, bwd) == (1282, 2566)
    assert bench.step_bytes_per_token_head(d) == fwd + bwd


def test_peaks_loader_reads_measured_file_and_falls_back(tmp_path, monkeypatch):
    """The roofline denominators: the measured file when present (keys found by name, nested or
    flat), the pool's earlier measurement when absent or unreadable."""
    import json
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_peaks()["source"] == "fallback"
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6431.7, "bf16_tflops": 1550.0, "bf16_tflops_sustained": 1380.0}))
    p = bench.load_peaks()
    assert (p["source"], p["hbm_gbs"], p["bf16_tflops"], p["sustained"]) == ("measured", 6431.7, 1550.0, 1380.0)
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm": {"copy_gbs": 6400}, "bf16": {"burst_tflops": 1500, "sustained_tflops": 1350}}))
    p = bench.load_peaks()
    assert (p["hbm_gbs"], p["bf16_tflops"], p["sustained"]) == (6400.0, 1500.0, 1350.0)
    (tmp_path / "MEASURED_PEAKS.json").write_text("{not json")
    assert bench.load_peaks()["source"] == "fallback"
