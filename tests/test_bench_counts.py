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
