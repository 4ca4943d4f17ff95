"""The shared input generator: Philox known answers, distributions, trees."""
import numpy as np

import synth


def test_philox_known_answers():
    # Known-answer vectors published with Philox4x32-10 (Random123 distribution)
    assert [int(x) for x in synth.philox4x32_10(0, 0, 0, 0, 0, 0)] == [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]
    f = 0xFFFFFFFF
    assert [int(x) for x in synth.philox4x32_10(f, f, f, f, f, f)] == [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]
    assert [int(x) for x in synth.philox4x32_10(0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344,
                                                0xA4093822, 0x299F31D0)] == [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]


def test_normal_moments_and_bf16_rounding():
    z = synth.normal_f64(5, 1, np.arange(200000))
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    b = synth.round_bf16(np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5]))
    assert b.tolist() == [1.0, 1.0 + 2 ** -6, -2.5]  # ties to even


def test_kda_inputs_distribution_and_row_independence():
    q, k, v, g, beta = synth.kda_inputs(0, np.arange(500), 2, 32, 32, "f32")
    assert np.allclose(np.linalg.norm(k, axis=-1), 1, atol=1e-6)
    assert np.all(g < 0) and np.all((beta > 0) & (beta < 1))
    # any subset of rows regenerates the same values
    sub = synth.kda_inputs(0, np.array([7, 400]), 2, 32, 32, "f32")
    assert np.array_equal(sub[1], k[[7, 400]]) and np.array_equal(sub[4], beta[[7, 400]])


def test_workload_trees():
    t = synth.workload("fig1").tree
    assert (t.n_rows, t.n_expanded()) == (121, 225)
    sf = synth.workload("single_fork").tree
    assert sf.n == 17 and sf.length[0] == 8192 and np.all((sf.length[1:] >= 512) & (sf.length[1:] <= 2048))
    ag = synth.workload("agentic").tree
    assert len(ag.leaves()) == 64 and np.all(ag.parent[1:] < np.arange(1, ag.n))
    wd = synth.workload("wide").tree
    assert wd.n == 585 and len(wd.leaves()) == 512
