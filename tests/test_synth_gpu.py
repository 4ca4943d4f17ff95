"""The device generator twin writes the same bits as the host generator."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def test_device_generator_matches_host():
    import torch
    import synth.gpu as sg
    sg.lib()
    rows = np.array([0, 1, 7, 123, 4095, 70000, 29072], np.int64)
    tr = torch.tensor(rows, dtype=torch.int32, device="cuda")
    for dtype in ("bf16", "f32"):
        dev = [x.float().cpu().numpy() for x in sg.kda_inputs(1, tr, 16, 128, 128, dtype)]
        host = synth.kda_inputs(1, rows, 16, 128, 128, dtype)
        for a, b in zip(dev, host):
            mism = int(np.sum(a != b.astype(np.float32)))
            assert mism == 0, (dtype, mism)
    d_o = sg.normal_rows(1, synth.STREAM["d_o"], tr, 16 * 128, "bf16").float().cpu().numpy()
    assert np.array_equal(d_o, synth.rows_normal(1, synth.STREAM["d_o"], rows, 16 * 128, "bf16").astype(np.float32))
    z = sg.normal_rows(3, 9, None, 64, "f32", scale=0.5, shape=(5,)).cpu().numpy()
    assert np.array_equal(z, synth.normal_tensor(3, 9, (5, 64), "f32", 0.5).astype(np.float32))
