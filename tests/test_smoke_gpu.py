"""The entry point's smoke check (one fp32 CUDA-core and one bf16 tensor-core forward + backward on the
Figure 1 tree, against the oracle) runs inside the GPU test tier as well."""
import os
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_smoke_entry_point():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    sys.path.insert(0, ROOT)
    import __graft_entry__ as entry
    entry.smoke()
