"""The device-side copy of the counter-based generator (torch int64 ops) draws the same stream as
the numpy one: identical integers, and normals equal to the last few fp64 bits.  Run on the CPU
device; the GPU uses the same code."""
import numpy as np
import torch

import synthetic as syn


def test_torch_stream_matches_numpy_stream():
    n, std = 10_001, 0.02
    for name, offset in (("x", 0), ("expert.3.gate_up", 12_345), ("router.w", 7)):
        host = (syn.normal(0, name, offset, n) * std).astype(np.float32)
        dev = syn.torch_normal_fp32(0, name, n, std, torch.device("cpu"), offset=offset).numpy()
        # same draws: equal after fp32 rounding except, rarely, one ulp
        diff = np.abs(dev.view(np.int32).astype(np.int64) - host.view(np.int32).astype(np.int64))
        assert diff.max() <= 1
        assert (diff == 0).mean() > 0.999


def test_streams_differ_by_name_and_seed():
    a = syn.torch_normal_fp32(0, "x", 64, 1.0, torch.device("cpu"))
    b = syn.torch_normal_fp32(0, "y", 64, 1.0, torch.device("cpu"))
    c = syn.torch_normal_fp32(1, "x", 64, 1.0, torch.device("cpu"))
    assert not torch.equal(a, b) and not torch.equal(a, c)
