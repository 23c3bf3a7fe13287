"""The canary-guarded output buffers of the GPU tests (helpers.Guarded), on
the CPU: writes inside the view pass, a write one element past either end is
reported with its side."""
import pytest
import torch

from helpers import Guarded


def test_guard_accepts_writes_inside_and_catches_overruns():
    g = Guarded((3, 5), torch.float32, fill=1.0, device="cpu")
    g.t.fill_(7.0)
    g.check()
    raw = g._raw
    after = Guarded.GUARD + g.t.numel() * 4
    raw[after] = 0  # one byte past the end
    with pytest.raises(AssertionError, match="after"):
        g.check()
    h = Guarded((4,), torch.int32, device="cpu")
    h._raw[Guarded.GUARD - 1] = 0  # one byte before the start
    with pytest.raises(AssertionError, match="before"):
        h.check()
