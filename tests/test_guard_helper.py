"""The sentinel guard that the GPU tests put around every output buffer (in
place of a memory sanitizer) detects a write one byte before or after the
buffer and passes when only the buffer itself is written; run on the CPU."""
import pytest
import torch

from nvfp4_testutil import GUARD_BYTES, Guarded


def test_guard_passes_writes_inside():
    g = Guarded((3, 5), torch.float32, fill=1.0, device="cpu")
    g.t.fill_(2.0)
    assert torch.equal(g.check("inside"), torch.full((3, 5), 2.0))
    assert g.t.data_ptr() % 16 == 0


@pytest.mark.parametrize("offset", [-1, 0])
def test_guard_catches_a_byte_outside(offset):
    g = Guarded(100, torch.uint8, device="cpu")
    i = GUARD_BYTES - 1 if offset < 0 else GUARD_BYTES + 100
    g.raw[i] = 0
    with pytest.raises(AssertionError):
        g.check("outside")
