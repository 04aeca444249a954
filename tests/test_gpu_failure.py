"""GPU failure detection without a GPU fault: a bounded pipeline wait that
runs out must end its kernel with an error status the host reads, and leave
the CUDA context usable for the next call."""
import pytest
import torch

import h3_inputs as hi
from joint_video_audio_b200 import _binding as B
from tests._parity import GpuCase

pytestmark = pytest.mark.gpu


def _stream():
    return torch.cuda.current_stream().cuda_stream


def test_wait_that_completes_reports_ok():
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert B.h3blk_selftest_wait(True, 50, word.data_ptr(), _stream()) == B.H3BLK_OK
    assert int(word.item()) == 0


def test_wait_that_never_completes_reports_timeout_and_context_survives():
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert B.h3blk_selftest_wait(False, 50, word.data_ptr(), _stream()) == B.H3BLK_ERR_TIMEOUT
    assert int(word.item()) != 0
    # the context still runs kernels: a whole block forward, error word clean
    c = GpuCase(hi.make_inputs("tiny_320"))
    out = c.run()
    assert torch.isfinite(out.float()).all()
    assert c.block.check(c.ws, c.n) == B.H3BLK_OK
    # and the self-test's own word is reset by the next call
    assert B.h3blk_selftest_wait(True, 50, word.data_ptr(), _stream()) == B.H3BLK_OK
