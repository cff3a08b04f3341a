"""Failure detection without a GPU fault: a bounded device-side wait that runs out (needs a B200)."""
import ctypes

import pytest
import torch

from sub_quadratic_two_squad_b200 import _lib
from test_gpu_parity import LG, run_fwd

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_survives():
    lib = _lib.load()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    # a wait on a barrier nothing completes, limited to 2 ms
    assert lib.squad_wait_selftest(ctypes.c_void_p(status.data_ptr()), 2_000_000, None) == _lib.SQUAD_OK
    torch.cuda.synchronize()
    assert int(status.item()) == _lib.SQUAD_ERR_TIMEOUT
    # the context is still usable and correct
    run_fwd(1, 2, 128, (21, 4, 8), (21, 2, 4), LG, torch.bfloat16)
