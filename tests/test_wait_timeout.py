"""Bounded device waits: a wait that nothing satisfies gives up with BSA_ERR_TIMEOUT and
leaves the context usable (no fault, trap or hang)."""
import ctypes
import time

import pytest

from view_transformers_b200 import _lib


def test_selftest_argument_validation():
    lib = _lib.load()
    E = _lib
    assert lib.bsa_selftest_wait_timeout(None, 1000, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_selftest_wait_timeout(0x10000, 0, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_selftest_wait_timeout(0x10000, 10_000_001, None) == E.BSA_ERR_INVALID_ARG
    assert lib.bsa_selftest_wait_timeout(0x10002, 1000, None) == E.BSA_ERR_INVALID_ARG   # misaligned


@pytest.mark.gpu
def test_wait_gives_up_with_timeout_status():
    import torch
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    _lib.bsa_selftest_wait_timeout(status.data_ptr(), 20_000, st)      # 20 ms limit
    code = _lib.bsa_check_status(status.data_ptr(), st)                # synchronises
    elapsed = time.perf_counter() - t0
    assert code == _lib.BSA_ERR_TIMEOUT
    assert elapsed < 5.0
    assert int(status.item()) == 0                                     # read and reset
    # the context is still usable: a plain launch and a second self-check both work
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float((x * 2).sum().item()) == 2 * 1023 * 1024 / 2
    _lib.bsa_selftest_wait_timeout(status.data_ptr(), 1_000, st)
    assert _lib.bsa_check_status(status.data_ptr(), st) == _lib.BSA_ERR_TIMEOUT
