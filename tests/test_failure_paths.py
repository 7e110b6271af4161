"""Failure detection without a GPU fault.

On the host: invalid arguments, shapes, cache states and workspace sizes are
refused before anything is enqueued (tests/test_abi.py). On the GPU: a kernel
whose bounded mbarrier wait can never complete gives up after a short limit,
raises the workspace's device error word and returns; the host reads it as
QI21_ERR_DEVICE_TIMEOUT and the context stays usable for the next call.
"""
import pytest
import torch


@pytest.fixture(scope="module")
def B():
    from prefix_kv_cached_b200 import build
    build.build()
    from prefix_kv_cached_b200 import binding
    return binding


def test_selftest_argument_checks(B):
    assert B.qi21_selftest_wait_timeout(0, 64, 1000, 0) == B.QI21_ERR_INVALID_ARG
    assert B.qi21_selftest_wait_timeout(0x10000, 64, 0, 0) == B.QI21_ERR_INVALID_ARG
    assert B.qi21_selftest_wait_timeout(0x10000, 64, 2_000_000_000, 0) == B.QI21_ERR_INVALID_ARG


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_context_survives(B):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert B.qi21_check_device_error(ws, ws.numel(), st) == B.QI21_OK
    assert B.qi21_selftest_wait_timeout(ws, ws.numel(), 2_000_000, st) == B.QI21_OK     # 2 ms limit
    assert B.qi21_check_device_error(ws, ws.numel(), st) == B.QI21_ERR_DEVICE_TIMEOUT
    # the word is cleared and the context still runs work
    assert B.qi21_check_device_error(ws, ws.numel(), st) == B.QI21_OK
    x = torch.ones(1024, device="cuda")
    out = torch.empty_like(x)
    B.check("euler", B.qi21_euler_update(x, x, 1.0, 0.5, out, 1024, st))
    torch.cuda.synchronize()
    assert float(out[0]) == 0.5
