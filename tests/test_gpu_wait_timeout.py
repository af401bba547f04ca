"""GPU: the bounded in-kernel wait and its flag.  A kernel waits, with the
layer kernels' own bounded mbarrier wait, on a barrier that nothing arrives
at: the wait gives up, the kernel returns, the host reads the flag, clears it,
and the library keeps working.  Nothing faults, traps or hangs."""
import numpy as np
import pytest

import oracle
import w8_quantized_linear_b200 as bn

pytestmark = pytest.mark.gpu
TOL = 1e-3

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from test_gpu_parity import Problem, host  # noqa: E402


def test_wait_that_runs_out_sets_the_flag_and_the_library_recovers():
    assert bn.device_wait_timeout(reset=True) == 0
    try:
        bn.debug_wait_probe()
        torch.cuda.synchronize()
        assert bn.device_wait_timeout(reset=True) == 1
        assert bn.device_wait_timeout() == 0
        p = Problem(4, 300, 1024, seed=12)
        for path in (bn.PATH_GEMV, bn.PATH_TC):
            y = host(bn.linear(1, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum, path=path))
            assert oracle.max_normalised_error(y, p.y_ref(1)) <= TOL
        torch.cuda.synchronize()
        assert bn.device_wait_timeout() == 0
    finally:
        bn.device_wait_timeout(reset=True)


def test_split_k_after_a_timeout_on_caller_and_static_scratch():
    """After the probe's wait ran out and the flag was cleared, split-K calls
    on caller scratch and on the library's static scratch match the oracle."""
    from test_gpu_parity import DEV

    M, N, K = 16, 300, 1024
    p = Problem(M, N, K, seed=41)
    try:
        bn.debug_wait_probe()
        torch.cuda.synchronize()
        assert bn.device_wait_timeout(reset=True) == 1
        for mode in (0, 1):
            ws = bn.workspace(bn.linear_ws_bytes(mode, M, N, K, bn.PATH_TC), DEV)
            args = (mode, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum)
            y_ws = bn.linear_ws(*args, ws, path=bn.PATH_TC)
            y_st = bn.linear_static_ws(*args, path=bn.PATH_TC)
            torch.cuda.synchronize()
            for y in (y_ws, y_st):
                assert oracle.max_normalised_error(host(y), p.y_ref(mode)) <= TOL
            assert torch.equal(y_ws, y_st)
        assert bn.device_wait_timeout() == 0
    finally:
        bn.device_wait_timeout(reset=True)


def test_split_k_call_that_gives_up_leaves_counters_at_zero():
    """A split-K call that starts while the flag of a run-out wait is still
    set gives up at its first wait that does not complete at once and winds
    down (its output is invalid).  Every warp still makes its arrival on the
    split counters, so the caller's scratch is left at zero and needs no
    clearing; clearing the flag also clears the static scratch's counters.
    Calls after that match the oracle."""
    from test_gpu_parity import DEV

    M, N, K = 16, 300, 1024
    p = Problem(M, N, K, seed=43)
    args = (1, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum)
    try:
        ws = bn.workspace(bn.linear_ws_bytes(1, M, N, K, bn.PATH_TC), DEV)
        bn.debug_wait_probe()
        bn.linear_ws(*args, ws, path=bn.PATH_TC)
        bn.linear_static_ws(*args, path=bn.PATH_TC)
        torch.cuda.synchronize()
        assert int(torch.count_nonzero(ws[:8192])) == 0
        assert bn.device_wait_timeout(reset=True) == 1
        y_ws = bn.linear_ws(*args, ws, path=bn.PATH_TC)
        y_st = bn.linear_static_ws(*args, path=bn.PATH_TC)
        torch.cuda.synchronize()
        assert oracle.max_normalised_error(host(y_ws), p.y_ref(1)) <= TOL
        assert torch.equal(y_ws, y_st)
        assert bn.device_wait_timeout() == 0
    finally:
        bn.device_wait_timeout(reset=True)
