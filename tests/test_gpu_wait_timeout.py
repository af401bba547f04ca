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
