"""GPU: the allocation-free split-K entry point (bitnest_linear_static_ws,
the library's own static device scratch) against the entry point that takes
caller scratch (bitnest_linear_ws), two calls in a row each.

Collected last on purpose: the static scratch is shared by every call in the
process, and these tests leave it as they found it (counters at zero)."""
import numpy as np
import pytest

import oracle
import w8_quantized_linear_b200 as bn

pytestmark = pytest.mark.gpu
TOL = 1e-3

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from test_gpu_parity import DEV, Problem, host  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _no_earlier_timeout():
    """The static scratch is shared by the whole process: start only from a
    clean state (no bounded wait has given up, so no split call has left
    arrivals behind), which a failure here would otherwise be blamed on."""
    assert bn.device_wait_timeout() == 0
    yield


@pytest.mark.parametrize("M,N,K,path", [(16, 300, 1024, bn.PATH_TC), (1, 100, 4096, bn.PATH_TC),
                                        (128, 256, 14336, bn.PATH_TC),
                                        (8, 4096, 14336, bn.PATH_AUTO)])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("act_group", [0, 128])
def test_static_scratch_matches_caller_scratch(M, N, K, path, mode, act_group):
    """The same split plan and summation order: bit-identical y from the two
    entry points, on each of two calls in a row, and y matches the oracle
    (8 tokens at K = 14336: the automatic choice with scratch splits K)."""
    p = Problem(M, N, K, seed=17 * M + N + K, act_group=act_group)
    nbytes = bn.linear_ws_bytes(mode, M, N, K, path)
    assert nbytes > 0
    ws = bn.workspace(nbytes, DEV)
    args = (mode, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum)
    ys = []
    for _ in range(2):
        ys.append(bn.linear_ws(*args, ws, act_group, path=path))
        ys.append(bn.linear_static_ws(*args, act_group, path=path))
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])
    assert oracle.max_normalised_error(host(ys[1]), p.y_ref(mode)) <= TOL
    assert bn.device_wait_timeout(reset=True) == 0


def test_static_scratch_without_split_is_linear():
    """Where nothing is split the call needs no scratch and is bitnest_linear."""
    p = Problem(4, 300, 4096, seed=9)
    assert bn.linear_ws_bytes(1, 4, 300, 4096) == 0
    y = bn.linear_static_ws(1, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum)
    y0 = bn.linear(1, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum)
    torch.cuda.synchronize()
    assert torch.equal(y, y0)


def test_static_scratch_shared_by_shapes():
    """Calls of different shapes in turn on the one static scratch each equal
    the caller-scratch result."""
    shapes = [(16, 300, 1024), (128, 256, 14336), (8, 4096, 14336)]
    probs = [Problem(M, N, K, seed=M + K) for M, N, K in shapes]
    for rnd in range(2):
        for p in probs:
            args = (0, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum)
            y = bn.linear_static_ws(*args, path=bn.PATH_TC)
            ws = bn.workspace(bn.linear_ws_bytes(0, p.M, p.N, p.K, bn.PATH_TC), DEV)
            y0 = bn.linear_ws(*args, ws, path=bn.PATH_TC)
            torch.cuda.synchronize()
            assert torch.equal(y, y0), (rnd, p.M, p.N, p.K)


def test_static_scratch_back_to_back_with_programmatic_launch():
    """Several static-scratch calls of different split shapes in a row on one
    stream, with programmatic dependent launch and no synchronisation between
    them: each y equals the caller-scratch result, and no wait gave up."""
    shapes = [(16, 300, 1024), (128, 256, 14336), (8, 4096, 14336), (33, 129, 2048)]
    probs = [Problem(M, N, K, seed=3 * M + K) for M, N, K in shapes]
    path = bn.PATH_TC | bn.PATH_OVERLAP
    ys = [bn.linear_static_ws(1, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum, path=path)
          for p in probs for _ in range(2)]
    torch.cuda.synchronize()
    for i, p in enumerate(probs):
        ws = bn.workspace(bn.linear_ws_bytes(1, p.M, p.N, p.K, bn.PATH_TC), DEV)
        y0 = bn.linear_ws(1, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum, ws, path=bn.PATH_TC)
        torch.cuda.synchronize()
        assert torch.equal(ys[2 * i], y0) and torch.equal(ys[2 * i + 1], y0), (p.M, p.N, p.K)
    assert bn.device_wait_timeout(reset=True) == 0
