"""GPU parity of the down_proj input path (online Hadamard rotation +
per-token quantisation, bitnest_hadamard_quantize_act) against the oracle.

The oracle rotates in fp64 by the definition (x H / sqrt(K)) and quantises
the fp32-rounded result; the GPU rotates in fp32 (Walsh-Hadamard per block,
then the order-28 mix).  So the per-token scale agrees to a relative 1e-5,
and a code may differ by one only where the exact rotated value sits within
1e-3 of a rounding tie of x_rot / s; elsewhere codes are equal.  The group
sums are exactly those of the GPU's codes, and the down_proj layer on them
matches the oracle's layer on its own codes."""
import numpy as np
import pytest

import oracle
import w8_quantized_linear_b200 as bn
from w8_quantized_linear_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 1e-3

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from test_gpu_parity import dev, host  # noqa: E402


def _check(x):
    M, K = x.shape
    xq, xs, xsum = bn.hadamard_quantize_act(dev(x))
    torch.cuda.synchronize()
    xq, xs, xsum = host(xq).astype(np.int64), host(xs), host(xsum)
    q_ref, xs_ref, xr = oracle.hadamard_quantize(x)
    assert np.all(np.abs(xs - xs_ref) <= 1e-5 * xs_ref)
    t = np.abs(xr / np.where(xs_ref > 0, xs_ref, 1.0)[:, None])
    near_tie = np.abs(t - np.floor(t) - 0.5) < 1e-3
    d = np.abs(xq - q_ref.astype(np.int64))
    assert np.all(d[~near_tie] == 0)
    assert np.all(d[near_tie] <= 1)
    assert np.array_equal(xsum, xq.reshape(M, K // 128, 128).sum(axis=2))
    return xq, xs, q_ref, xs_ref


@pytest.mark.parametrize("M,K", [(1, 14336), (4, 14336), (3, 1024), (2, 4096), (5, 3584),
                                 (1, 128), (2, 896), (9, 7168)])
def test_hadamard_quantize_matches_oracle(M, K):
    x = synth.activations(6000 + M + K, M, K)
    if M > 1:
        x[1] = 0  # an all-zero token: scale 0, codes 0
    _check(x)


def test_hadamard_quantize_then_down_proj_layer():
    """The rotated, quantised down_proj input through the target layer."""
    M, N, K = 4, 256, 14336
    x = synth.activations(6100, M, K)
    xq, xs, q_ref, xs_ref = _check(x)
    rng = np.random.default_rng(2)
    uh = rng.integers(0, 16, (N, K), dtype=np.uint8)
    ul = rng.integers(0, 16, (N, K), dtype=np.uint8)
    s = synth.group_scales(2100, N, K)
    d_hi, d_lo = bn.pack_planes(dev(uh), dev(ul))
    d_xq, d_xs, d_xsum = bn.hadamard_quantize_act(dev(x))
    y = bn.linear(1, d_hi, d_lo, dev(s), d_xq, d_xs, d_xsum)
    torch.cuda.synchronize()
    y_ref = oracle.linear(1, oracle.pack_plane(uh), oracle.pack_plane(ul), s,
                          q_ref.astype(np.int8), xs_ref, K)
    assert oracle.max_normalised_error(host(y), y_ref) <= TOL


def test_cluster_path_equals_one_cta_path():
    """Decode sizes of K = 28 x 512 run on a 7-CTA cluster per token, larger
    batches on one CTA per token; both take the same arithmetic in the same
    order, so the codes, scales and sums of the same rows are identical."""
    K = 14336
    x = synth.activations(6200, 20, K)
    x[3] = 0
    small = [host(t) for t in bn.hadamard_quantize_act(dev(x[:5]))]  # cluster kernel
    large = [host(t) for t in bn.hadamard_quantize_act(dev(x))]      # one CTA per token
    torch.cuda.synchronize()
    for a, b in zip(small, large):
        assert np.array_equal(a, b[:5])
    _check(x[:5])
