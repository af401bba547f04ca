"""GPU parity of the packer from fp16 weights (bitnest_pack_weights) against
the oracle: planes and fp16 scales bit for bit, on random weights of several
magnitudes, on values placed at the rounding ties of both nibbles, on
all-zero and subnormal groups, and on the full Llama-3-8B gate projection
(sampled rows); then the packed layer against the oracle's layer."""
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


def _check(w16):
    hi, lo, sc = bn.pack_weights(dev(w16))
    torch.cuda.synchronize()
    uh, ul, sc_ref = oracle.pack_weights(w16)
    assert np.array_equal(host(hi), oracle.pack_plane(uh))
    assert np.array_equal(host(lo), oracle.pack_plane(ul))
    assert np.array_equal(host(sc).view(np.uint16), sc_ref)


@pytest.mark.parametrize("N,K", [(1, 128), (3, 384), (64, 1024), (300, 4096), (17, 14336)])
@pytest.mark.parametrize("mag", [1e-3, 0.02, 3.0, 3000.0])
def test_pack_weights_bit_exact(N, K, mag):
    rng = np.random.default_rng(N + K)
    _check((rng.standard_normal((N, K)) * mag).astype(np.float16))


def test_pack_weights_ties_zero_and_subnormal_groups():
    rng = np.random.default_rng(8)
    K = 1024
    w = np.zeros((6, K))
    # s = 1: every half-integer t (ties of the high nibble) and every t whose
    # residual 16 (t - q4) lands on a tie or on +-8
    base = np.concatenate([np.arange(-13, 14) / 2.0, np.arange(-112, 113) / 16.0,
                           np.arange(-224, 225) / 32.0])
    w[0, :base.size] = base
    w[0, 0] = 7.0
    w[1] = rng.standard_normal(K) * 1e-6  # subnormal fp16 scales
    w[2, 128:256] = rng.standard_normal(128) * 0.01  # other groups all zero
    w[3] = rng.standard_normal(K) * 60000.0 / 5  # near the top of fp16
    w[4] = np.repeat(rng.choice([-7.0, 7.0], K // 4), 4)
    w[5] = rng.integers(-112, 113, K) / 16.0
    w = np.clip(w, -65504, 65504).astype(np.float16)
    _check(w)


def test_pack_weights_llama3_gate_sampled():
    N, K, _ = synth.LLAMA3_8B_PROJECTIONS["gate_proj"]
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    hi, lo, sc = bn.pack_weights(dev(w))
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, 1, N - 1], rng.choice(N, 64, replace=False)]))
    uh, ul, sc_ref = oracle.pack_weights(w[rows])
    assert np.array_equal(host(hi)[rows], oracle.pack_plane(uh))
    assert np.array_equal(host(lo)[rows], oracle.pack_plane(ul))
    assert np.array_equal(host(sc).view(np.uint16)[rows], sc_ref)


@pytest.mark.parametrize("mode", [0, 1])
def test_packed_layer_matches_oracle(mode):
    """Weights -> planes on the GPU -> the layer on the GPU, against the
    oracle's layer on the oracle's packing of the same weights."""
    M, N, K = 4, 200, 2048
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    x = synth.activations(77, M, K)
    hi, lo, sc = bn.pack_weights(dev(w))
    xq, xs, xsum = bn.quantize_act(dev(x), 0)
    y = bn.linear(mode, hi, lo, sc, xq, xs, xsum)
    torch.cuda.synchronize()
    uh, ul, sc_ref = oracle.pack_weights(w)
    q, xs_ref = oracle.quantize(x, 0)
    y_ref = oracle.linear(mode, oracle.pack_plane(uh), oracle.pack_plane(ul) if mode else None,
                          sc_ref, q, xs_ref, K)
    assert oracle.max_normalised_error(host(y), y_ref) <= TOL
