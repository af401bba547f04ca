"""GPU parity of decode attention over a nested KV cache
(bitnest_nested_attention) against the oracle: the cache is packed on the
GPU with bitnest_pack_weights (bit-exact with the oracle's packing), and the
fp32 attention output matches the oracle's fp64 one within the layer's
normalised-error bar, for the draft (KV4) and the target (KV8).  The cases
span one token, ragged tiles of 16, token ranges that leave some CTAs of a
KV head's cluster empty (T = 1025 over 16 CTAs of 80 tokens), a 16-CTA
cluster (T = 8192) and every group size (1, 2, 4, 8 query heads per KV
head)."""
import numpy as np
import pytest

import oracle
import w8_quantized_linear_b200 as bn

pytestmark = pytest.mark.gpu
TOL = 1e-3

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from test_gpu_parity import dev, host  # noqa: E402


@pytest.mark.parametrize("H,Hkv,T", [(32, 8, 1), (32, 8, 100), (8, 2, 2048), (4, 4, 37),
                                     (16, 2, 9), (8, 8, 300), (32, 8, 8192), (32, 8, 1025),
                                     (8, 1, 65), (16, 8, 4111)])
@pytest.mark.parametrize("mode", [0, 1])
def test_nested_attention_matches_oracle(H, Hkv, T, mode):
    D = 128
    rng = np.random.default_rng(H * 1000 + T)
    q = rng.standard_normal((H, D)).astype(np.float16)
    k = (rng.standard_normal((T * Hkv, D)) * 0.8).astype(np.float16)
    v = rng.standard_normal((T * Hkv, D)).astype(np.float16)
    kp, vp = bn.pack_weights(dev(k)), bn.pack_weights(dev(v))
    out = bn.nested_attention(mode, dev(q), kp, vp, Hkv)
    torch.cuda.synchronize()
    kp_ref, vp_ref = oracle.kv_pack(k), oracle.kv_pack(v)
    for got, ref in zip(kp + vp, kp_ref + vp_ref):
        assert np.array_equal(host(got).view(ref.dtype), ref)
    ref = oracle.nested_attention(mode, q, kp_ref, vp_ref, Hkv)
    assert oracle.max_normalised_error(host(out), ref) <= TOL
