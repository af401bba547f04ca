"""The bench's algorithmic byte counts (the numerators of every GB/s it
reports), checked against the sizes of the arrays one call actually reads
and writes, built with numpy at the workload's shapes (no GPU)."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from w8_quantized_linear_b200 import synth  # noqa: E402


def _nbytes(*shapes_dtypes):
    return sum(int(np.prod(s)) * np.dtype(d).itemsize for s, d in shapes_dtypes)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("M,N,K,g", [(1, 6144, 4096, 0), (4, 28672, 4096, 0), (4, 4096, 4096, 128),
                                     (1, 4096, 14336, 0)])
def test_quantise_plus_layer_bytes(mode, M, N, K, g):
    G = K // 128
    reads = [((N, K // 2), np.uint8)] * (1 if mode == 0 else 2)  # planes
    reads += [((N, G), np.float16), ((M, K), np.float16)]  # scales, activations
    writes = [((M, K), np.int8), ((M,) if g == 0 else (M, G), np.float32),
              ((M, N), np.float32)]  # codes, their scales, y (no group sums: the layer forms them)
    assert bench.fused_bytes(mode, M, N, K, g) == _nbytes(*reads, *writes)


@pytest.mark.parametrize("mode", [0, 1])
def test_layer_bytes(mode):
    M, N, K = 4, 14336, 4096
    G = K // 128
    arrays = [((N, K // 2), np.uint8)] * (1 if mode == 0 else 2)
    arrays += [((N, G), np.float16), ((M, K), np.int8), ((M,), np.float32), ((M, N), np.float32)]
    assert bench.linear_bytes(mode, M, N, K) == _nbytes(*arrays)


def test_step_and_round_bytes_cover_every_group_and_pass():
    per_pass = {mode: 0 for mode in bench.DECODE_M}
    for _, members in bench.LAYER_GROUPS:
        N = sum(synth.LLAMA3_8B_PROJECTIONS[m][0] for m in members)
        K, g = synth.LLAMA3_8B_PROJECTIONS[members[0]][1:]
        for mode, M in bench.DECODE_M.items():
            per_pass[mode] += bench.fused_bytes(mode, M, N, K, g)
    assert bench.decode_step_bytes() == per_pass[0] + per_pass[1]
    assert bench.round_bytes() == bench.ROUND_LAYERS * (bench.ROUND_DRAFT_PASSES * per_pass[0]
                                                        + per_pass[1])
    # the 7 projections' planes appear once per pass (hi; hi and lo)
    planes = sum(N * K // 2 for N, K, _ in synth.LLAMA3_8B_PROJECTIONS.values())
    assert per_pass[0] > planes and per_pass[1] > 2 * planes


@pytest.mark.parametrize("mode", [0, 1])
def test_attention_bytes(mode):
    H, Hkv, T, D = 32, 8, 2048, 128
    planes = [((T * Hkv, D // 2), np.uint8)] * (2 if mode == 0 else 4)  # K, V (hi; hi and lo)
    scales = [((T * Hkv, D // 128), np.float16)] * 2
    io = [((H, D), np.float16), ((H, D), np.float32)]
    assert bench.attention_bytes(mode, H, Hkv, T, D) == _nbytes(*planes, *scales, *io)
